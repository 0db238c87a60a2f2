// Channel scaling + krot Givens stages with tensor memory as the permutation
// network (sm_100a), for large token counts.
//
// Same arithmetic as rotate_kernel (GPTQModel wiki page "ParoQuant",
// "Pairwise Givens rotations" and "Activation and weight transforms"):
// X_r = X D^-1 R, a' = a cos t + b sin t, b' = -a sin t + b cos t, stages in
// order, pair indices local to the 128-channel group, fp32 on chip, one
// round-to-nearest to fp16 at the end.
//
// A CTA owns one 128-channel group and walks over 128-row tiles (blockIdx.y,
// blockIdx.y + gridDim.y, ...), so its stage tables are built once.  Row t of a
// tile lives in TMEM lane t; the 8 warps are (lane quadrant, half of the pairs).
// A stage needs, in every row, the two channels of each pair side by side;
// registers cannot be indexed by a runtime pair table, but a tcgen05.ld of one
// column per lane takes a warp-uniform column address.  So a warp gathers the
// 64 operands of its 32 pairs (one-column loads), rotates them in registers at
// compile-time register indices, and writes the results with bulk stores in
// that "slot" order into the other of two 128-column buffers; the next stage's
// gather table is composed with that order.  The two warps of a lane quadrant
// meet at a named barrier once per stage (four warps per quadrant measured
// slower: more barrier traffic, no better latency hiding).  The last stage scatters to the
// natural channel order and bulk loads bring each warp's half row back.
// Tensor memory is split between the SM sub-partitions, so a stage's data
// movement does not funnel through the one shared-memory pipe that bounds
// rotate_kernel.
//
// Slot order of a stage: pairs 2u and 2u+1 form unit u, whose four slots hold
// (a_2u, a_2u+1, b_2u, b_2u+1), so a unit is rotated with packed fp32x2 fmas.
//
// Factored rotations (the square-root-free Givens form of Gentleman, 1973):
// the value kept for a channel is its true value divided by a per-channel
// factor f that depends only on the tables, so it is known when they are
// built.  A pair (a, b) with factors (fa, fb) then takes two fmas,
// a' = a + kA b and b' = b + kB a.  If |cos| >= |sin|: kA = tan * fb / fa,
// kB = -tan * fa / fb and both factors take a cos.  Otherwise the two
// channels trade slots: the slot of a receives b's new value and the slot of
// b a's, with kA = -cot * fb / fa, kB = cot * fa / fb and factors (-sin fa)
// for b and (sin fb) for a (tan, cot here mean sin/cos, cos/sin).  Choosing
// the larger of |cos|, |sin| keeps |tan|, |cot| <= 1 and each factor within
// [2^(-s/2), 1] of its start after s stages.  The starting factor is the
// channel scale, so the input is not scaled; the final factors multiply the
// output once.
//
// With ABS the gather tables hold absolute TMEM addresses, one copy per lane
// quadrant, so a gather is a quarter of a table read and one load; without it
// (many stages) one table of columns is offset by the quadrant's lane base.
// Input tiles arrive by TMA (two 64-channel boxes, 128-byte swizzle, so the
// row-per-thread reads are conflict-free) into two buffers, two tiles ahead of
// use.
//
// With QUANT the rows are weight rows (out x in) and the kernel is the
// weight-side quantiser of the same page, section "Activation and weight
// transforms": W_r = W D R with D = 1 / channel_scales (the scaling step
// multiplies by D evaluated once per channel in fp32), then four-bit symmetric
// codes q = clamp(rint(W_r / s), -8, 7) + 8 with s the group scale bounded to
// [1e-5, 1e5] (the quotient as W_r times the fp32 reciprocal of s, rounded to
// nearest even), written straight into the AWQ layout: the codes of a tile go
// to shared memory transposed (channel-major bytes), and each packed word
// collects eight output rows' codes of one channel in the nibble order
// (0, 2, 4, 6, 1, 3, 5, 7).  qzeros gets the constant zero code 8.
#pragma once

#include "rotate.cuh"

namespace paro {

constexpr int kRtRows = 128;
constexpr int kRtWpq = 2;                // warps per TMEM lane quadrant (each takes 128/kRtWpq slots)
constexpr int kRtThreads = 128 * kRtWpq; // warps: (lane quadrant, slot range)
constexpr int kRtCols = 256;             // two 128-column buffers
constexpr int kRtMaxCtasPerSm = 2;       // 2 x 256 TMEM columns
constexpr int kRtAbsMaxKrot = 16;        // per-quadrant address tables up to this many stages
constexpr size_t kRtMinSmem = 80 * 1024; // above a third of an SM's shared memory: <= 2 CTAs/SM

// Output of the quantising instantiation (rows = N output channels).
struct RtQuant {
  const void* scales;     // [K/G, N] quantiser scales (activation type)
  int32_t* qweight;       // [K, N/8] AWQ words
  int32_t* qzeros;        // [K/G, N/8] AWQ words (all 8)
};

struct RtLayout {
  // IN tiles[2] | scale[128] | per stage (c0,c1,s0,s1)[32 units] |
  // gather addresses[Q][krot][128] | scatter addresses[Q][128] | raw pairs[krot][64] |
  // pos[128] | mbarriers[2] | tmem slot, abort flag
  // (Q = 4 lane quadrants for up to kRtAbsMaxKrot stages, else 1 table of columns)
  static constexpr size_t TILE = (size_t)kRtRows * 128 * 2;      // two 64-channel boxes
  static constexpr size_t BOX = TILE / 2;
  static constexpr size_t CS_STAGE = 32 * 16;
  __host__ __device__ static constexpr int copies(int krot) { return krot <= kRtAbsMaxKrot ? 4 : 1; }
  __host__ __device__ static constexpr size_t scale_off() { return 2 * TILE; }
  __host__ __device__ static constexpr size_t cs_off() { return scale_off() + 128 * 4; }
  __host__ __device__ static constexpr size_t g_off(int krot) { return cs_off() + (size_t)krot * CS_STAGE; }
  __host__ __device__ static constexpr size_t f_off(int krot) {
    return g_off(krot) + (size_t)copies(krot) * krot * 128 * 4;
  }
  __host__ __device__ static constexpr size_t praw_off(int krot) { return f_off(krot) + (size_t)copies(krot) * 128 * 4; }
  __host__ __device__ static constexpr size_t pos_off(int krot) { return praw_off(krot) + (size_t)krot * 64 * 4; }
  __host__ __device__ static constexpr size_t bar_off(int krot) { return pos_off(krot) + 128 * 4; }
  __host__ __device__ static constexpr size_t slot_off(int krot) { return bar_off(krot) + 16; }
  // quantiser only: the tile's codes, channel-major bytes [128 channels][128 rows]
  __host__ __device__ static constexpr size_t codes_off(int krot) { return slot_off(krot) + 16; }
  static constexpr size_t CODES = 128 * 128;
  // + 1 KB so the tiles can be aligned to the 1024 bytes the swizzle pattern needs
  __host__ __device__ static constexpr size_t bytes(int krot, bool quant = false) {
    return codes_off(krot) + (quant ? CODES : 0) + 1024 < kRtMinSmem
               ? kRtMinSmem
               : codes_off(krot) + (quant ? CODES : 0) + 1024;
  }
};

// The warps of lane quadrant qd: their TMEM accesses so far are complete
// and visible to each other.  Barrier ids are immediates (5 hardware barriers).
__device__ __forceinline__ void rt_quadrant_sync(int qd) {
  tmem_st_wait();
  tc_fence_before();
  switch (qd) {
    case 0: asm volatile("bar.sync 1, %0;" ::"n"(32 * kRtWpq) : "memory"); break;
    case 1: asm volatile("bar.sync 2, %0;" ::"n"(32 * kRtWpq) : "memory"); break;
    case 2: asm volatile("bar.sync 3, %0;" ::"n"(32 * kRtWpq) : "memory"); break;
    default: asm volatile("bar.sync 4, %0;" ::"n"(32 * kRtWpq) : "memory"); break;
  }
  tc_fence_after();
}

// Four-bit AWQ word of eight codes (bytes c0..c7 of output rows 8w .. 8w+7):
// nibble t holds the code of row 8w + (0, 2, 4, 6, 1, 3, 5, 7)[t].
__device__ __forceinline__ uint32_t rt_awq_word(uint32_t lo, uint32_t hi) {
  const uint32_t e = __byte_perm(lo, hi, 0x6420);   // c0 c2 c4 c6
  const uint32_t o = __byte_perm(lo, hi, 0x7531);   // c1 c3 c5 c7
  const uint32_t e4 = (e & 0xFu) | ((e >> 4) & 0xF0u) | ((e >> 8) & 0xF00u) | ((e >> 12) & 0xF000u);
  const uint32_t o4 = (o & 0xFu) | ((o >> 4) & 0xF0u) | ((o >> 8) & 0xF00u) | ((o >> 12) & 0xF000u);
  return e4 | (o4 << 16);
}

// grid: (K/128, row-tile slots), block 256.  tmX is x as [M, K] fp16 with box
// {64 channels, 128 rows}, 128-byte swizzle (rows past M read as zeros).
// QUANT: x is W [N = M, K], xr is unused and qo receives the packed codes.
template <bool ABS, bool QUANT, typename TA>
__global__ void __launch_bounds__(kRtThreads, kRtMaxCtasPerSm) rotate_tmem_kernel(
    const __grid_constant__ CUtensorMap tmX, TA* xr, const float* __restrict__ cs,
    const int16_t* __restrict__ pairs, const float* __restrict__ theta, int M, int K, int krot, int gsz,
    const RtQuant qo) {
  using L = RtLayout;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  unsigned char* const sb = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t in_base = smem_u32(sb);
  float* scale = reinterpret_cast<float*>(sb + L::scale_off());
  unsigned char* cstab = sb + L::cs_off();
  uint32_t* gtab = reinterpret_cast<uint32_t*>(sb + L::g_off(krot));
  uint32_t* ftab = reinterpret_cast<uint32_t*>(sb + L::f_off(krot));
  uint32_t* praw = reinterpret_cast<uint32_t*>(sb + L::praw_off(krot));
  int* pos = reinterpret_cast<int*>(sb + L::pos_off(krot));
  const uint32_t bar0 = smem_u32(sb + L::bar_off(krot));
  uint32_t* slot = reinterpret_cast<uint32_t*>(sb + L::slot_off(krot));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(slot + 1);

  const int grp = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, h = warp >> 2;            // lane quadrant, slot range
  const int ntiles = (M + kRtRows - 1) / kRtRows;
  const int gy = (int)gridDim.y;

  // Wait for the previous kernel before reading any input.  Tensor memory is
  // taken before dependents may launch: a dependent GEMM that allocates TMEM
  // early can then never hold what this kernel still needs.
  pdl_wait_primary();
  if (warp == 0) {
    tmem_alloc(smem_u32(slot), kRtCols);
    tmem_relinquish();
  }
  int issued = 0;                                    // tiles whose load thread 0 has issued
  if (tid == 0) {
    mbar_init(bar0, 1);
    mbar_init(bar0 + 8, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmX);
    // the first two tiles are in flight while the tables are built
    for (int b = 0; b < 2; ++b) {
      const int t = (int)blockIdx.y + b * gy;
      if (t >= ntiles) break;
      ++issued;
      mbar_arrive_expect_tx(bar0 + 8 * b, (uint32_t)L::TILE);
      tma_load_2d(in_base + b * (uint32_t)L::TILE, &tmX, bar0 + 8 * b, grp * kGroup, t * kRtRows);
      tma_load_2d(in_base + b * (uint32_t)L::TILE + (uint32_t)L::BOX, &tmX, bar0 + 8 * b,
                  grp * kGroup + 64, t * kRtRows);
    }
  }

  // ---- tables, 1: every stage's pairs and angles, loads issued together.
  // Indices outside the group are masked to 7 bits (every address stays inside
  // this CTA's allocation) and flagged.
  if (tid < 128) {
    const float c = cs != nullptr ? cs[grp * kGroup + tid] : 1.0f;
    scale[tid] = QUANT ? 1.0f / c : c;               // weights take D = 1 / channel_scales
  }
  for (int idx = tid; idx < krot * 64; idx += kRtThreads) {
    const int s = idx >> 6, p = idx & 63, u = p >> 1, w = p & 1;
    const uint32_t pr =
        *reinterpret_cast<const uint32_t*>(pairs + (size_t)s * K + (size_t)grp * kGroup + 2 * p);
    int i, j;
    tile_pair(pr, p, gsz, &i, &j);                   // tile channels of the pair's group
    praw[idx] = (uint32_t)i | ((uint32_t)j << 16);
    float sn, c;
    rot_sincos(theta[(size_t)s * (K / 2) + (size_t)grp * 64 + p], &sn, &c);
    float* csu = reinterpret_cast<float*>(cstab + s * L::CS_STAGE) + 4 * u;
    csu[w] = c;
    csu[2 + w] = sn;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // the quantiser writes layer constants (qweight, qzeros): it never releases
  // its dependents early, so a following call may read them before its wait
  if constexpr (!QUANT) pdl_launch_dependents();
  const uint32_t tmem0 = *slot;

  // ---- tables, 2 (warp 0): stage s reads buffer (s & 1) and writes buffer
  // ((s + 1) & 1); a slot's gather entry is where its channel sits in that
  // buffer: the channel index (s = 0) or its slot in stage s-1.  With ABS an
  // entry is the full TMEM address for each lane quadrant, else the column.
  // The unit table's (cos, sin) become the factored form's (kA, kB), and
  // scale[] follows every channel's factor (the final factors at the end).
  constexpr int Q = ABS ? 4 : 1;
  if (warp == 0) {
#pragma unroll
    for (int c = 0; c < 4; ++c) pos[lane + 32 * c] = lane + 32 * c;
    __syncwarp();
    for (int s = 0; s < krot; ++s) {
      int si[2], sj[2], ii[2], jj[2];
      bool tr[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int p = lane + 32 * e, u = p >> 1, w = p & 1;
        const uint32_t pr = praw[s * 64 + p];
        ii[e] = (int)(pr & 0xFFFFu);
        jj[e] = (int)(pr >> 16);
        si[e] = 4 * u + w;
        sj[e] = 4 * u + 2 + w;
        const uint32_t ci = (uint32_t)((s & 1) * 128 + pos[ii[e]]);
        const uint32_t cj = (uint32_t)((s & 1) * 128 + pos[jj[e]]);
        // factored form of this pair (each channel belongs to one pair of the
        // stage, so its factor is read and written by this lane only)
        float* csu = reinterpret_cast<float*>(cstab + s * L::CS_STAGE) + 4 * u;
        const float c = csu[w], sn = csu[2 + w];
        const float fa = scale[ii[e]], fb = scale[jj[e]];
        const bool trade = fabsf(sn) > fabsf(c);
        float ka, kb, nfa, nfb;
        if (!trade) {
          const float t = sn / c;
          ka = t * (fb / fa);
          kb = -t * (fa / fb);
          nfa = c * fa;
          nfb = c * fb;
        } else {
          const float t = c / sn;
          ka = -t * (fb / fa);
          kb = t * (fa / fb);
          nfa = sn * fb;                             // a's new value, now in b's slot
          nfb = -sn * fa;                            // b's new value, now in a's slot
        }
        csu[w] = ka;
        csu[2 + w] = kb;
        scale[ii[e]] = nfa;
        scale[jj[e]] = nfb;
        tr[e] = trade;
#pragma unroll
        for (int q = 0; q < Q; ++q) {
          const uint32_t lb = ABS ? tmem0 + ((uint32_t)(32 * q) << 16) : 0u;
          gtab[((size_t)q * krot + s) * 128 + si[e]] = lb + ci;
          gtab[((size_t)q * krot + s) * 128 + sj[e]] = lb + cj;
          if (s == krot - 1) {                       // the last stage scatters to channel order
            ftab[q * 128 + si[e]] = lb + (uint32_t)((krot & 1) * 128 + (trade ? jj[e] : ii[e]));
            ftab[q * 128 + sj[e]] = lb + (uint32_t)((krot & 1) * 128 + (trade ? ii[e] : jj[e]));
          }
        }
      }
      __syncwarp();
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        pos[ii[e]] = tr[e] ? sj[e] : si[e];
        pos[jj[e]] = tr[e] ? si[e] : sj[e];
      }
      __syncwarp();
    }
  }
  __syncthreads();

  constexpr int SW = 128 / kRtWpq;                   // slots (channels) per warp
  const int r = 32 * qd + lane;                      // row within the tile = TMEM lane
  const uint32_t lbase = tmem0 + ((uint32_t)(32 * qd) << 16);
  const uint32_t goff = ABS ? 0u : lbase;            // added to a table entry
  // this warp's SW slots of stage 0 and of the final scatter
  const uint32_t g_part = smem_u32(gtab + (ABS ? (size_t)qd * krot * 128 : 0) + SW * h);
  const uint32_t f_part = smem_u32(ftab + (ABS ? qd * 128 : 0) + SW * h);
  const uint32_t cs_part = smem_u32(cstab) + 4u * SW * h;            // units SW/4 * h ..
  const float4* scale4 = reinterpret_cast<const float4*>(scale + SW * h);
  const uint32_t rsw = (uint32_t)(r & 7);            // swizzle phase of row r

  int it = 0;
  for (int tile = blockIdx.y; tile < ntiles; tile += gy, ++it) {
    const int buf = it & 1;
    // ---- row r, channels SW*h .. SW*h+SW-1: swizzled 16-byte chunks, scaled
    if (!mbar_wait_bounded(bar0 + 8 * buf, (uint32_t)((it >> 1) & 1))) *abort_flag = 1;
    uint32_t v[SW];
    const unsigned char* rowp = sb + buf * L::TILE + ((SW * h) >> 6) * L::BOX + r * 128;
    const int q0 = ((SW * h) & 63) >> 3;             // first 16-byte chunk in the box row
#pragma unroll
    for (int q = 0; q < SW / 8; ++q) {
      const uint4 raw = *reinterpret_cast<const uint4*>(rowp + ((((uint32_t)(q0 + q)) ^ rsw) << 4));
      const uint32_t hv[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {                  // the channel scale is the starting factor
        const float2 f = Act<TA>::f2(hv[e]);
        v[8 * q + 2 * e] = __float_as_uint(f.x);
        v[8 * q + 2 * e + 1] = __float_as_uint(f.y);
      }
    }
    __syncthreads();                                 // every row read: this buffer is free
    if (*abort_flag) break;                          // uniform: set only before the barrier
    if (tid == 0 && tile + 2 * gy < ntiles) {
      ++issued;
      const int nrow = (tile + 2 * gy) * kRtRows;
      const uint32_t dstb = in_base + buf * (uint32_t)L::TILE;
      mbar_arrive_expect_tx(bar0 + 8 * buf, (uint32_t)L::TILE);
      tma_load_2d(dstb, &tmX, bar0 + 8 * buf, grp * kGroup, nrow);
      tma_load_2d(dstb + (uint32_t)L::BOX, &tmX, bar0 + 8 * buf, grp * kGroup + 64, nrow);
    }

    if (krot > 0) {
#pragma unroll
      for (int b = 0; b < SW / 32; ++b)
        tmem_st32(lbase + SW * h + 32 * b, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * b]));
      rt_quadrant_sync(qd);
      for (int s = 0; s < krot; ++s) {
        // gather this warp's SW slots; table reads run four 16-byte loads ahead
        const uint32_t gs = g_part + (uint32_t)s * 512u;
        uint4 g[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) g[k] = lds128(gs + 16 * k);
#pragma unroll
        for (int k = 0; k < SW / 4; ++k) {
          const uint4 a = g[k & 3];
          v[4 * k] = tmem_ld1(a.x + goff);
          v[4 * k + 1] = tmem_ld1(a.y + goff);
          v[4 * k + 2] = tmem_ld1(a.z + goff);
          v[4 * k + 3] = tmem_ld1(a.w + goff);
          if (k + 4 < SW / 4) g[k & 3] = lds128(gs + 16 * (k + 4));
        }
        tmem_ld_wait_tie(*reinterpret_cast<uint32_t(*)[32]>(&v[0]));
#pragma unroll
        for (int b = 1; b < SW / 32; ++b) tmem_tie(*reinterpret_cast<uint32_t(*)[32]>(&v[32 * b]));
        // rotate the SW/4 units (A = slots 0,1; B = slots 2,3), factored form
        const uint32_t cst = cs_part + (uint32_t)s * (uint32_t)L::CS_STAGE;
#pragma unroll
        for (int k = 0; k < SW / 4; ++k) {
          const uint4 t = lds128(cst + 16 * k);      // (kA0, kA1, kB0, kB1)
          const float2 KA = make_float2(__uint_as_float(t.x), __uint_as_float(t.y));
          const float2 KB = make_float2(__uint_as_float(t.z), __uint_as_float(t.w));
          const float2 A = make_float2(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]));
          const float2 B = make_float2(__uint_as_float(v[4 * k + 2]), __uint_as_float(v[4 * k + 3]));
          const float2 A2 = __ffma2_rn(B, KA, A);
          const float2 B2 = __ffma2_rn(A, KB, B);
          v[4 * k] = __float_as_uint(A2.x);
          v[4 * k + 1] = __float_as_uint(A2.y);
          v[4 * k + 2] = __float_as_uint(B2.x);
          v[4 * k + 3] = __float_as_uint(B2.y);
        }
        if (s + 1 < krot) {
          const uint32_t d = lbase + (uint32_t)((s + 1) & 1) * 128u + (uint32_t)(SW * h);
#pragma unroll
          for (int b = 0; b < SW / 32; ++b) tmem_st32(d + 32 * b, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * b]));
        } else {
          // last stage: scatter to the natural channel order
#pragma unroll
          for (int k = 0; k < SW / 4; ++k) {
            const uint4 f = lds128(f_part + 16 * k);
            tmem_st1(f.x + goff, v[4 * k]);
            tmem_st1(f.y + goff, v[4 * k + 1]);
            tmem_st1(f.z + goff, v[4 * k + 2]);
            tmem_st1(f.w + goff, v[4 * k + 3]);
          }
        }
        rt_quadrant_sync(qd);
      }
      const uint32_t fb = lbase + (uint32_t)(krot & 1) * 128u + (uint32_t)(SW * h);
#pragma unroll
      for (int b = 0; b < SW / 32; ++b) tmem_ld32(fb + 32 * b, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * b]));
      tmem_ld_wait_tie(*reinterpret_cast<uint32_t(*)[32]>(&v[0]));
#pragma unroll
      for (int b = 1; b < SW / 32; ++b) tmem_tie(*reinterpret_cast<uint32_t(*)[32]>(&v[32 * b]));
    }

    // ---- true values of channels SW*h .. SW*h+SW-1: times their final factors
#pragma unroll
    for (int q = 0; q < SW / 4; ++q) {
      const float4 f = scale4[q];
      const float2 lo = __fmul2_rn(make_float2(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1])),
                                   make_float2(f.x, f.y));
      const float2 hi = __fmul2_rn(make_float2(__uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3])),
                                   make_float2(f.z, f.w));
      v[4 * q] = __float_as_uint(lo.x);
      v[4 * q + 1] = __float_as_uint(lo.y);
      v[4 * q + 2] = __float_as_uint(hi.x);
      v[4 * q + 3] = __float_as_uint(hi.y);
    }
    const int row = tile * kRtRows + r;
    if constexpr (QUANT) {
      // ---- codes of row r (an output channel), channels SW*h .. SW*h+SW-1,
      // transposed into shared memory; then 8 AWQ words per thread
      // quantiser scale of each 16-channel chunk (a chunk lies in one group of
      // G >= 16 channels): scales row tile * 128 / G + channel / G
      float inv[SW / 16];
#pragma unroll
      for (int k = 0; k < SW / 16; ++k) {
        const int qg = (grp * kGroup + SW * h + 16 * k) / gsz;
        float sc = row < M ? Act<TA>::f1(static_cast<const TA*>(qo.scales)[(size_t)qg * M + row]) : 1.0f;
        sc = fminf(fmaxf(sc, 1e-5f), 1e5f);
        inv[k] = 1.0f / sc;
      }
      const uint32_t cb = smem_u32(sb + L::codes_off(krot)) + (uint32_t)(SW * h) * 128u + (uint32_t)r;
#pragma unroll
      for (int i = 0; i < SW; ++i) {
        int q = __float2int_rn(__uint_as_float(v[i]) * inv[i / 16]);
        q = min(max(q, -8), 7) + 8;
        asm volatile("st.shared.u8 [%0], %1;" ::"r"(cb + (uint32_t)i * 128u), "r"(q) : "memory");
      }
      __syncthreads();
      const uint32_t c0 = smem_u32(sb + L::codes_off(krot));
      const int nw = M / 8;                           // words per channel row of qweight
#pragma unroll
      for (int j = 0; j < (128 * 16) / kRtThreads; ++j) {
        const int idx = tid + kRtThreads * j, k = idx >> 4, w = idx & 15;
        const int wcol = tile * 16 + w;               // word column: rows 8 wcol .. 8 wcol + 7
        uint32_t lo, hi;
        asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(lo), "=r"(hi) : "r"(c0 + (uint32_t)k * 128u + 8u * w)
                     : "memory");
        if (wcol < nw) qo.qweight[(size_t)(grp * kGroup + k) * nw + wcol] = (int32_t)rt_awq_word(lo, hi);
      }
      // zero words of the tile's 128 / G quantisation groups: all code 8
      for (int z = tid; z < 16 * (kGroup / gsz); z += kRtThreads) {
        const int zr = z >> 4, zc = tile * 16 + (z & 15);
        if (zc < nw) qo.qzeros[(size_t)(grp * (kGroup / gsz) + zr) * nw + zc] = (int32_t)0x88888888u;
      }
    } else if (row < M) {
      // ---- fp16 (round to nearest), row r, channels SW*h .. SW*h+SW-1
      TA* dstp = xr + (size_t)row * K + (size_t)grp * kGroup + SW * h;
#pragma unroll
      for (int q = 0; q < SW / 8; ++q) {
        uint4 out;
        uint32_t* hv = &out.x;
#pragma unroll
        for (int e = 0; e < 4; ++e)
          hv[e] = Act<TA>::p2(__uint_as_float(v[8 * q + 2 * e]), __uint_as_float(v[8 * q + 2 * e + 1]));
        *reinterpret_cast<uint4*>(dstp + 8 * q) = out;
      }
    }
  }
  if (tid == 0 && *abort_flag) {
    // a wait gave up: let the loads still in flight land (bounded) before the
    // shared memory is released
    for (int t = it; t < issued; ++t)
      if (!mbar_wait_bounded(bar0 + 8 * (t & 1), (uint32_t)((t >> 1) & 1))) break;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem0, kRtCols);
  }
}

}  // namespace paro

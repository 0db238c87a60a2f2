// Channel scaling + krot Givens stages on the tensor cores (sm_100a), for
// large token counts.
//
// The stages of one 128-channel group are a fixed linear map of the group's
// channels (GPTQModel wiki page "ParoQuant", "Activation and weight
// transforms": X_r = X D^-1 R; "Pairwise Givens rotations": a' = a cos t +
// b sin t, b' = -a sin t + b cos t, stages in order, pair indices local to the
// group).  With the channel scale folded in, every token row x of group g
// becomes x R'_g with
//     R'_g = diag(cs_g) G_0 G_1 ... G_{krot-1}      (128 x 128, fp32),
// and row k of R'_g is the basis vector e_k, scaled by cs[k] and taken through
// the stages exactly as a token row would be.  So:
//   1. rmat_build_kernel rotates the 128 scaled basis rows of every group in
//      fp32 (the same per-pair arithmetic as the other rotation kernels) and
//      stores R'_g transposed, split into two fp16 parts
//      R'_g = Rhi + Rlo, Rlo = fp16(R'_g - Rhi);
//   2. rotate_tc_kernel computes the block-diagonal product X R' on the
//      tensor cores, X Rhi + X Rlo accumulated in fp32 in tensor memory, and
//      rounds X_r to fp16 once.
// X is fp16 and exact as an MMA operand, and Rhi + Rlo carries R' to about
// 2^-22 relative, so the result is the fp32 rotation up to summation order.
// The cost no longer grows with krot: 2 * 2 * M * 128 * K flops (two fp16
// products) against 4 * M * K bytes of HBM traffic, i.e. 512 flops per 4 bytes
// moved (about 2.1 GFLOP per 16 MB) -- less tensor-core time than the bytes
// take at HBM speed.
//
// The activation type (fp16 or bf16) is a template parameter: with bf16
// activations the parts are bf16 and carry R' to about 2^-16 relative, far
// below the bf16 rounding of X_r.
//
// Layout of the transposed parts in global memory: fp16 [2][K][128]; part 0 is
// Rhi, part 1 is Rlo; row g*128 + n, column k holds R'_g[k][n], i.e. each
// 128-row block is the K-major B operand (N = output channel, K = input
// channel) of one group.
#pragma once

#include "rotate.cuh"

namespace paro {

// ------------------------------------------------------------------ R' build
constexpr int kRbRows = 32;               // basis rows per CTA (4 CTAs per group), one per lane
constexpr int kRbThreads = 256;           // warp w applies pairs 8w .. 8w+7 of every stage
constexpr int kRbPitch = 129;             // fp32 words per row: lanes (rows) hit distinct banks

__host__ __device__ constexpr size_t rb_smem_bytes(int krot) {
  return (size_t)krot * (kGroup / 2) * sizeof(RotParam) + (size_t)kRbRows * kRbPitch * 4;
}

// Linears that rotate the same x (a decoder layer's q/k/v, or gate/up) are
// handled by one launch of each kernel: member i has its own tables, R' parts
// and X_r.
constexpr int kRcMaxMembers = 4;
struct RbOperand {
  const float* cs;         // [K] or nullptr
  const int16_t* pairs;    // [krot, K]
  const float* theta;      // [krot, K/2]
  void* rt;                // R' parts, [2][K][128] of the activation type
  int krot;
};
struct RbBatch {
  RbOperand op[kRcMaxMembers];
};

// grid (K/128, 128/kRbRows, members), block kRbThreads; dynamic shared memory
// for the largest krot of the batch.
// RELEASE: let the kernel that follows launch early (false when the parts are
// prepared layer constants, which later kernels read before they wait).
// INV: the basis rows are scaled by 1 / cs (the weight side, W_r = W D R with
// D = 1 / channel_scales), the reciprocal taken in fp32 as the weight
// quantiser takes it.
template <typename TA, bool RELEASE = true, bool INV = false>
__global__ void __launch_bounds__(kRbThreads) rmat_build_kernel(const __grid_constant__ RbBatch batch, int K,
                                                                int gsz) {
  // The rotation that follows waits for this kernel's completion; let it
  // launch and set itself up meanwhile.
  if constexpr (RELEASE) pdl_launch_dependents();
  const RbOperand& op = batch.op[blockIdx.z];
  const float* __restrict__ cs = op.cs;
  const int16_t* __restrict__ pairs = op.pairs;
  const float* __restrict__ theta = op.theta;
  TA* __restrict__ rt = static_cast<TA*>(op.rt);
  const int krot = op.krot;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  RotParam* prm = reinterpret_cast<RotParam*>(smem_raw);
  const uint32_t vbase = smem_u32(smem_raw + (size_t)krot * (kGroup / 2) * sizeof(RotParam));
  const int grp = blockIdx.x, r0 = blockIdx.y * kRbRows, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;

  // stage tables of the group (layer constants: read before waiting for the
  // kernel ahead); indices outside the group are masked and flagged
  load_rot_params(prm, pairs, theta, K, krot, grp, gsz, tid, kRbThreads);
  // basis rows r0 .. r0+31, scaled: row r has cs[r0 + r] at channel r0 + r
  for (int idx = tid; idx < kRbRows * kGroup; idx += kRbThreads) {
    const int r = idx >> 7, c = idx & (kGroup - 1);
    float val = 0.0f;
    if (c == r0 + r) {
      const float sc = cs != nullptr ? cs[(size_t)grp * kGroup + c] : 1.0f;
      val = INV ? 1.0f / sc : sc;
    }
    sts_f32(vbase + (uint32_t)(r * kRbPitch + c) * 4u, val);
  }
  __syncthreads();

  // stages: lane = basis row, warp = its eight pairs of the stage.  The pairs
  // of a stage are disjoint, so all sixteen operands are loaded before any
  // result is stored, and the warps of a stage never touch the same channel.
  const uint32_t row = vbase + (uint32_t)(lane * kRbPitch) * 4u;
  for (int s = 0; s < krot; ++s) {
    const RotParam* ps = prm + s * (kGroup / 2) + warp * 8;
    RotParam p[8];
    float a[8], b[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) p[q] = ps[q];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      a[q] = lds_f32(row + (uint32_t)p[q].i * 4u);
      b[q] = lds_f32(row + (uint32_t)p[q].j * 4u);
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      sts_f32(row + (uint32_t)p[q].i * 4u, fmaf(a[q], p[q].c, b[q] * p[q].s));
      sts_f32(row + (uint32_t)p[q].j * 4u, fmaf(b[q], p[q].c, -(a[q] * p[q].s)));
    }
    __syncthreads();
  }

  // The parts go into the caller's workspace, which the kernel ahead may
  // still be using.
  pdl_wait_primary();
  // thread (n, h): output channel n, basis rows r0 + 16h .. r0 + 16h + 15
  // (32 contiguous bytes of row g*128 + n of each part)
  const int n = tid & (kGroup - 1), h = tid >> 7;
  uint32_t hi[8], lo[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float va = lds_f32(vbase + (uint32_t)((16 * h + 2 * e) * kRbPitch + n) * 4u);
    const float vb = lds_f32(vbase + (uint32_t)((16 * h + 2 * e + 1) * kRbPitch + n) * 4u);
    // hi part rounded once to the activation type, lo part the remainder
    const TA ah = Act<TA>::from(va), bh = Act<TA>::from(vb);
    hi[e] = Act<TA>::p2(Act<TA>::f1(ah), Act<TA>::f1(bh));
    lo[e] = Act<TA>::p2(va - Act<TA>::f1(ah), vb - Act<TA>::f1(bh));
  }
  TA* dst = rt + ((size_t)grp * kGroup + n) * kGroup + r0 + 16 * h;
  uint4* dh = reinterpret_cast<uint4*>(dst);
  uint4* dl = reinterpret_cast<uint4*>(dst + (size_t)K * kGroup);
  dh[0] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
  dh[1] = make_uint4(hi[4], hi[5], hi[6], hi[7]);
  dl[0] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  dl[1] = make_uint4(lo[4], lo[5], lo[6], lo[7]);
}

// ------------------------------------------------------------------ X R'
// Work: jobs (member m, group g, 128-row tile t), member-major then
// group-major; CTA c of P (one per SM) takes the contiguous range
// [c J / P, (c+1) J / P), so every CTA moves the same number of tiles and
// holds one (member, group) R' at a time (a range crosses such a boundary at
// most a few times; R' is reloaded there).  All members read the same x.
//
// Warp roles: warp 0 = TMA producer (R' parts, x tiles through a
// kRcStages-deep ring), warp 1 = TMEM allocator and single-thread MMA issuer,
// warps 2..5 = epilogue (warp w reads TMEM lane quadrant w % 4: rows
// 32 (w % 4) .. +31 of the tile).  The epilogue rounds its rows to fp16 into a
// staging tile in shared memory (two boxes, 128-byte swizzle) and one thread
// writes the tile to X_r with two TMA stores (clipped at row M), so every
// global write is a full line; two staging tiles alternate.
//   A = x tile [128 rows][128 channels] fp16: two {64 channels, 128 rows}
//       boxes with the 128-byte swizzle (canonical K-major SW128 layout).
//   B = Rhi, Rlo of the group [128 n][128 k]: two boxes each, same layout.
//   D = fp32 [128 lanes = rows][128 columns = output channels], two buffers
//       (256 TMEM columns) so the epilogue of one tile overlaps the MMAs of
//       the next.
// Per tile: 8 k-steps of 16 channels, each one MMA with Rhi and one with Rlo
// into the same accumulator (M = 128, N = 128, K = 16, kind::f16).
constexpr int kRcStages = 3;
constexpr int kRcEpiWarps = 4;
constexpr int kRcThreads = 32 * (2 + kRcEpiWarps);
// The quantising variant has four times the epilogue warps (four per TMEM
// lane quadrant, 32 columns each): its epilogue does more work per value.
template <bool QUANT>
__host__ __device__ constexpr int rc_epi_warps() { return QUANT ? 4 * kRcEpiWarps : kRcEpiWarps; }
constexpr int kRcQuantCols = 128 / (4 * kRcEpiWarps / 4);   // columns per quantising epilogue warp
template <bool QUANT>
__host__ __device__ constexpr int rc_threads() { return 32 * (2 + rc_epi_warps<QUANT>()); }
constexpr int kRcCols = 256;

struct RcLayout {
  static constexpr int BOX = 128 * 64 * 2;                 // 16 KB
  static constexpr int R_OFF = 0;                          // Rhi 0, Rhi 1, Rlo 0, Rlo 1
  static constexpr int X_OFF = 4 * BOX;
  static constexpr int X_STAGE = 2 * BOX;
  static constexpr int O_OFF = X_OFF + kRcStages * X_STAGE;  // staging tiles [2]
  static constexpr int O_STAGE = 2 * BOX;
  static constexpr int BAR_OFF = O_OFF + 2 * O_STAGE;
  // x_full[S], x_empty[S], acc_full[2], acc_empty[2], r_full, r_free, mma_done
  static constexpr int NBARS = 2 * kRcStages + 7;
  static constexpr int MISC_OFF = BAR_OFF + 8 * NBARS;     // TMEM address, abort flag
  static constexpr int SMEM = MISC_OFF + 16 + 1024;        // + slack for 1024-byte alignment
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

// instruction descriptor: fp32 accumulate, fp16 A and B, both K-major, M = 128, N = 128
constexpr uint32_t kRcIdesc = (1u << 4) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

// 32 fp32 accumulator columns (chunk cb of 4) of tile row r -> fp16 (round to
// nearest) in the staging tile: 64-channel box cb / 2, 16-byte chunks
// 4 (cb % 2) .. +3 of the row, XOR-swizzled by (r & 7) as the 128-byte TMA
// swizzle expects.
template <typename TA>
__device__ __forceinline__ void rc_stage32(uint32_t tile, int r, int cb, const uint32_t (&v)[32]) {
  const uint32_t rowp = tile + (uint32_t)(cb >> 1) * RcLayout::BOX + (uint32_t)r * 128u;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint4 o;
    uint32_t* oh = &o.x;
#pragma unroll
    for (int e = 0; e < 4; ++e)
      oh[e] = Act<TA>::p2(__uint_as_float(v[8 * c + 2 * e]), __uint_as_float(v[8 * c + 2 * e + 1]));
    const uint32_t chunk = (uint32_t)(4 * (cb & 1) + c);
    sts128u(rowp + ((chunk ^ (uint32_t)(r & 7)) << 4), o);
  }
}

// The weight quantiser's outputs (QUANT variant): x is W [N, K] (weight rows),
// the product is W_r = W D R, and each tile is quantised with the quantiser
// scales [K/G, N] (bounded to [1e-5, 1e5]) into four-bit codes -8..7 + 8 and
// packed into AWQ words; y is then qweight [K, N/8] int32 with box {4 words,
// kRcQuantCols rows} (one epilogue warp's share of a tile), no swizzle, and qzeros
// [K/G, N/8] is filled with 0x88888888.
struct RcQuant {
  const void* scales;
  int32_t* qzeros;
  int n;                  // weight rows N
  int gsz;                // quantisation group size
};

// 32 fp32 values (channels k0 .. k0+31 of tile row r) -> four-bit codes
// clamp(rint(v / s), -8, 7) + 8, with inv0 / inv1 the reciprocals of the
// bounded scales of the two 16-channel chunks; bytes at codes[channel][row]
// (channel rows `pitch` bytes apart).
// The bounds are integers, so clamping before rounding gives the same code;
// rint is one fp32 addition of 1.5 * 2^23 (round to nearest even at unit
// spacing, exact for |v| <= 8), whose low mantissa bits are then the signed
// code, offset by 8 in the integer domain.  A NaN quotient gives level 0
// (code 8), infinities the clamped ends, as the stage-by-stage quantiser does.
__device__ __forceinline__ void rc_codes32(uint32_t codes, int r, int k0, const uint32_t (&v)[32], float inv0,
                                           float inv1, uint32_t pitch) {
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    const float x = __uint_as_float(v[e]) * (e < 16 ? inv0 : inv1);
    const float t = fminf(fmaxf(x == x ? x : 0.0f, -8.0f), 7.0f);   // NaN -> level 0, as rint + clamp gives
    const uint32_t q = (__float_as_uint(t + 12582912.0f) + 8u) & 0xFu;
    asm volatile("st.shared.u8 [%0], %1;" ::"r"(codes + (uint32_t)(k0 + e) * pitch + (uint32_t)r), "r"(q)
                 : "memory");
  }
}

// Per member: r = its R' parts as [2K, 128] fp16, y = its X_r [M, K] fp16
// (stores), both box {64, 128} with the 128-byte swizzle.
struct alignas(64) RcTarget {
  CUtensorMap r;
  CUtensorMap y;
};
struct RcBatch {
  RcTarget t[kRcMaxMembers];
};

// grid P <= number of SMs, block kRcThreads.  tmX: x [M, K] fp16, box {64, 128},
// 128-byte swizzle.  jobs = members * groups * tiles.
template <typename TA, bool QUANT = false>
__global__ void __launch_bounds__(rc_threads<QUANT>(), 1) rotate_tc_kernel(
    const __grid_constant__ CUtensorMap tmX, const __grid_constant__ RcBatch batch, int members, int K,
    int groups, int tiles, long long jobs, const RcQuant qo) {
  using L = RcLayout;
  constexpr int EPI = rc_epi_warps<QUANT>();
  extern __shared__ unsigned char smem_raw[];
  unsigned char* const sbase = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t base = smem_u32(sbase);
  const uint32_t x_full0 = base + L::BAR_OFF;
  const uint32_t x_empty0 = x_full0 + 8 * kRcStages;
  const uint32_t acc_full0 = x_empty0 + 8 * kRcStages;
  const uint32_t acc_empty0 = acc_full0 + 16;
  const uint32_t r_full = acc_empty0 + 16;
  const uint32_t r_free = r_full + 8;
  const uint32_t mma_done = r_free + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + L::MISC_OFF);
  volatile int* abort = reinterpret_cast<volatile int*>(sbase + L::MISC_OFF + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long P = gridDim.x, c = blockIdx.x;
  const long long j0 = c * jobs / P, j1 = (c + 1) * jobs / P;
  const int nj = (int)(j1 - j0);

  if (tid == 0) {
    for (int s = 0; s < kRcStages; ++s) {
      mbar_init(x_full0 + 8 * s, 1);
      mbar_init(x_empty0 + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(acc_full0 + 8 * a, 1);
      mbar_init(acc_empty0 + 8 * a, EPI);
    }
    mbar_init(r_full, 1);
    mbar_init(r_free, 1);
    mbar_init(mma_done, 1);
    *abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmX);
    for (int m = 0; m < members; ++m) {
      tma_prefetch_desc(&batch.t[m].r);
      tma_prefetch_desc(&batch.t[m].y);
    }
  }
  if (warp == 1) {                         // the whole warp allocates the two accumulators
    tmem_alloc(smem_u32(tmem_slot), kRcCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // tensor memory is held: a dependent kernel may launch now without ever
  // taking columns this one still needs (not the quantiser: its outputs are
  // layer constants that the kernels after it read before they wait)
  if constexpr (!QUANT) pdl_launch_dependents();
  const uint32_t tmem0 = *tmem_slot;
  // R' comes from the build kernel, x from the kernel before it (the build
  // kernel completes only after that one has)
  pdl_wait_primary();

  int issued = 0, r_loads = 0;             // producer's count of x tiles and R' loads
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      long long cur_u = -1;
      for (int i = 0; i < nj; ++i) {
        const long long j = j0 + i;
        const long long u = j / tiles;                 // (member, group) unit
        const int m = (int)(u / groups), g = (int)(u % groups), t = (int)(j % tiles);
        if (u != cur_u) {
          // every MMA that reads the previous unit's R' has completed
          if (r_loads > 0 && !tc_wait(r_free, (uint32_t)((r_loads - 1) & 1), abort)) break;
          const CUtensorMap* tmR = &batch.t[m].r;
          mbar_arrive_expect_tx(r_full, 4 * L::BOX);
          tma_load_2d(base + L::R_OFF + 0 * L::BOX, tmR, r_full, 0, g * 128);
          tma_load_2d(base + L::R_OFF + 1 * L::BOX, tmR, r_full, 64, g * 128);
          tma_load_2d(base + L::R_OFF + 2 * L::BOX, tmR, r_full, 0, K + g * 128);
          tma_load_2d(base + L::R_OFF + 3 * L::BOX, tmR, r_full, 64, K + g * 128);
          ++r_loads;
          cur_u = u;
        }
        const int s = i % kRcStages;
        if (i >= kRcStages && !tc_wait(x_empty0 + 8 * s, (uint32_t)(((i / kRcStages) - 1) & 1), abort)) break;
        const uint32_t dst = base + L::X_OFF + s * L::X_STAGE;
        mbar_arrive_expect_tx(x_full0 + 8 * s, L::X_STAGE);
        tma_load_2d(dst, &tmX, x_full0 + 8 * s, g * 128, t * 128);
        tma_load_2d(dst + L::BOX, &tmX, x_full0 + 8 * s, g * 128 + 64, t * 128);
        ++issued;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      long long cur_u = -1;
      int gi = -1;
      for (int i = 0; i < nj; ++i) {
        const long long j = j0 + i;
        const long long u = j / tiles;                 // (member, group) unit
        if (u != cur_u) {
          ++gi;
          cur_u = u;
          if (!tc_wait(r_full, (uint32_t)(gi & 1), abort)) break;
        }
        const int s = i % kRcStages, a = i & 1;
        if (!tc_wait(x_full0 + 8 * s, (uint32_t)((i / kRcStages) & 1), abort)) break;
        if (i >= 2 && !tc_wait(acc_empty0 + 8 * a, (uint32_t)(((i >> 1) - 1) & 1), abort)) break;
        tc_fence_after();
        const uint32_t d = tmem0 + (uint32_t)(a * 128);
        const uint32_t xs = base + L::X_OFF + s * L::X_STAGE;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          // 128-byte swizzled rows, 8-row groups 1024 B apart; +32 B per 16 channels
          const uint32_t box = (uint32_t)(ks >> 2) * L::BOX, off = (uint32_t)(ks & 3) * 32;
          const uint64_t ad = umma_desc(xs + box + off, 16, 1024, 2);
          const uint64_t bh = umma_desc(base + L::R_OFF + box + off, 16, 1024, 2);
          const uint64_t bl = umma_desc(base + L::R_OFF + 2 * L::BOX + box + off, 16, 1024, 2);
          umma_f16(d, ad, bh, kRcIdesc | Act<TA>::kIdescAB, ks > 0 ? 1u : 0u);
          umma_f16(d, ad, bl, kRcIdesc | Act<TA>::kIdescAB, 1u);
        }
        umma_commit(x_empty0 + 8 * s);    // the x stage and ...
        umma_commit(acc_full0 + 8 * a);   // ... the accumulator, once these MMAs finish
        if (i + 1 == nj || (j + 1) / tiles != u) umma_commit(r_free);   // last tile of the unit
      }
      // every MMA issued here has completed before tensor memory is released
      umma_commit(mma_done);
      mbar_wait_bounded(mma_done, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                // TMEM lane quadrant of this warp
    const int r = 32 * q + lane;           // tile row of this thread
    const bool leader = warp == 2 && lane == 0;   // issues the TMA stores
    // quantising: warps 2..5 take columns 0..31, 6..9 columns 32..63, and so on
    const int c0 = QUANT ? kRcQuantCols * ((warp - 2) >> 2) : 0;
    // All epilogue warps take part in every named barrier of every tile, even
    // after a wait has given up (the work is skipped, the barriers are not),
    // so no warp can be left at a barrier; a given-up wait returns at once.
    for (int i = 0; i < nj; ++i) {
      const long long j = j0 + i;
      const long long u = j / tiles;
      const int m = (int)(u / groups), g = (int)(u % groups), t = (int)(j % tiles);
      const int a = i & 1;
      // quantiser scales of this thread's row and 16-channel chunks, requested
      // before the wait for the accumulator (a chunk lies in one group of G >= 16)
      float inv[kRcQuantCols / 16];        // this warp's 16-channel chunks
      if constexpr (QUANT) {
        const int n = t * 128 + r;
#pragma unroll
        for (int kk = 0; kk < kRcQuantCols / 16; ++kk) {
          const int qg = (g * kGroup + c0 + 16 * kk) / qo.gsz;
          float sc = n < qo.n ? Act<TA>::f1(static_cast<const TA*>(qo.scales)[(size_t)qg * qo.n + n]) : 1.0f;
          sc = fminf(fmaxf(sc, 1e-5f), 1e5f);
          inv[kk] = 1.0f / sc;
        }
      }
      // warp-uniform (tcgen05.ld is a warp-wide instruction)
      const bool ok = __all_sync(0xffffffffu, tc_wait(acc_full0 + 8 * a, (uint32_t)((i >> 1) & 1), abort));
      uint32_t v0[32], v1[32], v2[32], v3[32];
      if (ok) {
        tc_fence_after();
        const uint32_t ta = tmem0 + ((uint32_t)(32 * q) << 16) + (uint32_t)(a * 128 + c0);
        tmem_ld32(ta, v0);
        if constexpr (!QUANT) {
          tmem_ld32(ta + 32, v1);
          tmem_ld32(ta + 64, v2);
          tmem_ld32(ta + 96, v3);
        }
        tmem_ld_wait_tie(v0);
        if constexpr (!QUANT) {
          tmem_tie(v1);
          tmem_tie(v2);
          tmem_tie(v3);
        }
      }
      // the accumulator may be overwritten once every warp has read it
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && ok) mbar_arrive(acc_empty0 + 8 * a);
      const uint32_t tile = base + L::O_OFF + (uint32_t)(i & 1) * L::O_STAGE;
      if constexpr (QUANT) {
        // Each warp packs its own 32 rows x 32 channels: codes as bytes
        // [32 channels][32 rows], then 4 AWQ words per channel [32][4]
        // (16-byte rows), written by the warp with one TMA store of a
        // {4 words, 32 rows} box; no CTA-wide barrier.
        const int ew = warp - 2;                                  // 0 .. EPI - 1
        constexpr uint32_t kCodes = 32u * kRcQuantCols, kWarpArea = kCodes + 16u * kRcQuantCols;
        const uint32_t codes = base + L::O_OFF + (uint32_t)(i & 1) * L::O_STAGE + (uint32_t)ew * kWarpArea;
        const uint32_t words = codes + kCodes;
        if (lane == 0) bulk_wait_group_read<1>();                 // this warp's store of tile i - 2 has read them
        __syncwarp();
        if (ok) rc_codes32(codes, lane, 0, v0, inv[0], inv[1], 32);
        __syncwarp();
        if (ok) {
          // word (k, w): rows 8w .. 8w+7 of channel k, row 8w + i at nibble
          // (i >> 1) + 4 (i & 1): the even rows' codes fill the low half-word,
          // the odd rows' the high one
#pragma unroll
          for (int it = 0; it < kRcQuantCols * 4 / 32; ++it) {
            const int idx = lane + 32 * it, k = idx >> 2, w = idx & 3;
            uint32_t lo, hi;
            asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(lo), "=r"(hi)
                         : "r"(codes + (uint32_t)k * 32u + 8u * (uint32_t)w));
            const uint32_t ev = prmt(lo, hi, 0x6420), od = prmt(lo, hi, 0x7531);   // bytes of rows 0,2,4,6 / 1,3,5,7
            const uint32_t e2 = ev | (ev >> 4), o2 = od | (od >> 4);              // two nibbles per even byte
            sts_f32(words + (uint32_t)k * 16u + 4u * (uint32_t)w, __uint_as_float(prmt(e2, o2, 0x6420)));
          }
          if (ew == 0) {
            // the tile's zero words: rows of its quantisation groups, its 16 word columns
            const int zrows = kGroup / qo.gsz, zw = qo.n / 8;
            for (int idx = lane; idx < zrows * 16; idx += 32) {
              const int wc = t * 16 + (idx & 15);
              if (wc < zw) qo.qzeros[(size_t)((g * kGroup) / qo.gsz + (idx >> 4)) * zw + wc] = (int32_t)0x88888888u;
            }
          }
        }
        fence_proxy_async_smem();          // the words are read by the TMA (async proxy)
        __syncwarp();
        if (lane == 0 && ok && !*abort) {
          tma_store_2d(&batch.t[m].y, words, t * 16 + 4 * q, g * 128 + c0);
          bulk_commit_group();
        }
      } else {
        // staging tile i & 1 is free once the stores of tile i - 2 have read it
        if (leader) bulk_wait_group_read<1>();
        named_bar_sync(1, 32 * EPI);
        if (ok) {
          rc_stage32<TA>(tile, r, 0, v0);
          rc_stage32<TA>(tile, r, 1, v1);
          rc_stage32<TA>(tile, r, 2, v2);
          rc_stage32<TA>(tile, r, 3, v3);
        }
        fence_proxy_async_smem();          // the tile is read by the TMA (async proxy)
        named_bar_sync(2, 32 * EPI);
        if (leader && !*abort) {
          tma_store_2d(&batch.t[m].y, tile, g * 128, t * 128);
          tma_store_2d(&batch.t[m].y, tile + L::BOX, g * 128 + 64, t * 128);
          bulk_commit_group();
        }
      }
    }
    // the stores have written X_r (the words) before the kernel completes
    if (QUANT ? lane == 0 : leader) bulk_wait_group_all();
  }

  if (warp == 0 && lane == 0 && *abort) {
    // a wait gave up: let this thread's copies still in flight land (bounded)
    // before the shared memory is released
    for (int i = issued > kRcStages ? issued - kRcStages : 0; i < issued; ++i)
      if (!mbar_wait_bounded(x_full0 + 8 * (i % kRcStages), (uint32_t)((i / kRcStages) & 1))) break;
    if (r_loads > 0) mbar_wait_bounded(r_full, (uint32_t)((r_loads - 1) & 1));
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem0, kRcCols);
  }
}

}  // namespace paro

// Decode W4 GEMV (M <= 16 token rows), warp-specialised, on warp-level tensor-core
// MMA (m16n8k16, fp16 in, fp32 accumulate), reading AWQ-packed weights directly.
//
// What it computes (GPTQModel wiki page "ParoQuant", "Activation and weight
// transforms" and "Triton plans and tuning"):
//   Y[m, n] = sum_g s[g, n] * sum_{k in g} X_r[m, k] * (q[k, n] - z[g, n]) + b[n]
//
// Work layout.  A CTA owns 256 output columns (32 packed words = one 128-byte
// line of every qweight row) and a contiguous range of 128-row groups of K.
// Warp 0 is the producer: one lane streams each group through a ring of STAGES
// shared-memory stages with TMA (qweight 128 rows x 128 B, 128-byte swizzle;
// the group's 256 scales and 32 zero words; the matching 128 columns of X_r),
// signalling "full" mbarriers; consumers release a stage on its "empty"
// mbarrier.  Weights, scales and zeros do not depend on the previous kernel, so
// the producer streams them before griddepcontrol.wait (programmatic dependent
// launch) and only the X_r loads wait for the rotation kernel.
// Consumer warps are 4 column slices (64 columns each) x KP k-parts; k-part p
// takes the CTA's groups p, p+KP, ... so every warp works on whole groups.
//
// MMA mapping (Y^T = W^T X_r^T: weights are the 16-row A operand, tokens the
// 8-wide B operand).  Thread (g = lane/4, t = lane%4) of column slice c owns
// word column wcol = 8c + g, i.e. columns 8*wcol .. 8*wcol+7; m-tile j's rows g
// and g+8 are columns 2j and 2j+1 of that word, which the AWQ nibble order puts
// at nibbles j and j+4.  A byte permute of the words of rows k and k+1 puts both
// k's of one column into the two halves of a register, and
//   (v & 0x000F000F) | 0x64006400  ->  fp16 pair 1024 + q      (nibbles 0, 2)
//   (v & 0x00F000F0) | 0x64006400  ->  fp16 pair 1024 + 16 q   (nibbles 1, 3)
// are exact.  The zero point is not subtracted per weight: one more MMA with an
// all-ones A operand gives the group row sums r[m] = sum_{k in g} X_r[m, k], and
// at the end of the group
//   sum_k X_r (q - z) = C - (1024 + z) r       (16 (q - z) and 1024 + 16 z for odd j)
// in fp32, then times the group scale (s / 16 for odd j, an exact power of two).
//
// Split-K: the S CTAs that share an output tile form a thread-block cluster
// along K.  CTA r owns columns [r*NTILE/S, (r+1)*NTILE/S): every CTA pushes its
// fp32 partial of each slice into the owner's inbox (a dedicated shared-memory
// area, one slot per sender) with distributed-shared-memory stores; after one
// cluster barrier each owner sums its inbox in sender order, adds the bias and
// writes fp16 Y.  No global scratch, no atomics, deterministic.
#pragma once

#include "common.cuh"

namespace paro {

constexpr int kGvMaxStages = 8;
constexpr uint32_t kGvMagic = 0x64006400u;  // fp16 pair (1024, 1024)
constexpr uint32_t kGvOnes = 0x3C003C00u;   // fp16 pair (1, 1)

// NTILE output columns per CTA (64 per column-slice warp), KP k-parts, STAGES
// groups in flight.
template <int NT, int KP, int NTILE, int STAGES>
struct GemvLayout {
  static constexpr int CSL = NTILE / 64;                  // column-slice warps per k-part
  static constexpr int WORDS = NTILE / 8;                 // packed words per row segment
  static constexpr int THREADS = 32 * (1 + CSL * KP);
  static constexpr int MP = 8 * NT;                       // token rows per CTA
  static constexpr int W_BYTES = 128 * WORDS * 4;         // one group of qweight
  static constexpr int X_BYTES = 2 * MP * 128;            // two 64-column boxes
  static constexpr int S_BYTES = NTILE * 2;
  static constexpr int Z_BYTES = WORDS * 4;
  static constexpr int X_OFF = W_BYTES;
  static constexpr int S_OFF = X_OFF + ((X_BYTES + 1023) / 1024) * 1024;
  static constexpr int Z_OFF = S_OFF + S_BYTES;
  static constexpr int STAGE = ((Z_OFF + Z_BYTES + 1023) / 1024) * 1024;
  static constexpr int TX_BYTES = W_BYTES + S_BYTES + Z_BYTES + X_BYTES;
  static constexpr int RED_BYTES = KP * MP * NTILE * 4;     // k-part partial tiles
  static constexpr int INBOX_OFF = STAGES * STAGE;          // split-K inbox [S][MP][NTILE/S]
  static constexpr int INBOX_BYTES = MP * NTILE * 4;
  static constexpr int BAR_OFF = INBOX_OFF + INBOX_BYTES;   // full[], empty[] mbarriers
  static constexpr int SMEM = BAR_OFF + 16 * STAGES + 1024;
  static_assert(RED_BYTES <= STAGES * STAGE, "reduction tiles must fit in stage memory");
  static_assert(STAGES <= kGvMaxStages, "too many stages");
  // 128-byte swizzle needs 128-byte rows; 64-byte rows use the 64-byte swizzle
  static constexpr int ROW_BYTES = WORDS * 4;
};

__device__ __forceinline__ void gv_unpack4(uint32_t m, uint32_t (&e)[4]) {
  const uint32_t m8 = m >> 8;
  e[0] = and_or(m, 0x000F000Fu, kGvMagic);
  e[1] = and_or(m, 0x00F000F0u, kGvMagic);
  e[2] = and_or(m8, 0x000F000Fu, kGvMagic);
  e[3] = and_or(m8, 0x00F000F0u, kGvMagic);
}

template <int NT, int KP, int NTILE, int STAGES>
__global__ void __launch_bounds__(32 * (1 + (NTILE / 64) * KP)) w4_gemv_kernel(
    const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
    const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmZ,
    const __half* __restrict__ bias, __half* __restrict__ Y, int M, int N, int K) {
  using L = GemvLayout<NT, KP, NTILE, STAGES>;
  constexpr int kGvStages = STAGES;
  constexpr int kGvTile = NTILE;
  // The next kernel in the stream may launch now; it waits for our completion
  // before it touches anything we read or write.
  pdl_launch_dependents();

  extern __shared__ unsigned char smem_raw[];
  // 1024-byte aligned base, derived on the shared array so every access stays LDS/STS
  unsigned char* const sbase = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t base = smem_u32(sbase);
  const uint32_t full0 = base + L::BAR_OFF;
  const uint32_t empty0 = full0 + 8 * kGvStages;

  const int ntile = blockIdx.x, split = blockIdx.y;
  const int n0 = ntile * kGvTile;
  const int groups = K / 128;
  const int g_begin = (int)(((long long)split * groups) / gridDim.y);
  const int g_end = (int)(((long long)(split + 1) * groups) / gridDim.y);
  const int ng = g_end - g_begin;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < kGvStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, L::CSL);  // the column-slice warps of one k-part
    }
    fence_barrier_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmS);
    tma_prefetch_desc(&tmZ);
  }
  __syncthreads();

  float acc[4][NT][4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[j][nt][e] = 0.f;
  const int cw = warp - 1;                 // consumer index (warp 0 produces)
  const int cslice = cw % L::CSL, kpart = cw / L::CSL;
  const int g = lane >> 2, t = lane & 3;
  const int wcol = 8 * cslice + g;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      const int pre = min(kGvStages, ng);
      for (int i = 0; i < pre; ++i) {
        const uint32_t st = base + i * L::STAGE, bar = full0 + 8 * i;
        const int kg = g_begin + i;
        mbar_arrive_expect_tx(bar, L::TX_BYTES);
        tma_load_2d_hint(st, &tmW, bar, n0 / 8, kg * 128, pol);
        tma_load_2d(st + L::S_OFF, &tmS, bar, n0, kg);
        tma_load_2d(st + L::Z_OFF, &tmZ, bar, n0 / 8, kg);
      }
      pdl_wait_primary();                  // X_r comes from the rotation kernel
      for (int i = 0; i < pre; ++i) {
        const uint32_t st = base + i * L::STAGE, bar = full0 + 8 * i;
        const int kg = g_begin + i;
        tma_load_2d(st + L::X_OFF, &tmX, bar, kg * 128, 0);
        tma_load_2d(st + L::X_OFF + L::MP * 128, &tmX, bar, kg * 128 + 64, 0);
      }
      for (int i = pre; i < ng; ++i) {
        const int s = i % kGvStages;
        if (!mbar_wait_bounded(empty0 + 8 * s, ((i / kGvStages) - 1) & 1)) break;
        const uint32_t st = base + s * L::STAGE, bar = full0 + 8 * s;
        const int kg = g_begin + i;
        mbar_arrive_expect_tx(bar, L::TX_BYTES);
        tma_load_2d_hint(st, &tmW, bar, n0 / 8, kg * 128, pol);
        tma_load_2d(st + L::S_OFF, &tmS, bar, n0, kg);
        tma_load_2d(st + L::Z_OFF, &tmZ, bar, n0 / 8, kg);
        tma_load_2d(st + L::X_OFF, &tmX, bar, kg * 128, 0);
        tma_load_2d(st + L::X_OFF + L::MP * 128, &tmX, bar, kg * 128 + 64, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    // Swizzled offsets that do not change from group to group.  qweight rows
    // 16 ks + 2t + {0, 1, 8, 9} have (row & 7) = 2t + {0, 1, 0, 1}.
    const int wchunk = wcol >> 2, wword = (wcol & 3) * 4;
    constexpr int RB = L::ROW_BYTES;
    // 128-byte rows: chunk ^ (row & 7); 64-byte rows (64-byte swizzle): chunk ^ ((row >> 1) & 3)
    auto swz = [&](int row) -> int { return RB == 128 ? (row & 7) : ((row >> 1) & 3); };
    const uint32_t wo0 = (uint32_t)((2 * t) * RB + ((wchunk ^ swz(2 * t)) << 4) + wword);
    const uint32_t wo1 = (uint32_t)((2 * t + 1) * RB + ((wchunk ^ swz(2 * t + 1)) << 4) + wword);
    // X_r tile: token rows of 128 B per 64-column box; columns 16 ks + 2t (+8)
    // sit in 16-byte chunk 2 (ks & 3) (+1), swizzled with (token & 7).
    uint32_t xo[4][NT][2];
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int tok = 8 * nt + g;
        const int c0 = 2 * q;
        xo[q][nt][0] = (uint32_t)(L::X_OFF + tok * 128 + (((c0) ^ (tok & 7)) << 4) + 4 * t);
        xo[q][nt][1] = (uint32_t)(L::X_OFF + tok * 128 + (((c0 + 1) ^ (tok & 7)) << 4) + 4 * t);
      }
    const uint32_t ones[4] = {kGvOnes, kGvOnes, kGvOnes, kGvOnes};

    for (int i = kpart; i < ng; i += KP) {
      const int s = i % kGvStages;
      const unsigned char* stp = sbase + s * L::STAGE;
      const bool ready = mbar_wait_bounded(full0 + 8 * s, (i / kGvStages) & 1);
      if (ready) {
        // group constants for this thread's 8 columns
        const uint32_t zw = *reinterpret_cast<const uint32_t*>(stp + L::Z_OFF + wcol * 4);
        const uint4 s8 = *reinterpret_cast<const uint4*>(stp + L::S_OFF + wcol * 16);
        float cg[4][NT][4];
        float rs[NT][4];
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const unsigned char* wrow = stp + ks * 16 * RB;
          const uint32_t w0 = *reinterpret_cast<const uint32_t*>(wrow + wo0);
          const uint32_t w1 = *reinterpret_cast<const uint32_t*>(wrow + wo1);
          const uint32_t w8 = *reinterpret_cast<const uint32_t*>(wrow + 8 * RB + wo0);
          const uint32_t w9 = *reinterpret_cast<const uint32_t*>(wrow + 8 * RB + wo1);
          uint32_t b0[NT], b1[NT];
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const unsigned char* xb = stp + (ks >> 2) * (L::MP * 128);
            b0[nt] = *reinterpret_cast<const uint32_t*>(xb + xo[ks & 3][nt][0]);
            b1[nt] = *reinterpret_cast<const uint32_t*>(xb + xo[ks & 3][nt][1]);
          }
          uint32_t elo01[4], ehi01[4], elo89[4], ehi89[4];
          gv_unpack4(prmt(w0, w1, 0x5410), elo01);
          gv_unpack4(prmt(w0, w1, 0x7632), ehi01);
          gv_unpack4(prmt(w8, w9, 0x5410), elo89);
          gv_unpack4(prmt(w8, w9, 0x7632), ehi89);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t a[4] = {elo01[j], ehi01[j], elo89[j], ehi89[j]};
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              if (ks == 0) mma_16816_zc(cg[j][nt], a, b0[nt], b1[nt]);
              else mma_16816(cg[j][nt], a, b0[nt], b1[nt]);
            }
          }
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            if (ks == 0) mma_16816_zc(rs[nt], ones, b0[nt], b1[nt]);
            else mma_16816(rs[nt], ones, b0[nt], b1[nt]);
          }
        }
        // this warp is done reading the stage
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * s);
        // zero-point correction and group scale, in fp32
        const uint32_t sw[4] = {s8.x, s8.y, s8.z, s8.w};   // (s[2j], s[2j+1])
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int sh = (j & 1) ? 4 : 0;
          const float zl = 1024.f + (float)(((zw >> (4 * j)) & 0xFu) << sh);
          const float zh = 1024.f + (float)(((zw >> (16 + 4 * j)) & 0xFu) << sh);
          float2 sf = __half22float2(*reinterpret_cast<const __half2*>(&sw[j]));
          if (j & 1) sf.x *= 0.0625f, sf.y *= 0.0625f;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const float r0 = rs[nt][0], r1 = rs[nt][1];   // row sums of tokens 2t, 2t+1
            acc[j][nt][0] = fmaf(sf.x, fmaf(-zl, r0, cg[j][nt][0]), acc[j][nt][0]);
            acc[j][nt][1] = fmaf(sf.x, fmaf(-zl, r1, cg[j][nt][1]), acc[j][nt][1]);
            acc[j][nt][2] = fmaf(sf.y, fmaf(-zh, r0, cg[j][nt][2]), acc[j][nt][2]);
            acc[j][nt][3] = fmaf(sf.y, fmaf(-zh, r1, cg[j][nt][3]), acc[j][nt][3]);
          }
        }
      } else {
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * s);   // keep the producer moving
      }
    }
  }

  // Everything before us in the stream is complete before anyone writes Y.
  pdl_wait_primary();
  __syncthreads();

  // ---------------- reduction over k-parts (shared memory, fixed order)
  float* red = reinterpret_cast<float*>(sbase);
  if (warp != 0) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int tt = 0; tt < 2; ++tt) {
        const int tl = 8 * nt + 2 * t + tt;
        float* p = red + ((size_t)kpart * L::MP + tl) * kGvTile + 8 * wcol;
        *reinterpret_cast<float4*>(p) =
            make_float4(acc[0][nt][tt], acc[0][nt][2 + tt], acc[1][nt][tt], acc[1][nt][2 + tt]);
        *reinterpret_cast<float4*>(p + 4) =
            make_float4(acc[2][nt][tt], acc[2][nt][2 + tt], acc[3][nt][tt], acc[3][nt][2 + tt]);
      }
  }
  __syncthreads();
  const int mrows = min(L::MP, M);
  const int S = gridDim.y;
  const int cols = kGvTile / S;                    // columns owned by each CTA of the cluster
  const uint32_t rank = S > 1 ? cluster_ctarank() : 0u;
  const uint32_t inbox = base + L::INBOX_OFF;
  // fold the k-parts (fixed order); write Y directly or push to the slice owner
  for (int idx = tid; idx < mrows * kGvTile / 4; idx += L::THREADS) {
    float4 v = reinterpret_cast<const float4*>(red)[idx];
#pragma unroll
    for (int kp = 1; kp < KP; ++kp) {
      const float4 u = reinterpret_cast<const float4*>(red + (size_t)kp * L::MP * kGvTile)[idx];
      v.x += u.x; v.y += u.y; v.z += u.z; v.w += u.w;
    }
    const int tl = idx / (kGvTile / 4);
    const int col = 4 * (idx % (kGvTile / 4));
    if (S > 1) {
      const int owner = col / cols;
      const uint32_t off = inbox + (uint32_t)(((int)rank * L::MP + tl) * cols + (col - owner * cols)) * 4u;
      st_cluster_f4(mapa_shared(off, (uint32_t)owner), v);
      continue;
    }
    const int n = n0 + col;
    if (n >= N) continue;
    if (bias != nullptr) {
      v.x += __half2float(bias[n]); v.y += __half2float(bias[n + 1]);
      v.z += __half2float(bias[n + 2]); v.w += __half2float(bias[n + 3]);
    }
    const __half2 h0 = __floats2half2_rn(v.x, v.y), h1 = __floats2half2_rn(v.z, v.w);
    uint2 out;
    out.x = *reinterpret_cast<const uint32_t*>(&h0);
    out.y = *reinterpret_cast<const uint32_t*>(&h1);
    *reinterpret_cast<uint2*>(Y + (size_t)tl * N + n) = out;
  }
  if (S == 1) return;

  // every partial pushed into this CTA's inbox is complete and visible after this
  cluster_sync();
  const float* box = reinterpret_cast<const float*>(sbase + L::INBOX_OFF);
  for (int idx = tid; idx < mrows * (cols / 4); idx += L::THREADS) {
    const int tl = idx / (cols / 4);
    const int c = 4 * (idx % (cols / 4));
    const int n = n0 + (int)rank * cols + c;
    if (n >= N) continue;
    float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int q = 0; q < S; ++q) {
      const float4 v = *reinterpret_cast<const float4*>(box + ((size_t)q * L::MP + tl) * cols + c);
      sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
    }
    if (bias != nullptr) {
      sum.x += __half2float(bias[n]); sum.y += __half2float(bias[n + 1]);
      sum.z += __half2float(bias[n + 2]); sum.w += __half2float(bias[n + 3]);
    }
    const __half2 h0 = __floats2half2_rn(sum.x, sum.y), h1 = __floats2half2_rn(sum.z, sum.w);
    uint2 out;
    out.x = *reinterpret_cast<const uint32_t*>(&h0);
    out.y = *reinterpret_cast<const uint32_t*>(&h1);
    *reinterpret_cast<uint2*>(Y + (size_t)tl * N + n) = out;
  }
}

}  // namespace paro

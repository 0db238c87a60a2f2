// W4 GEMV / small-tile GEMM on warp-level tensor-core MMA (m16n8k16, fp16 in,
// fp32 accumulate), reading AWQ-packed weights directly.
//
// What it computes (GPTQModel wiki page "ParoQuant", "Activation and weight
// transforms" and "Triton plans and tuning"):
//   Y[m, n] = sum_k X_r[m, k] * (q[k, n] - z[k/128, n]) * s[k/128, n] + b[n]
//
// Layout of the work.  A CTA owns 256 output columns (32 packed words = one
// 128-byte line of every qweight row) and a contiguous range of 128-row
// groups.  Each pipeline stage is one group: TMA brings 128 x 128 B of
// qweight (128-byte swizzle), the group's 256 scales and 32 zero words, and
// the matching 128 columns of X_r for the CTA's token rows.  Warps are laid out
// 4 (column slices of 64) x KSPLIT (interleaved k-steps of each group).
//
// The MMA runs transposed, Y^T = W^T X_r^T: the weights are the 16-row "A"
// operand and the tokens the 8-wide "B" operand, so decode (M <= 16) wastes at
// most half of an 8-wide token tile instead of 15/16 of a 16-row tile.  The
// A-row <-> column mapping is chosen so that one packed word feeds one thread:
// thread (g = lane/4, t = lane%4) of column slice c owns word column
// wcol = 8c + g, i.e. columns 8*wcol .. 8*wcol+7, and m-tile j's rows g and g+8
// are columns 2j and 2j+1 of that word.  With the AWQ nibble order those two
// columns sit at nibbles j and j+4; a byte permute of the words of rows k and
// k+1 puts both k's of one column into the two halves of a register, and
//   (v & 0x000F000F) | 0x64006400  ->  fp16 pair 1024 + q        (nibble 0)
//   (v & 0x00F000F0) | 0x64006400  ->  fp16 pair 1024 + 16 q     (nibble 1)
// (nibbles 2, 3 the same after one 8-bit shift) are exact.  Subtracting the
// fp16 pair (1024 + z) or (1024 + 16 z) leaves q - z or 16 (q - z) exactly; the
// factor 16 is folded into the group scale.  The group scale is applied either
// to the fp32 group partial sums (decode: exact) or to the fp16 weights before
// the MMA (large token tiles: one fp16 rounding of (q - z) * s).
//
// Split-K (decode): the S CTAs that share an output tile form one thread-block
// cluster along K.  Each leaves its fp32 partial tile in its own shared memory;
// after a cluster barrier, CTA r sums columns [r*256/S, (r+1)*256/S) over the
// S partials through distributed shared memory, in split order, adds the bias
// and writes fp16 Y.  No global scratch, no atomics, deterministic.
#pragma once

#include "common.cuh"

namespace paro {

constexpr int kNTile = 256;             // output columns per CTA
constexpr int kNWords = kNTile / 8;     // packed words per qweight row segment
constexpr int kMmaStages = 5;     // groups in flight per CTA (two CTAs per SM for decode)
constexpr uint32_t kMagic = 0x64006400u;   // fp16 pair (1024, 1024)

template <int NT, int KSPLIT>
struct MmaLayout {
  static constexpr int THREADS = 128 * KSPLIT;
  static constexpr int MP = 8 * NT;                      // token rows per CTA tile
  static constexpr int W_BYTES = 128 * kNWords * 4;      // 16 KB
  static constexpr int X_BYTES = 2 * MP * 128;           // two 64-column boxes
  static constexpr int S_BYTES = kNTile * 2;
  static constexpr int Z_BYTES = kNWords * 4;
  static constexpr int X_OFF = W_BYTES;
  static constexpr int S_OFF = X_OFF + ((X_BYTES + 1023) / 1024) * 1024;
  static constexpr int Z_OFF = S_OFF + S_BYTES;
  static constexpr int STAGE = ((Z_OFF + Z_BYTES + 1023) / 1024) * 1024;
  static constexpr int TX_BYTES = W_BYTES + X_BYTES + S_BYTES + Z_BYTES;
  // partial tiles for the k-split / cluster reductions reuse stage memory
  static constexpr int RED_BYTES = KSPLIT * MP * kNTile * 4;
  static constexpr int SMEM = kMmaStages * STAGE + 1024 + 128;
  static_assert(RED_BYTES <= kMmaStages * STAGE, "reduction tile must fit in stage memory");
};

// The four nibble pairs of a merged word: e[0] = 1024+q (nib 0), e[1] = 1024+16q
// (nib 1), e[2] = 1024+q (nib 2), e[3] = 1024+16q (nib 3) per 16-bit half.
__device__ __forceinline__ void unpack4(uint32_t m, uint32_t (&e)[4]) {
  const uint32_t m8 = m >> 8;
  e[0] = and_or(m, 0x000F000Fu, kMagic);
  e[1] = and_or(m, 0x00F000F0u, kMagic);
  e[2] = and_or(m8, 0x000F000Fu, kMagic);
  e[3] = and_or(m8, 0x00F000F0u, kMagic);
}

template <int NT, int KSPLIT, bool SCALE_IN_A>
__global__ void __launch_bounds__(128 * KSPLIT) w4_mma_kernel(
    const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
    const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmZ,
    const __half* __restrict__ bias, __half* __restrict__ Y, int M, int N, int K) {
  using L = MmaLayout<NT, KSPLIT>;
  constexpr int KSTEPS = 8 / KSPLIT;       // 16-row k-steps per warp per group
  extern __shared__ unsigned char smem_raw[];
  // 1024-byte aligned base, derived by pointer arithmetic on the shared array so
  // the compiler keeps every access in the shared window (LDS, not generic LD)
  unsigned char* const sbase = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t base = smem_u32(sbase);
  const uint32_t bar0 = base + kMmaStages * L::STAGE;   // kMmaStages x 8 bytes

  const int ntile = blockIdx.x, split = blockIdx.y, mtile = blockIdx.z;
  const int n0 = ntile * kNTile;
  const int tok0 = mtile * L::MP;
  const int groups = K / 128;
  // balanced split of the groups over gridDim.y CTAs (each gets >= 1 when S <= groups)
  const int g_begin = (int)(((long long)split * groups) / gridDim.y);
  const int g_end = (int)(((long long)(split + 1) * groups) / gridDim.y);
  const int ng = g_end - g_begin;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int cslice = warp & 3, kpart = warp >> 2;
  const int wcol = 8 * cslice + g;

  if (tid == 0) {
    for (int s = 0; s < kMmaStages; ++s) mbar_init(bar0 + 8 * s, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmS);
    tma_prefetch_desc(&tmZ);
  }
  __syncthreads();

  const uint64_t pol_stream = policy_evict_first();
  const int npro = min(kMmaStages, ng);
  // Weights, scales and zeros do not depend on the kernel before us: start
  // streaming them before waiting for it.
  if (tid == 0) {
    for (int i = 0; i < npro; ++i) {
      const uint32_t st = base + i * L::STAGE, bar = bar0 + 8 * i;
      const int kg = g_begin + i;
      mbar_arrive_expect_tx(bar, L::TX_BYTES);
      tma_load_2d_hint(st, &tmW, bar, n0 / 8, kg * 128, pol_stream);
      tma_load_2d(st + L::S_OFF, &tmS, bar, n0, kg);
      tma_load_2d(st + L::Z_OFF, &tmZ, bar, n0 / 8, kg);
    }
  }
  pdl_wait_primary();
  if (tid == 0) {
    for (int i = 0; i < npro; ++i) {
      const uint32_t st = base + i * L::STAGE, bar = bar0 + 8 * i;
      const int kg = g_begin + i;
      tma_load_2d(st + L::X_OFF, &tmX, bar, kg * 128, tok0);
      tma_load_2d(st + L::X_OFF + L::MP * 128, &tmX, bar, kg * 128 + 64, tok0);
    }
  }

  // Per-thread smem offsets that do not change from k-step to k-step: the
  // 128-byte swizzle XORs the 16-byte chunk with (row & 7), and rows
  // 16*ks + 2t + {0, 1, 8, 9} have (row & 7) = 2t + {0, 1, 0, 1}.
  const int wchunk = wcol >> 2, wword = (wcol & 3) * 4;
  const uint32_t wo0 = (uint32_t)((2 * t) * 128 + ((wchunk ^ (2 * t)) << 4) + wword);
  const uint32_t wo1 = (uint32_t)((2 * t + 1) * 128 + ((wchunk ^ (2 * t + 1)) << 4) + wword);

  float acc[4][NT][4];
  float cg[4][NT][4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[j][nt][e] = 0.f, cg[j][nt][e] = 0.f;

  int issued = npro, consumed = 0;
  for (int i = 0; i < ng; ++i) {
    const int s = i % kMmaStages;
    const unsigned char* stp = sbase + s * L::STAGE;
    const bool ready = mbar_wait_bounded(bar0 + 8 * s, (i / kMmaStages) & 1);
    if (ready) {
      // group constants for this thread's 8 columns
      const uint32_t zw = *reinterpret_cast<const uint32_t*>(stp + L::Z_OFF + wcol * 4);
      const uint4 s8 = *reinterpret_cast<const uint4*>(stp + L::S_OFF + wcol * 16);
      const uint32_t sw[4] = {s8.x, s8.y, s8.z, s8.w};   // (s[2j], s[2j+1]) pairs
      uint32_t zz_lo[4], zz_hi[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t sh = (j & 1) ? 4u : 0u;          // odd m-tiles carry 16 (q - z)
        const uint32_t zl = ((zw >> (4 * j)) & 0xFu) << sh;
        const uint32_t zh = ((zw >> (16 + 4 * j)) & 0xFu) << sh;
        zz_lo[j] = (zl | (zl << 16)) | kMagic;
        zz_hi[j] = (zh | (zh << 16)) | kMagic;
      }
      uint32_t ss_lo[4], ss_hi[4];
      if (SCALE_IN_A) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          // odd m-tiles: s / 16 (exact power-of-two scaling of a normal fp16)
          const uint32_t sj = (j & 1) ? hmul2_u32(sw[j], 0x2C002C00u) : sw[j];
          ss_lo[j] = prmt(sj, sj, 0x1010);   // (s[2j], s[2j])
          ss_hi[j] = prmt(sj, sj, 0x3232);   // (s[2j+1], s[2j+1])
        }
      }

#pragma unroll
      for (int q = 0; q < KSTEPS; ++q) {
        const int ks = q * KSPLIT + kpart;           // interleaved k-steps
        const unsigned char* wrow = stp + ks * 2048;
        const uint32_t w0 = *reinterpret_cast<const uint32_t*>(wrow + wo0);
        const uint32_t w1 = *reinterpret_cast<const uint32_t*>(wrow + wo1);
        const uint32_t w8 = *reinterpret_cast<const uint32_t*>(wrow + 1024 + wo0);
        const uint32_t w9 = *reinterpret_cast<const uint32_t*>(wrow + 1024 + wo1);
        uint32_t elo01[4], ehi01[4], elo89[4], ehi89[4];
        unpack4(prmt(w0, w1, 0x5410), elo01);
        unpack4(prmt(w0, w1, 0x7632), ehi01);
        unpack4(prmt(w8, w9, 0x5410), elo89);
        unpack4(prmt(w8, w9, 0x7632), ehi89);
        uint32_t b0[NT], b1[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int tok = 8 * nt + g;
          const int k0 = 16 * ks + 2 * t;              // even; k0 + 8 in the next chunk
          const int box = k0 >> 6, c0 = (k0 & 63) >> 3;
          const unsigned char* xrow = stp + L::X_OFF + box * (L::MP * 128) + tok * 128;
          b0[nt] = *reinterpret_cast<const uint32_t*>(xrow + (((c0) ^ (tok & 7)) << 4) + (k0 & 7) * 2);
          b1[nt] = *reinterpret_cast<const uint32_t*>(xrow + (((c0 + 1) ^ (tok & 7)) << 4) + (k0 & 7) * 2);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t a[4];
          a[0] = hsub2_u32(elo01[j], zz_lo[j]);
          a[1] = hsub2_u32(ehi01[j], zz_hi[j]);
          a[2] = hsub2_u32(elo89[j], zz_lo[j]);
          a[3] = hsub2_u32(ehi89[j], zz_hi[j]);
          if (SCALE_IN_A) {
            a[0] = hmul2_u32(a[0], ss_lo[j]);
            a[1] = hmul2_u32(a[1], ss_hi[j]);
            a[2] = hmul2_u32(a[2], ss_lo[j]);
            a[3] = hmul2_u32(a[3], ss_hi[j]);
          }
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            if (SCALE_IN_A) mma_16816(acc[j][nt], a, b0[nt], b1[nt]);
            else mma_16816(cg[j][nt], a, b0[nt], b1[nt]);
          }
        }
      }
      if (!SCALE_IN_A) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float2 sf = __half22float2(*reinterpret_cast<const __half2*>(&sw[j]));
          if (j & 1) sf.x *= 0.0625f, sf.y *= 0.0625f;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            acc[j][nt][0] = fmaf(cg[j][nt][0], sf.x, acc[j][nt][0]);
            acc[j][nt][1] = fmaf(cg[j][nt][1], sf.x, acc[j][nt][1]);
            acc[j][nt][2] = fmaf(cg[j][nt][2], sf.y, acc[j][nt][2]);
            acc[j][nt][3] = fmaf(cg[j][nt][3], sf.y, acc[j][nt][3]);
#pragma unroll
            for (int e = 0; e < 4; ++e) cg[j][nt][e] = 0.f;
          }
        }
      }
    }
    // every thread is done with stage s: refill it (or stop on a timeout)
    if (__syncthreads_or(!ready)) break;
    consumed = i + 1;
    if (i + kMmaStages < ng) ++issued;
    if (tid == 0 && i + kMmaStages < ng) {
      const uint32_t st = base + s * L::STAGE, bar = bar0 + 8 * s;
      const int kg = g_begin + i + kMmaStages;
      mbar_arrive_expect_tx(bar, L::TX_BYTES);
      tma_load_2d_hint(st, &tmW, bar, n0 / 8, kg * 128, pol_stream);
      tma_load_2d(st + L::S_OFF, &tmS, bar, n0, kg);
      tma_load_2d(st + L::Z_OFF, &tmZ, bar, n0 / 8, kg);
      tma_load_2d(st + L::X_OFF, &tmX, bar, kg * 128, tok0);
      tma_load_2d(st + L::X_OFF + L::MP * 128, &tmX, bar, kg * 128 + 64, tok0);
    }
  }

  // A timed-out wait left copies in flight: give them (bounded) time to land
  // before this CTA reuses or releases its shared memory.
  if (consumed < ng && tid == 0)
    for (int i = consumed; i < issued; ++i)
      mbar_wait_bounded(bar0 + 8 * (i % kMmaStages), (i / kMmaStages) & 1);
  __syncthreads();

  // ---------------- epilogue
  // partial tile of each k-part: red[kpart][token][256 columns] fp32 (stage memory)
  float* red = reinterpret_cast<float*>(sbase);
  const bool reduce_cta = (KSPLIT > 1) || (gridDim.y > 1);
  if (reduce_cta) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int tt = 0; tt < 2; ++tt) {
        const int tl = 8 * nt + 2 * t + tt;
        float* p = red + ((size_t)kpart * L::MP + tl) * kNTile + 8 * wcol;
        *reinterpret_cast<float4*>(p) =
            make_float4(acc[0][nt][tt], acc[0][nt][2 + tt], acc[1][nt][tt], acc[1][nt][2 + tt]);
        *reinterpret_cast<float4*>(p + 4) =
            make_float4(acc[2][nt][tt], acc[2][nt][2 + tt], acc[3][nt][tt], acc[3][nt][2 + tt]);
      }
    __syncthreads();
    if (KSPLIT > 1) {   // fold the k-parts into part 0, fixed order
      for (int idx = tid; idx < L::MP * kNTile / 4; idx += L::THREADS) {
        float4 v = reinterpret_cast<float4*>(red)[idx];
#pragma unroll
        for (int kp = 1; kp < KSPLIT; ++kp) {
          const float4 u = reinterpret_cast<const float4*>(red + (size_t)kp * L::MP * kNTile)[idx];
          v.x += u.x; v.y += u.y; v.z += u.z; v.w += u.w;
        }
        reinterpret_cast<float4*>(red)[idx] = v;
      }
    }
  }

  const int mrows = min(L::MP, M - tok0);
  if (gridDim.y == 1) {
    if (!reduce_cta) {
      const int ncol = n0 + 8 * wcol;   // this thread's 8 columns
      if (ncol >= N) return;            // N % 32 == 0: all 8 in range together
      float bb[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) bb[c] = bias != nullptr ? __half2float(bias[ncol + c]) : 0.f;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
          const int tok = tok0 + 8 * nt + 2 * t + tt;
          if (tok >= M) continue;
          uint4 out;
          __half2* h = reinterpret_cast<__half2*>(&out);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            h[j] = __floats2half2_rn(acc[j][nt][tt] + bb[2 * j], acc[j][nt][2 + tt] + bb[2 * j + 1]);
          *reinterpret_cast<uint4*>(Y + (size_t)tok * N + ncol) = out;
        }
      return;
    }
    __syncthreads();
    for (int idx = tid; idx < mrows * (kNTile / 4); idx += L::THREADS) {
      const int tl = idx / (kNTile / 4);
      const int n = n0 + 4 * (idx % (kNTile / 4));
      if (n >= N) continue;
      float4 v = reinterpret_cast<const float4*>(red)[idx];
      if (bias != nullptr) {
        v.x += __half2float(bias[n]); v.y += __half2float(bias[n + 1]);
        v.z += __half2float(bias[n + 2]); v.w += __half2float(bias[n + 3]);
      }
      const __half2 h0 = __floats2half2_rn(v.x, v.y), h1 = __floats2half2_rn(v.z, v.w);
      uint2 out;
      out.x = *reinterpret_cast<const uint32_t*>(&h0);
      out.y = *reinterpret_cast<const uint32_t*>(&h1);
      *reinterpret_cast<uint2*>(Y + (size_t)(tok0 + tl) * N + n) = out;
    }
    return;
  }

  // split-K over the cluster: CTA r reduces its column slice over all S partials
  cluster_sync();
  const int S = gridDim.y;
  const uint32_t rank = cluster_ctarank();
  const int cols = kNTile / S;
  const int c_begin = (int)rank * cols;
  const uint32_t red_addr = base;
  for (int idx = tid; idx < mrows * (cols / 4); idx += L::THREADS) {
    const int tl = idx / (cols / 4);
    const int col = c_begin + 4 * (idx % (cols / 4));
    const int n = n0 + col;
    if (n >= N) continue;
    const uint32_t off = red_addr + (uint32_t)(tl * kNTile + col) * 4u;
    float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int q = 0; q < S; ++q) {
      const float4 v = ld_cluster_f4(mapa_shared(off, (uint32_t)q));
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
    *reinterpret_cast<uint2*>(Y + (size_t)(tok0 + tl) * N + n) = out;
  }
  // keep this CTA's partial tile alive until every CTA of the cluster has read it
  cluster_sync();
}

}  // namespace paro

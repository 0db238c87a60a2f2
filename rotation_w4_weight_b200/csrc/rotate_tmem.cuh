// Channel scaling + krot Givens stages with tensor memory as the permutation
// network (sm_100a), for large token counts.
//
// Same arithmetic as rotate_kernel (GPTQModel wiki page "ParoQuant",
// "Pairwise Givens rotations" and "Activation and weight transforms"):
// X_r = X D^-1 R, a' = a cos t + b sin t, b' = -a sin t + b cos t, stages in
// order, pair indices local to the 128-channel group, fp32 on chip, one
// round-to-nearest to fp16 at the end.
//
// A CTA of 4 warps owns one group of 128 token rows: thread t holds row t, i.e.
// TMEM lane t, 128 fp32 columns.  A stage needs, in every row, the two channels
// of each pair side by side; registers cannot be indexed by a runtime pair
// table, but a tcgen05.ld of one column per lane takes a warp-uniform column
// address.  So each stage gathers its 128 operands in pair order (128 one-column
// loads), rotates them in registers with compile-time register indices, and
// writes the 128 results back in that pair order with bulk stores; the next
// stage's gather addresses are composed with that order once per CTA, in a
// shared-memory table.  The last stage scatters to
// the natural channel order instead, and a bulk load brings the row back.
// Tensor memory is split between the four SM sub-partitions, so the data
// movement of a stage no longer funnels through the single shared-memory pipe
// that bounds rotate_kernel.
#pragma once

#include "rotate.cuh"

namespace paro {

constexpr int kRtRows = 128;
constexpr int kRtThreads = 128;
constexpr int kRtCols = 128;             // TMEM columns per CTA (one fp32 per channel)
constexpr int kRtMinSmem = 48 * 1024;    // at most 4 CTAs (4 x 128 TMEM columns) per SM

struct RtLayout {
  // float2 (cos, sin)[krot][64] | uint32 gather column[krot][128] | int pos[2][128] |
  // uint32 final scatter column[128] | tmem slot
  __host__ __device__ static size_t cs_off() { return 0; }
  __host__ __device__ static size_t gather_off(int krot) { return (size_t)krot * 64 * 8; }
  __host__ __device__ static size_t pos_off(int krot) { return gather_off(krot) + (size_t)krot * 128 * 4; }
  __host__ __device__ static size_t fin_off(int krot) { return pos_off(krot) + 2 * 128 * 4; }
  __host__ __device__ static size_t slot_off(int krot) { return fin_off(krot) + 128 * 4; }
  __host__ __device__ static size_t bytes(int krot) {
    const size_t b = slot_off(krot) + 16;
    return b < (size_t)kRtMinSmem ? (size_t)kRtMinSmem : b;
  }
};

__global__ void __launch_bounds__(kRtThreads) rotate_tmem_kernel(
    const __half* x, __half* xr, const float* __restrict__ cs, const int16_t* __restrict__ pairs,
    const float* __restrict__ theta, int M, int K, int krot) {
  // Wait for the previous kernel before reading any input, then let the GEMM
  // that follows start streaming its weights (see rotate_kernel).
  pdl_wait_primary();
  pdl_launch_dependents();

  extern __shared__ __align__(16) unsigned char smem_raw[];
  float2* cstab = reinterpret_cast<float2*>(smem_raw + RtLayout::cs_off());
  uint32_t* gather = reinterpret_cast<uint32_t*>(smem_raw + RtLayout::gather_off(krot));
  int* pos = reinterpret_cast<int*>(smem_raw + RtLayout::pos_off(krot));
  uint32_t* fin = reinterpret_cast<uint32_t*>(smem_raw + RtLayout::fin_off(krot));
  uint32_t* slot = reinterpret_cast<uint32_t*>(smem_raw + RtLayout::slot_off(krot));

  const int grp = blockIdx.x;
  const int row0 = blockIdx.y * kRtRows;
  const int tid = threadIdx.x, warp = tid >> 5;

  if (warp == 0) {
    tmem_alloc(smem_u32(slot), kRtCols);
    tmem_relinquish();
  }

  // ---- tables: (cos, sin) per pair; gather columns per stage.  Stage s reads
  // channel ch from column ch (s = 0) or from its position in stage s-1's pair
  // order (2p for the pair's a, 2p+1 for its b).  Indices outside the group are
  // masked to 7 bits (every column stays inside this CTA's allocation) and flagged.
  for (int idx = tid; idx < krot * 64; idx += kRtThreads) {
    const int s = idx >> 6, p = idx & 63;
    float sn, c;
    sincosf(theta[(size_t)s * (K / 2) + (size_t)grp * 64 + p], &sn, &c);
    cstab[idx] = make_float2(c, sn);
  }
  for (int s = 0; s < krot; ++s) {
    int* cur = pos + (s & 1) * 128;          // positions in stage s's pair order
    const int* prev = pos + ((s + 1) & 1) * 128;
    if (s > 0) __syncthreads();              // prev written, cur free to overwrite
    for (int e = tid; e < 128; e += kRtThreads) cur[e] = e;   // defined even for bad tables
    __syncthreads();
    for (int p = tid; p < 64; p += kRtThreads) {
      const int16_t* ps = pairs + (size_t)s * K + (size_t)grp * kGroup + 2 * p;
      int i = ps[0], j = ps[1];
      if ((unsigned)i >= 128u || (unsigned)j >= 128u) {
        flag_error(kErrPairIndex);
        i &= 127;
        j &= 127;
      }
      gather[s * 128 + 2 * p] = (uint32_t)(s == 0 ? i : prev[i]);
      gather[s * 128 + 2 * p + 1] = (uint32_t)(s == 0 ? j : prev[j]);
      if (s == krot - 1) {                    // the last stage scatters to channel order
        fin[2 * p] = (uint32_t)i;
        fin[2 * p + 1] = (uint32_t)j;
      }
      cur[i] = 2 * p;
      cur[j] = 2 * p + 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *slot + ((uint32_t)(32 * warp) << 16);   // this warp's 32 lanes

  // ---- load the row, scale, store to TMEM in natural channel order
  const int row = row0 + tid;
  uint32_t v[128];
  {
    const __half* src = x + (size_t)row * K + (size_t)grp * kGroup;
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      uint4 raw = make_uint4(0, 0, 0, 0);
      if (row < M) raw = *reinterpret_cast<const uint4*>(src + 8 * q);
      const __half2* h = reinterpret_cast<const __half2*>(&raw);
      float sc[8];
      if (cs != nullptr) {
        const float4 a = *reinterpret_cast<const float4*>(cs + grp * kGroup + 8 * q);
        const float4 b = *reinterpret_cast<const float4*>(cs + grp * kGroup + 8 * q + 4);
        sc[0] = a.x; sc[1] = a.y; sc[2] = a.z; sc[3] = a.w;
        sc[4] = b.x; sc[5] = b.y; sc[6] = b.z; sc[7] = b.w;
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) sc[e] = 1.0f;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(h[e]);
        v[8 * q + 2 * e] = __float_as_uint(f.x * sc[2 * e]);
        v[8 * q + 2 * e + 1] = __float_as_uint(f.y * sc[2 * e + 1]);
      }
    }
  }
  if (krot > 0) {
#pragma unroll
    for (int b = 0; b < 4; ++b) tmem_st32(tbase + 32 * b, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * b]));
    tmem_st_wait();

    for (int s = 0; s < krot; ++s) {
      // gather the stage's operands in pair order
      const uint4* gs = reinterpret_cast<const uint4*>(gather + s * 128);
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        const uint4 g4 = gs[q];
        v[4 * q] = tmem_ld1(tbase + g4.x);
        v[4 * q + 1] = tmem_ld1(tbase + g4.y);
        v[4 * q + 2] = tmem_ld1(tbase + g4.z);
        v[4 * q + 3] = tmem_ld1(tbase + g4.w);
      }
      tmem_ld_wait_tie(*reinterpret_cast<uint32_t(*)[32]>(&v[0]));
      tmem_tie(*reinterpret_cast<uint32_t(*)[32]>(&v[32]));
      tmem_tie(*reinterpret_cast<uint32_t(*)[32]>(&v[64]));
      tmem_tie(*reinterpret_cast<uint32_t(*)[32]>(&v[96]));
      // rotate every pair (registers 2p, 2p+1)
      const float4* cs4 = reinterpret_cast<const float4*>(cstab + s * 64);
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        const float4 t = cs4[q];             // (cos, sin) of pairs 2q and 2q+1
        float a = __uint_as_float(v[4 * q]), b = __uint_as_float(v[4 * q + 1]);
        v[4 * q] = __float_as_uint(fmaf(a, t.x, b * t.y));
        v[4 * q + 1] = __float_as_uint(fmaf(b, t.x, -(a * t.y)));
        a = __uint_as_float(v[4 * q + 2]);
        b = __uint_as_float(v[4 * q + 3]);
        v[4 * q + 2] = __float_as_uint(fmaf(a, t.z, b * t.w));
        v[4 * q + 3] = __float_as_uint(fmaf(b, t.z, -(a * t.w)));
      }
      if (s + 1 < krot) {
        // write back in this stage's pair order (the next gather composes with it)
#pragma unroll
        for (int b = 0; b < 4; ++b)
          tmem_st32(tbase + 32 * b, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * b]));
      } else {
        // last stage: scatter to the natural channel order
        const uint4* f4 = reinterpret_cast<const uint4*>(fin);
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const uint4 f = f4[q];
          tmem_st1(tbase + f.x, v[4 * q]);
          tmem_st1(tbase + f.y, v[4 * q + 1]);
          tmem_st1(tbase + f.z, v[4 * q + 2]);
          tmem_st1(tbase + f.w, v[4 * q + 3]);
        }
      }
      tmem_st_wait();
    }
#pragma unroll
    for (int b = 0; b < 4; ++b) tmem_ld32(tbase + 32 * b, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * b]));
    tmem_ld_wait_tie(*reinterpret_cast<uint32_t(*)[32]>(&v[0]));
    tmem_tie(*reinterpret_cast<uint32_t(*)[32]>(&v[32]));
    tmem_tie(*reinterpret_cast<uint32_t(*)[32]>(&v[64]));
    tmem_tie(*reinterpret_cast<uint32_t(*)[32]>(&v[96]));
  }

  // ---- fp16 (round to nearest) row out
  if (row < M) {
    __half* dst = xr + (size_t)row * K + (size_t)grp * kGroup;
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      uint4 out;
      __half2* h = reinterpret_cast<__half2*>(&out);
#pragma unroll
      for (int e = 0; e < 4; ++e)
        h[e] = __floats2half2_rn(__uint_as_float(v[8 * q + 2 * e]), __uint_as_float(v[8 * q + 2 * e + 1]));
      *reinterpret_cast<uint4*>(dst + 8 * q) = out;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(*slot, kRtCols);
  }
}

}  // namespace paro

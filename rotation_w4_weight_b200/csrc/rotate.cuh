// Channel scaling + krot stages of group-local Givens pair rotations
// (GPTQModel wiki page "ParoQuant", sections "Pairwise Givens rotations" and
// "Activation and weight transforms": X_r = X D^-1 R, a' = a cos t + b sin t,
// b' = -a sin t + b cos t, stages in order, pair indices local to the group).
//
// One CTA owns one 128-channel group of a tile of ROWS token rows.  The tile
// lives in shared memory channel-major (xs[channel][row]) in fp32.  A warp
// instruction covers PPI = 32/RL pairs x RL rows (RL = min(ROWS, 32)): with
// 32 rows per pair every access is 32 consecutive words, conflict-free for any
// pair table; the 4-row tile used for decode batches trades some bank
// conflicts for 8 pairs per instruction and many more CTAs.  Every stage's
// (cos, sin, i, j) is computed once per CTA into shared memory and read as a
// broadcast.  Global traffic is one fp16 read and one fp16 write per element
// (16-byte vectors).
#pragma once

#include "common.cuh"

namespace paro {

constexpr int kGroup = 128;
constexpr int kMaxKrot = 64;
constexpr int kRotThreads = 256;

struct RotParam {
  float c, s;
  int i, j;
};

// Stage tables of group `grp` -> shared memory.  Indices outside 0..127 are
// masked (so no access can leave the tile) and flagged in the status word.
__device__ __forceinline__ void load_rot_params(RotParam* prm, const int16_t* __restrict__ pairs,
                                                const float* __restrict__ theta, int K, int krot,
                                                int grp, int tid, int nthreads) {
  for (int idx = tid; idx < krot * (kGroup / 2); idx += nthreads) {
    const int s = idx / (kGroup / 2);
    const int p = idx % (kGroup / 2);
    const int16_t* ps = pairs + (size_t)s * K + (size_t)grp * kGroup + 2 * p;
    int i = ps[0], j = ps[1];
    if ((unsigned)i >= (unsigned)kGroup || (unsigned)j >= (unsigned)kGroup) {
      flag_error(kErrPairIndex);
      i &= kGroup - 1;
      j &= kGroup - 1;
    }
    float sn, cs;
    rot_sincos(theta[(size_t)s * (K / 2) + (size_t)grp * (kGroup / 2) + p], &sn, &cs);
    prm[idx] = RotParam{cs, sn, i, j};
  }
}

template <int ROWS>
struct RotTile {
  static constexpr int RL = ROWS < 32 ? ROWS : 32;     // rows per lane group
  static constexpr int PPI = 32 / RL;                  // pairs per warp instruction
  static constexpr int R = ROWS / RL;                  // rows per lane
  static constexpr int PITCH = ROWS < 32 ? ROWS + 1 : ROWS;
};

// grid: (K/128, ceil(M/ROWS)), block 256.  Dynamic smem: krot*64*16 bytes of
// RotParam + the fp32 tile (rotate_smem_bytes).
template <int ROWS>
__global__ void __launch_bounds__(kRotThreads) rotate_kernel(
    const __half* x, __half* xr, const float* __restrict__ cs,
    const int16_t* __restrict__ pairs, const float* __restrict__ theta, int M, int K, int krot) {
  using T = RotTile<ROWS>;
  // Programmatic dependent launch: the GEMV that follows may launch at once and
  // stream its weights while this kernel works.  The stage tables are layer
  // constants (read-only for the call, not written by the previous kernel), so
  // they are read before waiting for the previous kernel; x is read after.
  pdl_launch_dependents();

  extern __shared__ __align__(16) unsigned char smem_raw[];
  RotParam* prm = reinterpret_cast<RotParam*>(smem_raw);
  float* xs = reinterpret_cast<float*>(smem_raw + (size_t)krot * (kGroup / 2) * sizeof(RotParam));

  const int grp = blockIdx.x;
  const int row0 = blockIdx.y * ROWS;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  load_rot_params(prm, pairs, theta, K, krot, grp, tid, kRotThreads);
  pdl_wait_primary();

  // ---- load + scale: item = (8-channel chunk v, row r), rows fastest
  for (int idx = tid; idx < 16 * ROWS; idx += kRotThreads) {
    const int v = idx / ROWS, r = idx % ROWS;
    const int row = row0 + r;
    const int ch0 = grp * kGroup + 8 * v;
    uint4 raw = make_uint4(0, 0, 0, 0);
    if (row < M) raw = *reinterpret_cast<const uint4*>(x + (size_t)row * K + ch0);
    float sc[8];
    if (cs != nullptr) {
      const float4 a = *reinterpret_cast<const float4*>(cs + ch0);
      const float4 b = *reinterpret_cast<const float4*>(cs + ch0 + 4);
      sc[0] = a.x; sc[1] = a.y; sc[2] = a.z; sc[3] = a.w;
      sc[4] = b.x; sc[5] = b.y; sc[6] = b.z; sc[7] = b.w;
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) sc[e] = 1.0f;
    }
    const __half2* h = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __half22float2(h[e]);
      xs[(8 * v + 2 * e) * T::PITCH + r] = f.x * sc[2 * e];
      xs[(8 * v + 2 * e + 1) * T::PITCH + r] = f.y * sc[2 * e + 1];
    }
  }
  __syncthreads();

  // ---- stages: warp w applies pairs 8w..8w+7; lane = (pair sub-index, row)
  const int pq = lane / T::RL, rl = lane % T::RL;
  for (int s = 0; s < krot; ++s) {
    const RotParam* ps = prm + s * (kGroup / 2) + warp * 8;
#pragma unroll
    for (int q = 0; q < 8 / T::PPI; ++q) {
      const RotParam p = ps[q * T::PPI + pq];
      float* xi = xs + p.i * T::PITCH + rl;
      float* xj = xs + p.j * T::PITCH + rl;
#pragma unroll
      for (int rr = 0; rr < T::R; ++rr) {
        const float a = xi[rr * 32];
        const float b = xj[rr * 32];
        xi[rr * 32] = fmaf(a, p.c, b * p.s);
        xj[rr * 32] = fmaf(b, p.c, -(a * p.s));
      }
    }
    __syncthreads();
  }

  // ---- store fp16 (round to nearest), same item mapping as the load
  for (int idx = tid; idx < 16 * ROWS; idx += kRotThreads) {
    const int v = idx / ROWS, r = idx % ROWS;
    const int row = row0 + r;
    if (row >= M) continue;
    const int ch0 = grp * kGroup + 8 * v;
    uint4 out;
    __half2* h = reinterpret_cast<__half2*>(&out);
#pragma unroll
    for (int e = 0; e < 4; ++e)
      h[e] = __floats2half2_rn(xs[(8 * v + 2 * e) * T::PITCH + r],
                               xs[(8 * v + 2 * e + 1) * T::PITCH + r]);
    *reinterpret_cast<uint4*>(xr + (size_t)row * K + ch0) = out;
  }
}

inline size_t rotate_smem_bytes(int rows, int krot) {
  const size_t tile = rows < 32 ? (size_t)kGroup * (rows + 1) * 4 : (size_t)kGroup * rows * 4;
  return (size_t)krot * (kGroup / 2) * sizeof(RotParam) + tile;
}

}  // namespace paro

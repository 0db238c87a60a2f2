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

// The kernels work on 128-channel tiles; a tile holds 128 / G rotation groups
// (G = 16, 32, 64 or 128).  Pair p of a tile's stage (entries 2p, 2p+1 of the
// tile's slice of the pair table, angle p of its slice of theta) belongs to
// the tile's group 2p / G, and its group-local indices become tile channels
// by that group's offset.  An index outside 0..G-1 is masked to the group (so
// no access can leave it) and flagged in the status word.
__device__ __forceinline__ void tile_pair(uint32_t raw, int p, int gsz, int* i, int* j) {
  uint32_t a = raw & 0xFFFFu, b = raw >> 16;
  if ((a | b) >= (uint32_t)gsz) {
    flag_error(kErrPairIndex);
    a &= (uint32_t)(gsz - 1);
    b &= (uint32_t)(gsz - 1);
  }
  const int off = (2 * p) & ~(gsz - 1);           // first channel of the pair's group in the tile
  *i = (int)a + off;
  *j = (int)b + off;
}

// Stage tables of tile `grp` -> shared memory.
__device__ __forceinline__ void load_rot_params(RotParam* prm, const int16_t* __restrict__ pairs,
                                                const float* __restrict__ theta, int K, int krot,
                                                int grp, int gsz, int tid, int nthreads) {
  for (int idx = tid; idx < krot * (kGroup / 2); idx += nthreads) {
    const int s = idx / (kGroup / 2);
    const int p = idx % (kGroup / 2);
    const uint32_t raw =
        *reinterpret_cast<const uint32_t*>(pairs + (size_t)s * K + (size_t)grp * kGroup + 2 * p);
    int i, j;
    tile_pair(raw, p, gsz, &i, &j);
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
template <int ROWS, typename TA>
__global__ void __launch_bounds__(kRotThreads) rotate_kernel(
    const TA* x, TA* xr, const float* __restrict__ cs,
    const int16_t* __restrict__ pairs, const float* __restrict__ theta, int M, int K, int krot, int gsz) {
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

  load_rot_params(prm, pairs, theta, K, krot, grp, gsz, tid, kRotThreads);
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
    const uint32_t h[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = Act<TA>::f2(h[e]);
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
    uint32_t h[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      h[e] = Act<TA>::p2(xs[(8 * v + 2 * e) * T::PITCH + r], xs[(8 * v + 2 * e + 1) * T::PITCH + r]);
    *reinterpret_cast<uint4*>(xr + (size_t)row * K + ch0) = make_uint4(h[0], h[1], h[2], h[3]);
  }
}

// ---------------------------------------------------------------------------
// Decode batches (M <= 16, krot <= 8): one warp per token row of a group, so
// no block-wide barrier sits between stages.  The CTA first turns the stage
// tables into per-channel form (partner channel, cos, signed sin: channel i of
// pair (i, j) gets +sin, channel j gets -sin, so both updates read
// x' = x cos + x_partner sin_signed, the same fma order as rotate_kernel); a
// lane keeps its four channels' entries for every stage in registers.  Per
// stage a warp publishes its row (128 fp32) in its own shared buffer, reads the
// four partner values and updates its channels.  Tables are layer constants,
// built before waiting for the previous kernel; x is read after.
// Two warps (token rows) per CTA: small enough in registers to share an SM
// with two decode-GEMV CTAs of the kernel ahead, so the next call's table
// build overlaps its tail (8 warps: decoder-layer decode rotation overhead
// 13.2 %, 2 warps: 10.3 %, 1 warp: 14.2 %, the build no longer hidden).
constexpr int kRrWarps = 2;                // token rows per CTA
constexpr int kRrMaxKrot = 8;              // stages kept in registers

struct RrLayout {
  // partner[krot][128] u8 | cos[krot][128] f32 | signed sin[krot][128] f32 | row buffers[kRrWarps][128] f32
  __host__ __device__ static constexpr size_t cos_off(int krot) { return ((size_t)krot * 128 + 15) / 16 * 16; }
  __host__ __device__ static constexpr size_t sin_off(int krot) { return cos_off(krot) + (size_t)krot * 512; }
  __host__ __device__ static constexpr size_t row_off(int krot) { return sin_off(krot) + (size_t)krot * 512; }
  // two row buffers per warp, alternating by stage
  __host__ __device__ static constexpr size_t bytes(int krot) { return row_off(krot) + kRrWarps * 1024; }
};

// Rotation tables and output of one linear; a launch rotates the same x for up
// to kRrMaxLinears linears (blockIdx.z), each with its own tables.
constexpr int kRrMaxLinears = 4;
struct RrOperand {
  void* xr;                // X_r of the activation type
  const float* cs;
  const int16_t* pairs;
  const float* theta;
  int krot;
};
struct RrBatch {
  RrOperand op[kRrMaxLinears];
};

template <typename TA>
__global__ void __launch_bounds__(32 * kRrWarps) rotate_rows_kernel(const RrBatch batch, const TA* x,
                                                                    int M, int K, int gsz) {
  pdl_launch_dependents();                         // the GEMV may start streaming weights
  RrOperand o = batch.op[0];
#pragma unroll
  for (int i = 1; i < kRrMaxLinears; ++i)
    if ((int)blockIdx.z == i) o = batch.op[i];
  TA* const xr = static_cast<TA*>(o.xr);
  const float* __restrict__ const cs = o.cs;
  const int16_t* __restrict__ const pairs = o.pairs;
  const float* __restrict__ const theta = o.theta;
  const int krot = o.krot;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  uint8_t* partner = smem_raw;
  float* cosv = reinterpret_cast<float*>(smem_raw + RrLayout::cos_off(krot));
  float* sinv = reinterpret_cast<float*>(smem_raw + RrLayout::sin_off(krot));
  const int grp = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row = blockIdx.y * kRrWarps + warp;

  // ---- per-channel tables (identity first, so every entry is defined)
  for (int idx = tid; idx < krot * 128; idx += blockDim.x) {
    partner[idx] = (uint8_t)(idx & 127);
    cosv[idx] = 1.f;
    sinv[idx] = 0.f;
  }
  __syncthreads();
  for (int idx = tid; idx < krot * 64; idx += blockDim.x) {
    const int st = idx >> 6, p = idx & 63;
    const uint32_t pr = *reinterpret_cast<const uint32_t*>(pairs + (size_t)st * K + (size_t)grp * kGroup + 2 * p);
    int i, j;
    tile_pair(pr, p, gsz, &i, &j);                 // masked to the group, flagged
    float sn, c;
    rot_sincos(theta[(size_t)st * (K / 2) + (size_t)grp * 64 + p], &sn, &c);
    partner[st * 128 + i] = (uint8_t)j;
    cosv[st * 128 + i] = c;
    sinv[st * 128 + i] = sn;
    partner[st * 128 + j] = (uint8_t)i;
    cosv[st * 128 + j] = c;
    sinv[st * 128 + j] = -sn;
  }
  __syncthreads();
  const int ch = 4 * lane;                         // this lane's channels ch .. ch+3
  uint32_t pw[kRrMaxKrot];
  float4 cf[kRrMaxKrot], sf[kRrMaxKrot];
#pragma unroll
  for (int st = 0; st < kRrMaxKrot; ++st) {
    if (st < krot) {
      pw[st] = *reinterpret_cast<const uint32_t*>(partner + st * 128 + ch);
      cf[st] = *reinterpret_cast<const float4*>(cosv + st * 128 + ch);
      sf[st] = *reinterpret_cast<const float4*>(sinv + st * 128 + ch);
    }
  }
  float4 csv = make_float4(1.f, 1.f, 1.f, 1.f);
  if (cs != nullptr) csv = *reinterpret_cast<const float4*>(cs + (size_t)grp * kGroup + ch);

  pdl_wait_primary();                              // x may come from the previous kernel
  if (row >= M) return;
  const uint2 raw = *reinterpret_cast<const uint2*>(x + (size_t)row * K + (size_t)grp * kGroup + ch);
  const float2 lo = Act<TA>::f2(raw.x);
  const float2 hi = Act<TA>::f2(raw.y);
  float v[4] = {lo.x * csv.x, lo.y * csv.y, hi.x * csv.z, hi.y * csv.w};
  // Stage st publishes into buffer st & 1: the barrier after a publish also
  // orders every lane's reads of the stage before (the other buffer), so the
  // buffer a publish overwrites was last read two stages ago, behind that
  // barrier; one warp barrier per stage.
  const uint32_t rb0 = smem_u32(smem_raw + RrLayout::row_off(krot) + warp * 1024);
#pragma unroll
  for (int st = 0; st < kRrMaxKrot; ++st) {
    if (st < krot) {
      const uint32_t rb = rb0 + 512u * (uint32_t)(st & 1);
      sts128(rb + 4u * ch, make_float4(v[0], v[1], v[2], v[3]));
      __syncwarp();
      float xp[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) xp[k] = __uint_as_float(lds32(rb + 4u * ((pw[st] >> (8 * k)) & 0xFFu)));
      const float c4[4] = {cf[st].x, cf[st].y, cf[st].z, cf[st].w};
      const float s4[4] = {sf[st].x, sf[st].y, sf[st].z, sf[st].w};
#pragma unroll
      for (int k = 0; k < 4; ++k) v[k] = fmaf(v[k], c4[k], xp[k] * s4[k]);
    }
  }
  uint2 out;
  out.x = Act<TA>::p2(v[0], v[1]);
  out.y = Act<TA>::p2(v[2], v[3]);
  *reinterpret_cast<uint2*>(xr + (size_t)row * K + (size_t)grp * kGroup + ch) = out;
}

inline size_t rotate_smem_bytes(int rows, int krot) {
  const size_t tile = rows < 32 ? (size_t)kGroup * (rows + 1) * 4 : (size_t)kGroup * rows * 4;
  return (size_t)krot * (kGroup / 2) * sizeof(RotParam) + tile;
}

}  // namespace paro

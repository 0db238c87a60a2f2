// Stacked experts sharing one rotation: routing on the device.
//
// What the layer computes (brain.gartu.xyz ParoQuant page, MLX section: the
// experts' weights are stacked in one tensor and their rotations are shared;
// each projection is the rotated W4 linear of the GPTQModel wiki page
// "ParoQuant", "Activation and weight transforms"):
//   X_r = rotate(x * channel_scales)                 once, for every expert
//   y[t, j] = X_r[t] . dequant(W[e]) + b[e],         e = expert_idx[t, j]
//
// The calls that follow need the routed rows of each expert contiguous.  The
// route kernel (one CTA) counts the slots of every expert, scans the counts
// into offsets, cuts each expert's rows into segments of at most 8 rows (the
// decode GEMV's token tile) and tiles of at most 256 rows (the prefill GEMM's
// tile), and places every valid slot at offset[e] + (its rank among the
// earlier slots of e): a stable counting sort, so the order is the slots'
// order and the result is deterministic.  X_r[token(slot)] is then copied
// into the sorted rows: by the route kernel itself when they are few (decode),
// else by the gather kernel.  A slot whose index lies outside
// 0..E-1 is flagged in the status word and its output row is written as 0.
#pragma once

#include "common.cuh"

namespace paro {

constexpr int kMoeRouteThreads = 1024;
constexpr int kMoeMaxExperts = kMoeRouteThreads;   // one expert per thread in the scans
constexpr int kMoeGvRows = 8;                       // rows per decode GEMV segment
constexpr int kMoeTcRows = 256;                     // rows per prefill GEMM tile
// Routed rows up to this many bytes are gathered by the route kernel (one CTA
// copies them in a few microseconds at most), saving the gather launch.
constexpr size_t kMoeRouteGatherBytes = 256 * 1024;

// Routing results, in the caller's workspace.
struct MoeHead {
  int valid;      // routed slots (indices inside 0..E-1)
  int n_gv;       // decode segments
  int n_tc;       // prefill tiles
  int pad;
};

// Exclusive scan over the block (one value per thread); `tot` gets the total.
__device__ __forceinline__ int moe_block_scan(int v, int* warp_sums, int* tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, inc, d);
    if (lane >= d) inc += u;
  }
  if (lane == 31) warp_sums[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    int w = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, w, d);
      if (lane >= d) w += u;
    }
    if (lane < nw) warp_sums[lane] = w;           // inclusive over warps
  }
  __syncthreads();
  const int before = (warp > 0 ? warp_sums[warp - 1] : 0) + inc - v;
  *tot = warp_sums[(blockDim.x >> 5) - 1];
  __syncthreads();                                 // warp_sums may be reused
  return before;
}

// One CTA of kMoeRouteThreads threads.  idx [S] (S = T * topk slots, slot
// p = t * topk + j); y [S, N] of the activation type, 16-byte aligned.  With
// `xg` set, sorted row q of xg [S, K] <- row perm[q] / topk of xr [T, K]
// (rows of x_chunks 16-byte chunks).
__global__ void __launch_bounds__(kMoeRouteThreads) moe_route_kernel(const int* __restrict__ idx, int S, int E,
                                                                    MoeHead* head, int* __restrict__ perm,
                                                                    int4* __restrict__ gv, int4* __restrict__ tc,
                                                                    void* y, int row_bytes, const uint4* xr,
                                                                    uint4* xg, int x_chunks, int topk) {
  __shared__ int cnt[kMoeMaxExperts];
  __shared__ int off[kMoeMaxExperts];
  __shared__ int warp_sums[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_launch_dependents();                         // the gather may launch; it waits for us
  pdl_wait_primary();                              // the indices may come from the kernel ahead
  for (int e = tid; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  for (int p = tid; p < S; p += blockDim.x) {
    const int e = idx[p];
    if (e >= 0 && e < E) {
      atomicAdd(&cnt[e], 1);                       // counts only: the order comes below
    } else {
      flag_error(kErrExpertIndex);
      uint4* row = reinterpret_cast<uint4*>(static_cast<unsigned char*>(y) + (size_t)p * row_bytes);
      for (int c = 0; c < row_bytes / 16; ++c) row[c] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  __syncthreads();
  // scans over the experts: row offsets, decode segments, prefill tiles
  const int c = tid < E ? cnt[tid] : 0;
  const int ngv = (c + kMoeGvRows - 1) / kMoeGvRows, ntc = (c + kMoeTcRows - 1) / kMoeTcRows;
  int valid, tot_gv, tot_tc;
  const int o = moe_block_scan(c, warp_sums, &valid);
  const int ogv = moe_block_scan(ngv, warp_sums, &tot_gv);
  const int otc = moe_block_scan(ntc, warp_sums, &tot_tc);
  if (tid < E) {
    off[tid] = o;
    for (int i = 0; i < ngv; ++i) gv[ogv + i] = make_int4(tid, o + kMoeGvRows * i, min(kMoeGvRows, c - kMoeGvRows * i), 0);
    for (int i = 0; i < ntc; ++i) tc[otc + i] = make_int4(tid, o + kMoeTcRows * i, min(kMoeTcRows, c - kMoeTcRows * i), 0);
  }
  if (tid == 0) *head = MoeHead{valid, tot_gv, tot_tc, 0};
  __syncthreads();
  // stable placement: warp w places experts w, w + 32, ...; a ballot over 32
  // consecutive slots ranks the hits in slot order
  for (int e = warp; e < E; e += blockDim.x >> 5) {
    const int n = cnt[e];
    if (n == 0) continue;
    int run = 0;
    for (int p0 = 0; p0 < S && run < n; p0 += 32) {
      const int p = p0 + lane;
      const bool hit = p < S && idx[p] == e;
      const unsigned m = __ballot_sync(0xffffffffu, hit);
      if (hit) perm[off[e] + run + __popc(m & ((1u << lane) - 1u))] = p;
      run += __popc(m);
    }
  }
  if (xg == nullptr) return;
  // the gather, for few rows: perm is complete (and visible to the CTA) after
  // the barrier; X_r was written by the kernel ahead (waited for above)
  __syncthreads();
  const int64_t chunks = (int64_t)valid * x_chunks;
  for (int64_t i = tid; i < chunks; i += blockDim.x) {
    const int q = (int)(i / x_chunks), c = (int)(i - (int64_t)q * x_chunks);
    xg[i] = xr[(int64_t)(perm[q] / topk) * x_chunks + c];
  }
}

// Sorted row q (q < valid) <- X_r[perm[q] / topk]: one warp per row, 16-byte
// chunks.  grid ceil(S / 8), block 256.
template <typename TA>
__global__ void __launch_bounds__(256) moe_gather_kernel(const MoeHead* head, const int* __restrict__ perm,
                                                         const TA* __restrict__ xr, TA* __restrict__ xg, int K,
                                                         int topk) {
  pdl_launch_dependents();                         // the expert GEMV / GEMM may start; it waits for us
  pdl_wait_primary();                              // the routing and X_r are written by the kernels ahead
  const int q = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (q >= head->valid) return;
  const int t = perm[q] / topk;
  const uint4* src = reinterpret_cast<const uint4*>(xr + (size_t)t * K);
  uint4* dst = reinterpret_cast<uint4*>(xg + (size_t)q * K);
  for (int c = lane; c < K / 8; c += 32) dst[c] = src[c];
}

}  // namespace paro

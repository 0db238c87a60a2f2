// C ABI of the library (declarations and contracts in include/paro.h):
// host-side validation, workspace planning, TMA descriptor encoding and
// kernel dispatch.  Every error is reported as a status code before any launch.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cstring>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/paro.h"
#include "common.cuh"
#include "pack.cuh"
#include "rotate.cuh"
#include "rotate_tmem.cuh"
#include "rotate_tc.cuh"
#include "moe.cuh"
#include "w4_gemv.cuh"
#include "w4_tc.cuh"

using namespace paro;

namespace {

constexpr int kMaxDecodeM = 16;      // M <= 16: split-K GEMV path
constexpr int kDecodeTargetCtas = 296;   // two decode CTAs per SM
constexpr int kMaxSplits = 8;         // cluster size along K (portable maximum)
// M >= this: paro_w4_linear rotates on the tensor cores (R' built per call into
// the workspace; measured faster than the pair-by-pair tensor-memory kernel from
// one 128-row tile up); below it the shared-memory / warp-per-row kernels
constexpr int64_t kRotTcMinM = 65;
// longest wait paro_selftest_wait_timeout accepts (it holds the stream that long)
constexpr uint64_t kSelftestMaxLimitNs = 100000000ull;   // 100 ms

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ---------------------------------------------------------------- activation type
// TMA element type of the activation type (loads and stores copy the bits).
template <typename TA>
constexpr CUtensorMapDataType tma_dt() {
  return Act<TA>::kBf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
}

// ---------------------------------------------------------------- TMA encode
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D row-major tensor [rows, cols] of `esize`-byte elements, box [box_rows, box_cols].
bool encode_2d(CUtensorMap* map, CUtensorMapDataType dt, size_t esize, const void* ptr,
               uint64_t rows, uint64_t cols, uint32_t box_rows, uint32_t box_cols,
               CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * esize};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// X as [K/64 chunks][rows][64] (chunk stride 128 bytes, row stride K*2 bytes):
// box {64 columns, box_rows rows, box_chunks chunks}, 128-byte swizzle.  One
// copy brings several groups' activation columns in the layout the GEMV reads.
bool encode_x_chunks(CUtensorMap* map, CUtensorMapDataType dt, const void* x, uint64_t rows, uint64_t K,
                     uint32_t box_rows, uint32_t box_chunks) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {64, rows, K / 64};
  cuuint64_t strides[2] = {K * 2, 128};
  cuuint32_t box[3] = {64, box_rows, box_chunks};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, dt, 3, const_cast<void*>(x), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- device facts
struct DeviceInfo {
  int sms = 0;
  size_t smem_per_sm = 0, smem_reserved_per_block = 0, smem_optin = 0;
};

// SM count and shared-memory capacity of the current device, queried once per
// device (entries are never moved, so returned references stay valid).
const DeviceInfo& device_info() {
  constexpr int kDevs = 64;
  static std::mutex mu;
  static DeviceInfo table[kDevs];
  static const DeviceInfo none;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kDevs) return none;
  std::lock_guard<std::mutex> lock(mu);
  DeviceInfo& d = table[dev];
  if (d.sms != 0) return d;
  int sms = 0, per_sm = 0, reserved = 0, optin = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess)
    return none;
  d.smem_per_sm = (size_t)per_sm;
  d.smem_reserved_per_block = (size_t)reserved;
  d.smem_optin = (size_t)optin;
  d.sms = sms;
  return d;
}

// ---------------------------------------------------------------- launches
template <typename Kern, typename... Args>
int launch_ex(Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream, bool pdl,
              unsigned cluster_y, bool balance, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[3];
  unsigned n = 0;
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster_y > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = 1;
    attr[n].val.clusterDim.y = cluster_y;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  if (cluster_y > 1 && balance) {
    // let the hardware place a cluster's CTAs by load rather than packing them
    attr[n].id = cudaLaunchAttributeClusterSchedulingPolicyPreference;
    attr[n].val.clusterSchedulingPolicyPreference = cudaClusterSchedulingPolicyLoadBalancing;
    ++n;
  }
  cfg.attrs = n ? attr : nullptr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, args...) == cudaSuccess ? PARO_OK : PARO_ERR_CUDA;
}

template <typename Kern, typename... Args>
int launch(Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream, bool pdl,
           Args... args) {
  return launch_ex(kernel, grid, block, smem, stream, pdl, 1u, false, args...);
}

// Raise the dynamic shared memory limit of a kernel once per device (callers
// pass the largest size the kernel is ever launched with) and ask for the
// largest shared-memory carveout.
template <typename Kern>
bool allow_smem(Kern kernel, size_t bytes) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  static std::mutex mu;
  static std::vector<std::pair<const void*, int>> done;
  std::lock_guard<std::mutex> lock(mu);
  const void* key = reinterpret_cast<const void*>(kernel);
  for (auto& d : done)
    if (d.first == key && d.second == dev) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) !=
      cudaSuccess)
    return false;
  // every kernel here stages its operands in shared memory: prefer the largest carveout
  // (occupancy queries then see the configuration the launches get)
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared) != cudaSuccess)
    return false;
  done.emplace_back(key, dev);
  return true;
}

// Group sizes the kernels implement: every power of two that divides their
// 128-channel tiles down to 16 (the rotation groups and the quantisation
// groups share G; K must be a multiple of 128).
inline bool supported_group(int G, int64_t K) {
  return (G == 16 || G == 32 || G == 64 || G == 128) && K % kGroup == 0;
}

// The group size of a call whose arguments passed the checks (-1 is K).
inline int group_of(int group_size, int64_t K) { return group_size == -1 ? (int)K : group_size; }

int normalize_group(int group_size, int64_t K, int* G) {
  const int64_t g = (group_size == -1) ? K : group_size;
  if (g <= 0 || (g % 2) != 0 || K <= 0 || (K % g) != 0) return PARO_ERR_INVALID_ARG;
  *G = static_cast<int>(g);
  return PARO_OK;
}

// ---------------------------------------------------------------- rotation
int check_rotation_args(const void* x, const void* xr, int64_t M, int64_t K, const float* cs,
                        const int16_t* pairs, const float* theta, int group_size, int krot) {
  if (M < 0 || K <= 0 || krot < 0) return PARO_ERR_INVALID_ARG;
  int G = 0;
  if (int st = normalize_group(group_size, K, &G)) return st;
  if (!supported_group(G, K) || krot > kMaxKrot) return PARO_ERR_UNSUPPORTED;
  if (M == 0) return PARO_OK;   // nothing to touch: NULL data pointers are fine
  if (x == nullptr || xr == nullptr) return PARO_ERR_INVALID_ARG;
  if (krot > 0 && (pairs == nullptr || theta == nullptr)) return PARO_ERR_INVALID_ARG;
  if (M * K >= (int64_t(1) << 31)) return PARO_ERR_UNSUPPORTED;
  if (!aligned(x, 16) || !aligned(xr, 16)) return PARO_ERR_ALIGNMENT;
  if (cs != nullptr && !aligned(cs, 16)) return PARO_ERR_ALIGNMENT;
  if (krot > 0 && (!aligned(pairs, 4) || !aligned(theta, 4))) return PARO_ERR_ALIGNMENT;
  return PARO_OK;
}

// Warp-per-row rotation of one x for `count` linears (blockIdx.z), decode sizes
// (M <= 16, every krot <= kRrMaxKrot; max_krot sizes the tables).
template <typename TA>
int launch_rotate_rows(const TA* x, const RrBatch& b, int count, int64_t M, int64_t K, int max_krot,
                       int gsz, cudaStream_t stream) {
  // always kRrWarps warps: all of them build the tables, warps past the batch then leave
  const dim3 grid((unsigned)(K / kGroup), (unsigned)((M + kRrWarps - 1) / kRrWarps), (unsigned)count);
  if (!allow_smem(rotate_rows_kernel<TA>, RrLayout::bytes(kRrMaxKrot))) return PARO_ERR_CUDA;
  return launch(rotate_rows_kernel<TA>, grid, dim3(32 * kRrWarps), RrLayout::bytes(max_krot), stream, true, b,
                x, (int)M, (int)K, gsz);
}

// Tensor-memory rotation kernel (and, with QUANT, the weight quantiser): CTAs
// stay resident over several 128-row tiles of one group (one wave of at most
// 2 CTAs per SM: the shared-memory floor of the kernel guarantees no more fit).
template <bool QUANT, typename TA>
int launch_rotate_tmem(const TA* x, TA* xr, int64_t M, int64_t K, const float* cs,
                       const int16_t* pairs, const float* theta, int krot, int gsz, const RtQuant& qo,
                       cudaStream_t stream) {
  const size_t smem = RtLayout::bytes(krot, QUANT);
  const DeviceInfo& di = device_info();
  if (di.sms == 0) return PARO_ERR_CUDA;
  const bool abs_tables = krot <= kRtAbsMaxKrot;
  if (abs_tables ? !allow_smem(rotate_tmem_kernel<true, QUANT, TA>, RtLayout::bytes(kRtAbsMaxKrot, QUANT))
                 : !allow_smem(rotate_tmem_kernel<false, QUANT, TA>, RtLayout::bytes(kMaxKrot, QUANT)))
    return PARO_ERR_CUDA;
  const size_t per_block = smem + di.smem_reserved_per_block;
  int per_sm = (int)(di.smem_per_sm / per_block);
  per_sm = per_sm < 1 ? 1 : (per_sm > kRtMaxCtasPerSm ? kRtMaxCtasPerSm : per_sm);
  // one wave: gridDim.y row-tile slots per group, then as few tiles per CTA
  // as that allows, spread evenly
  const int64_t groups = K / kGroup, ntiles = (M + kRtRows - 1) / kRtRows;
  const int64_t slots = (int64_t)di.sms * per_sm;
  int64_t gy = slots / groups;
  gy = gy < 1 ? 1 : (gy > ntiles ? ntiles : gy);
  const int64_t per_cta = (ntiles + gy - 1) / gy;
  gy = (ntiles + per_cta - 1) / per_cta;
  if (gy > 65535) gy = 65535;
  CUtensorMap tmX;
  if (!encode_2d(&tmX, tma_dt<TA>(), 2, x, M, K, kRtRows, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return PARO_ERR_CUDA;
  const dim3 grid((unsigned)groups, (unsigned)gy);
  if (abs_tables)
    return launch(rotate_tmem_kernel<true, QUANT, TA>, grid, dim3(kRtThreads), smem, stream, true, tmX, xr, cs,
                  pairs, theta, (int)M, (int)K, krot, gsz, qo);
  return launch(rotate_tmem_kernel<false, QUANT, TA>, grid, dim3(kRtThreads), smem, stream, true, tmX, xr, cs,
                pairs, theta, (int)M, (int)K, krot, gsz, qo);
}

template <typename TA>
int launch_rotate(const TA* x, TA* xr, int64_t M, int64_t K, const float* cs,
                  const int16_t* pairs, const float* theta, int krot, int gsz, cudaStream_t stream) {
  // Large batches: tensor memory as the permutation network.
  if (M > 64) return launch_rotate_tmem<false, TA>(x, xr, M, K, cs, pairs, theta, krot, gsz, RtQuant{}, stream);
  // Decode batches with few stages: one warp per row, no block barrier per stage.
  if (M <= 16 && krot <= kRrMaxKrot) {
    RrBatch b;
    std::memset(&b, 0, sizeof(b));
    b.op[0] = RrOperand{xr, cs, pairs, theta, krot};
    return launch_rotate_rows<TA>(x, b, 1, M, K, krot, gsz, stream);
  }
  // rows per CTA: 4 for decode-sized batches (more CTAs, shorter latency),
  // 32..64 otherwise (conflict-free 32-row warp accesses)
  const int rows = M <= 16 ? 4 : (M <= 32 ? 32 : (M <= 64 ? 64 : 128));
  const size_t smem = rotate_smem_bytes(rows, krot);
  const dim3 grid((unsigned)(K / kGroup), (unsigned)((M + rows - 1) / rows));
  const dim3 block(kRotThreads);
  if (grid.y > 65535u) return PARO_ERR_UNSUPPORTED;
  // the limit is raised once to what the largest krot needs
  switch (rows) {
    case 4:
      if (!allow_smem(rotate_kernel<4, TA>, rotate_smem_bytes(4, kMaxKrot))) return PARO_ERR_CUDA;
      return launch(rotate_kernel<4, TA>, grid, block, smem, stream, true, x, xr, cs, pairs, theta,
                    (int)M, (int)K, krot, gsz);
    case 32:
      if (!allow_smem(rotate_kernel<32, TA>, rotate_smem_bytes(32, kMaxKrot))) return PARO_ERR_CUDA;
      return launch(rotate_kernel<32, TA>, grid, block, smem, stream, true, x, xr, cs, pairs, theta,
                    (int)M, (int)K, krot, gsz);
    case 64:
      if (!allow_smem(rotate_kernel<64, TA>, rotate_smem_bytes(64, kMaxKrot))) return PARO_ERR_CUDA;
      return launch(rotate_kernel<64, TA>, grid, block, smem, stream, true, x, xr, cs, pairs, theta,
                    (int)M, (int)K, krot, gsz);
    default:
      if (!allow_smem(rotate_kernel<128, TA>, rotate_smem_bytes(128, kMaxKrot))) return PARO_ERR_CUDA;
      return launch(rotate_kernel<128, TA>, grid, block, smem, stream, true, x, xr, cs, pairs, theta,
                    (int)M, (int)K, krot, gsz);
  }
}

// Rotation as X R' on the tensor cores for `count` linears that read the same
// x: one launch builds every member's R' (fp16 parts, transposed) into its `rt`,
// a second computes every member's X_r = X R'.
struct RotTcMember {
  const float* cs;
  const int16_t* pairs;
  const float* theta;
  int krot;
  void* xr;         // X_r [M, K]
  void* rt;         // R' parts [2][K][128]
  bool prebuilt;    // rt already holds R' (paro_rotation_matrix_prepare): no build
};

template <typename TA>
int launch_rotate_tc(const TA* x, const RotTcMember* mem, int count, int64_t M, int64_t K, int gsz,
                     cudaStream_t stream) {
  const DeviceInfo& di = device_info();
  if (di.sms == 0) return PARO_ERR_CUDA;
  if (count < 1 || count > kRcMaxMembers) return PARO_ERR_UNSUPPORTED;
  const int64_t groups = K / kGroup, tiles = (M + 127) / 128;
  RbBatch rb;
  std::memset(&rb, 0, sizeof(rb));
  RcBatch rc;
  std::memset(&rc, 0, sizeof(rc));
  int max_krot = 0, nb = 0;
  for (int i = 0; i < count; ++i) {
    if (!mem[i].prebuilt) {      // members without a prepared R' build it now
      rb.op[nb++] = RbOperand{mem[i].cs, mem[i].pairs, mem[i].theta, mem[i].rt, mem[i].krot};
      max_krot = std::max(max_krot, mem[i].krot);
    }
    if (!encode_2d(&rc.t[i].r, tma_dt<TA>(), 2, mem[i].rt, 2 * K, kGroup, 128, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d(&rc.t[i].y, tma_dt<TA>(), 2, mem[i].xr, M, K, 128, 64, CU_TENSOR_MAP_SWIZZLE_128B))
      return PARO_ERR_CUDA;
  }
  if (nb > 0) {
    if (!allow_smem(rmat_build_kernel<TA>, rb_smem_bytes(kMaxKrot))) return PARO_ERR_CUDA;
    if (int st = launch(rmat_build_kernel<TA>, dim3((unsigned)groups, (unsigned)(kGroup / kRbRows), (unsigned)nb),
                        dim3(kRbThreads), rb_smem_bytes(max_krot), stream, true, rb, (int)K, gsz))
      return st;
  }
  CUtensorMap tmX;
  if (!encode_2d(&tmX, tma_dt<TA>(), 2, x, M, K, 128, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return PARO_ERR_CUDA;
  if (!allow_smem(rotate_tc_kernel<TA>, RcLayout::SMEM)) return PARO_ERR_CUDA;
  const int64_t jobs = (int64_t)count * groups * tiles;
  const int64_t ctas = jobs < di.sms ? jobs : di.sms;
  return launch(rotate_tc_kernel<TA>, dim3((unsigned)ctas), dim3(kRcThreads), RcLayout::SMEM, stream, true, tmX,
                rc, count, (int)K, (int)groups, (int)tiles, (long long)jobs, RcQuant{});
}

// Weight quantiser on the tensor cores: R'' = diag(1 / cs) G_0 ... G_{krot-1}
// per group (the build kernel with inverted scales) into the workspace, then
// W_r = W R'' with the quantising epilogue (codes and AWQ words straight from
// the fp32 accumulators).  fp16 weights only: R'' in two fp16 parts keeps
// W_r to about 2^-22 relative, within the fp32 rounding the codes are judged
// by; bf16 parts would keep only 2^-16.
int launch_quantize_tc(const __half* w, const float* cs, const int16_t* pairs, const float* theta,
                       const __half* scales, int32_t* qweight, int32_t* qzeros, int64_t N, int64_t K, int gsz,
                       int krot, void* rt, cudaStream_t s) {
  const DeviceInfo& di = device_info();
  if (di.sms == 0) return PARO_ERR_CUDA;
  const int64_t groups = K / kGroup, tiles = (N + 127) / 128;
  RbBatch rb;
  std::memset(&rb, 0, sizeof(rb));
  rb.op[0] = RbOperand{cs, pairs, theta, rt, krot};
  if (!allow_smem(rmat_build_kernel<__half, true, true>, rb_smem_bytes(kMaxKrot))) return PARO_ERR_CUDA;
  if (int st = launch(rmat_build_kernel<__half, true, true>, dim3((unsigned)groups, (unsigned)(kGroup / kRbRows), 1),
                      dim3(kRbThreads), rb_smem_bytes(krot), s, true, rb, (int)K, gsz))
    return st;
  RcBatch rc;
  std::memset(&rc, 0, sizeof(rc));
  CUtensorMap tmX;
  if (!encode_2d(&rc.t[0].r, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, rt, 2 * K, kGroup, 128, 64,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&rc.t[0].y, CU_TENSOR_MAP_DATA_TYPE_INT32, 4, qweight, K, N / 8, kRcQuantCols, 4,
                 CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, w, N, K, 128, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return PARO_ERR_CUDA;
  auto k = rotate_tc_kernel<__half, true>;
  if (!allow_smem(k, RcLayout::SMEM)) return PARO_ERR_CUDA;
  const int64_t jobs = groups * tiles;
  const int64_t ctas = jobs < di.sms ? jobs : di.sms;
  return launch(k, dim3((unsigned)ctas), dim3(rc_threads<true>()), RcLayout::SMEM, s, true, tmX, rc, 1, (int)K,
                (int)groups, (int)tiles, (long long)jobs, RcQuant{scales, qzeros, (int)N, gsz});
}

// ---------------------------------------------------------------- linear plan
struct LinearPlan {
  bool decode = false;
  int nt = 1;              // decode: 8-token MMA tiles per CTA
  int n_tiles = 0;         // decode column tiles
  int splits = 1;          // decode split-K factor = cluster size along K
  int variant = 0;         // decode kernel configuration (tile, k-parts, stages)
  bool rot_tc = false;     // the rotation runs on the tensor cores (R' in the workspace)
  int gsz = kGroup;        // group size (rotation and quantisation)
  size_t off_xr = 0, off_rt = 0, total = 0;
};

int check_linear_shape(int64_t M, int64_t K, int64_t N, int group_size) {
  if (M < 0 || K <= 0 || N <= 0) return PARO_ERR_INVALID_ARG;
  int G = 0;
  if (int st = normalize_group(group_size, K, &G)) return st;
  if (N % 8 != 0) return PARO_ERR_INVALID_ARG;
  if (!supported_group(G, K) || N % 32 != 0) return PARO_ERR_UNSUPPORTED;
  if (M * K >= (int64_t(1) << 31) || M * N >= (int64_t(1) << 31) || K * N >= (int64_t(1) << 34) ||
      M > (int64_t(1) << 22))
    return PARO_ERR_UNSUPPORTED;
  return PARO_OK;
}

// Shared memory of a decode GEMV configuration (variant, token tiles) for
// `gmax` 128-row groups and `gr` quantisation-group rows per CTA.
size_t gemv_layout_bytes(int variant, int nt, int gmax, int gr) {
  const bool one = nt == 1;
  switch (variant) {
    case 0: return one ? GemvLayout<1, 2, 256, 4>::smem(gmax, gr) : GemvLayout<2, 2, 256, 4>::smem(gmax, gr);
    case 6: return one ? GemvLayout<1, 2, 256, 2>::smem(gmax, gr) : 0;
    case 2: return one ? GemvLayout<1, 4, 128, 8>::smem(gmax, gr) : GemvLayout<2, 4, 128, 8>::smem(gmax, gr);
    case 5: return one ? GemvLayout<1, 4, 64, 8>::smem(gmax, gr) : GemvLayout<2, 4, 64, 8>::smem(gmax, gr);
    default: return one ? GemvLayout<1, 2, 128, 4>::smem(gmax, gr) : GemvLayout<2, 2, 128, 4>::smem(gmax, gr);
  }
}
constexpr size_t kSmemPerCta = 227 * 1024;   // dynamic shared memory a CTA may use (sm_100)

// The split is a function of the shape only (not of the device), so the
// workspace size query and the call agree everywhere.
LinearPlan make_plan(int64_t M, int64_t K, int64_t N, int gsz) {
  LinearPlan p;
  p.gsz = gsz;
  const int groups = (int)(K / kGroup);
  p.decode = M <= kMaxDecodeM;
  p.off_xr = 0;
  p.total = round_up((size_t)M * K * 2, 256);   // X_r, written when rotating
  if (M >= kRotTcMinM) {                          // R' parts: fp16 [2][K][128]
    p.rot_tc = true;
    p.off_rt = p.total;
    p.total += (size_t)K * kGroup * 2 * 2;
  }
  if (p.decode) {
    p.nt = M <= 8 ? 1 : 2;
    // Configuration by shape class, from sweeps on B200 over the Llama-3-8B
    // decode shapes (column tile, k-parts, stages, split along K):
    //   wide (N > 4096, e.g. gate/up):      256 columns, 2 k-parts, 4-stage ring, split 4 for
    //                                        M <= 4 (two CTAs on most SMs: gate 10.2 -> 9.8 us at
    //                                        M = 1), split 2 above (M = 8: split 4 is 4 % slower)
    //   deep (N <= 4096, K > 4096, down):   128 columns, 2 k-parts, 4-stage ring, split 8
    //   square/narrow (q, o, k, v), M <= 8: 128 columns, 4 k-parts, 8 stages, split 4 (8 if N <= 2048)
    //   square, 8 < M <= 16:                64 columns, 4 k-parts, 8 stages, split 2
    //   narrow (N <= 2048), 8 < M <= 16:    128 columns, 2 k-parts, 4 stages, split 8
    // Grouped wide members (gate + up) at M <= 8 take a 2-stage variant of the
    // wide plan in group_plan, so the pair fits one wave.
    int tile, want;
    if (N > 4096) {
      tile = 256; p.variant = 0; want = M <= 4 ? 4 : 2;
    } else if (K > 4096) {
      tile = 128; p.variant = 3; want = 8;
    } else if (M <= 8) {
      tile = 128; p.variant = 2; want = N <= 2048 ? 8 : 4;
    } else if (N <= 2048) {
      tile = 128; p.variant = 3; want = 8;
    } else {
      tile = 64; p.variant = 5; want = 2;
    }
    p.n_tiles = (int)((N + tile - 1) / tile);
    int s = 1;
    while (s * 2 <= want && s * 2 <= kMaxSplits && s * 2 <= groups && p.n_tiles * s * 2 <= kDecodeTargetCtas) s *= 2;
    // a CTA holds at most kGvMaxGroups groups of activations and constants,
    // and its layout (with 128 / G rows of scales and zero words per group)
    // must fit the shared memory of one CTA
    const int gq = kGroup / gsz;
    auto bytes = [&](int sp) {
      const int gm = (groups + sp - 1) / sp;
      return gemv_layout_bytes(p.variant, p.nt, gm, gm * gq);
    };
    while (((groups + s - 1) / s > kGvMaxGroups || bytes(s) > kSmemPerCta) && s < kMaxSplits) s *= 2;
    p.splits = s;
    // deeper than the GEMV's reach (K > 16384, or small groups of a very deep
    // K): the tensor-core GEMM serves it
    if ((groups + s - 1) / s > kGvMaxGroups || bytes(s) > kSmemPerCta) p.decode = false;
  }
  return p;
}

// Routing of a stacked-expert launch (segment variants of the GEMV / GEMM).
struct SegRouting {
  const int4* segs;       // {expert, first sorted row, rows}
  const int* count;       // segments written by the routing (device)
  const int* perm;        // sorted row -> output row
  int max_segs;           // grid bound on the segment count
  int experts;            // E: the weight, scale and zero maps cover E stacked experts
};

// One linear of a prefill GEMM launch.
struct PrefillLinear {
  const void* x;          // the activations the GEMM reads (X_r, or x itself)
  void* y;
  int64_t N;
  const int32_t* qweight;
  const int32_t* qzeros;
  const void* scales;
  const void* bias;
};

// Prefill (M > 16): tcgen05 GEMM, 256 token rows x 256 output columns per CTA,
// one launch over the column tiles of `count` (<= NL) linears sharing M and K.
template <int SR, typename TA, int NL, bool SEG = false>
int launch_w4_prefill_nl(const PrefillLinear* lin, int count, int64_t M, int64_t K, int gsz, cudaStream_t s,
                         bool pdl, const SegRouting* seg = nullptr) {
  if (count < 1 || count > NL) return PARO_ERR_UNSUPPORTED;
  TcBatch<NL> b;
  std::memset(&b, 0, sizeof(b));
  int64_t tiles = 0;
  for (int i = 0; i < NL; ++i) {
    TcOperand& o = b.op[i];
    if (i >= count) {
      o.tile_begin = INT_MAX;                   // never selected
      continue;
    }
    const int64_t N = lin[i].N;
    const int64_t E = SEG ? seg->experts : 1;     // stacked experts along the rows
    const bool ok =
        encode_2d(&o.a, tma_dt<TA>(), 2, lin[i].x, M, K, kTcMB * kTcBM, kTcBK, CU_TENSOR_MAP_SWIZZLE_128B) &&
        encode_2d(&o.w, CU_TENSOR_MAP_DATA_TYPE_INT32, 4, lin[i].qweight, E * K, N / 8, kTcBK, kTcBN / 8,
                  CU_TENSOR_MAP_SWIZZLE_128B) &&
        encode_2d(&o.s, tma_dt<TA>(), 2, lin[i].scales, E * (K / gsz), N, SR, kTcBN, CU_TENSOR_MAP_SWIZZLE_NONE) &&
        encode_2d(&o.z, CU_TENSOR_MAP_DATA_TYPE_INT32, 4, lin[i].qzeros, E * (K / gsz), N / 8, SR, kTcBN / 8,
                  CU_TENSOR_MAP_SWIZZLE_NONE) &&
        (SEG || encode_2d(&o.y, tma_dt<TA>(), 2, lin[i].y, M, N, kTcMB * kTcBM, 64, CU_TENSOR_MAP_SWIZZLE_128B));
    if (!ok) return PARO_ERR_CUDA;
    o.bias = lin[i].bias;
    o.n = (int)N;
    o.tile_begin = (int)tiles;
    tiles += (N + kTcBN - 1) / kTcBN;
    if (SEG) {
      o.segs = seg->segs;
      o.seg_count = seg->count;
      o.perm = seg->perm;
      o.yptr = lin[i].y;
    }
  }
  const dim3 grid((unsigned)tiles, SEG ? (unsigned)seg->max_segs
                                       : (unsigned)((M + kTcMB * kTcBM - 1) / (kTcMB * kTcBM)), 1);
  if (tiles > INT_MAX / 2 || grid.y > 65535u) return PARO_ERR_UNSUPPORTED;
  using L = TcLayoutT<SR>;
  auto k = w4_tc_gemm_kernel<SR, TA, NL, SEG>;
  if (!allow_smem(k, L::SMEM)) return PARO_ERR_CUDA;
  return launch(k, grid, dim3(kTcThreads), L::SMEM, s, pdl, b, (int)M, (int)K, gsz);
}

template <int SR, typename TA>
int launch_w4_prefill_sr(const PrefillLinear* lin, int count, int64_t M, int64_t K, int gsz, cudaStream_t s,
                         bool pdl) {
  return count == 1 ? launch_w4_prefill_nl<SR, TA, 1>(lin, count, M, K, gsz, s, pdl)
                    : launch_w4_prefill_nl<SR, TA, kTcMaxLinears>(lin, count, M, K, gsz, s, pdl);
}

// One stacked-expert linear: tiles of the routed rows sorted by expert.
template <typename TA>
int launch_w4_prefill_seg(const PrefillLinear& lin, int64_t M, int64_t K, int gsz, cudaStream_t s,
                          const SegRouting& seg) {
  switch (gsz) {
    case 32: return launch_w4_prefill_nl<2, TA, 1, true>(&lin, 1, M, K, gsz, s, true, &seg);
    case 16: return launch_w4_prefill_nl<4, TA, 1, true>(&lin, 1, M, K, gsz, s, true, &seg);
    default: return launch_w4_prefill_nl<1, TA, 1, true>(&lin, 1, M, K, gsz, s, true, &seg);
  }
}

template <typename TA>
int launch_w4_prefill(const PrefillLinear* lin, int count, int64_t M, int64_t K, int gsz, cudaStream_t s,
                      bool pdl) {
  // scale rows per 64-row k-block: 64 / G groups below G = 64
  switch (gsz) {
    case 32: return launch_w4_prefill_sr<2, TA>(lin, count, M, K, gsz, s, pdl);
    case 16: return launch_w4_prefill_sr<4, TA>(lin, count, M, K, gsz, s, pdl);
    default: return launch_w4_prefill_sr<1, TA>(lin, count, M, K, gsz, s, pdl);
  }
}

// Shared memory a GEMV CTA is launched with: at least what its group range
// needs, padded so that no more than ceil(ctas / SMs) CTAs of the grid fit on
// one SM.  CTAs of one grid packed onto an SM stream slower than the same CTAs
// spread out, while a grid larger than the SM count must still fit in one wave.
// Returns 0 when the device's limits are unknown.
size_t gemv_footprint(size_t need, int64_t ctas) {
  const DeviceInfo& dev = device_info();
  if (dev.sms <= 0 || dev.smem_per_sm == 0 || dev.smem_optin < need) return 0;
  const int64_t per_sm = (ctas + dev.sms - 1) / dev.sms;      // CTAs each SM must hold
  const size_t pad = dev.smem_per_sm / (size_t)(per_sm + 1) + 1;  // one more no longer fits
  const size_t want = pad > dev.smem_reserved_per_block ? pad - dev.smem_reserved_per_block : 0;
  return std::min(dev.smem_optin, std::max(need, want));
}

// One linear of a decode GEMV launch.
struct GemvLinearArgs {
  const void* qweight;
  const void* qzeros;
  const void* scales;
  const void* x;          // the activations the GEMV reads (X_r, or x itself)
  const void* bias;
  void* y;
  int64_t N;
};

// Decode GEMV launch over `count` (<= NL) linears sharing M and K: grid
// (column tiles of every linear, splits), one cluster of `splits` CTAs along K
// per column tile.  With SEG, one stacked-expert linear: grid (segments x
// column tiles, splits), x = the routed rows sorted by expert.
template <int NT, int KP, int NTILE, int STAGES, int NL, typename TA, bool SEG = false>
int launch_gemv(const LinearPlan& plan, const GemvLinearArgs* lin, int count, int64_t M, int64_t K,
                cudaStream_t s, bool pdl, const SegRouting* seg = nullptr) {
  using L = GemvLayout<NT, KP, NTILE, STAGES>;
  const int groups = (int)(K / kGroup);
  const int gmax = (groups + plan.splits - 1) / plan.splits;   // largest group range of a CTA
  const int gq = kGroup / plan.gsz;                             // quantisation groups per 128 rows
  if (gmax > kGvMaxGroups || count < 1 || count > NL) return PARO_ERR_UNSUPPORTED;
  GemvBatch<NL> b;
  std::memset(&b, 0, sizeof(b));
  int64_t tiles = 0;
  for (int i = 0; i < NL; ++i) {
    GemvOperand& o = b.op[i];
    if (i >= count) {
      o.tile_begin = INT_MAX;                   // never selected
      continue;
    }
    const int64_t N = lin[i].N;
    const int64_t E = SEG ? seg->experts : 1;     // stacked experts along the rows
    const bool ok =
        encode_2d(&o.w, CU_TENSOR_MAP_DATA_TYPE_INT32, 4, lin[i].qweight, E * K, N / 8, 128, L::WORDS,
                  L::ROW_BYTES == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                      : (L::ROW_BYTES == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE)) &&
        encode_2d(&o.s, tma_dt<TA>(), 2, lin[i].scales, E * (K / plan.gsz), N,
                  (uint32_t)(gmax * gq), NTILE, CU_TENSOR_MAP_SWIZZLE_NONE) &&
        encode_2d(&o.z, CU_TENSOR_MAP_DATA_TYPE_INT32, 4, lin[i].qzeros, E * (K / plan.gsz), N / 8,
                  (uint32_t)(gmax * gq), L::WORDS, CU_TENSOR_MAP_SWIZZLE_NONE) &&
        encode_x_chunks(&o.x, tma_dt<TA>(), lin[i].x, (uint64_t)M, (uint64_t)K, (uint32_t)L::MP,
                        (uint32_t)(2 * gmax));
    if (!ok) return PARO_ERR_CUDA;
    o.bias = lin[i].bias;
    o.y = lin[i].y;
    o.n = (int)N;
    o.tile_begin = (int)tiles;
    tiles += (N + NTILE - 1) / NTILE;
    if (SEG) {
      o.segs = seg->segs;
      o.seg_count = seg->count;
      o.perm = seg->perm;
      o.seg_tiles = (int)((N + NTILE - 1) / NTILE);
    }
  }
  if (SEG) tiles *= seg->max_segs;
  if (tiles > INT_MAX / 2) return PARO_ERR_UNSUPPORTED;
  // G = 128 takes the kernel with the group layout fixed at compile time
  auto k = plan.gsz == kGroup ? w4_gemv_kernel<NT, KP, NTILE, STAGES, NL, TA, 1, SEG>
                              : w4_gemv_kernel<NT, KP, NTILE, STAGES, NL, TA, 0, SEG>;
  const dim3 grid((unsigned)tiles, (unsigned)plan.splits, 1);
  const size_t smem = gemv_footprint((size_t)L::smem(gmax, gmax * gq), (int64_t)grid.x * grid.y);
  if (smem == 0 || !allow_smem(k, device_info().smem_optin)) return PARO_ERR_CUDA;
  // a grid larger than the SM count places its clusters by load (measured:
  // 256-CTA grids of 8-CTA clusters ran 1-10 % faster; one-per-SM grids did not gain)
  const bool balance = (int64_t)grid.x * grid.y > device_info().sms;
  return launch_ex(k, grid, dim3(L::THREADS), smem, s, pdl, (unsigned)plan.splits, balance, b, (int)M,
                   (int)K, gmax, gq);
}

template <int NT, int NL, typename TA>
int dispatch_gemv_nl(const LinearPlan& plan, const GemvLinearArgs* lin, int count, int64_t M, int64_t K,
                     cudaStream_t s, bool pdl) {
  switch (plan.variant) {
    case 0: return launch_gemv<NT, 2, 256, 4, NL, TA>(plan, lin, count, M, K, s, pdl);
    case 2: return launch_gemv<NT, 4, 128, 8, NL, TA>(plan, lin, count, M, K, s, pdl);
    case 5: return launch_gemv<NT, 4, 64, 8, NL, TA>(plan, lin, count, M, K, s, pdl);
    case 6:   // grouped wide members in one wave (group_plan): 2-stage ring
      if constexpr (NT == 1 && NL > 1) return launch_gemv<NT, 2, 256, 2, NL, TA>(plan, lin, count, M, K, s, pdl);
      return PARO_ERR_UNSUPPORTED;
    default: return launch_gemv<NT, 2, 128, 4, NL, TA>(plan, lin, count, M, K, s, pdl);
  }
}

// One stacked-expert linear, segments of one token tile.
template <typename TA>
int dispatch_gemv_seg(const LinearPlan& plan, const GemvLinearArgs& lin, int64_t M, int64_t K, cudaStream_t s,
                      const SegRouting& seg) {
  if (plan.nt != 1) return PARO_ERR_UNSUPPORTED;
  switch (plan.variant) {
    case 0: return launch_gemv<1, 2, 256, 4, 1, TA, true>(plan, &lin, 1, M, K, s, true, &seg);
    case 2: return launch_gemv<1, 4, 128, 8, 1, TA, true>(plan, &lin, 1, M, K, s, true, &seg);
    case 5: return launch_gemv<1, 4, 64, 8, 1, TA, true>(plan, &lin, 1, M, K, s, true, &seg);
    default: return launch_gemv<1, 2, 128, 4, 1, TA, true>(plan, &lin, 1, M, K, s, true, &seg);
  }
}

template <typename TA>
int dispatch_gemv(const LinearPlan& plan, const GemvLinearArgs* lin, int count, int64_t M, int64_t K,
                  cudaStream_t s, bool pdl) {
  if (count == 1)
    return plan.nt == 1 ? dispatch_gemv_nl<1, 1, TA>(plan, lin, count, M, K, s, pdl)
                        : dispatch_gemv_nl<2, 1, TA>(plan, lin, count, M, K, s, pdl);
  return plan.nt == 1 ? dispatch_gemv_nl<1, kGvMaxLinears, TA>(plan, lin, count, M, K, s, pdl)
                      : dispatch_gemv_nl<2, kGvMaxLinears, TA>(plan, lin, count, M, K, s, pdl);
}

}  // namespace

// =================================================================== entry bodies
// The entry points below are these bodies for one activation type: fp16 for
// the plain names, fp16 or bf16 by `dtype` for the *_dt names.
namespace {
template <typename TA>
int rotate_impl(const void* x, void* x_r, int64_t M, int64_t K, const float* channel_scales,
                const int16_t* pairs, const float* theta, int group_size, int krot, cudaStream_t s) {
  if (int st = check_rotation_args(x, x_r, M, K, channel_scales, pairs, theta, group_size, krot))
    return st;
  if (M == 0) return PARO_OK;
  return launch_rotate<TA>(static_cast<const TA*>(x), static_cast<TA*>(x_r), M, K, channel_scales, pairs, theta,
                           krot, group_of(group_size, K), s);
}

template <typename TA>
int quantize_impl(const void* w, const float* channel_scales, const int16_t* pairs, const float* theta,
                  const void* scales, int32_t* qweight, int32_t* qzeros, int64_t N, int64_t K, int group_size,
                  int krot, cudaStream_t s) {
  if (N < 0 || K <= 0 || krot < 0 || N % 8 != 0) return PARO_ERR_INVALID_ARG;
  int G = 0;
  if (int st = normalize_group(group_size, K, &G)) return st;
  if (!supported_group(G, K) || krot > kMaxKrot) return PARO_ERR_UNSUPPORTED;
  if (N == 0) return PARO_OK;   // nothing to touch: NULL data pointers are fine
  if (w == nullptr || scales == nullptr || qweight == nullptr || qzeros == nullptr) return PARO_ERR_INVALID_ARG;
  if (krot > 0 && (pairs == nullptr || theta == nullptr)) return PARO_ERR_INVALID_ARG;
  if (N * K >= (int64_t(1) << 31)) return PARO_ERR_UNSUPPORTED;
  if (!aligned(w, 16) || !aligned(scales, 2) || !aligned(qweight, 4) || !aligned(qzeros, 4))
    return PARO_ERR_ALIGNMENT;
  if (channel_scales != nullptr && !aligned(channel_scales, 4)) return PARO_ERR_ALIGNMENT;
  if (krot > 0 && (!aligned(pairs, 4) || !aligned(theta, 4))) return PARO_ERR_ALIGNMENT;
  const RtQuant qo{scales, qweight, qzeros};
  return launch_rotate_tmem<true, TA>(static_cast<const TA*>(w), nullptr, N, K, channel_scales, pairs, theta,
                                      krot, G, qo, s);
}
}  // namespace

// =================================================================== C ABI
extern "C" {

const char* paro_status_string(int status) {
  switch (status) {
    case PARO_OK: return "ok";
    case PARO_ERR_INVALID_ARG: return "invalid argument";
    case PARO_ERR_UNSUPPORTED: return "unsupported configuration";
    case PARO_ERR_ALIGNMENT: return "misaligned pointer";
    case PARO_ERR_WORKSPACE: return "workspace missing or too small";
    case PARO_ERR_CUDA: return "CUDA error";
    case PARO_ERR_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
  }
}

const char* paro_version(void) { return "0.1.0"; }

int paro_rotate(const void* x, void* x_r, int64_t M, int64_t K, const float* channel_scales,
                const int16_t* pairs, const float* theta, int group_size, int krot,
                paro_stream_t stream) {
  return paro_rotate_dt(x, x_r, M, K, channel_scales, pairs, theta, group_size, krot, PARO_DTYPE_F16, stream);
}

int paro_rotate_dt(const void* x, void* x_r, int64_t M, int64_t K, const float* channel_scales,
                   const int16_t* pairs, const float* theta, int group_size, int krot, int dtype,
                   paro_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (dtype) {
    case PARO_DTYPE_F16:
      return rotate_impl<__half>(x, x_r, M, K, channel_scales, pairs, theta, group_size, krot, s);
    case PARO_DTYPE_BF16:
      return rotate_impl<__nv_bfloat16>(x, x_r, M, K, channel_scales, pairs, theta, group_size, krot, s);
    default: return PARO_ERR_INVALID_ARG;
  }
}

int paro_rotate_rmat(const void* x, void* x_r, int64_t M, int64_t K, const void* rmat, int dtype,
                     paro_stream_t stream) {
  if (dtype != PARO_DTYPE_F16 && dtype != PARO_DTYPE_BF16) return PARO_ERR_INVALID_ARG;
  if (M < 0 || K <= 0) return PARO_ERR_INVALID_ARG;
  if (K % kGroup != 0 || K >= (int64_t(1) << 24) || M * K >= (int64_t(1) << 31)) return PARO_ERR_UNSUPPORTED;
  if (M == 0) return PARO_OK;
  if (x == nullptr || x_r == nullptr || rmat == nullptr) return PARO_ERR_INVALID_ARG;
  if (x == x_r) return PARO_ERR_INVALID_ARG;      // tiles are read and written by different stages of one pass
  if (!aligned(x, 16) || !aligned(x_r, 16) || !aligned(rmat, 256)) return PARO_ERR_ALIGNMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const RotTcMember one{nullptr, nullptr, nullptr, 0, x_r, const_cast<void*>(rmat), true};
  if (dtype == PARO_DTYPE_F16) return launch_rotate_tc<__half>(static_cast<const __half*>(x), &one, 1, M, K, kGroup, s);
  return launch_rotate_tc<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(x), &one, 1, M, K, kGroup, s);
}

int paro_quantize_w4(const void* w, const float* channel_scales, const int16_t* pairs,
                     const float* theta, const void* scales, int32_t* qweight, int32_t* qzeros,
                     int64_t N, int64_t K, int group_size, int krot, paro_stream_t stream) {
  return paro_quantize_w4_dt(w, channel_scales, pairs, theta, scales, qweight, qzeros, N, K, group_size, krot,
                             PARO_DTYPE_F16, stream);
}

int paro_quantize_w4_dt(const void* w, const float* channel_scales, const int16_t* pairs,
                        const float* theta, const void* scales, int32_t* qweight, int32_t* qzeros,
                        int64_t N, int64_t K, int group_size, int krot, int dtype, paro_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (dtype) {
    case PARO_DTYPE_F16:
      return quantize_impl<__half>(w, channel_scales, pairs, theta, scales, qweight, qzeros, N, K, group_size,
                                   krot, s);
    case PARO_DTYPE_BF16:
      return quantize_impl<__nv_bfloat16>(w, channel_scales, pairs, theta, scales, qweight, qzeros, N, K,
                                          group_size, krot, s);
    default: return PARO_ERR_INVALID_ARG;
  }
}

size_t paro_quantize_w4_workspace_size(int64_t K) {
  if (K <= 0 || K % kGroup != 0 || K >= (int64_t(1) << 24)) return 0;
  return (size_t)K * kGroup * 2 * 2;
}

int paro_quantize_w4_tc(const void* w, const float* channel_scales, const int16_t* pairs, const float* theta,
                        const void* scales, int32_t* qweight, int32_t* qzeros, int64_t N, int64_t K,
                        int group_size, int krot, void* workspace, size_t workspace_bytes, paro_stream_t stream) {
  if (N < 0 || K <= 0 || krot < 0 || N % 8 != 0) return PARO_ERR_INVALID_ARG;
  int G = 0;
  if (int st = normalize_group(group_size, K, &G)) return st;
  if (!supported_group(G, K) || krot > kMaxKrot || N % 32 != 0 || K >= (int64_t(1) << 24))
    return PARO_ERR_UNSUPPORTED;
  if (N == 0) return PARO_OK;   // nothing to touch: NULL data pointers are fine
  if (w == nullptr || scales == nullptr || qweight == nullptr || qzeros == nullptr || workspace == nullptr)
    return PARO_ERR_INVALID_ARG;
  if (krot > 0 && (pairs == nullptr || theta == nullptr)) return PARO_ERR_INVALID_ARG;
  if (N * K >= (int64_t(1) << 31)) return PARO_ERR_UNSUPPORTED;
  if (workspace_bytes < paro_quantize_w4_workspace_size(K)) return PARO_ERR_WORKSPACE;
  if (!aligned(w, 16) || !aligned(scales, 2) || !aligned(qweight, 16) || !aligned(qzeros, 4) ||
      !aligned(workspace, 256))
    return PARO_ERR_ALIGNMENT;
  if (channel_scales != nullptr && !aligned(channel_scales, 4)) return PARO_ERR_ALIGNMENT;
  if (krot > 0 && (!aligned(pairs, 4) || !aligned(theta, 4))) return PARO_ERR_ALIGNMENT;
  return launch_quantize_tc(static_cast<const __half*>(w), channel_scales, pairs, theta,
                            static_cast<const __half*>(scales), qweight, qzeros, N, K, G, krot, workspace,
                            reinterpret_cast<cudaStream_t>(stream));
}

int paro_pack_awq(const uint8_t* codes, const uint8_t* zero_codes, int32_t* qweight,
                  int32_t* qzeros, int64_t N, int64_t K, int group_size, paro_stream_t stream) {
  if (N <= 0 || K <= 0 || N % 8 != 0) return PARO_ERR_INVALID_ARG;
  int G = 0;
  if (int st = normalize_group(group_size, K, &G)) return st;
  if (codes == nullptr || qweight == nullptr) return PARO_ERR_INVALID_ARG;
  if ((zero_codes == nullptr) != (qzeros == nullptr)) return PARO_ERR_INVALID_ARG;
  if (N / 8 > 65535) return PARO_ERR_UNSUPPORTED;
  if (!aligned(qweight, 4) || (qzeros != nullptr && !aligned(qzeros, 4))) return PARO_ERR_ALIGNMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (int st = launch(pack_rows_kernel, dim3((unsigned)((K + 255) / 256), (unsigned)(N / 8)),
                      dim3(256), 0, s, false, codes, qweight, N, K))
    return st;
  if (qzeros != nullptr) {
    const int64_t R = K / G;
    return launch(pack_rows_kernel, dim3((unsigned)((R + 255) / 256), (unsigned)(N / 8)),
                  dim3(256), 0, s, false, zero_codes, qzeros, N, R);
  }
  return PARO_OK;
}

int paro_unpack_awq(const int32_t* qweight, const int32_t* qzeros, uint8_t* codes,
                    uint8_t* zero_codes, int64_t N, int64_t K, int group_size,
                    paro_stream_t stream) {
  if (N <= 0 || K <= 0 || N % 8 != 0) return PARO_ERR_INVALID_ARG;
  int G = 0;
  if (int st = normalize_group(group_size, K, &G)) return st;
  if (codes == nullptr || qweight == nullptr) return PARO_ERR_INVALID_ARG;
  if ((zero_codes == nullptr) != (qzeros == nullptr)) return PARO_ERR_INVALID_ARG;
  if (N / 8 > 65535) return PARO_ERR_UNSUPPORTED;
  if (!aligned(qweight, 4) || (qzeros != nullptr && !aligned(qzeros, 4))) return PARO_ERR_ALIGNMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (int st = launch(unpack_rows_kernel, dim3((unsigned)((K + 255) / 256), (unsigned)(N / 8)),
                      dim3(256), 0, s, false, qweight, codes, N, K))
    return st;
  if (qzeros != nullptr) {
    const int64_t R = K / G;
    return launch(unpack_rows_kernel, dim3((unsigned)((R + 255) / 256), (unsigned)(N / 8)),
                  dim3(256), 0, s, false, qzeros, zero_codes, N, R);
  }
  return PARO_OK;
}

size_t paro_w4_linear_workspace_size(int64_t M, int64_t K, int64_t N, int group_size) {
  if (check_linear_shape(M, K, N, group_size) != PARO_OK) return 0;
  return make_plan(M, K, N, group_of(group_size, K)).total;
}

size_t paro_rotation_matrix_size(int64_t K) {
  if (K <= 0 || K % kGroup != 0 || K >= (int64_t(1) << 24)) return 0;
  return (size_t)K * kGroup * 2 * 2;
}

int paro_rotation_matrix_prepare(const float* channel_scales, const int16_t* pairs, const float* theta,
                                 int64_t K, int group_size, int krot, int dtype, void* rmat, size_t rmat_bytes,
                                 paro_stream_t stream) {
  if (dtype != PARO_DTYPE_F16 && dtype != PARO_DTYPE_BF16) return PARO_ERR_INVALID_ARG;
  if (K <= 0 || krot < 0) return PARO_ERR_INVALID_ARG;
  int G = 0;
  if (int st = normalize_group(group_size, K, &G)) return st;
  if (!supported_group(G, K) || krot > kMaxKrot || K >= (int64_t(1) << 24)) return PARO_ERR_UNSUPPORTED;
  if (rmat == nullptr || (krot > 0 && (pairs == nullptr || theta == nullptr))) return PARO_ERR_INVALID_ARG;
  if (rmat_bytes < paro_rotation_matrix_size(K)) return PARO_ERR_WORKSPACE;
  if (!aligned(rmat, 256) || (channel_scales != nullptr && !aligned(channel_scales, 4)) ||
      (krot > 0 && (!aligned(pairs, 4) || !aligned(theta, 4))))
    return PARO_ERR_ALIGNMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  RbBatch rb;
  std::memset(&rb, 0, sizeof(rb));
  rb.op[0] = RbOperand{channel_scales, pairs, theta, rmat, krot};
  const dim3 grid((unsigned)(K / kGroup), (unsigned)(kGroup / kRbRows), 1);
  // the build kernel that does not release its dependents early: R' is a
  // layer constant that later calls read before they wait for the kernel ahead
  if (dtype == PARO_DTYPE_F16) {
    if (!allow_smem(rmat_build_kernel<__half, false>, rb_smem_bytes(kMaxKrot))) return PARO_ERR_CUDA;
    return launch(rmat_build_kernel<__half, false>, grid, dim3(kRbThreads), rb_smem_bytes(krot), s, false, rb,
                  (int)K, G);
  }
  if (!allow_smem(rmat_build_kernel<__nv_bfloat16, false>, rb_smem_bytes(kMaxKrot))) return PARO_ERR_CUDA;
  return launch(rmat_build_kernel<__nv_bfloat16, false>, grid, dim3(kRbThreads), rb_smem_bytes(krot), s, false, rb,
                (int)K, G);
}

}  // extern "C"

namespace {
// Every check of paro_w4_linear that does not involve the workspace.
int check_linear_args(const void* x, const void* y, int64_t M, int64_t K, int64_t N, const int32_t* qweight,
                      const int32_t* qzeros, const void* scales, const void* bias, const float* channel_scales,
                      const int16_t* pairs, const float* theta, int group_size, int krot) {
  if (int st = check_linear_shape(M, K, N, group_size)) return st;
  if (krot < 0) return PARO_ERR_INVALID_ARG;
  if (krot > kMaxKrot) return PARO_ERR_UNSUPPORTED;
  if (M == 0) return PARO_OK;   // empty batch: nothing to read or write
  if (x == nullptr || y == nullptr || qweight == nullptr || qzeros == nullptr || scales == nullptr)
    return PARO_ERR_INVALID_ARG;
  if (krot > 0 && (pairs == nullptr || theta == nullptr)) return PARO_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(y, 16) || !aligned(qweight, 16) || !aligned(qzeros, 16) ||
      !aligned(scales, 16) || (bias != nullptr && !aligned(bias, 4)))
    return PARO_ERR_ALIGNMENT;
  if (channel_scales != nullptr && !aligned(channel_scales, 16)) return PARO_ERR_ALIGNMENT;
  if (krot > 0 && (!aligned(pairs, 4) || !aligned(theta, 4))) return PARO_ERR_ALIGNMENT;
  return PARO_OK;
}

// Shared memory of the GEMV layout of a plan, for `gmax` groups per CTA.
size_t gemv_smem(const LinearPlan& p, int gmax) {
  return gemv_layout_bytes(p.variant, p.nt, gmax, gmax * (kGroup / p.gsz));
}

int plan_tile(const LinearPlan& p) { return p.variant == 0 || p.variant == 6 ? 256 : (p.variant == 5 ? 64 : 128); }

// Whether a decode GEMV grid of `ctas` CTAs with plan p is resident at once
// (false when the device's limits are unknown).
bool gemv_one_wave(const LinearPlan& p, int64_t K, int64_t ctas) {
  const DeviceInfo& dev = device_info();
  if (dev.sms <= 0) return false;
  const int groups = (int)(K / kGroup);
  const int gmax = (groups + p.splits - 1) / p.splits;
  if (gmax > kGvMaxGroups) return false;
  const size_t need = gemv_smem(p, gmax);
  if (need == 0 || need > kSmemPerCta) return false;
  const size_t fp = gemv_footprint(need, ctas);
  if (fp == 0) return false;
  const int64_t per_sm = (int64_t)(dev.smem_per_sm / (fp + dev.smem_reserved_per_block));
  return ctas <= per_sm * dev.sms;
}

// A wide plan (256 columns, 4-stage ring) whose grid of `units` x splits CTAs
// is not resident at once: the 2-stage ring (one stage per k-part) puts two
// CTAs on an SM, at the same split or at half of it.  Returns whether *p (as
// possibly changed) fits one wave.
bool wide_one_wave(LinearPlan* p, int64_t K, int64_t units) {
  if (gemv_one_wave(*p, K, units * p->splits)) return true;
  if (p->variant != 0 || p->nt != 1) return false;
  for (int sp = p->splits; sp >= 1 && 2 * sp >= p->splits; sp /= 2) {
    LinearPlan q = *p;
    q.variant = 6;
    q.splits = sp;
    if (gemv_one_wave(q, K, units * sp)) {
      *p = q;
      return true;
    }
  }
  return false;
}

// One GEMV launch for a group of decode linears sharing x: the plan of the
// widest member for all of them, taken only when the whole grid is resident
// at once with that plan's footprint (larger groups gain nothing from sharing
// a launch: each member already fills the GPU).
bool group_plan(int64_t M, int64_t K, const paro_linear* lin, int count, int gsz, LinearPlan* out) {
  int64_t widest = 0;
  for (int i = 0; i < count; ++i) widest = std::max(widest, lin[i].N);
  LinearPlan p = make_plan(M, K, widest, gsz);
  if (!p.decode) return false;
  // (variant 6 keeps 256-column tiles, so the tile count does not change)
  const int tile = plan_tile(p);
  int64_t tiles = 0;
  for (int i = 0; i < count; ++i) tiles += (lin[i].N + tile - 1) / tile;
  // wide members (gate and up, say) at up to 8 tokens share one launch on
  // the 2-stage ring
  if (!wide_one_wave(&p, K, tiles)) return false;
  p.n_tiles = (int)tiles;
  *out = p;
  return true;
}

template <typename TA>
// rmat: this linear's prepared R' parts (paro_rotation_matrix_prepare) or nullptr.
int linear_impl(const void* x, void* y, int64_t M, int64_t K, int64_t N, const int32_t* qweight,
                const int32_t* qzeros, const void* scales, const void* bias, const float* channel_scales,
                const int16_t* pairs, const float* theta, int group_size, int krot, void* workspace,
                size_t workspace_bytes, cudaStream_t s, const void* rmat = nullptr) {
  if (int st = check_linear_args(x, y, M, K, N, qweight, qzeros, scales, bias, channel_scales, pairs, theta,
                                 group_size, krot))
    return st;
  if (rmat != nullptr && !aligned(rmat, 256)) return PARO_ERR_ALIGNMENT;
  if (M == 0) return PARO_OK;   // empty batch: nothing to read or write

  const int G = group_of(group_size, K);
  const LinearPlan plan = make_plan(M, K, N, G);

  const bool rotate = krot > 0 || channel_scales != nullptr;
  if (rotate && (workspace == nullptr || workspace_bytes < plan.total)) return PARO_ERR_WORKSPACE;
  if (rotate && !aligned(workspace, 256)) return PARO_ERR_ALIGNMENT;
  const TA* xa = static_cast<const TA*>(x);
  // Programmatic dependent launch throughout: the GEMV/GEMM requests weights,
  // scales and zero points before it waits for the kernel ahead of it (the
  // rotation, or whatever preceded the call), and reads activations after.
  const bool pdl = true;
  if (rotate) {
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    TA* xr = reinterpret_cast<TA*>(ws + plan.off_xr);
    if (plan.rot_tc) {
      const bool pre = rmat != nullptr;
      const RotTcMember one{channel_scales, pairs, theta, krot, xr,
                            pre ? const_cast<void*>(rmat) : static_cast<void*>(ws + plan.off_rt), pre};
      if (int st = launch_rotate_tc<TA>(xa, &one, 1, M, K, G, s)) return st;
    } else if (int st = launch_rotate<TA>(xa, xr, M, K, channel_scales, pairs, theta, krot, G, s)) {
      return st;
    }
    xa = xr;
  }

  if (!plan.decode) {
    const PrefillLinear one{xa, y, N, qweight, qzeros, scales, bias};
    return launch_w4_prefill<TA>(&one, 1, M, K, G, s, pdl);
  }

  const GemvLinearArgs one{qweight, qzeros, scales, xa, bias, y, N};
  return dispatch_gemv<TA>(plan, &one, 1, M, K, s, pdl);
}
}  // namespace

extern "C" {

int paro_w4_linear(const void* x, void* y, int64_t M, int64_t K, int64_t N,
                   const int32_t* qweight, const int32_t* qzeros, const void* scales,
                   const void* bias, const float* channel_scales, const int16_t* pairs,
                   const float* theta, int group_size, int krot, void* workspace,
                   size_t workspace_bytes, paro_stream_t stream) {
  return paro_w4_linear_dt(x, y, M, K, N, qweight, qzeros, scales, bias, channel_scales, pairs, theta, group_size,
                           krot, PARO_DTYPE_F16, workspace, workspace_bytes, stream);
}

int paro_w4_linear_dt(const void* x, void* y, int64_t M, int64_t K, int64_t N,
                      const int32_t* qweight, const int32_t* qzeros, const void* scales,
                      const void* bias, const float* channel_scales, const int16_t* pairs,
                      const float* theta, int group_size, int krot, int dtype, void* workspace,
                      size_t workspace_bytes, paro_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (dtype) {
    case PARO_DTYPE_F16:
      return linear_impl<__half>(x, y, M, K, N, qweight, qzeros, scales, bias, channel_scales, pairs, theta,
                                 group_size, krot, workspace, workspace_bytes, s);
    case PARO_DTYPE_BF16:
      return linear_impl<__nv_bfloat16>(x, y, M, K, N, qweight, qzeros, scales, bias, channel_scales, pairs,
                                        theta, group_size, krot, workspace, workspace_bytes, s);
    default: return PARO_ERR_INVALID_ARG;
  }
}

static_assert(PARO_MAX_GROUP == kGvMaxLinears && PARO_MAX_GROUP == kRrMaxLinears && PARO_MAX_GROUP == kRcMaxMembers &&
                  PARO_MAX_GROUP == kTcMaxLinears,
              "one launch holds every member of a group");

}  // extern "C"

namespace {
bool rotates(const paro_linear& l) { return l.krot > 0 || l.channel_scales != nullptr; }

// The member whose X_r member i reads: the first member with the same rotation
// (same krot and the same channel_scales, pairs and theta tensors — experts
// that share one rotation rotate x once), or -1 when member i does not rotate.
int rotation_owner(const paro_linear* l, int i) {
  if (!rotates(l[i])) return -1;
  for (int j = 0; j < i; ++j)
    if (rotates(l[j]) && l[j].krot == l[i].krot && l[j].channel_scales == l[i].channel_scales &&
        (l[i].krot == 0 || (l[j].pairs == l[i].pairs && l[j].theta == l[i].theta)))
      return j;
  return i;
}
}  // namespace

extern "C" {

size_t paro_w4_linear_group_workspace_size(int64_t M, int64_t K, int count, const paro_linear* linears,
                                           int group_size) {
  if (count < 1 || count > PARO_MAX_GROUP || linears == nullptr) return 0;
  size_t total = 0;
  for (int i = 0; i < count; ++i) {
    if (check_linear_shape(M, K, linears[i].N, group_size) != PARO_OK) return 0;
    total += make_plan(M, K, linears[i].N, group_of(group_size, K)).total;
  }
  return total;
}

int paro_w4_linear_group_launches(int64_t M, int64_t K, int count, const paro_linear* linears,
                                  int group_size) {
  if (count < 1 || count > PARO_MAX_GROUP || linears == nullptr) return 0;
  int rot = 0;
  bool rows_ok = M <= 16;
  for (int i = 0; i < count; ++i) {
    if (check_linear_shape(M, K, linears[i].N, group_size) != PARO_OK || linears[i].krot < 0 ||
        linears[i].krot > kMaxKrot)
      return 0;
    if (rotation_owner(linears, i) == i) {       // one rotation per distinct set of tables
      ++rot;
      rows_ok = rows_ok && linears[i].krot <= kRrMaxKrot;
    }
  }
  if (M == 0) return 0;
  // prefill batches rotating on the tensor cores: one R' build and one X R'
  // launch for all rotating members, then one GEMM each
  const int G = group_of(group_size, K);
  const LinearPlan first = make_plan(M, K, linears[0].N, G);
  if (!first.decode) {
    // prefill: one GEMM launch for the whole group.  Above 64 rows one X R'
    // launch for all rotating members, after one R' build for those without
    // a prepared R'; below, a launch per distinct rotation.
    if (!first.rot_tc) return rot + 1;
    bool build = false;
    for (int i = 0; i < count; ++i) build = build || (rotation_owner(linears, i) == i && linears[i].rmat == nullptr);
    return (rot > 0 ? (build ? 2 : 1) : 0) + 1;
  }
  LinearPlan gp;
  // one GEMV per member: several members still share one warp-per-row
  // rotation launch when every rotation fits it, else each rotates alone
  if (count == 1 || !group_plan(M, K, linears, count, G, &gp))
    return (count > 1 && rows_ok && rot > 0 ? 1 : rot) + count;
  return (rot > 0 ? (rows_ok ? 1 : rot) : 0) + 1;
}

}  // extern "C"

namespace {
template <typename TA>
int group_impl(const void* x, int64_t M, int64_t K, int count, const paro_linear* linears, int group_size,
               void* workspace, size_t workspace_bytes, cudaStream_t s) {
  if (count < 1 || linears == nullptr) return PARO_ERR_INVALID_ARG;
  if (count > PARO_MAX_GROUP) return PARO_ERR_UNSUPPORTED;
  bool any_rotate = false;
  for (int i = 0; i < count; ++i) {
    const paro_linear& l = linears[i];
    if (int st = check_linear_args(x, l.y, M, K, l.N, l.qweight, l.qzeros, l.scales, l.bias, l.channel_scales,
                                   l.pairs, l.theta, group_size, l.krot))
      return st;
    if (l.rmat != nullptr && !aligned(l.rmat, 256)) return PARO_ERR_ALIGNMENT;
    any_rotate = any_rotate || l.krot > 0 || l.channel_scales != nullptr;
  }
  if (M == 0) return PARO_OK;
  const size_t need = paro_w4_linear_group_workspace_size(M, K, count, linears, group_size);
  if (any_rotate && (workspace == nullptr || workspace_bytes < need)) return PARO_ERR_WORKSPACE;
  if (any_rotate && !aligned(workspace, 256)) return PARO_ERR_ALIGNMENT;
  // member i's X_r lives at workspace + i * per (all members share M and K)
  const int G = group_of(group_size, K);
  const size_t per = make_plan(M, K, linears[0].N, G).total;
  unsigned char* ws = static_cast<unsigned char*>(workspace);

  const LinearPlan first = make_plan(M, K, linears[0].N, G);
  if (count > 1 && !first.decode) {
    // prefill: every distinct rotation's X_r, then one GEMM launch over every
    // member's column tiles.  Above 64 rows the rotating members share one
    // R' build (members with a prepared R' skip it) and one X R' launch (x
    // is read once per tile for all of them); below, each distinct rotation
    // is its own launch.
    RotTcMember rm[PARO_MAX_GROUP];
    int nrot = 0;
    const TA* xs[PARO_MAX_GROUP];
    for (int i = 0; i < count; ++i) {
      const paro_linear& l = linears[i];
      const int o = rotation_owner(linears, i);
      xs[i] = static_cast<const TA*>(x);
      if (o < 0) continue;
      TA* xr = reinterpret_cast<TA*>(ws + o * per + first.off_xr);
      if (o == i) {
        if (first.rot_tc) {
          const bool pre = l.rmat != nullptr;
          rm[nrot++] = RotTcMember{l.channel_scales, l.pairs, l.theta, l.krot, xr,
                                   pre ? const_cast<void*>(l.rmat) : static_cast<void*>(ws + i * per + first.off_rt),
                                   pre};
        } else if (int st = launch_rotate<TA>(static_cast<const TA*>(x), xr, M, K, l.channel_scales, l.pairs,
                                              l.theta, l.krot, G, s)) {
          return st;
        }
      }
      xs[i] = xr;
    }
    if (nrot > 0)
      if (int st = launch_rotate_tc<TA>(static_cast<const TA*>(x), rm, nrot, M, K, G, s)) return st;
    PrefillLinear pl[PARO_MAX_GROUP];
    for (int i = 0; i < count; ++i) {
      const paro_linear& l = linears[i];
      pl[i] = PrefillLinear{xs[i], l.y, l.N, l.qweight, l.qzeros, l.scales, l.bias};
    }
    return launch_w4_prefill<TA>(pl, count, M, K, G, s, true);
  }

  LinearPlan gp;
  if (count == 1 || !group_plan(M, K, linears, count, G, &gp)) {
    // Decode members that need a GEMV launch each (the group does not fit one
    // wave) still share one warp-per-row rotation launch for every distinct
    // rotation; each GEMV then reads its rotation's X_r.
    if (count > 1 && M <= 16) {
      RrBatch rb;
      std::memset(&rb, 0, sizeof(rb));
      int nrot = 0, max_krot = 0;
      bool rows_ok = true;
      for (int i = 0; i < count; ++i) {
        const paro_linear& l = linears[i];
        if (rotation_owner(linears, i) != i) continue;
        rows_ok = rows_ok && l.krot <= kRrMaxKrot;
        rb.op[nrot++] = RrOperand{ws + i * per + first.off_xr, l.channel_scales, l.pairs, l.theta, l.krot};
        max_krot = std::max(max_krot, l.krot);
      }
      if (rows_ok && nrot > 0) {
        if (int st = launch_rotate_rows<TA>(static_cast<const TA*>(x), rb, nrot, M, K, max_krot, G, s)) return st;
        for (int i = 0; i < count; ++i) {
          const paro_linear& l = linears[i];
          const int o = rotation_owner(linears, i);
          const void* src = o >= 0 ? static_cast<const void*>(ws + o * per + first.off_xr) : x;
          if (int st = linear_impl<TA>(src, l.y, M, K, l.N, l.qweight, l.qzeros, l.scales, l.bias, nullptr, nullptr,
                                       nullptr, group_size, 0, nullptr, 0, s))
            return st;
        }
        return PARO_OK;
      }
    }
    // one call per member, each with its own slice of the workspace; a member
    // that shares an earlier member's rotation reads that member's X_r
    for (int i = 0; i < count; ++i) {
      const paro_linear& l = linears[i];
      const int o = rotation_owner(linears, i);
      int st;
      if (o >= 0 && o != i)
        st = linear_impl<TA>(ws + o * per + first.off_xr, l.y, M, K, l.N, l.qweight, l.qzeros, l.scales, l.bias,
                             nullptr, nullptr, nullptr, group_size, 0, nullptr, 0, s);
      else
        st = linear_impl<TA>(x, l.y, M, K, l.N, l.qweight, l.qzeros, l.scales, l.bias, l.channel_scales, l.pairs,
                             l.theta, group_size, l.krot, ws ? ws + i * per : nullptr, ws ? per : 0, s, l.rmat);
      if (st) return st;
    }
    return PARO_OK;
  }

  // every member's rotation of x: one warp-per-row launch when all fit it
  const TA* xa = static_cast<const TA*>(x);
  GemvLinearArgs lin[PARO_MAX_GROUP];
  RrBatch rb;
  std::memset(&rb, 0, sizeof(rb));
  int nrot = 0, max_krot = 0;
  bool rows_ok = M <= 16;
  for (int i = 0; i < count; ++i) {
    const paro_linear& l = linears[i];
    const int o = rotation_owner(linears, i);
    TA* xr = o >= 0 ? reinterpret_cast<TA*>(ws + o * per) : nullptr;
    if (o == i) {
      rb.op[nrot++] = RrOperand{xr, l.channel_scales, l.pairs, l.theta, l.krot};
      max_krot = std::max(max_krot, l.krot);
      rows_ok = rows_ok && l.krot <= kRrMaxKrot;
    }
    lin[i] = GemvLinearArgs{l.qweight, l.qzeros, l.scales, o >= 0 ? static_cast<const void*>(xr) : xa, l.bias,
                            l.y, l.N};
  }
  if (nrot > 0) {
    if (rows_ok) {
      if (int st = launch_rotate_rows<TA>(xa, rb, nrot, M, K, max_krot, G, s)) return st;
    } else {
      for (int r = 0; r < nrot; ++r)
        if (int st = launch_rotate<TA>(xa, static_cast<TA*>(rb.op[r].xr), M, K, rb.op[r].cs, rb.op[r].pairs,
                                       rb.op[r].theta, rb.op[r].krot, G, s))
          return st;
    }
  }
  return dispatch_gemv<TA>(gp, lin, count, M, K, s, true);
}
}  // namespace

extern "C" {

int paro_w4_linear_group(const void* x, int64_t M, int64_t K, int count, const paro_linear* linears,
                         int group_size, void* workspace, size_t workspace_bytes, paro_stream_t stream) {
  return paro_w4_linear_group_dt(x, M, K, count, linears, group_size, PARO_DTYPE_F16, workspace, workspace_bytes,
                                 stream);
}

int paro_w4_linear_group_dt(const void* x, int64_t M, int64_t K, int count, const paro_linear* linears,
                            int group_size, int dtype, void* workspace, size_t workspace_bytes,
                            paro_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (dtype) {
    case PARO_DTYPE_F16:
      return group_impl<__half>(x, M, K, count, linears, group_size, workspace, workspace_bytes, s);
    case PARO_DTYPE_BF16:
      return group_impl<__nv_bfloat16>(x, M, K, count, linears, group_size, workspace, workspace_bytes, s);
    default: return PARO_ERR_INVALID_ARG;
  }
}

}  // extern "C"

// ------------------------------------------------------------ stacked experts
namespace {
constexpr int kMoeMaxTopk = 64;
constexpr int kMoeDecodeMaxT = kMaxDecodeM;    // tokens up to which the segment GEMV runs

// Workspace of a stacked-expert call: X_r [T, K] (when rotating), the sorted
// rows Xg [S, K], the routing head, perm [S], decode segments [S] and prefill
// tiles [S] (each segment or tile has at least one row), and above 64 tokens
// the R' parts [2][K][128] of the tensor-core rotation; 256-byte aligned.
struct MoePlan {
  size_t off_xr = 0, off_xg = 0, off_head = 0, off_perm = 0, off_gv = 0, off_tc = 0, off_rt = 0, total = 0;
  bool rot_tc = false;
};
MoePlan moe_plan(int64_t T, int64_t K, int64_t S) {
  MoePlan p;
  p.off_xr = 0;
  p.rot_tc = T >= kRotTcMinM;
  p.off_xg = round_up((size_t)T * K * 2, 256);
  p.off_head = p.off_xg + round_up((size_t)S * K * 2, 256);
  p.off_perm = p.off_head + 256;
  p.off_gv = p.off_perm + round_up((size_t)S * 4, 256);
  p.off_tc = p.off_gv + round_up((size_t)S * 16, 256);
  p.off_rt = p.off_tc + round_up((size_t)S * 16, 256);
  p.total = p.off_rt + (p.rot_tc ? (size_t)K * kGroup * 2 * 2 : 0);
  return p;
}

int check_moe_shape(int64_t T, int64_t K, int64_t N, int E, int topk, int group_size) {
  if (T < 0 || E < 1 || topk < 1) return PARO_ERR_INVALID_ARG;
  if (E > kMoeMaxExperts || topk > kMoeMaxTopk) return PARO_ERR_UNSUPPORTED;
  const int64_t S = T * topk;
  if (int st = check_linear_shape(S, K, N, group_size)) return st;
  // TMA row coordinates of the stacked weights are 32-bit
  if ((int64_t)E * K >= (int64_t(1) << 31) || S >= (int64_t(1) << 24)) return PARO_ERR_UNSUPPORTED;
  return PARO_OK;
}

template <typename TA>
int moe_impl(const void* x, void* y, int64_t T, int64_t K, int64_t N, int E, int topk, const int32_t* expert_idx,
             const int32_t* qweight, const int32_t* qzeros, const void* scales, const void* bias,
             const float* channel_scales, const int16_t* pairs, const float* theta, int group_size, int krot,
             void* workspace, size_t workspace_bytes, cudaStream_t s) {
  if (int st = check_moe_shape(T, K, N, E, topk, group_size)) return st;
  if (krot < 0) return PARO_ERR_INVALID_ARG;
  if (krot > kMaxKrot) return PARO_ERR_UNSUPPORTED;
  if (T == 0) return PARO_OK;
  if (x == nullptr || y == nullptr || expert_idx == nullptr || qweight == nullptr || qzeros == nullptr ||
      scales == nullptr || workspace == nullptr)
    return PARO_ERR_INVALID_ARG;
  if (krot > 0 && (pairs == nullptr || theta == nullptr)) return PARO_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(y, 16) || !aligned(qweight, 16) || !aligned(qzeros, 16) || !aligned(scales, 16) ||
      !aligned(expert_idx, 4) || (bias != nullptr && !aligned(bias, 4)) || !aligned(workspace, 256))
    return PARO_ERR_ALIGNMENT;
  if (channel_scales != nullptr && !aligned(channel_scales, 16)) return PARO_ERR_ALIGNMENT;
  if (krot > 0 && (!aligned(pairs, 4) || !aligned(theta, 4))) return PARO_ERR_ALIGNMENT;
  const int64_t S = T * topk;
  const MoePlan mp = moe_plan(T, K, S);
  if (workspace_bytes < mp.total) return PARO_ERR_WORKSPACE;
  const int G = group_of(group_size, K);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  const TA* xr = static_cast<const TA*>(x);
  // the rotation is shared by every expert: once, on the T tokens (above 64
  // tokens as X R' on the tensor cores, as paro_w4_linear does)
  if (krot > 0 || channel_scales != nullptr) {
    TA* out = reinterpret_cast<TA*>(ws + mp.off_xr);
    if (mp.rot_tc) {
      const RotTcMember one{channel_scales, pairs, theta, krot, out, ws + mp.off_rt, false};
      if (int st = launch_rotate_tc<TA>(static_cast<const TA*>(x), &one, 1, T, K, G, s)) return st;
    } else if (int st = launch_rotate<TA>(static_cast<const TA*>(x), out, T, K, channel_scales, pairs, theta, krot,
                                          G, s)) {
      return st;
    }
    xr = out;
  }
  MoeHead* head = reinterpret_cast<MoeHead*>(ws + mp.off_head);
  int* perm = reinterpret_cast<int*>(ws + mp.off_perm);
  int4* gv = reinterpret_cast<int4*>(ws + mp.off_gv);
  int4* tc = reinterpret_cast<int4*>(ws + mp.off_tc);
  TA* xg = reinterpret_cast<TA*>(ws + mp.off_xg);
  // few routed rows (decode): the route kernel gathers them itself
  const bool route_gathers = (size_t)S * K * 2 <= kMoeRouteGatherBytes;
  if (int st = launch(moe_route_kernel, dim3(1), dim3(kMoeRouteThreads), 0, s, true, expert_idx, (int)S, E, head,
                      perm, gv, tc, y, (int)(N * 2), reinterpret_cast<const uint4*>(xr),
                      route_gathers ? reinterpret_cast<uint4*>(xg) : static_cast<uint4*>(nullptr), (int)(K / 8),
                      topk))
    return st;
  if (!route_gathers)
    if (int st = launch(moe_gather_kernel<TA>, dim3((unsigned)((S + 7) / 8)), dim3(256), 0, s, true,
                        static_cast<const MoeHead*>(head), static_cast<const int*>(perm), xr, xg, (int)K, topk))
      return st;
  const int64_t used = std::min<int64_t>(E, S);   // experts that can hold a row
  if (T <= kMoeDecodeMaxT) {
    // segments of at most 8 rows: one token tile of the decode GEMV each
    const LinearPlan plan = make_plan(kMoeGvRows, K, N, G);
    if (plan.decode) {
      // (the 2-stage ring that puts a grouped gate/up pair in one wave was
      // measured slower here: 1707 vs 2047 GB/s for two gate-shaped experts
      // at one token; the segment GEMV requests no weights before its wait,
      // so the deeper ring matters more than the second wave)
      const int max_segs = (int)std::min<int64_t>(S, S / kMoeGvRows + used);
      const SegRouting seg{gv, &head->n_gv, perm, max_segs, E};
      const GemvLinearArgs lin{qweight, qzeros, scales, xg, bias, y, N};
      return dispatch_gemv_seg<TA>(plan, lin, S, K, s, seg);
    }
  }
  const SegRouting seg{tc, &head->n_tc, perm, (int)std::min<int64_t>(S, S / kMoeTcRows + used), E};
  const PrefillLinear lin{xg, y, N, qweight, qzeros, scales, bias};
  return launch_w4_prefill_seg<TA>(lin, S, K, G, s, seg);
}
}  // namespace

extern "C" {

size_t paro_w4_moe_workspace_size(int64_t T, int64_t K, int64_t N, int E, int topk, int group_size) {
  if (check_moe_shape(T, K, N, E, topk, group_size) != PARO_OK) return 0;
  return moe_plan(T, K, T * topk).total;
}

int paro_w4_moe_linear(const void* x, void* y, int64_t T, int64_t K, int64_t N, int E, int topk,
                       const int32_t* expert_idx, const int32_t* qweight, const int32_t* qzeros, const void* scales,
                       const void* bias, const float* channel_scales, const int16_t* pairs, const float* theta,
                       int group_size, int krot, int dtype, void* workspace, size_t workspace_bytes,
                       paro_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (dtype) {
    case PARO_DTYPE_F16:
      return moe_impl<__half>(x, y, T, K, N, E, topk, expert_idx, qweight, qzeros, scales, bias, channel_scales,
                              pairs, theta, group_size, krot, workspace, workspace_bytes, s);
    case PARO_DTYPE_BF16:
      return moe_impl<__nv_bfloat16>(x, y, T, K, N, E, topk, expert_idx, qweight, qzeros, scales, bias,
                                     channel_scales, pairs, theta, group_size, krot, workspace, workspace_bytes, s);
    default: return PARO_ERR_INVALID_ARG;
  }
}

int paro_w4_moe_launches(int64_t T, int64_t K, int64_t N, int E, int topk, int group_size, int krot,
                         int rotate) {
  if (check_moe_shape(T, K, N, E, topk, group_size) != PARO_OK || T == 0 || krot < 0 || krot > kMaxKrot) return 0;
  // rotation (two launches above 64 tokens: R' build and X R'), route, gather
  // (folded into the route for few rows), expert GEMV or GEMM
  const bool route_gathers = (size_t)(T * topk) * K * 2 <= kMoeRouteGatherBytes;
  return (rotate ? (T >= kRotTcMinM ? 2 : 1) : 0) + (route_gathers ? 2 : 3);
}

}  // extern "C"

// ------------------------------------------------------------ no-allocation variant
// Scratch for paro_w4_linear_noalloc: a file-scope device array (every GPU that
// loads the library holds it until exit).  Host code must not pass the symbol
// itself to a kernel — on the host it is only a stand-in; the device address
// comes from cudaGetSymbolAddress, looked up once per device and cached.
static __device__ __align__(256) unsigned char g_noalloc_scratch[PARO_W4_LINEAR_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;

// Device address of g_noalloc_scratch on the current device (nullptr on failure).
void* noalloc_scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}
}  // namespace

extern "C" {

int paro_w4_linear_noalloc(const void* x, void* y, int64_t M, int64_t K, int64_t N,
                           const int32_t* qweight, const int32_t* qzeros, const void* scales,
                           const void* bias, const float* channel_scales, const int16_t* pairs,
                           const float* theta, int group_size, int krot, paro_stream_t stream) {
  return paro_w4_linear_noalloc_dt(x, y, M, K, N, qweight, qzeros, scales, bias, channel_scales, pairs, theta,
                                   group_size, krot, PARO_DTYPE_F16, stream);
}

int paro_w4_linear_noalloc_dt(const void* x, void* y, int64_t M, int64_t K, int64_t N,
                              const int32_t* qweight, const int32_t* qzeros, const void* scales,
                              const void* bias, const float* channel_scales, const int16_t* pairs,
                              const float* theta, int group_size, int krot, int dtype, paro_stream_t stream) {
  if (dtype != PARO_DTYPE_F16 && dtype != PARO_DTYPE_BF16) return PARO_ERR_INVALID_ARG;
  // the same argument checks, in the same order, as paro_w4_linear
  if (int st = check_linear_args(x, y, M, K, N, qweight, qzeros, scales, bias, channel_scales, pairs, theta,
                                 group_size, krot))
    return st;
  if (M == 0) return PARO_OK;
  // only a call that rotates (krot > 0 or channel scales) stages anything
  const bool rotate = krot > 0 || channel_scales != nullptr;
  if (!rotate)
    return paro_w4_linear_dt(x, y, M, K, N, qweight, qzeros, scales, bias, nullptr, pairs, theta, group_size, 0,
                             dtype, nullptr, 0, stream);
  if (paro_w4_linear_workspace_size(M, K, N, group_size) > (size_t)PARO_W4_LINEAR_NOALLOC_SCRATCH_BYTES)
    return PARO_ERR_WORKSPACE;
  void* scratch = noalloc_scratch_address();
  if (scratch == nullptr) return PARO_ERR_CUDA;
  return paro_w4_linear_dt(x, y, M, K, N, qweight, qzeros, scales, bias, channel_scales, pairs, theta,
                           group_size, krot, dtype, scratch, (size_t)PARO_W4_LINEAR_NOALLOC_SCRATCH_BYTES, stream);
}

int paro_validate_pairs(const int16_t* pairs_host, int64_t K, int group_size, int krot) {
  if (pairs_host == nullptr || krot < 0) return PARO_ERR_INVALID_ARG;
  int G = 0;
  if (int st = normalize_group(group_size, K, &G)) return st;
  std::vector<unsigned char> seen((size_t)G);
  for (int s = 0; s < krot; ++s)
    for (int64_t g = 0; g < K / G; ++g) {
      std::fill(seen.begin(), seen.end(), 0);
      const int16_t* p = pairs_host + (size_t)s * K + (size_t)g * G;
      for (int e = 0; e < G; ++e) {
        const int v = p[e];
        if (v < 0 || v >= G || seen[(size_t)v]) return PARO_ERR_INVALID_ARG;
        seen[(size_t)v] = 1;
      }
    }
  return PARO_OK;
}

int paro_device_status(int clear) {
  if (cudaDeviceSynchronize() != cudaSuccess) return PARO_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, paro::g_status, sizeof(v)) != cudaSuccess) return PARO_ERR_CUDA;
  if (clear) {
    const unsigned z = 0;
    if (cudaMemcpyToSymbol(paro::g_status, &z, sizeof(z)) != cudaSuccess) return PARO_ERR_CUDA;
  }
  if (v & kErrTimeout) return PARO_ERR_TIMEOUT;
  if (v & (kErrPairIndex | kErrExpertIndex)) return PARO_ERR_INVALID_ARG;
  return PARO_OK;
}

int paro_selftest_wait_timeout(uint64_t limit_ns, uint64_t* elapsed_ns, paro_stream_t stream) {
  if (limit_ns == 0 || limit_ns > kSelftestMaxLimitNs) return PARO_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  wait_selftest_kernel<<<1, 32, 0, s>>>((unsigned long long)limit_ns);
  if (cudaGetLastError() != cudaSuccess) return PARO_ERR_CUDA;
  unsigned long long e = 0;
  if (cudaMemcpyFromSymbolAsync(&e, g_selftest_elapsed_ns, sizeof(e), 0, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return PARO_ERR_CUDA;
  if (elapsed_ns != nullptr) *elapsed_ns = (uint64_t)e;
  return PARO_OK;
}

}  // extern "C"

// Prefill W4 GEMM on the sm_100a tensor cores (tcgen05 / TMEM), M > 16 token rows.
// Quantisation groups of G = 128, 64, 32 or 16 rows (scales and zero words of
// the 64-row k-block's max(1, 64 / G) groups come with each TMA stage).
// Activations, weights as dequantised, scales, bias and Y are fp16 or bf16
// (template type TA; bf16 unpacks every nibble to 128 + q and runs the MMA
// with bf16 A and B).
//
// What it computes (GPTQModel wiki page "ParoQuant", "Activation and weight
// transforms" and "Triton plans and tuning"):
//   Y[m, n] = sum_k X_r[m, k] * (q[k, n] - z[k/G, n]) * s[k/G, n] + b[n]
//
// CTA tile: 256 token rows x 256 output columns, K in blocks of 64, as two
// 128-token accumulators that share every dequantised weight tile (the int4
// -> fp16 work per tensor-core FLOP is half that of a 128-token tile).
//   A = X_r tile [256 tokens][64 k] fp16, K-major, brought by TMA with the
//       128-byte swizzle (the UMMA canonical K-major SW128 layout); token block
//       b starts 16 KB in.
//   B = W^T tile [256 columns][64 k] fp16, K-major, written by the dequant warps
//       from the AWQ words in the canonical no-swizzle layout: 8x8 core matrices
//       of 128 contiguous bytes, k-chunks 128 B apart (LBO), 8-row groups
//       1040 B apart (SBO: one extra 16 bytes per group so the dequant stores
//       of eight neighbouring groups hit eight different bank groups).
//   D = two fp32 accumulators [128 lanes = tokens][256 columns] in tensor
//       memory (all 512 columns; one CTA per SM).
// Warp roles (18 warps): warp 0 = TMA producer, warp 1 = TMEM allocator and
// single-thread MMA issuer, warps 2..17 = dequant (k-chunk (warp-2)/2, 16 word
// columns, 4 rows per lane) and then epilogue.  Two rings: a 3-deep TMA ring (A, the packed qweight tile
// [64 rows][32 words] with 128-byte swizzle, the group's scales and zero words),
// deep enough to cover the TMA round trip, and a 3-deep ring of dequantised B
// tiles so the dequant warps run ahead of the tensor core.  Barriers: tma_full / tma_empty per TMA stage (bytes
// landed / MMAs done), b_full / b_empty per B buffer (8 dequant warps / MMAs
// done); tcgen05.commit signals the "empty" ones when the MMAs complete.
//
// Dequantisation of one packed word column w for 4 rows of k-chunk c: a byte
// permute of rows (k, k+1) puts both k's of one column in one register;
// (v & 0x000F000F) | 0x64006400 and (v & 0x00F000F0) | 0x64006400 give the fp16
// pairs 1024 + q and 1024 + 16 q exactly; subtracting (1024 + z) or (1024 + 16 z)
// leaves q - z or 16 (q - z) exactly, and multiplying by s or s/16 rounds
// (q - z) s to fp16 once.  One 8-byte store per column writes its 4 k's.
#pragma once

#include "common.cuh"

namespace paro {

constexpr int kTcBM = 128;               // token rows per accumulator (UMMA M)
constexpr int kTcMB = 2;                 // accumulators (token blocks) per CTA
constexpr int kTcBN = 256;               // output columns per CTA
constexpr int kTcBK = 64;                // k per stage (128-byte rows)
constexpr int kTcStages = 3;             // TMA ring: A, packed weights, scales, zeros
constexpr int kTcBBufs = 3;              // dequantised B ring
constexpr int kTcDequantWarps = 16;      // (k-chunk, half of its 8 rows) per warp
constexpr int kTcThreads = 32 * (2 + kTcDequantWarps);
constexpr int kTcBSbo = 1040;            // B: bytes between 8-row groups
constexpr int kTcBLbo = 128;             // B: bytes between k-chunks

// SR = scale / zero rows per 64-row k-block: 1 for G >= 64, 64 / G below
// (G = 32: 2, G = 16: 4, which leaves room for only 2 dequantised B buffers).
template <int SR>
struct TcLayoutT {
  static constexpr int BBUFS = SR >= 4 ? 2 : kTcBBufs;
  // TMA stage (1024-aligned): A | packed weights | scales | zeros
  static constexpr int A_OFF = 0;                          // 32768 B
  static constexpr int A_BLOCK = kTcBM * kTcBK * 2;         // one token block
  static constexpr int A_BYTES = kTcMB * A_BLOCK;
  static constexpr int WQ_OFF = A_OFF + A_BYTES;           // 8192 B, 1024-aligned
  static constexpr int WQ_BYTES = kTcBK * (kTcBN / 8) * 4;
  static constexpr int S_OFF = WQ_OFF + WQ_BYTES;          // SR x 512 B
  static constexpr int S_ROW = kTcBN * 2;
  static constexpr int S_BYTES = SR * S_ROW;
  static constexpr int Z_OFF = S_OFF + S_BYTES;            // SR x 128 B
  static constexpr int Z_ROW = (kTcBN / 8) * 4;
  static constexpr int Z_BYTES = SR * Z_ROW;
  static constexpr int STAGE = ((Z_OFF + Z_BYTES + 1023) / 1024) * 1024;
  static constexpr int TX_BYTES = A_BYTES + WQ_BYTES + S_BYTES + Z_BYTES;
  // dequantised B buffers after the TMA ring
  static constexpr int B_RING = kTcStages * STAGE;
  static constexpr int B_BYTES = (kTcBN / 8) * kTcBSbo;   // 33280 B
  static constexpr int B_STRIDE = ((B_BYTES + 127) / 128) * 128;
  static constexpr int BAR_OFF = B_RING + BBUFS * B_STRIDE;
  // barriers: tma_full[S], tma_empty[S], b_full[B], b_empty[B], accum_full
  static constexpr int NBARS = 2 * kTcStages + 2 * BBUFS + 1;
  static constexpr int MISC_OFF = BAR_OFF + 8 * NBARS;
  static constexpr int SMEM = MISC_OFF + 16 + 1024;
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
  // epilogue staging of the fp16 output tile, over the (then idle) TMA ring
  // and the start of the B ring: four {64 columns, 256 rows} boxes
  static constexpr int O_BOX = kTcMB * kTcBM * 64 * 2;     // 32 KB
  static_assert((kTcBN / 64) * O_BOX <= BAR_OFF, "output staging fits before the barriers");
};

// instruction descriptor: fp32 accumulate, fp16 A and B, both K-major, M=128, N=256
constexpr uint32_t kTcIdesc = (1u << 4) | ((uint32_t)(kTcBN >> 3) << 17) | ((uint32_t)(kTcBM >> 4) << 24);

// Operands of one linear of a launch.  A launch covers NL linears that share
// M and K (a decoder layer's q/k/v, say), each with its own activations (its
// X_r), weights and output: the column tiles of linear l are blockIdx.x =
// tile_begin .. tile_begin + ceil(n / 256) - 1.
struct alignas(64) TcOperand {
  CUtensorMap a;          // X_r [M, K], box {64, 256}, 128-byte swizzle
  CUtensorMap w;          // qweight [K, N/8] int32, box {32 words, 64 rows}, 128-byte swizzle
  CUtensorMap s;          // scales [K/G, N], box {256, SR}
  CUtensorMap z;          // qzeros [K/G, N/8] int32, box {32, SR}
  CUtensorMap y;          // Y [M, N], box {64, 256}, 128-byte swizzle
  const void* bias;       // [N] or nullptr (activation type)
  int n;                  // output columns
  int tile_begin;         // first column tile of this linear in the grid
  // Segment variant (stacked experts): the maps cover all E experts (weights
  // [E*K, N/8], scales and zero words [E*K/G, ...]; a = the routed rows sorted
  // by expert), and blockIdx.y is the tile: segs[y] = {expert, first sorted
  // row, rows <= 256}; sorted row q is output row perm[q] of y (written with
  // plain stores, row by row); bias is [E, N].
  const int4* segs;
  const int* seg_count;   // tiles written by the routing (device)
  const int* perm;
  void* yptr;             // y [rows of y, N] (activation type)
};
constexpr int kTcMaxLinears = 4;
template <int NL>
struct TcBatch {
  TcOperand op[NL];
};

template <int SR, typename TA, int NL, bool SEG = false>
__global__ void __launch_bounds__(kTcThreads, 1) w4_tc_gemm_kernel(const __grid_constant__ TcBatch<NL> ops,
                                                                   int M, int K, int gsz) {
  using L = TcLayoutT<SR>;
  // this CTA's linear (selected by constant offsets into the parameter block)
  const TcOperand* op = &ops.op[0];
#pragma unroll
  for (int i = 1; i < NL; ++i)
    if ((int)blockIdx.x >= ops.op[i].tile_begin) op = &ops.op[i];
  const CUtensorMap* const tmA = &op->a;
  const CUtensorMap* const tmW = &op->w;
  const CUtensorMap* const tmS = &op->s;
  const CUtensorMap* const tmZ = &op->z;
  const CUtensorMap* const tmY = &op->y;
  const TA* __restrict__ bias = static_cast<const TA*>(op->bias);
  const int N = op->n;
  // Segment variant: the tile's expert and rows are written by the kernels
  // ahead, so the whole CTA waits for them first (before any setup).
  int expert = 0, tok0 = blockIdx.y * (kTcMB * kTcBM), tile_rows = 0;
  if constexpr (SEG) {
    pdl_wait_primary();
    if ((int)blockIdx.y >= *op->seg_count) return;
    const int4 sg = op->segs[blockIdx.y];
    expert = sg.x;
    tok0 = sg.y;
    tile_rows = sg.z;
    if (bias != nullptr) bias += (size_t)expert * N;
  }
  const int wrow0 = expert * K, qrow0 = expert * (K / gsz);   // the expert's weight / scale rows
  constexpr int kTcBBufs = L::BBUFS;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* const sbase = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t base = smem_u32(sbase);
  const uint32_t tma_full0 = base + L::BAR_OFF;
  const uint32_t tma_empty0 = tma_full0 + 8 * kTcStages;
  const uint32_t b_full0 = tma_empty0 + 8 * kTcStages;
  const uint32_t b_empty0 = b_full0 + 8 * kTcBBufs;
  const uint32_t accum_full = b_empty0 + 8 * kTcBBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + L::MISC_OFF);
  volatile int* abort = reinterpret_cast<volatile int*>(sbase + L::MISC_OFF + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = ((int)blockIdx.x - op->tile_begin) * kTcBN;
  const int nk = K / kTcBK;

  if (tid == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(tma_full0 + 8 * s, 1);
      mbar_init(tma_empty0 + 8 * s, 1);
    }
    for (int b = 0; b < kTcBBufs; ++b) {
      mbar_init(b_full0 + 8 * b, kTcDequantWarps);
      mbar_init(b_empty0 + 8 * b, 1);
    }
    mbar_init(accum_full, 1);
    *abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(tmA);
    tma_prefetch_desc(tmW);
    tma_prefetch_desc(tmS);
    tma_prefetch_desc(tmZ);
    tma_prefetch_desc(tmY);
  }
  if (warp == 1) {                      // the whole warp allocates 2 x 256 TMEM columns
    tmem_alloc(smem_u32(tmem_slot), kTcMB * kTcBN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const int pre = min(kTcStages, nk);
      // weights, scales and zeros do not depend on the previous kernel
      for (int kb = 0; kb < pre; ++kb) {
        const uint32_t st = base + kb * L::STAGE, bar = tma_full0 + 8 * kb;
        mbar_arrive_expect_tx(bar, L::TX_BYTES);
        tma_load_2d(st + L::WQ_OFF, tmW, bar, n0 / 8, wrow0 + kb * kTcBK);
        tma_load_2d(st + L::S_OFF, tmS, bar, n0, qrow0 + (kb * kTcBK) / gsz);
        tma_load_2d(st + L::Z_OFF, tmZ, bar, n0 / 8, qrow0 + (kb * kTcBK) / gsz);
      }
      pdl_wait_primary();               // X_r is written by the rotation kernel
      for (int kb = 0; kb < pre; ++kb)
        tma_load_2d(base + kb * L::STAGE + L::A_OFF, tmA, tma_full0 + 8 * kb, kb * kTcBK, tok0);
      for (int kb = pre; kb < nk; ++kb) {
        const int s = kb % kTcStages;
        if (!tc_wait(tma_empty0 + 8 * s, ((kb / kTcStages) - 1) & 1, abort)) break;
        const uint32_t st = base + s * L::STAGE, bar = tma_full0 + 8 * s;
        mbar_arrive_expect_tx(bar, L::TX_BYTES);
        tma_load_2d(st + L::WQ_OFF, tmW, bar, n0 / 8, wrow0 + kb * kTcBK);
        tma_load_2d(st + L::S_OFF, tmS, bar, n0, qrow0 + (kb * kTcBK) / gsz);
        tma_load_2d(st + L::Z_OFF, tmZ, bar, n0 / 8, qrow0 + (kb * kTcBK) / gsz);
        tma_load_2d(st + L::A_OFF, tmA, bar, kb * kTcBK, tok0);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % kTcStages, b = kb % kTcBBufs;
        if (!tc_wait(tma_full0 + 8 * s, (kb / kTcStages) & 1, abort)) break;
        if (!tc_wait(b_full0 + 8 * b, (kb / kTcBBufs) & 1, abort)) break;
        tc_fence_after();
        const uint32_t a0 = base + s * L::STAGE + L::A_OFF;
        const uint32_t b0 = base + L::B_RING + b * L::B_STRIDE;
#pragma unroll
        for (int ks = 0; ks < kTcBK / 16; ++ks) {
          // B: no swizzle, k-chunks LBO apart, 8-row groups SBO apart; 2 chunks per 16 k
          const uint64_t bd = umma_desc(b0 + ks * 2 * kTcBLbo, kTcBLbo, kTcBSbo, 0);
#pragma unroll
          for (int mb = 0; mb < kTcMB; ++mb) {
            // A: 128-byte swizzled rows, 8-row groups 1024 B apart; +32 B per 16 k
            const uint64_t ad = umma_desc(a0 + mb * L::A_BLOCK + ks * 32, 16, 1024, 2);
            umma_f16(tmem_d + (uint32_t)(mb * kTcBN), ad, bd, kTcIdesc | Act<TA>::kIdescAB,
                     (kb > 0 || ks > 0) ? 1u : 0u);
          }
        }
        umma_commit(tma_empty0 + 8 * s);   // the TMA stage and ...
        umma_commit(b_empty0 + 8 * b);     // ... the B buffer are free once these MMAs finish
      }
      umma_commit(accum_full);          // all MMAs of the tile are done
    }
  } else {
    // ------------------------------------------------------------ dequant warps
    // warp (c, wh): k-chunk c (rows 8c .. 8c+7), word columns 16 wh .. 16 wh + 15;
    // lane (w, h): word column w, rows 8c + 4h .. +3.  Neighbouring lanes differ in
    // h, so the 8-byte stores of a half-warp land in 16 different 8-byte slots.
    const int dw = warp - 2;
    const int c = dw >> 1;
    const int w = 16 * (dw & 1) + (lane >> 1);   // packed word column: output columns 8w .. 8w+7
    const int h = lane & 1;
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % kTcStages, bb = kb % kTcBBufs;
      if (!tc_wait(tma_full0 + 8 * s, (kb / kTcStages) & 1, abort)) break;
      if (kb >= kTcBBufs && !tc_wait(b_empty0 + 8 * bb, ((kb / kTcBBufs) - 1) & 1, abort)) break;
      // shared-memory addresses (explicit ld/st.shared: no generic-address path)
      const uint32_t stp = base + (uint32_t)(s * L::STAGE);
      const uint32_t btile = base + (uint32_t)(L::B_RING + bb * L::B_STRIDE);
      // 4 words of rows 8c+4h .. +3, word column w (128-byte swizzled rows)
      uint32_t wv[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int row = 8 * c + 4 * h + r;
        wv[r] = lds32(stp + (uint32_t)(L::WQ_OFF + row * 128 + ((((w >> 2) ^ (row & 7))) << 4) + (w & 3) * 4));
      }
      // group zero points and scales of the 8 columns (column j at nibble j/2 + 4 (j & 1));
      // rows 8c .. 8c+7 of the block lie in quantisation group (8 c) / G of its SR
      const int sr = SR > 1 ? (8 * c) / gsz : 0;
      const uint32_t zw = lds32(stp + (uint32_t)(L::Z_OFF + sr * L::Z_ROW + w * 4));
      const uint4 s8 = lds128(stp + (uint32_t)(L::S_OFF + sr * L::S_ROW + w * 16));
      const uint32_t sw[4] = {s8.x, s8.y, s8.z, s8.w};
      uint32_t outv[8][2];
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        uint32_t elo[4], ehi[4];
        const uint32_t mlo = prmt(wv[2 * p], wv[2 * p + 1], 0x5410);
        const uint32_t mhi = prmt(wv[2 * p], wv[2 * p + 1], 0x7632);
        if constexpr (Act<TA>::kBf16) {
          // bf16 (7 mantissa bits): every nibble moved to bits 0..3, 128 + q
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            elo[j] = and_or(mlo >> (4 * j), 0x000F000Fu, 0x43004300u);
            ehi[j] = and_or(mhi >> (4 * j), 0x000F000Fu, 0x43004300u);
          }
        } else {
          const uint32_t mlo8 = mlo >> 8, mhi8 = mhi >> 8;
          elo[0] = and_or(mlo, 0x000F000Fu, 0x64006400u);
          elo[1] = and_or(mlo, 0x00F000F0u, 0x64006400u);
          elo[2] = and_or(mlo8, 0x000F000Fu, 0x64006400u);
          elo[3] = and_or(mlo8, 0x00F000F0u, 0x64006400u);
          ehi[0] = and_or(mhi, 0x000F000Fu, 0x64006400u);
          ehi[1] = and_or(mhi, 0x00F000F0u, 0x64006400u);
          ehi[2] = and_or(mhi8, 0x000F000Fu, 0x64006400u);
          ehi[3] = and_or(mhi8, 0x00F000F0u, 0x64006400u);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          outv[2 * j][p] = elo[j];        // column 2j   (nibble j)
          outv[2 * j + 1][p] = ehi[j];    // column 2j+1 (nibble j + 4)
        }
      }
#pragma unroll
      for (int col = 0; col < 8; ++col) {
        const int j = col >> 1;
        const int nib = j + 4 * (col & 1);
        uint32_t sc = prmt(sw[j], sw[j], (col & 1) ? 0x3232 : 0x1010);   // (s, s)
        uint2 o;
        if constexpr (Act<TA>::kBf16) {
          const uint32_t z = (zw >> (4 * nib)) & 0xFu;
          const uint32_t zz = (z | (z << 16)) | 0x43004300u;              // 128 + z
          o.x = bmul2_u32(bsub2_u32(outv[col][0], zz), sc);
          o.y = bmul2_u32(bsub2_u32(outv[col][1], zz), sc);
        } else {
          const uint32_t sh = (j & 1) ? 4u : 0u;
          const uint32_t z = ((zw >> (4 * nib)) & 0xFu) << sh;
          const uint32_t zz = (z | (z << 16)) | 0x64006400u;
          if (j & 1) sc = hmul2_u32(sc, 0x2C002C00u);                      // s / 16
          o.x = hmul2_u32(hsub2_u32(outv[col][0], zz), sc);
          o.y = hmul2_u32(hsub2_u32(outv[col][1], zz), sc);
        }
        sts64(btile + (uint32_t)(w * kTcBSbo + c * kTcBLbo + col * 16 + h * 8), o);
      }
      fence_proxy_async_smem();         // make the B tile visible to the tensor core
      __syncwarp();
      if (lane == 0) mbar_arrive(b_full0 + 8 * bb);
    }

    // ------------------------------------------------------------ epilogue
    // warp w reads TMEM lanes 32*(w%4) .. +31 (its token rows of a block);
    // warps 2..5 take block 0 columns 0..127, 6..9 block 0 columns 128..255,
    // 10..13 and 14..17 the same halves of block 1.  The fp16 tile (+ bias) is
    // staged in shared memory — the TMA ring, idle once every MMA is done — as
    // four {64 columns, 256 rows} boxes with the 128-byte swizzle, and one
    // thread writes it with four TMA stores (clipped at row M and column N),
    // so every global write is a full line.
    pdl_wait_primary();                 // previous kernels are complete before Y is written
    const bool ok = __all_sync(0xffffffffu, tc_wait(accum_full, 0, abort));   // warp-uniform
    tc_fence_after();
    const int quarter = warp & 3;
    const int cq = (warp - 2) >> 2;                 // 0..3
    const int mb = cq >> 1, chalf = cq & 1;
    const int row = mb * kTcBM + 32 * quarter + lane;   // token row within the tile
    if (ok) {
#pragma unroll 1
      for (int cb = 0; cb < 4; ++cb) {
        const int col0 = chalf * 128 + cb * 32;
        uint32_t r[32];
        tmem_ld32(tmem_d + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(mb * kTcBN + col0), r);
        tmem_ld_wait_tie(r);
        const int n = n0 + col0;
        // box col0 / 64, 16-byte chunks (col0 % 64) / 8 .. +3 of this row
        const uint32_t rowp = base + (uint32_t)(col0 >> 6) * L::O_BOX + (uint32_t)row * 128u;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float v[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) v[e] = __uint_as_float(r[8 * q + e]);
          if (bias != nullptr && n < N) {   // bias is only 4-byte aligned: pair loads
            const uint32_t* bh = reinterpret_cast<const uint32_t*>(bias + n + 8 * q);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = Act<TA>::f2(bh[e]);
              v[2 * e] += f.x;
              v[2 * e + 1] += f.y;
            }
          }
          uint4 o;
          uint32_t* oh = &o.x;
#pragma unroll
          for (int e = 0; e < 4; ++e) oh[e] = Act<TA>::p2(v[2 * e], v[2 * e + 1]);
          const uint32_t chunk = (uint32_t)(((col0 & 63) >> 3) + q);
          sts128u(rowp + ((chunk ^ (uint32_t)(row & 7)) << 4), o);
        }
      }
    }
    fence_proxy_async_smem();           // the staged tile is read by the TMA (async proxy)
    named_bar_sync(1, 32 * kTcDequantWarps);
    if constexpr (SEG) {
      // the tile's rows go to their slots: 16-byte chunks of the staged boxes,
      // row by row, only the tile's own rows and columns below N
      if (!*abort) {
        TA* const Yp = static_cast<TA*>(op->yptr);
        const int et = tid - 64;                  // epilogue thread 0 .. 511
        for (int idx = et; idx < tile_rows * (kTcBN / 8); idx += 32 * kTcDequantWarps) {
          const int r = idx / (kTcBN / 8), ch = idx % (kTcBN / 8);
          const int n = n0 + 8 * ch;
          if (n >= N) continue;
          const uint32_t src = base + (uint32_t)(ch >> 3) * L::O_BOX + (uint32_t)r * 128u +
                               ((uint32_t)((ch & 7) ^ (r & 7)) << 4);
          *reinterpret_cast<uint4*>(Yp + (size_t)op->perm[tok0 + r] * N + n) = lds128(src);
        }
      }
    } else if (warp == 2 && lane == 0 && !*abort) {
#pragma unroll
      for (int b = 0; b < kTcBN / 64; ++b)
        if (n0 + 64 * b < N) tma_store_2d(tmY, base + (uint32_t)b * L::O_BOX, n0 + 64 * b, tok0);
      bulk_commit_group();
      bulk_wait_group_all();            // written before the kernel completes
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_d, kTcMB * kTcBN);
  }
}

}  // namespace paro

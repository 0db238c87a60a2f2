// Decode W4 GEMV (M <= 16 token rows), warp-specialised, on warp-level tensor-core
// MMA (m16n8k16, fp16 in, fp32 accumulate), reading AWQ-packed weights directly.
//
// What it computes (GPTQModel wiki page "ParoQuant", "Activation and weight
// transforms" and "Triton plans and tuning"):
//   Y[m, n] = sum_g s[g, n] * sum_{k in g} X_r[m, k] * (q[k, n] - z[g, n]) + b[n]
//
// Work layout.  A CTA owns NTILE output columns (NTILE/8 packed words of every
// qweight row) and a contiguous range of at most kGvMaxGroups 128-row groups of
// K.  Warp 0 is the producer.  One lane streams each group's qweight block
// (128 rows, 64- or 128-byte swizzle) through a ring of STAGES shared-memory
// stages with TMA, signalling "full" mbarriers; consumers release a stage on its
// "empty" mbarrier.  The CTA's scales, zero words and X_r columns are each one
// TMA copy for the whole range (a TMA instruction costs tens of cycles to issue
// whatever its size, so few large copies start the stream sooner), resident
// for the whole kernel.  Weights, scales and zeros do not depend on the
// previous kernel, so they are requested before griddepcontrol.wait
// (programmatic dependent launch); only the X_r copy waits for the rotation.
// Consumer warps are 4 column slices (64 columns each) x KP k-parts; k-part p
// takes the CTA's groups p, p+KP, ... so every warp works on whole groups.
//
// Activations, scales, bias and Y are fp16 or bf16 (template type TA); with
// bf16 every nibble is unpacked to 128 + q (bf16 has 7 mantissa bits) and the
// MMA runs on bf16 operands.
//
// Quantisation groups of G = 128, 64, 32 or 16 rows: the fold below runs at
// the end of every G / 16 k-steps with that group's scales and zero words.
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
// along K.  CTA r owns columns [r*NTILE/S, (r+1)*NTILE/S): every consumer warp
// pushes its fp32 partials of each slice straight from registers into the
// owner's inbox (a dedicated shared-memory area, one slot per sender CTA and
// k-part) with distributed-shared-memory stores; after one cluster barrier
// each owner sums its inbox in a fixed order, adds the bias and writes fp16 Y.
// No global scratch, no atomics, deterministic.  A second cluster-barrier phase
// (each CTA arrives once all bytes addressed to it have landed, and waits at
// exit) keeps every CTA resident until every push of the cluster has landed, so
// no st.async is ever in flight from or to a CTA that has left.
#pragma once

#include "common.cuh"

namespace paro {

constexpr int kGvMaxStages = 8;
constexpr int kGvMaxGroups = 16;            // 128-row groups of K per CTA
constexpr uint32_t kGvMagic = 0x64006400u;  // fp16 pair (1024, 1024)
constexpr uint32_t kGvMagicBf = 0x43004300u;   // bf16 pair (128, 128)

// NTILE output columns per CTA (64 per column-slice warp), KP k-parts, STAGES
// groups in flight.
template <int NT, int KP, int NTILE, int STAGES>
struct GemvLayout {
  static constexpr int CSL = NTILE / 64;                  // column-slice warps per k-part
  static constexpr int WORDS = NTILE / 8;                 // packed words per row segment
  static constexpr int THREADS = 32 * (1 + CSL * KP);
  static constexpr int MP = 8 * NT;                       // token rows per CTA
  static constexpr int W_BYTES = 128 * WORDS * 4;         // one group of qweight
  static constexpr int STAGE = ((W_BYTES + 1023) / 1024) * 1024;
  // resident for the whole kernel, laid out for the launch's largest group
  // range gmax: X_r as [64-column chunk][token][64] (two chunks per group),
  // scales [group][NTILE], zero words [group][WORDS]; then the split-K inbox
  // and the barriers.
  static constexpr int XG_BYTES = 2 * MP * 128;           // X_r of one group
  static constexpr int X_OFF = STAGES * STAGE;
  static constexpr int INBOX_BYTES = KP * MP * NTILE * 4;   // partials [S][KP][MP][NTILE/S]
  // scales and zero words hold gr = gmax * 128 / G quantisation-group rows
  __host__ __device__ static constexpr int s_off(int gmax) { return X_OFF + gmax * XG_BYTES; }
  __host__ __device__ static constexpr int z_off(int gmax, int gr) { return s_off(gmax) + gr * NTILE * 2; }
  __host__ __device__ static constexpr int inbox_off(int gmax, int gr) {
    return ((z_off(gmax, gr) + gr * WORDS * 4 + 1023) / 1024) * 1024;
  }
  // barriers: full[STAGES], empty[STAGES], consts, X_r, inbox
  __host__ __device__ static constexpr int bar_off(int gmax, int gr) { return inbox_off(gmax, gr) + INBOX_BYTES; }
  __host__ __device__ static constexpr int smem(int gmax, int gr) {
    return bar_off(gmax, gr) + 8 * (2 * STAGES + 3) + 1024;
  }
  static_assert(STAGES <= kGvMaxStages, "too many stages");
  // k-part p consumes groups p, p + KP, ...: with STAGES a multiple of KP every
  // stage (group i sits in stage i % STAGES) belongs to one k-part, so its
  // mbarrier phases are waited on in order and never aliased by parity
  static_assert(STAGES % KP == 0, "each stage must belong to one k-part");
  // 128-byte swizzle needs 128-byte rows; 64-byte rows use the 64-byte swizzle
  static constexpr int ROW_BYTES = WORDS * 4;
};

// Operands of one linear of a launch.  A launch covers NL linears that share
// the token count and K (a decoder layer's q/k/v, say): the column tiles of
// linear l are blockIdx.x = tile_begin .. tile_begin + ceil(n / NTILE) - 1.
struct alignas(64) GemvOperand {
  CUtensorMap w;          // qweight [K, N/8] int32, box {NTILE/8 words, 128 rows}
  CUtensorMap x;          // X_r [M, K] fp16 as [K/64][M][64], box {64, MP, 2 gmax}
  CUtensorMap s;          // scales [K/G, N] fp16, box {NTILE, gmax * 128 / G}
  CUtensorMap z;          // qzeros [K/G, N/8] int32, box {NTILE/8, gmax * 128 / G}
  const void* bias;       // [N] or nullptr (activation type)
  void* y;                // [M, N] (activation type)
  int n;                  // output columns
  int tile_begin;         // first column tile of this linear in the grid
  // Segment variant (stacked experts): the maps cover all E experts (weights
  // [E*K, N/8], scales and zero words [E*K/G, ...]; x = the routed rows sorted
  // by expert), and CTA x = segment * seg_tiles + column tile.  Segment s is
  // segs[s] = {expert, first sorted row, rows <= 8}; sorted row q is output
  // row perm[q] of y; bias is [E, N].
  const int4* segs;
  const int* seg_count;   // segments written by the routing (device)
  const int* perm;
  int seg_tiles;
};
template <int NL>
struct GemvBatch {
  GemvOperand op[NL];
};
constexpr int kGvMaxLinears = 4;

// Nibbles j = 0..3 of the two 16-bit halves of m.  fp16: 1024 + q for even j
// and 1024 + 16 q for odd j (the nibble read in place, 10 mantissa bits);
// bf16 (7 mantissa bits): every nibble moved to bits 0..3, 128 + q.
template <typename TA>
__device__ __forceinline__ void gv_unpack4(uint32_t m, uint32_t (&e)[4]) {
  if constexpr (Act<TA>::kBf16) {
    e[0] = and_or(m, 0x000F000Fu, kGvMagicBf);
    e[1] = and_or(m >> 4, 0x000F000Fu, kGvMagicBf);
    e[2] = and_or(m >> 8, 0x000F000Fu, kGvMagicBf);
    e[3] = and_or(m >> 12, 0x000F000Fu, kGvMagicBf);
  } else {
    const uint32_t m8 = m >> 8;
    e[0] = and_or(m, 0x000F000Fu, kGvMagic);
    e[1] = and_or(m, 0x00F000F0u, kGvMagic);
    e[2] = and_or(m8, 0x000F000Fu, kGvMagic);
    e[3] = and_or(m8, 0x00F000F0u, kGvMagic);
  }
}

template <typename TA>
__device__ __forceinline__ void gv_mma(bool first, float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if constexpr (Act<TA>::kBf16) {
    if (first) mma_16816_bf_zc(d, a, b0, b1);
    else mma_16816_bf(d, a, b0, b1);
  } else {
    if (first) mma_16816_zc(d, a, b0, b1);
    else mma_16816(d, a, b0, b1);
  }
}

// GQ: quantisation groups per 128 rows fixed at compile time (1: G = 128),
// or 0 to take them from gq_arg (G = 64, 32, 16).  SEG: the segment variant
// (one operand, stacked experts, routing read after the kernel ahead).
template <int NT, int KP, int NTILE, int STAGES, int NL, typename TA, int GQ, bool SEG = false>
__global__ void __launch_bounds__(32 * (1 + (NTILE / 64) * KP), 1) w4_gemv_kernel(
    const __grid_constant__ GemvBatch<NL> ops, int M, int K, int gmax, int gq_arg) {
  using L = GemvLayout<NT, KP, NTILE, STAGES>;
  // this CTA's linear (selected by constant offsets into the parameter block)
  const GemvOperand* op = &ops.op[0];
#pragma unroll
  for (int i = 1; i < NL; ++i)
    if ((int)blockIdx.x >= ops.op[i].tile_begin) op = &ops.op[i];
  const CUtensorMap* const tmW = &op->w;
  const CUtensorMap* const tmX = &op->x;
  const CUtensorMap* const tmS = &op->s;
  const CUtensorMap* const tmZ = &op->z;
  const TA* bias = static_cast<const TA*>(op->bias);
  TA* const Y = static_cast<TA*>(op->y);
  const int N = op->n;
  constexpr int kGvStages = STAGES;
  constexpr int kGvTile = NTILE;
  // The next kernel in the stream may launch now; it waits for our completion
  // before it touches anything we read or write.
  pdl_launch_dependents();

  // Segment variant: this CTA's expert and routed rows are written by the
  // kernels ahead, so everything (weights included) waits for them.  Every
  // CTA of a cluster has the same segment, so a cluster leaves as a whole.
  int ntile = (int)blockIdx.x - op->tile_begin;
  int expert = 0, row0 = 0, seg_rows = M;
  if constexpr (SEG) {
    pdl_wait_primary();
    const int seg = (int)blockIdx.x / op->seg_tiles;
    ntile = (int)blockIdx.x - seg * op->seg_tiles;
    if (seg >= *op->seg_count) return;
    const int4 sg = op->segs[seg];
    expert = sg.x;
    row0 = sg.y;
    seg_rows = sg.z;
    if (bias != nullptr) bias += (size_t)expert * N;
  }

  extern __shared__ unsigned char smem_raw[];
  // 1024-byte aligned base, derived on the shared array so every access stays LDS/STS
  unsigned char* const sbase = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t base = smem_u32(sbase);
  // gq = 128 / G quantisation groups per 128-row group (G = 128, 64, 32, 16);
  // spq = G / 16 k-steps of 16 rows each
  const int gq = GQ > 0 ? GQ : gq_arg;
  const int gr = gmax * gq, spq = 8 / gq;
  const uint32_t full0 = base + L::bar_off(gmax, gr);
  const uint32_t empty0 = full0 + 8 * kGvStages;
  const uint32_t cbar = empty0 + 8 * kGvStages;   // scales + zero words
  const uint32_t xbar = cbar + 8;                  // X_r
  const uint32_t inbar = xbar + 8;                 // peers' split-K partials landed

  const int split = blockIdx.y;
  const int n0 = ntile * kGvTile;
  const int groups = K / 128;
  // 32-bit arithmetic (groups <= 2^16, splits <= 8): no 64-bit division routine
  const int g_begin = (int)(((unsigned)split * (unsigned)groups) / gridDim.y);
  const int g_end = (int)(((unsigned)(split + 1) * (unsigned)groups) / gridDim.y);
  const int ng = g_end - g_begin;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = gridDim.y;                          // CTAs of the cluster along K
  const int mrows = min(L::MP, seg_rows);
  // stacked experts: the expert's first weight row and first scale / zero row
  const int wrow0 = expert * K, qrow0 = expert * (K / 128) * gq;

  if (tid == 0) {
    for (int s = 0; s < kGvStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, L::CSL);  // the column-slice warps of one k-part
    }
    mbar_init(cbar, 1);
    mbar_init(xbar, 1);
    mbar_init(inbar, 1);
    fence_barrier_init();
    // every peer's k-part partials of this CTA's columns, counted in bytes
    if (S > 1) mbar_arrive_expect_tx(inbar, (uint32_t)((S - 1) * KP * mrows * (kGvTile / S) * 4));
    tma_prefetch_desc(tmW);
    tma_prefetch_desc(tmX);
    tma_prefetch_desc(tmS);
    tma_prefetch_desc(tmZ);
  }
  __syncthreads();
  // the peers may address this CTA's inbox barrier once every CTA has set its own up
  if (S > 1) cluster_arrive_release();

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
      // the tensor maps' boxes hold gmax groups (the largest range of any CTA;
      // rows past this CTA's range are loaded and not used)
      mbar_arrive_expect_tx(cbar, (uint32_t)(gr * (NTILE * 2 + L::WORDS * 4)));
      tma_load_2d(base + L::s_off(gmax), tmS, cbar, n0, qrow0 + g_begin * gq);
      tma_load_2d(base + L::z_off(gmax, gr), tmZ, cbar, n0 / 8, qrow0 + g_begin * gq);
      for (int i = 0; i < pre; ++i) {
        const uint32_t bar = full0 + 8 * i;
        mbar_arrive_expect_tx(bar, L::W_BYTES);
        tma_load_2d_hint(base + i * L::STAGE, tmW, bar, n0 / 8, wrow0 + (g_begin + i) * 128, pol);
      }
      pdl_wait_primary();                  // X_r comes from the rotation kernel
      mbar_arrive_expect_tx(xbar, (uint32_t)(gmax * L::XG_BYTES));
      tma_load_3d(base + L::X_OFF, tmX, xbar, 0, row0, 2 * g_begin);
      for (int i = pre; i < ng; ++i) {
        const int s = i % kGvStages;
        if (!mbar_wait_bounded(empty0 + 8 * s, ((i / kGvStages) - 1) & 1)) break;
        const uint32_t bar = full0 + 8 * s;
        mbar_arrive_expect_tx(bar, L::W_BYTES);
        tma_load_2d_hint(base + s * L::STAGE, tmW, bar, n0 / 8, wrow0 + (g_begin + i) * 128, pol);
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    // Swizzled offsets that do not change from group to group.  qweight rows
    // 16 ks + 2t + {0, 1, 8, 9} have (row & 7) = 2t + {0, 1, 0, 1}.
    const int wchunk = wcol >> 2, wword = (wcol & 3) * 4;
    constexpr int RB = L::ROW_BYTES;
    // 128-byte rows: chunk ^ (row & 7); 64-byte rows (64-byte swizzle): chunk ^ ((row >> 1) & 3);
    // 32-byte rows are not swizzled (four rows of a warp's load already span all banks)
    auto swz = [&](int row) -> int { return RB == 128 ? (row & 7) : (RB == 64 ? ((row >> 1) & 3) : 0); };
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
        xo[q][nt][0] = (uint32_t)(tok * 128 + (((c0) ^ (tok & 7)) << 4) + 4 * t);
        xo[q][nt][1] = (uint32_t)(tok * 128 + (((c0 + 1) ^ (tok & 7)) << 4) + 4 * t);
      }
    const uint32_t ones[4] = {Act<TA>::kOnes, Act<TA>::kOnes, Act<TA>::kOnes, Act<TA>::kOnes};
    const uint32_t sq = base + (uint32_t)L::s_off(gmax);   // scales of the range
    const uint32_t zq = base + (uint32_t)L::z_off(gmax, gr);   // zero words of the range

    // scales, zero words and X_r of every group of the range (once)
    bool consts_ready = mbar_wait_bounded(cbar, 0);
    consts_ready = mbar_wait_bounded(xbar, 0) && consts_ready;
    for (int i = kpart; i < ng; i += KP) {
      const int s = i % kGvStages;
      // explicit ld.shared: generic loads of shared memory take the long-latency path
      const uint32_t stq = base + (uint32_t)(s * L::STAGE);
      const bool ready = mbar_wait_bounded(full0 + 8 * s, (i / kGvStages) & 1) && consts_ready;
      if (ready) {
        float cg[4][NT][4];
        float rs[NT][4];
        // end of the quantisation group that closes at k-step ks: zero-point
        // correction and group scale, in fp32, with this thread's 8 columns'
        // constants
        auto fold = [&](int ks) {
          const int qrow = i * gq + ks / spq;
          const uint32_t zw = lds32(zq + (uint32_t)((qrow * L::WORDS + wcol) * 4));
          const uint4 s8 = lds128(sq + (uint32_t)(qrow * NTILE * 2 + wcol * 16));
          const uint32_t sw[4] = {s8.x, s8.y, s8.z, s8.w};   // (s[2j], s[2j+1])
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            // fp16: 1024 + z (16 z and s / 16 for odd j); bf16: 128 + z
            const int sh = (!Act<TA>::kBf16 && (j & 1)) ? 4 : 0;
            const float mg = Act<TA>::kBf16 ? 128.f : 1024.f;
            const float zl = mg + (float)(((zw >> (4 * j)) & 0xFu) << sh);
            const float zh = mg + (float)(((zw >> (16 + 4 * j)) & 0xFu) << sh);
            float2 sf = Act<TA>::f2(sw[j]);
            if (sh) sf.x *= 0.0625f, sf.y *= 0.0625f;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              const float r0 = rs[nt][0], r1 = rs[nt][1];   // row sums of tokens 2t, 2t+1
              acc[j][nt][0] = fmaf(sf.x, fmaf(-zl, r0, cg[j][nt][0]), acc[j][nt][0]);
              acc[j][nt][1] = fmaf(sf.x, fmaf(-zl, r1, cg[j][nt][1]), acc[j][nt][1]);
              acc[j][nt][2] = fmaf(sf.y, fmaf(-zh, r0, cg[j][nt][2]), acc[j][nt][2]);
              acc[j][nt][3] = fmaf(sf.y, fmaf(-zh, r1, cg[j][nt][3]), acc[j][nt][3]);
            }
          }
        };
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t wrow = stq + (uint32_t)(ks * 16 * RB);
          const uint32_t w0 = lds32(wrow + wo0);
          const uint32_t w1 = lds32(wrow + wo1);
          const uint32_t w8 = lds32(wrow + 8 * RB + wo0);
          const uint32_t w9 = lds32(wrow + 8 * RB + wo1);
          uint32_t b0[NT], b1[NT];
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const uint32_t xb = base + (uint32_t)(L::X_OFF + i * L::XG_BYTES + (ks >> 2) * (L::MP * 128));
            b0[nt] = lds32(xb + xo[ks & 3][nt][0]);
            b1[nt] = lds32(xb + xo[ks & 3][nt][1]);
          }
          uint32_t elo01[4], ehi01[4], elo89[4], ehi89[4];
          gv_unpack4<TA>(prmt(w0, w1, 0x5410), elo01);
          gv_unpack4<TA>(prmt(w0, w1, 0x7632), ehi01);
          gv_unpack4<TA>(prmt(w8, w9, 0x5410), elo89);
          gv_unpack4<TA>(prmt(w8, w9, 0x7632), ehi89);
          // the first k-step starts the sums at zero (a known constant of the
          // unrolled loop, so no branch between the two MMA forms)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t a[4] = {elo01[j], ehi01[j], elo89[j], ehi89[j]};
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) gv_mma<TA>(ks == 0, cg[j][nt], a, b0[nt], b1[nt]);
          }
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) gv_mma<TA>(ks == 0, rs[nt], ones, b0[nt], b1[nt]);
          // a quantisation group that closes inside the 128 rows (G < 128):
          // fold it and restart the sums at zero
          if (ks != 7 && (ks & (spq - 1)) == spq - 1) {
            fold(ks);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                rs[nt][e] = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) cg[j][nt][e] = 0.f;
              }
            }
          }
        }
        // this warp is done reading the stage; the last group folds from registers
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * s);
        fold(7);
      } else {
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * s);   // keep the producer moving
      }
    }
  }

  // Everything before us in the stream is complete before anyone writes Y.
  pdl_wait_primary();

  // ---------------- reduction over k-parts and the split along K.  Every
  // consumer thread holds 8 consecutive columns for each of its tokens; it
  // writes them straight into the inbox of the CTA that owns those columns
  // (slot [sender rank][k-part]): its own with plain stores, a peer's with
  // st.async counted on the peer's inbox barrier.  Each owner waits for its
  // own stores (CTA barrier) and the peers' bytes (its mbarrier), then folds
  // the inbox in a fixed order (deterministic), adds the bias and writes Y.
  // No cluster-wide barrier at the end; a CTA leaves only once every byte
  // addressed to it has landed.
  const int cols = kGvTile / S;                    // columns owned by each CTA of the cluster
  const uint32_t rank = S > 1 ? cluster_ctarank() : 0u;
  const uint32_t inbox = base + L::inbox_off(gmax, gr);  // fp32 [S][KP][MP][cols]
  __syncwarp();
  if (S > 1) cluster_wait_acquire();               // every peer's inbox barrier is set up
  if (warp != 0) {
    const int owner = (8 * wcol) / cols;
    const int c0 = 8 * wcol - owner * cols;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int tt = 0; tt < 2; ++tt) {
        const int tl = 8 * nt + 2 * t + tt;
        if (tl >= mrows) continue;
        const uint32_t off = inbox + (uint32_t)(((((int)rank * KP + kpart) * L::MP + tl) * cols + c0) * 4);
        const float4 v0 =
            make_float4(acc[0][nt][tt], acc[0][nt][2 + tt], acc[1][nt][tt], acc[1][nt][2 + tt]);
        const float4 v1 =
            make_float4(acc[2][nt][tt], acc[2][nt][2 + tt], acc[3][nt][tt], acc[3][nt][2 + tt]);
        if (owner != (int)rank) {
          const uint32_t rbar = mapa_shared(inbar, (uint32_t)owner);
          st_async_f4(mapa_shared(off, (uint32_t)owner), v0, rbar);
          st_async_f4(mapa_shared(off + 16, (uint32_t)owner), v1, rbar);
        } else {
          sts128(off, v0);
          sts128(off + 16, v1);
        }
      }
  }
  // this thread's first output (the bias load overlaps the barrier)
  const int nq = mrows * (cols / 4);
  float4 bv = make_float4(0.f, 0.f, 0.f, 0.f);
  if (bias != nullptr && tid < nq) {
    const int n = n0 + (int)rank * cols + 4 * (tid % (cols / 4));
    if (n < N) {
      const float2 b0 = Act<TA>::f2(*reinterpret_cast<const uint32_t*>(bias + n));
      const float2 b1 = Act<TA>::f2(*reinterpret_cast<const uint32_t*>(bias + n + 2));
      bv = make_float4(b0.x, b0.y, b1.x, b1.y);
    }
  }
  // this CTA's own partials (CTA barrier) and every peer's (the inbox barrier)
  __syncthreads();
  const bool landed = S == 1 || mbar_wait_bounded(inbar, 0);   // a timeout is flagged inside
  // second cluster-barrier phase: a CTA arrives once every byte addressed to it
  // has landed, and waits on the phase before it exits; so when any CTA leaves,
  // every push of the cluster has landed and no st.async is still in flight
  // (from it or to it)
  __syncwarp();
  if (S > 1) cluster_arrive_release();
  const uint32_t box = base + (uint32_t)L::inbox_off(gmax, gr);
  for (int idx = tid; idx < nq; idx += L::THREADS) {
    const int tl = idx / (cols / 4);
    const int c = 4 * (idx % (cols / 4));
    const int n = n0 + (int)rank * cols + c;
    if (n >= N) continue;
    float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
    // slots in order (sender rank, k-part); the KP slots of a rank are loaded
    // together so their latencies overlap
    for (int r = 0; r < S; ++r) {
      uint4 v[KP];
#pragma unroll
      for (int p = 0; p < KP; ++p) v[p] = lds128(box + (uint32_t)((((r * KP + p) * L::MP + tl) * cols + c) * 4));
#pragma unroll
      for (int p = 0; p < KP; ++p) {
        sum.x += __uint_as_float(v[p].x); sum.y += __uint_as_float(v[p].y);
        sum.z += __uint_as_float(v[p].z); sum.w += __uint_as_float(v[p].w);
      }
    }
    if (bias != nullptr) {
      if (idx != tid) {
        const float2 b0 = Act<TA>::f2(*reinterpret_cast<const uint32_t*>(bias + n));
        const float2 b1 = Act<TA>::f2(*reinterpret_cast<const uint32_t*>(bias + n + 2));
        bv = make_float4(b0.x, b0.y, b1.x, b1.y);
      }
      sum.x += bv.x; sum.y += bv.y; sum.z += bv.z; sum.w += bv.w;
    }
    uint2 out;
    out.x = Act<TA>::p2(sum.x, sum.y);
    out.y = Act<TA>::p2(sum.z, sum.w);
    const int yrow = SEG ? op->perm[row0 + tl] : tl;
    *reinterpret_cast<uint2*>(Y + (size_t)yrow * N + n) = out;
  }
  if (S > 1) {
    // returns once every CTA of the cluster has received all its bytes (each
    // arrives after finitely many bounded waits); if this CTA's own bytes had
    // not all landed, give the late ones one more bounded wait before its
    // shared memory goes away
    __syncwarp();
    cluster_wait_acquire();
    if (!landed) mbar_wait_bounded(inbar, 0);
  }
}

}  // namespace paro

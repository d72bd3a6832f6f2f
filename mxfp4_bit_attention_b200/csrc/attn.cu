// attn.cu -- fused MXFP4 attention with Pre-Normalization Quantization on tcgen05.
//
// Method: "MXAttention: Data-Free Optimal Scaling and Pre-Normalization Quantization for
// MXFP4 Attention" -- Pith review page, Fig. 4 (FlashAttention loop; PNQ quantizes the
// unnormalized exponential tile once and feeds the same quantized tile to the row sum l and
// to the output update; direct placement uses the unquantized tile for l) and Fig. 1 (UOS
// scaling for every MXFP4 tensor in attention); 10100.com article (same mechanism).
//
// One CTA owns 128 query rows of one head and sweeps all keys in tiles of 64:
//   warp 4 (one lane)  bulk-copies Q^ once and K^/V^ tiles + their scale atoms into a
//                      4-stage shared-memory ring;
//   warp 5             issues S = Q^ K^T (tcgen05.mma kind::mxf4 block-scaled, fp32 in TMEM);
//   warp 6             issues O~ += P^ V^ (same kind, fp32 in TMEM); the two issuers split the
//                      serial per-tile cost of tcgen05 issue and mbarrier waits;
//   warps 0-3          one query row per thread: read S from TMEM, online max (optionally lazy,
//                      threshold tau in log2 units), P~ = 2^(S*c - m) folded with the MXFP4 scale
//                      of each 32-key group, E2M1 codes of P~ written to shared memory in the
//                      MMA operand layout, group scales written as a scale atom, O~ rescaled in
//                      TMEM when the running max moves, and finally O = O~ / l.
// PNQ row sum: V^'s operand image carries 16 extra rows after its d channel rows, the first
// all ones (scale 2^0), so the PV MMA also accumulates l = sum_k P^_k into O~ column d, with the
// same codes, the same scales and the same rescaling as the output: the row sum is the sum of
// the quantized tile by construction.  Direct placement (pnq = 0) sums P~ in registers instead.
// The exp2s are split between MUFU (ex2.approx) and an FMA-pipe polynomial so that neither
// pipe alone bounds the softmax.
// Two CTAs share an SM (256 TMEM columns each), so one CTA's softmax overlaps the other's MMAs.
// Every wait is bounded; on expiry the CTA records a status word, drains its in-flight copies
// and MMAs, frees its TMEM and exits.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <type_traits>

#include "kernels.cuh"
#include "ptx.cuh"

namespace mxattn {

constexpr int kBM = 128;        // query rows per CTA
constexpr int kBN = 64;         // keys per tile
// Kernel variants: the fixed-shape full-attention pass (timed), the same with the diagnostic dump
// of one CTA, and the masked variant (causal masking and/or a packed varlen batch).
enum { kModeFull = 0, kModeDump = 1, kModeMasked = 2 };
constexpr int kStages = 4;      // K/V shared-memory ring depth
// Warps 0-3 run the softmax (warp w reads TMEM lanes 32w..32w+31); the producer and the two MMA
// issuers take three of the warps after them (where they sit was measured not to matter).
#ifndef MXATTN_PRODUCER_WARP
#define MXATTN_PRODUCER_WARP 4
#endif
#ifndef MXATTN_QK_WARP
#define MXATTN_QK_WARP 5
#endif
#ifndef MXATTN_PV_WARP
#define MXATTN_PV_WARP 6
#endif
constexpr int kProducerWarp = MXATTN_PRODUCER_WARP;
constexpr int kQkWarp = MXATTN_QK_WARP;
constexpr int kPvWarp = MXATTN_PV_WARP;
constexpr int kWarps = 1 + (kProducerWarp > kQkWarp ? (kProducerWarp > kPvWarp ? kProducerWarp : kPvWarp)
                                                    : (kQkWarp > kPvWarp ? kQkWarp : kPvWarp));
constexpr int kThreads = 32 * kWarps;  // 224 with the default roles
static_assert(kProducerWarp >= 4 && kQkWarp >= 4 && kPvWarp >= 4 && kProducerWarp != kQkWarp &&
                  kProducerWarp != kPvWarp && kQkWarp != kPvWarp, "warp roles");
constexpr int kOnesRows = 16;   // rows appended to V^: row 0 all ones, rows 1..15 zero
constexpr uint32_t kTmemCols = 256;
// Budget of the waits that drain in-flight copies and MMAs before a CTA exits (normal or
// aborted): they always complete, so they get the full default budget whatever the caller set.
constexpr long long kDrainBudgetCycles = 2000000000LL;
#ifndef MXATTN_POLY_WORDS
#define MXATTN_POLY_WORDS 1
#endif
// Of the four 8-key words of each 32-key group, this many take their exp2 from the FMA-pipe
// polynomial instead of MUFU.
constexpr int kPolyWords = MXATTN_POLY_WORDS;

// NVF: the NVFP4 comparison format (E4M3 scales per 16 elements: one 512-byte scale atom per
// 64 contraction elements, so Q/K carry D/64 atoms per tile and V one atom per 64-key tile).
template <int D, bool NVF = false>
struct Layout {
  // K/V scale-factor slots in TMEM, reused every SLOTS tiles.  A slot's last reader, QK(j-SLOTS)
  // or PV(j-SLOTS), is complete when it is overwritten for any SLOTS >= 2 (see the issuers);
  // NVFP4's larger scale atoms fit the 256 columns with 2.
  static constexpr int SLOTS = NVF ? 2 : 3;
  static constexpr int QK_ATOMS = NVF ? D / 64 : 1;  // scale atoms of a Q tile / 128-key K tile
  static constexpr int SFQ_BYTES = 512 * QK_ATOMS;
  static constexpr int SFK_BYTES = 512 * QK_ATOMS;
  static constexpr uint32_t ONES_SCALE = NVF ? 0x38383838u : 0x7F7F7F7Fu;  // 1.0 in E4M3 / E8M0
  // shared memory, byte offsets from a 1024-byte aligned base
  static constexpr int Q_BYTES = kBM * D / 2;
  static constexpr int K_BYTES = kBN * D / 2;
  static constexpr int V_BYTES = D * kBN / 2;
  static constexpr int ONES_BYTES = kOnesRows * kBN / 2;
  static constexpr int STAGE_BYTES = K_BYTES + V_BYTES + ONES_BYTES;
  static constexpr int Q_CODES = 0;
  static constexpr int STAGE0 = Q_BYTES;
  static constexpr int P_BYTES = kBM * kBN / 2;
  static constexpr int P_CODES = STAGE0 + kStages * STAGE_BYTES;  // two P buffers
  static constexpr int SF_Q = P_CODES + 2 * P_BYTES;
  static constexpr int SF_P = SF_Q + SFQ_BYTES;                   // two scale atoms
  static constexpr int SF_ONES = SF_P + 2 * 512;  // scale atom of the ones rows (constant)
  static constexpr int SF_K = SF_ONES + 512;
  static constexpr int SF_V = SF_K + kStages * SFK_BYTES;
  static constexpr int BARS = SF_V + kStages * 512;
  enum {
    B_Q = 0,
    B_KV_FULL = 1,
    B_KV_EMPTY = 1 + kStages,
    B_S_FULL = 1 + 2 * kStages,
    B_S_FREE,
    B_P_FULL,                 // two: one per P buffer
    B_O_DONE = B_P_FULL + 2,  // two: PV MMAs of even and odd tiles
    B_DRAIN = B_O_DONE + 2,
    NUM_BARS
  };
  static constexpr int TMEM_SLOT = BARS + NUM_BARS * 8;
  static constexpr int ABORT = TMEM_SLOT + 4;
  static constexpr int TOTAL = ABORT + 4;
  // slack for aligning the base; at least 80 KB so that no third CTA (which would block in
  // tcgen05.alloc until a neighbour frees its columns) becomes resident on an SM
  static constexpr int DYN_SMEM = TOTAL + 1024 > 80 * 1024 ? TOTAL + 1024 : 80 * 1024;
  static_assert(STAGE_BYTES % 512 == 0, "K tiles need 512-byte alignment");
  // tensor memory columns
  static constexpr uint32_t T_S = 0;
  static constexpr uint32_t T_O = 64;                      // O~: D columns, then l at column D
  static constexpr uint32_t T_SFQ = T_O + D + kOnesRows;
  static constexpr uint32_t T_SFP = T_SFQ + 4 * QK_ATOMS;     // 2 x 4 columns
  static constexpr uint32_t T_SFK = T_SFP + 8;                // SLOTS x (4 QK_ATOMS) columns
  static constexpr uint32_t SFK_COLS = 4 * QK_ATOMS;
  static constexpr uint32_t T_SFV = T_SFK + SFK_COLS * SLOTS;  // SLOTS x 8 columns (V atom + ones atom)
  static_assert(T_SFV + 8 * SLOTS <= kTmemCols, "TMEM budget");
  static constexpr uint32_t QK_LAYOUT = D == 128 ? kLayoutSW64 : kLayoutSW32;
};

__device__ __forceinline__ void raise_abort(volatile int* flag, int* status, int where) {
  *flag = 1;
  if (atomicCAS(status, 0, kStatusTimeout) == 0) atomicExch(status + 1, where);
}

// Group maximum of 32 raw S values (MASK: keys at index >= valid are excluded).
#ifndef MXATTN_MAX_CHAINS
#define MXATTN_MAX_CHAINS 2
#endif
template <bool MASK>
__device__ __forceinline__ float group_max(const uint32_t (&s)[32], int base, int valid) {
  constexpr int C = MXATTN_MAX_CHAINS;  // independent max chains
  float m[C];
#pragma unroll
  for (int k = 0; k < C; k++) m[k] = -INFINITY;
#pragma unroll
  for (int i = 0; i < 32; i += 2 * C) {
#pragma unroll
    for (int k = 0; k < C; k++) {
      float v0 = __uint_as_float(s[i + 2 * k]), v1 = __uint_as_float(s[i + 2 * k + 1]);
      if (MASK) {
        v0 = base + i + 2 * k < valid ? v0 : -INFINITY;
        v1 = base + i + 2 * k + 1 < valid ? v1 : -INFINITY;
      }
      m[k] = fmax3(m[k], v0, v1);
    }
  }
#pragma unroll
  for (int k = 1; k < C; k++) m[0] = fmaxf(m[0], m[k]);
  return m[0];
}

// E2M1 codes of one group of 32: p = 2^((S - sm) c - e), 4 packed words.  S - sm is formed first,
// exactly for every score near the running max (and 0 for a score equal to it), as the oracle's
// exp(x - m) is: a score equal to the running max gives 2^-e exactly, which for e = 2 is the
// E2M1 midpoint 0.25 that rounds to 0.  Direct placement also accumulates the unquantized p.
template <bool MASK, bool SUM>
__device__ __forceinline__ void group_codes(const uint32_t (&s)[32], int base, int valid, float c, float sm,
                                            float e, uint32_t* w, float& psum) {
  const float2 cc = make_float2(c, c);
  const float2 ne = make_float2(-e, -e);
  const float2 nsm = make_float2(-sm, -sm);
#pragma unroll
  for (int q = 0; q < 4; q++) {
    float p[8];
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      const float2 d = __fadd2_rn(make_float2(__uint_as_float(s[q * 8 + i]), __uint_as_float(s[q * 8 + i + 1])), nsm);
      const float2 x = __ffma2_rn(d, cc, ne);
      if (q >= 4 - kPolyWords) {
        const float2 y = exp2_poly2(x);
        p[i] = y.x;
        p[i + 1] = y.y;
      } else {
        p[i] = ex2_approx(x.x);
        p[i + 1] = ex2_approx(x.y);
      }
      if (MASK) {
        p[i] = base + q * 8 + i < valid ? p[i] : 0.f;
        p[i + 1] = base + q * 8 + i + 1 < valid ? p[i + 1] : 0.f;
      }
      if (SUM) psum += p[i] + p[i + 1];
    }
    w[q] = cvt_e2m1x8(p[0], p[1], p[2], p[3], p[4], p[5], p[6], p[7]);
  }
}

// NVFP4 (comparison format) blocks of 16 keys: s[off..off+15] holds keys base..base+15.
template <bool MASK>
__device__ __forceinline__ float block16_max(const uint32_t (&s)[32], int off, int base, int valid) {
  float m[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int i = 0; i < 16; i += 4) {
#pragma unroll
    for (int k = 0; k < 2; k++) {
      float v0 = __uint_as_float(s[off + i + 2 * k]), v1 = __uint_as_float(s[off + i + 2 * k + 1]);
      if (MASK) {
        v0 = base + i + 2 * k < valid ? v0 : -INFINITY;
        v1 = base + i + 2 * k + 1 < valid ? v1 : -INFINITY;
      }
      m[k] = fmax3(m[k], v0, v1);
    }
  }
  return fmaxf(m[0], m[1]);
}

// E2M1 codes of one block of 16: p = 2^(S*c - bias), 2 packed words (POLY: the second word's
// exp2 from the FMA-pipe polynomial).
template <bool MASK, bool SUM, bool POLY>
__device__ __forceinline__ void block16_codes(const uint32_t (&s)[32], int off, int base, int valid, float c,
                                              float bias, uint32_t* w, float& psum) {
  const float2 cc = make_float2(c, c);
  const float2 nb = make_float2(-bias, -bias);
#pragma unroll
  for (int q = 0; q < 2; q++) {
    float p[8];
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      const float2 x = __ffma2_rn(
          make_float2(__uint_as_float(s[off + q * 8 + i]), __uint_as_float(s[off + q * 8 + i + 1])), cc, nb);
      if (POLY && q == 1) {
        const float2 y = exp2_poly2(x);
        p[i] = y.x;
        p[i + 1] = y.y;
      } else {
        p[i] = ex2_approx(x.x);
        p[i + 1] = ex2_approx(x.y);
      }
      if (MASK) {
        p[i] = base + q * 8 + i < valid ? p[i] : 0.f;
        p[i + 1] = base + q * 8 + i + 1 < valid ? p[i + 1] : 0.f;
      }
      if (SUM) psum += p[i] + p[i + 1];
    }
    w[q] = cvt_e2m1x8(p[0], p[1], p[2], p[3], p[4], p[5], p[6], p[7]);
  }
}

// NVFP4 exponential tiles: P~ <= 1 is scaled by 448 * 6 before its blocks take their E4M3
// scales, so that the block holding the running max (P~ = 1) gets scale 448 and code 6; the
// factor cancels in O~ / l (both accumulate the scaled codes).
constexpr float kLog2NvScale = 11.392317422778760f;  // log2(448 * 6)
constexpr float kLog2E4m3Max = 8.807354922057604f;   // log2(448)

template <int D, int DT, bool PNQ, int MODE, bool NVF>
__global__ void __launch_bounds__(kThreads, 2) mxattn_fwd_kernel(const AttnArgs a) {
  using L = Layout<D, NVF>;
  constexpr bool DUMP = MODE == kModeDump;
  constexpr bool MASKED = MODE == kModeMasked;
  constexpr int NV = PNQ ? D + kOnesRows : D;  // N of the PV MMA
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool causal = MASKED && a.causal;
  // The problem of this CTA: query tile qt (rows 128qt..) of head bh, with Nq query rows and Nk
  // keys; the packed operand tiles it reads and where its output rows go.  Under causal masking
  // the longest query tiles (the last ones) are launched first, so that the short ones fill in
  // behind them.
  const int bh = blockIdx.y;
  int Nq = a.N, Nk = a.Nk, qt;
  size_t q_tile, k_tile0, v_tile0;  // Q tile, first 128-key K tile / scale atom, first 64-key V tile
  size_t out_row0, out_step;        // output element offset of query row 0, and per row
  if (MASKED && a.vl.cu_seqlens != nullptr) {
    // packed varlen batch: blockIdx.x runs over the tiles of all sequences; token-major [T, H, d]
    const int g = causal ? a.vl.tiles_per_head - 1 - (int)blockIdx.x : (int)blockIdx.x;
    if (g >= __ldg(a.vl.tile_off + a.vl.nseq)) return;  // past the last sequence: the whole CTA
    const int sq = varlen_sequence(a.vl, g);
    const int start = __ldg(a.vl.cu_seqlens + sq);
    Nq = Nk = __ldg(a.vl.cu_seqlens + sq + 1) - start;
    const int t0 = __ldg(a.vl.tile_off + sq);
    qt = g - t0;
    q_tile = (size_t)bh * a.vl.tiles_per_head + g;
    k_tile0 = (size_t)bh * a.vl.tiles_per_head + t0;
    v_tile0 = 2 * k_tile0;
    out_row0 = ((size_t)start * a.BH + bh) * D;
    out_step = (size_t)a.BH * D;
  } else {
    const int T128 = (a.N + 127) / 128;
    qt = causal ? T128 - 1 - (int)blockIdx.x : (int)blockIdx.x;
    q_tile = (size_t)bh * T128 + qt;
    k_tile0 = (size_t)bh * ((a.Nk + 127) / 128);
    v_tile0 = (size_t)bh * ((a.Nk + 63) / 64);
    out_row0 = (size_t)bh * a.N * D;
    out_step = D;
  }
  const int T64 = (Nk + 63) / 64;  // 64-key tiles of the problem
  // tiles the CTA sweeps: all, or under causal masking those up to its diagonal
  const int TJ = causal ? (2 * qt + 2 < T64 ? 2 * qt + 2 : T64) : T64;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::ABORT);
  __shared__ int never;  // a flag nothing sets: drains ignore the abort flag
  auto bar = [&](int i) -> uint32_t { return sb + L::BARS + 8 * i; };

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    never = 0;
    mbar_init(bar(L::B_Q), 1);
    for (int s = 0; s < kStages; s++) {
      mbar_init(bar(L::B_KV_FULL + s), 1);
      mbar_init(bar(L::B_KV_EMPTY + s), 1);
    }
    mbar_init(bar(L::B_S_FULL), 1);
    mbar_init(bar(L::B_S_FREE), 4);
    mbar_init(bar(L::B_P_FULL), 4);
    mbar_init(bar(L::B_P_FULL + 1), 4);
    mbar_init(bar(L::B_O_DONE), 1);
    mbar_init(bar(L::B_O_DONE + 1), 1);
    mbar_init(bar(L::B_DRAIN), 2);  // one commit from each issuer
    fence_mbar_init();
  }
  if (PNQ) {
    // the ones rows of every stage (row 0: code 1.0 = 0x2 in every nibble; rows 1..15: zero) and
    // their scale atom (row 0, every key group: 2^0; everything else zero)
    for (int i = threadIdx.x; i < kStages * L::ONES_BYTES / 4; i += kThreads) {
      const int st = i / (L::ONES_BYTES / 4), off = i % (L::ONES_BYTES / 4);
      reinterpret_cast<uint32_t*>(smem + L::STAGE0 + st * L::STAGE_BYTES + L::K_BYTES + L::V_BYTES)[off] =
          off < (kBN / 2) / 4 ? 0x22222222u : 0u;
    }
    for (int i = threadIdx.x; i < 512 / 4; i += kThreads)
      reinterpret_cast<uint32_t*>(smem + L::SF_ONES)[i] = i == 0 ? L::ONES_SCALE : 0u;
    fence_proxy_async_smem();
  }
  if (warp == kQkWarp) {
    tmem_alloc(sb + L::TMEM_SLOT, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + L::TMEM_SLOT);
  const volatile int* no_abort = &never;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      bool ok = true;
      int issued = 0;
      mbar_arrive_expect_tx(bar(L::B_Q), L::Q_BYTES + L::SFQ_BYTES);
      bulk_g2s(sb + L::Q_CODES, a.q_codes + q_tile * (size_t)L::Q_BYTES, L::Q_BYTES, bar(L::B_Q));
      bulk_g2s(sb + L::SF_Q, a.q_scales + q_tile * L::SFQ_BYTES, L::SFQ_BYTES, bar(L::B_Q));
      for (int j = 0; j < TJ; j++) {
        const int s = j % kStages;
        if (j >= kStages) {
          ok = mbar_wait(bar(L::B_KV_EMPTY + s), ((j / kStages) - 1) & 1, abort_flag, a.wait_budget);
          if (!ok) break;
        }
        const uint32_t fb = bar(L::B_KV_FULL + s);
        const size_t t128 = k_tile0 + j / 2;
        mbar_arrive_expect_tx(fb, L::K_BYTES + L::V_BYTES + L::SFK_BYTES + 512);
        bulk_g2s(sb + L::STAGE0 + s * L::STAGE_BYTES,
                 a.k_codes + (t128 * kBM + (j % 2) * kBN) * (size_t)(D / 2), L::K_BYTES, fb);
        bulk_g2s(sb + L::SF_K + s * L::SFK_BYTES, a.k_scales + t128 * L::SFK_BYTES, L::SFK_BYTES, fb);
        bulk_g2s(sb + L::STAGE0 + s * L::STAGE_BYTES + L::K_BYTES,
                 a.v_codes + (v_tile0 + j) * (size_t)L::V_BYTES, L::V_BYTES, fb);
        // V scales: MXFP4 one atom per 128-key tile (both 64-key halves), NVFP4 one per 64-key tile
        bulk_g2s(sb + L::SF_V + s * 512, a.v_scales + (NVF ? v_tile0 + j : t128) * 512, 512, fb);
        issued = j + 1;
      }
      if (!ok) raise_abort(abort_flag, a.status, 1);
      // Let every copy issued land before the CTA can exit, whichever warp gave up (another warp
      // may abort after this loop finished).  In a normal run these phases have long completed
      // and nothing newer was issued, so each wait returns at once.
      mbar_wait(bar(L::B_Q), 0, no_abort, kDrainBudgetCycles);
      for (int j = (issued > kStages ? issued - kStages : 0); j < issued; j++)
        mbar_wait(bar(L::B_KV_FULL + j % kStages), (j / kStages) & 1, no_abort, kDrainBudgetCycles);
    }
  } else if (warp == kQkWarp) {
    // ------------------------------------------------------------------ QK issuer
    // The warp runs the loop converged (waits and descriptor arithmetic stay warp-uniform); lane 0
    // alone issues its tcgen05 operations, so that each of its commits covers all of them.
    const bool leader = lane == 0;
    bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar(L::B_Q), 0, abort_flag, a.wait_budget));
    if (ok) {
      tc_fence_after();
      if (leader)
        for (int at = 0; at < L::QK_ATOMS; at++) tmem_cp_sf_atom(tmem + L::T_SFQ + 4 * at, sb + L::SF_Q + 512 * at);
      __syncwarp();
      const uint64_t qdesc = smem_desc(sb + L::Q_CODES, 16, 8 * (D / 2), L::QK_LAYOUT);
      for (int j = 0; j < TJ; j++) {
        const int s = j % kStages, f = j % L::SLOTS;
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar(L::B_KV_FULL + s), (j / kStages) & 1, abort_flag, a.wait_budget));
        if (!ok) break;
        tc_fence_after();
        // K scale slot f was last read by QK(j - SLOTS), complete since the softmax read that S
        // before releasing it, which this warp waited for before issuing QK(j - 1)
        if (leader)
          for (int at = 0; at < L::QK_ATOMS; at++)
            tmem_cp_sf_atom(tmem + L::T_SFK + L::SFK_COLS * f + 4 * at, sb + L::SF_K + L::SFK_BYTES * s + 512 * at);
        if (j > 0) {
          ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar(L::B_S_FREE), (j - 1) & 1, abort_flag, a.wait_budget));
          if (!ok) break;
          tc_fence_after();
        }
        const uint64_t kdesc = smem_desc(sb + L::STAGE0 + s * L::STAGE_BYTES, 16, 8 * (D / 2), L::QK_LAYOUT);
        if (leader) {
#pragma unroll
          for (int kb = 0; kb < D / 64; kb++) {
            // K block kb covers head dims 64kb..64kb+63: 32 bytes further along each row;
            // MXFP4: scale bytes 2kb and 2kb+1 of each row's scale word; NVFP4: scale atom kb.
            // The K tile's 64 keys are rows 64(j&1).. of its 128-key atom: columns 2(j&1)..
            if (NVF)
              mma_nvf4(tmem + L::T_S, qdesc + (uint64_t)(kb * 2), kdesc + (uint64_t)(kb * 2), nvf4_idesc(kBM, kBN),
                       tmem + L::T_SFQ + 4 * kb, tmem + L::T_SFK + L::SFK_COLS * f + 4 * kb + 2 * (j & 1),
                       kb > 0 ? 1u : 0u);
            else
              mma_mxf4(tmem + L::T_S, qdesc + (uint64_t)(kb * 2), kdesc + (uint64_t)(kb * 2),
                       mxf4_idesc(kBM, kBN, 2 * kb, 2 * kb), tmem + L::T_SFQ,
                       tmem + L::T_SFK + 4 * f + 2 * (j & 1), kb > 0 ? 1u : 0u);
          }
        }
        if (j >= 2) {
          // S(j) also tells the softmax that P buffer j&1 (last read by PV(j-2)) is free: see
          // PV(j-2) complete before committing S(j) (the MMAs above, which touch neither P nor O~,
          // already run meanwhile).  Each O_DONE barrier is at most one phase away from it.
          ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar(L::B_O_DONE + (j & 1)), ((j - 2) >> 1) & 1, abort_flag, a.wait_budget));
          if (!ok) break;
          tc_fence_after();
        }
        if (leader) mma_commit(bar(L::B_S_FULL));
        __syncwarp();
      }
    }
    if (!ok && leader) raise_abort(abort_flag, a.status, 2);
    // wait for every tcgen05 operation of both issuers before TMEM is released
    if (leader) mma_commit(bar(L::B_DRAIN));
    __syncwarp();
    mbar_wait(bar(L::B_DRAIN), 0, no_abort, kDrainBudgetCycles);
  } else if (warp == kPvWarp) {
    // ------------------------------------------------------------------ PV issuer (same scheme)
    const bool leader = lane == 0;
    if (PNQ && leader)
      for (int f = 0; f < L::SLOTS; f++) tmem_cp_sf_atom(tmem + L::T_SFV + 8 * f + 4, sb + L::SF_ONES);
    __syncwarp();
    bool ok = true;
    // With three scale slots the V atom of tile jp is copied before P(jp) is awaited, off the path
    // from P(jp) to PV(jp): its slot was last read by PV(jp-3), complete once S(jp-1) was committed
    // (the QK issuer saw PV(jp-3) finish first), which P(jp-1) arriving implies.
    constexpr bool kEarlyV = L::SLOTS >= 3;
    auto copy_v_scales = [&](int sp, int fp) {
      if (PNQ && D == 64) {
        // with d = 64 the ones row is B-operand row 64, inside the V scale atom (whose
        // channels >= d are zero): give it scale 1 for all four key groups
        *reinterpret_cast<volatile uint32_t*>(smem + L::SF_V + 512 * sp + 8) = L::ONES_SCALE;
        fence_proxy_async_smem();
      }
      tmem_cp_sf_atom(tmem + L::T_SFV + 8 * fp, sb + L::SF_V + 512 * sp);
    };
    for (int jp = 0; jp < TJ; jp++) {
      const int sp = jp % kStages, fp = jp % L::SLOTS, pb = jp & 1;
      // V^(jp) landed with K^(jp), before S(jp) and so before P(jp); this warp also waits for the
      // stage itself (it cannot have been refilled: that needs this warp's commit below)
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar(L::B_KV_FULL + sp), (jp / kStages) & 1, abort_flag, a.wait_budget));
      if (!ok) break;
      tc_fence_after();
      if (kEarlyV && leader) copy_v_scales(sp, fp);
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar(L::B_P_FULL + pb), (jp >> 1) & 1, abort_flag, a.wait_budget));
      if (!ok) break;
      tc_fence_after();
      const uint64_t pdesc = smem_desc(sb + L::P_CODES + pb * L::P_BYTES, 16, 8 * (kBN / 2), kLayoutSW32);
      const uint64_t vdesc =
          smem_desc(sb + L::STAGE0 + sp * L::STAGE_BYTES + L::K_BYTES, 16, 8 * (kBN / 2), kLayoutSW32);
      if (leader) {
        // P scale slot pb (and, without the early copy, V scale slot fp) were last read by PV(jp-2)
        // (and PV(jp-SLOTS)), complete before S(jp) was committed, which the softmax saw before
        // writing P(jp)
        tmem_cp_sf_atom(tmem + L::T_SFP + 4 * pb, sb + L::SF_P + 512 * pb);
        if (!kEarlyV) copy_v_scales(sp, fp);
        if (NVF)
          mma_nvf4(tmem + L::T_O, pdesc, vdesc, nvf4_idesc(kBM, NV), tmem + L::T_SFP + 4 * pb, tmem + L::T_SFV + 8 * fp,
                   jp > 0 ? 1u : 0u);
        else
          mma_mxf4(tmem + L::T_O, pdesc, vdesc, mxf4_idesc(kBM, NV, 0, 2 * (jp & 1)), tmem + L::T_SFP + 4 * pb,
                   tmem + L::T_SFV + 8 * fp, jp > 0 ? 1u : 0u);
        mma_commit(bar(L::B_O_DONE + (jp & 1)));
        // QK(jp) read the stage too: complete, since the softmax saw S(jp) before P(jp)
        mma_commit(bar(L::B_KV_EMPTY + sp));
      }
      __syncwarp();
    }
    if (!ok && leader) raise_abort(abort_flag, a.status, 4);
    if (leader) mma_commit(bar(L::B_DRAIN));
    __syncwarp();
    mbar_wait(bar(L::B_DRAIN), 0, no_abort, kDrainBudgetCycles);
  } else if (warp < 4) {
    // ------------------------------------------------------------------ softmax (warps 0-3)
    const int row = threadIdx.x;  // TMEM lane and query row within the tile
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    const float c = a.scale_log2;
    const bool dumping = DUMP && bh == a.dump_bh && qt == a.dump_qt;
    const DumpLayout dl(D, T64);
    // keys this row sees: all Nk, or under causal masking those up to its own position
    const int kmax = causal ? (qt * kBM + row + 1 < Nk ? qt * kBM + row + 1 : Nk) : Nk;
    float sm = -INFINITY;  // running max of S used for the exponent (raw MMA units)
    float m2 = -INFINITY;  // the same in log2 units, fl32(sm * c)
    float l = 0.f;         // direct placement only (PNQ keeps l in O~ column D)
    bool ok = true;
    bool s_ready = false;  // S(j) was seen complete by the early test during tile j-1
    // one key tile; FULL: all 64 keys are inside N (every tile but possibly the last), so the
    // main loop carries no masking
    auto tile = [&](int j, auto full_tag) -> bool {
      constexpr bool FULL = decltype(full_tag)::value;
      if (!__all_sync(0xFFFFFFFFu, s_ready)) {
        ok = mbar_wait(bar(L::B_S_FULL), j & 1, abort_flag, a.wait_budget);
        if (!__all_sync(0xFFFFFFFFu, ok)) return false;
      }
      tc_fence_after();
      uint32_t s0[32], s1[32];
      tmem_ld64_wait(tl + L::T_S, tl + L::T_S + 32, s0, s1);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::B_S_FREE));
      if (dumping && j < 2) {
        float* ds = reinterpret_cast<float*>(a.dump + dl.s) + ((size_t)j * 128 + row) * 64;
        for (int i = 0; i < 32; i++) {
          ds[i] = __uint_as_float(s0[i]);
          ds[32 + i] = __uint_as_float(s1[i]);
        }
      }

      const int valid = FULL ? kBN : kmax - j * kBN;  // this row's keys in the tile (may be <= 0)
      constexpr int NG = NVF ? 4 : 2;  // scale groups of the tile (MXFP4: 32 keys, NVFP4: 16)
      float gmax[NG];
      if constexpr (NVF) {
        gmax[0] = block16_max<!FULL>(s0, 0, 0, valid);
        gmax[1] = block16_max<!FULL>(s0, 16, 16, valid);
        gmax[2] = block16_max<!FULL>(s1, 0, 32, valid);
        gmax[3] = block16_max<!FULL>(s1, 16, 48, valid);
      } else if (FULL) {
        gmax[0] = group_max<false>(s0, 0, valid);
        gmax[1] = group_max<false>(s1, 32, valid);
      } else {
        gmax[0] = group_max<true>(s0, 0, valid);
        gmax[1] = group_max<true>(s1, 32, valid);
      }
      // Running max kept in raw S units (sm) and in log2 units (m2 = fl32(sm * c)).  A group's
      // maximum is taken as 2^((gmax - sm) * c): exactly 1 for the group that holds the running
      // max, as exp(0) is in the oracle, so scale rules whose boundaries sit on powers of two
      // (OCP, q = 4 or 8) decide it the same way.
      float mt_raw = fmaxf(gmax[0], gmax[1]);
      if constexpr (NVF) mt_raw = fmaxf(mt_raw, fmaxf(gmax[2], gmax[3]));
      const bool move = j == 0 || (mt_raw * c > m2 + a.tau);
      // O~ and l are rescaled by alpha = 2^(m_old - m_new) only when some row of the warp moves
      // its max (alpha = 1 elsewhere); tile 0 starts both at zero
      const bool any_move = j > 0 && __any_sync(0xFFFFFFFFu, move);
      const float sm_old = sm;
      if (move) sm = mt_raw;
      m2 = sm * c;
      float alpha = 1.f;
      if (any_move && move) alpha = ex2_approx((sm_old - sm) * c);

      uint32_t eb[NG];  // scale bytes (E8M0; NVFP4: E4M3)
      float bias[NG];   // MXFP4: the groups' exponents e; NVFP4: the exp2 argument's offset
      float sc[NG];     // NVFP4: the scales' values
      (void)sc;
      if constexpr (NVF) {
        // block b: y = P~ * 448 * 6, scale = E4M3(max y / 6) = E4M3(2^((gmax - sm) c + log2 448)),
        // codes of y / scale = 2^(S c - m2 + log2(448 * 6) - log2 scale); a zero scale (a block
        // far below the running max, or all masked) zeroes the block
#pragma unroll
        for (int g = 0; g < 4; g += 2) {
          const uint32_t b2 = cvt_e4m3x2(ex2_approx((gmax[g] - sm) * c + kLog2E4m3Max),
                                         ex2_approx((gmax[g + 1] - sm) * c + kLog2E4m3Max));
          const float2 sv = e4m3x2_to_float2(b2);
          eb[g] = b2 & 0xFFu;
          eb[g + 1] = b2 >> 8;
          sc[g] = sv.x;
          sc[g + 1] = sv.y;
          bias[g] = sv.x > 0.f ? m2 - kLog2NvScale + lg2_approx(sv.x) : INFINITY;
          bias[g + 1] = sv.y > 0.f ? m2 - kLog2NvScale + lg2_approx(sv.y) : INFINITY;
        }
      } else {
#pragma unroll
        for (int g = 0; g < 2; g++) bias[g] = shared_exponent_log2f((gmax[g] - sm) * c, a.rule, eb[g]);  // e
      }
      uint32_t w[8];
      float psum[NG] = {};
      if constexpr (NVF) {
        block16_codes<!FULL, !PNQ, false>(s0, 0, 0, valid, c, bias[0], w, psum[0]);
        block16_codes<!FULL, !PNQ, true>(s0, 16, 16, valid, c, bias[1], w + 2, psum[1]);
        block16_codes<!FULL, !PNQ, false>(s1, 0, 32, valid, c, bias[2], w + 4, psum[2]);
        block16_codes<!FULL, !PNQ, true>(s1, 16, 48, valid, c, bias[3], w + 6, psum[3]);
      } else if (FULL) {
        group_codes<false, !PNQ>(s0, 0, valid, c, sm, bias[0], w, psum[0]);
        group_codes<false, !PNQ>(s1, 32, valid, c, sm, bias[1], w + 4, psum[1]);
      } else {
        group_codes<true, !PNQ>(s0, 0, valid, c, sm, bias[0], w, psum[0]);
        group_codes<true, !PNQ>(s1, 32, valid, c, sm, bias[1], w + 4, psum[1]);
      }
      // P buffer pb was last read by PV(j-2), which the QK issuer saw complete before it
      // committed S(j).  With MXFP4 P the stores go before the S test below, whose memory clobber
      // would otherwise hold them behind it (2.5% at 720p); with NVFP4 P they go after the
      // rescale, which measured 2.5% faster for that format.
      const int pb = j & 1;
      auto store_p = [&]() {
        uint8_t* prow = smem + L::P_CODES + pb * L::P_BYTES + row * (kBN / 2);
        const int sw = (row >> 2) & 1;
        *reinterpret_cast<uint4*>(prow + (sw * 16)) = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4*>(prow + ((1 ^ sw) * 16)) = make_uint4(w[4], w[5], w[6], w[7]);
        if constexpr (NVF)
          *reinterpret_cast<uint32_t*>(smem + L::SF_P + pb * 512 + (row % 32) * 16 + (row / 32) * 4) =
              eb[0] | (eb[1] << 8) | (eb[2] << 16) | (eb[3] << 24);
        else
          *reinterpret_cast<uint16_t*>(smem + L::SF_P + pb * 512 + (row % 32) * 16 + (row / 32) * 4) =
              (uint16_t)(eb[0] | (eb[1] << 8));
      };
      if constexpr (!NVF) store_p();
      // test S(j+1) now, so that the test's latency overlaps the work below
      s_ready = j + 1 < TJ && mbar_test(bar(L::B_S_FULL), (j + 1) & 1);
      if (!PNQ) {
        float lsum = 0.f;
        if constexpr (NVF) {
#pragma unroll
          for (int g = 0; g < 4; g++) lsum += psum[g] * sc[g];  // in units of y, as the PNQ sum
        } else {
#pragma unroll
          for (int g = 0; g < 2; g++) lsum += psum[g] * __uint_as_float(eb[g] << 23);  // byte 0: 2^-127 -> 0
        }
        l = alpha * l + lsum;
      }

      // Rescaling O~ needs PV(j-1) complete.  Each O_DONE barrier (even / odd tiles) can be at
      // most one phase behind or ahead of the phase waited for here.
      if (any_move) {
        ok = mbar_wait(bar(L::B_O_DONE + ((j - 1) & 1)), ((j - 1) >> 1) & 1, abort_flag, a.wait_budget);
        if (!__all_sync(0xFFFFFFFFu, ok)) return false;
        tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < D / 32; cc++) {
          uint32_t o[32];
          tmem_ld32(tl + L::T_O + 32 * cc, o);
          tmem_wait_ld();
          pin32(o);
#pragma unroll
          for (int i = 0; i < 32; i++) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tl + L::T_O + 32 * cc, o);
        }
        if (PNQ) {
          uint32_t lv;
          tmem_ld1(tl + L::T_O + D, lv);
          tmem_wait_ld();
          pin1(lv);
          tmem_st1(tl + L::T_O + D, __float_as_uint(__uint_as_float(lv) * alpha));
        }
        tmem_wait_st();
      }
      if constexpr (NVF) store_p();
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::B_P_FULL + pb));
      if (dumping) {
        uint32_t* dp = reinterpret_cast<uint32_t*>(a.dump + dl.p_codes + ((size_t)j * 128 + row) * 32);
        for (int i = 0; i < 8; i++) dp[i] = w[i];
        uint8_t* dsf = a.dump + dl.p_scales + ((size_t)j * 128 + row) * 2;
        dsf[0] = (uint8_t)eb[0];
        dsf[1] = (uint8_t)eb[1];
        // the unquantized tile, relative to this tile's running max (dump only)
        float* dpt = reinterpret_cast<float*>(a.dump + dl.p_tilde) + ((size_t)j * 128 + row) * 64;
        for (int i = 0; i < 32; i++) {
          dpt[i] = i < valid ? ex2_approx(__fmaf_rn(__uint_as_float(s0[i]), c, -m2)) : 0.f;
          dpt[32 + i] = 32 + i < valid ? ex2_approx(__fmaf_rn(__uint_as_float(s1[i]), c, -m2)) : 0.f;
        }
        reinterpret_cast<float*>(a.dump + dl.m_tiles)[(size_t)j * 128 + row] = m2;
      }
      return true;
    };
    // tiles every row of the CTA sees in full, then the masked ones (the ragged last tile of the
    // keys; under causal masking the two diagonal tiles)
    int full_tiles = (Nk % kBN == 0) ? T64 : T64 - 1;
    if (causal && full_tiles > 2 * qt) full_tiles = 2 * qt;
    for (int j = 0; ok && j < full_tiles; j++) ok = tile(j, std::true_type{});
    if (MASKED) {
      for (int j = full_tiles; ok && j < TJ; j++) ok = tile(j, std::false_type{});
    } else if (ok && full_tiles < T64) {
      ok = tile(T64 - 1, std::false_type{});  // the ragged last tile
    }
    if (ok && TJ >= 2) {  // the last two PV MMAs, one on each O_DONE barrier
      ok = mbar_wait(bar(L::B_O_DONE + (TJ & 1)), ((TJ - 2) >> 1) & 1, abort_flag, a.wait_budget);
      ok = __all_sync(0xFFFFFFFFu, ok);
    }
    if (ok) {
      ok = mbar_wait(bar(L::B_O_DONE + ((TJ - 1) & 1)), ((TJ - 1) >> 1) & 1, abort_flag, a.wait_budget);
      ok = __all_sync(0xFFFFFFFFu, ok);
    }
    if (ok) {
      tc_fence_after();
      if (PNQ) {
        uint32_t lv;
        tmem_ld1(tl + L::T_O + D, lv);
        tmem_wait_ld();
        pin1(lv);
        l = __uint_as_float(lv);
      }
      const float inv_l = 1.f / l;
      const int qrow = qt * kBM + row;
      const bool store = qrow < Nq;
      const size_t obase = out_row0 + (size_t)(store ? qrow : 0) * out_step;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; cc++) {
        uint32_t o[32];
        tmem_ld32(tl + L::T_O + 32 * cc, o);
        tmem_wait_ld();
        pin32(o);
        if (dumping) {
          float* d_o = reinterpret_cast<float*>(a.dump + dl.o) + (size_t)row * D + 32 * cc;
          for (int i = 0; i < 32; i++) d_o[i] = __uint_as_float(o[i]);
          if (cc == 0) {
            reinterpret_cast<float*>(a.dump + dl.l)[row] = l;
            reinterpret_cast<float*>(a.dump + dl.m)[row] = m2;
          }
        }
        if (store) {
          if (DT == kBF16) {
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + obase + 32 * cc);
#pragma unroll
            for (int v = 0; v < 4; v++) {
              uint32_t pk[4];
#pragma unroll
              for (int i = 0; i < 4; i++) {
                const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(o[v * 8 + 2 * i]) * inv_l,
                                                                __uint_as_float(o[v * 8 + 2 * i + 1]) * inv_l);
                pk[i] = *reinterpret_cast<const uint32_t*>(&b2);
              }
              dst[v] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
          } else {
            float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + obase + 32 * cc);
#pragma unroll
            for (int v = 0; v < 8; v++)
              dst[v] = make_float4(__uint_as_float(o[4 * v]) * inv_l, __uint_as_float(o[4 * v + 1]) * inv_l,
                                   __uint_as_float(o[4 * v + 2]) * inv_l, __uint_as_float(o[4 * v + 3]) * inv_l);
          }
        }
      }
    }
    if (!ok) raise_abort(abort_flag, a.status, 3);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kQkWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, int DT, bool PNQ, bool NVF>
static cudaError_t launch_attention_t(const AttnArgs& a, cudaStream_t s) {
  using L = Layout<D, NVF>;
  // the diagnostic dump and the masking are separate instantiations, so the timed kernel carries
  // none of them; the NVFP4 comparison format runs full attention only
  const bool masked = a.causal || a.vl.cu_seqlens != nullptr;
  if (NVF && (masked || a.dump != nullptr)) return cudaErrorNotSupported;
  auto kern = NVF                 ? mxattn_fwd_kernel<D, DT, PNQ, kModeFull, NVF>
              : a.dump != nullptr ? mxattn_fwd_kernel<D, DT, PNQ, kModeDump, false>
              : masked            ? mxattn_fwd_kernel<D, DT, PNQ, kModeMasked, false>
                                  : mxattn_fwd_kernel<D, DT, PNQ, kModeFull, false>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::DYN_SMEM);
  if (err != cudaSuccess) return err;
  const unsigned qtiles = a.vl.cu_seqlens != nullptr ? (unsigned)a.vl.tiles_per_head : (unsigned)((a.N + kBM - 1) / kBM);
  dim3 grid(qtiles, (unsigned)a.BH);
  kern<<<grid, kThreads, L::DYN_SMEM, s>>>(a);
  return cudaGetLastError();
}

template <int D, int DT>
static cudaError_t launch_attention_d(const AttnArgs& a, cudaStream_t s) {
  const bool nv = a.fmt == kFmtNVFP4;
  if (a.pnq) return nv ? launch_attention_t<D, DT, true, true>(a, s) : launch_attention_t<D, DT, true, false>(a, s);
  return nv ? launch_attention_t<D, DT, false, true>(a, s) : launch_attention_t<D, DT, false, false>(a, s);
}

cudaError_t launch_attention(const AttnArgs& a, int D, int dtype, cudaStream_t s) {
  if (D == 128) return dtype == kBF16 ? launch_attention_d<128, kBF16>(a, s) : launch_attention_d<128, kFP32>(a, s);
  return dtype == kBF16 ? launch_attention_d<64, kBF16>(a, s) : launch_attention_d<64, kFP32>(a, s);
}

static_assert(Layout<128, true>::DYN_SMEM <= 113 * 1024 && Layout<128, false>::DYN_SMEM <= 113 * 1024,
              "two CTAs per SM");

}  // namespace mxattn

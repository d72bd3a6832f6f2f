// attn_wide.cu -- fused MXFP4 attention with Pre-Normalization Quantization on tcgen05, keys in
// tiles of 128 (opts.key_tile = 128).
//
// Method: "MXAttention: Data-Free Optimal Scaling and Pre-Normalization Quantization for
// MXFP4 Attention" -- Pith review page, Fig. 4 (FlashAttention loop; PNQ quantizes the
// unnormalized exponential tile once and feeds the same quantized tile to the row sum l and
// to the output update; direct placement uses the unquantized tile for l) and Fig. 1 (UOS
// scaling for every MXFP4 tensor in attention); 10100.com article (same mechanism).
//
// One CTA per SM owns 128 query rows of one head and sweeps all keys in tiles of 128.  The
// element work of the softmax (an exponential, a quantization and a share of a maximum per
// score) is what bounds MXFP4 attention, so the design spends the SM's issue slots on it:
//   warps 0-3 (softmax group 0) take the even key tiles and warps 4-7 (group 1) the odd ones,
//                      each with its own S buffer in TMEM (2 x 128 columns), so the S = Q^ K^T of
//                      a group's next tile runs while it works on the current one; warp w and
//                      warp w+4 own the same 32 query rows (TMEM lanes 32(w%4)..).  The running
//                      max passes from one group to the other once per tile through shared
//                      memory (one 64-bit slot per row, tagged with the tile index and polled
//                      by the reader), right after the tile's max is known, so the groups
//                      overlap everything else;
//   warp 8 (one lane)  bulk-copies Q^ once and K^/V^ tiles + their scale atoms into a ring;
//   warps 9, 10        issue S = Q^ K^T (tcgen05.mma kind::mxf4 block-scaled, M128 N128) for the
//                      tiles of softmax group 0 and 1 respectively, so that neither group's next
//                      S waits behind the other's buffer release;
//   warp 11            issues O~ += P^ V^ (two K = 64 MMAs per tile, M128 N = d + 16).
// P^ is written in four shared-memory buffers (two per group), so the softmax never waits for
// the PV MMA of its own previous tile.  PNQ row sum: V^'s operand image carries 16 extra rows
// after its d channel rows, the first all ones (scale 2^0), so the PV MMA also accumulates
// l = sum_k P^_k into O~ column d, with the same codes, scales and rescaling as the output.
// Direct placement (pnq = 0) sums P~ in registers instead.  Exponentials: MUFU ex2 for most
// 8-key words; the rest use an FMA-pipe stand-in that yields the same E2M1 code as 2^x
// (e2m1_exp2_stand_in), so neither pipe alone bounds the softmax.
// Every wait is bounded; on expiry the CTA records a status word, drains its in-flight copies and
// MMAs, frees its TMEM and exits.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <type_traits>

#include "kernels.cuh"
#include "ptx.cuh"

namespace mxattn {
namespace wide {

constexpr int kBM = 128;   // query rows per CTA
constexpr int kBN = 128;   // keys per tile
enum { kModeFull = 0, kModeDump = 1, kModeMasked = 2 };
constexpr int kStages = 5;  // K/V shared-memory ring depth
constexpr int kPBufs = 4;   // P^ buffers (tile j uses j % 4)
// Softmax groups: group g (warps 4g..4g+3) takes the key tiles j with j % kGroups == g.  (A third
// group would need the registers of 128 scores per thread in 16 warps, more than a CTA has.)
constexpr int kGroups = 2;
constexpr int kSoftWarps = 4 * kGroups;
// the warpgroup after the softmax warps: the producer, two QK issuers (tiles of even and odd
// index, S buffer j % 2) and the PV issuer
constexpr int kProducerWarp = kSoftWarps, kQkWarp = kSoftWarps + 1, kPvWarp = kSoftWarps + 3;
constexpr int kWarps = kSoftWarps + 4;
constexpr int kThreads = 32 * kWarps;
// S_FULL barriers: tile j commits to j % kSFullSlots, so that a group testing its next tile
// (kGroups ahead) never sees an older phase of the same barrier
constexpr int kSFullSlots = 2 * kGroups;

constexpr int kOnesRows = 16;  // rows appended to each 64-key half of V^: row 0 all ones, rows 1..15 zero
constexpr uint32_t kTmemCols = 512;
constexpr long long kDrainBudgetCycles = 2000000000LL;
// Suspend-time hint of the producer's and the MMA issuers' waits (nanoseconds): their work has a
// tile or more of slack, and a sleeping warp leaves its SM sub-partition's issue slots to the
// softmax warps there.
#ifndef MXATTN_ISSUER_SLEEP_NS
#define MXATTN_ISSUER_SLEEP_NS 1000
#endif
constexpr uint32_t kIssuerSleepNs = MXATTN_ISSUER_SLEEP_NS;
// 8-key words (of the 16 in a tile, word i = keys 8i..8i+7) whose exponentials come from the
// FMA-pipe stand-in instead of MUFU; PNQ only (direct placement needs the exact exponentials).
#ifndef MXATTN_WIDE_POLY_MASK
#define MXATTN_WIDE_POLY_MASK 0x8888u
#endif
constexpr uint32_t kPolyMask = MXATTN_WIDE_POLY_MASK;

template <int D>
struct Layout {
  static constexpr int K_SLOTS = 4;  // K scale-factor slots in TMEM: two per QK issuer
  static constexpr int V_SLOTS = 5;  // V scale-factor slots in TMEM (slot j % 5)
  // shared memory, byte offsets from a 1024-byte aligned base
  static constexpr int Q_BYTES = kBM * D / 2;
  static constexpr int K_BYTES = kBN * D / 2;
  static constexpr int VH_BYTES = D * 32;  // one 64-key half of V^: D channel rows of 32 bytes
  static constexpr int ONES_BYTES = kOnesRows * 32;
  static constexpr int VH_STRIDE = VH_BYTES + ONES_BYTES;
  static constexpr int STAGE_BYTES = K_BYTES + 2 * VH_STRIDE;
  static constexpr int Q_CODES = 0;
  static constexpr int STAGE0 = Q_BYTES;
  static constexpr int P_BYTES = kBM * kBN / 2;
  static constexpr int P_CODES = STAGE0 + kStages * STAGE_BYTES;
  static constexpr int SF_Q = P_CODES + kPBufs * P_BYTES;
  static constexpr int SF_P = SF_Q + 512;
  static constexpr int SF_ONES = SF_P + kPBufs * 512;  // scale atom of the ones rows (constant)
  static constexpr int SF_K = SF_ONES + 512;
  static constexpr int SF_V = SF_K + kStages * 512;
  // running max handed between the groups: per query row one 64-bit slot holding the tile index
  // (high word) and the max after that tile (low word)
  static constexpr int MX = SF_V + kStages * 512;
  static constexpr int LX = MX + 8 * kBM;             // epilogue: per group l and its frame [kGroups][2][128]
  static constexpr int BARS = LX + 1024 * kGroups;
  enum {
    B_Q = 0,
    B_KV_FULL = 1,
    B_KV_EMPTY = 1 + kStages,
    B_S_FULL = 1 + 2 * kStages,  // kSFullSlots
    B_S_FREE = B_S_FULL + kSFullSlots,  // two: one per S buffer (tile parity)
    B_P_FULL = B_S_FREE + 2,     // kPBufs
    B_O_DONE = B_P_FULL + kPBufs,  // kPBufs: PV(j) commits to O_DONE[j % kPBufs]
    B_EPI = B_O_DONE + kPBufs,   // every group ready for the epilogue
    B_DRAIN = B_EPI + 1,
    NUM_BARS
  };
  static constexpr int TMEM_SLOT = BARS + NUM_BARS * 8;
  static constexpr int ABORT = TMEM_SLOT + 4;
  static constexpr int TOTAL = ABORT + 4;
  // one CTA per SM: it allocates all 512 TMEM columns, and more than half the shared memory
  // keeps a second CTA (which would block in tcgen05.alloc) off the SM
  static constexpr int DYN_SMEM = TOTAL + 1024 > 116 * 1024 ? TOTAL + 1024 : 116 * 1024;
  static_assert(STAGE_BYTES % 1024 == 0 && VH_STRIDE % 256 == 0, "operand image alignment");
  static_assert(DYN_SMEM <= 227 * 1024, "shared memory");
  // tensor memory columns
  static constexpr uint32_t T_S = 0;                  // S buffers: group g at 128 g
  static constexpr uint32_t T_O = 256;                // O~: D columns, then l at column D
  static constexpr uint32_t T_SFQ = T_O + D + kOnesRows;  // Q scales, one copy per QK issuer
  static constexpr uint32_t T_SFP = T_SFQ + 8;        // kPBufs x 4 columns
  static constexpr uint32_t T_SFK = T_SFP + 4 * kPBufs;  // K_SLOTS x 4 columns
  static constexpr uint32_t T_SFV = T_SFK + 4 * K_SLOTS; // V_SLOTS x 8 columns (V atom + ones atom)
  static_assert(T_SFV + 8 * V_SLOTS <= kTmemCols, "TMEM budget");
  static constexpr uint32_t QK_LAYOUT = D == 128 ? kLayoutSW64 : kLayoutSW32;
};

__device__ __forceinline__ void raise_abort(volatile int* flag, int* status, int where) {
  *flag = 1;
  if (atomicCAS(status, 0, kStatusTimeout) == 0) atomicExch(status + 1, where);
}

// Maxima of the four 32-key groups of a 128-key tile, eight independent chains of three-input
// maxima advanced together so that their latencies overlap.
__device__ __forceinline__ void group_maxima(const uint32_t (&s)[128], float (&gmax)[4]) {
  float a[4], b[4];
#pragma unroll
  for (int g = 0; g < 4; g++) a[g] = b[g] = -INFINITY;
#pragma unroll
  for (int i = 0; i < 32; i += 4) {
#pragma unroll
    for (int g = 0; g < 4; g++) {
      a[g] = fmax3(a[g], __uint_as_float(s[32 * g + i]), __uint_as_float(s[32 * g + i + 1]));
      b[g] = fmax3(b[g], __uint_as_float(s[32 * g + i + 2]), __uint_as_float(s[32 * g + i + 3]));
    }
  }
#pragma unroll
  for (int g = 0; g < 4; g++) gmax[g] = fmaxf(a[g], b[g]);
}

// E2M1 codes of one 8-key word, p = 2^((S - sm) c - e).  S - sm is formed first, exactly for every
// score near the running max (and 0 for a score equal to it), as the oracle's exp(x - m) is, so a
// score equal to the running max gives 2^-e exactly (for e = 2 the E2M1 midpoint 0.25, which
// rounds to 0).  MUFU ex2, or (POLY) the FMA-pipe stand-in fed with
// w = clamp(((S - sm) c - e + 2.5) / 8, 0, 1) = sat((S - sm) cs + bs).  SUM: direct placement,
// also accumulates the unquantized p.
template <bool POLY, bool SUM>
__device__ __forceinline__ uint32_t word_codes(const uint32_t* s, float sm, float c, float e, float cs, float bs,
                                               float& psum) {
  float p[8];
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const float2 d = __fadd2_rn(make_float2(__uint_as_float(s[i]), __uint_as_float(s[i + 1])), make_float2(-sm, -sm));
    if (POLY) {
      const float2 y = e2m1_exp2_stand_in(make_float2(fma_sat(d.x, cs, bs), fma_sat(d.y, cs, bs)));
      p[i] = y.x;
      p[i + 1] = y.y;
    } else {
      const float2 x = __ffma2_rn(d, make_float2(c, c), make_float2(-e, -e));
      p[i] = ex2_approx(x.x);
      p[i + 1] = ex2_approx(x.y);
      if (SUM) psum += p[i] + p[i + 1];
    }
  }
  return cvt_e2m1x8(p[0], p[1], p[2], p[3], p[4], p[5], p[6], p[7]);
}

// the four words of 32-key group G (words 4G..4G+3 of the tile)
template <int G, bool PNQ>
__device__ __forceinline__ void group_codes(const uint32_t (&s)[128], float sm, float c, float e, uint32_t* w,
                                            float& psum) {
  const float cs = c * 0.125f;
  const float bs = (-kStandInLo - e) * 0.125f;  // exact: e is a small integer
#pragma unroll
  for (int q = 0; q < 4; q++) {
    constexpr uint32_t mask = PNQ ? kPolyMask : 0u;
    if ((mask >> (4 * G + q)) & 1u)
      w[q] = word_codes<true, false>(s + 32 * G + 8 * q, sm, c, e, cs, bs, psum);
    else
      w[q] = word_codes<false, !PNQ>(s + 32 * G + 8 * q, sm, c, e, cs, bs, psum);
  }
}

template <int D, int DT, bool PNQ, int MODE>
__global__ void __launch_bounds__(kThreads, 1) mxattn_fwd_wide_kernel(const AttnArgs a) {
  using L = Layout<D>;
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
  // the longest query tiles (the last ones) are launched first.
  const int bh = blockIdx.y;
  int Nq = a.N, Nk = a.Nk, qt;
  size_t q_tile, k_tile0, v_tile0;  // Q tile, first 128-key K tile / scale atom, first 64-key V half
  int v_halves;                     // 64-key V halves of this problem present in memory
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
    v_halves = 2 * ((Nk + 127) / 128);  // every sequence owns whole 128-key tiles of halves
    out_row0 = ((size_t)start * a.BH + bh) * D;
    out_step = (size_t)a.BH * D;
  } else {
    const int T128q = (a.N + 127) / 128;
    qt = causal ? T128q - 1 - (int)blockIdx.x : (int)blockIdx.x;
    q_tile = (size_t)bh * T128q + qt;
    k_tile0 = (size_t)bh * ((a.Nk + 127) / 128);
    v_halves = (a.Nk + 63) / 64;
    v_tile0 = (size_t)bh * v_halves;
    out_row0 = (size_t)bh * a.N * D;
    out_step = D;
  }
  const int T = (Nk + kBN - 1) / kBN;  // key tiles of the problem
  // tiles the CTA sweeps: all, or under causal masking those up to its diagonal
  const int TJ = causal ? (qt + 1 < T ? qt + 1 : T) : T;
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
    for (int i = 0; i < kSFullSlots; i++) mbar_init(bar(L::B_S_FULL + i), 1);
    for (int b = 0; b < 2; b++) mbar_init(bar(L::B_S_FREE + b), 128);  // every thread of a group
    for (int b = 0; b < kPBufs; b++) {
      mbar_init(bar(L::B_P_FULL + b), 4);
      mbar_init(bar(L::B_O_DONE + b), 1);
    }
    mbar_init(bar(L::B_EPI), kSoftWarps);
    mbar_init(bar(L::B_DRAIN), 3);  // one commit from each issuer
    fence_mbar_init();
  }
  if (PNQ) {
    // the ones rows after each V^ half of every stage (row 0: code 1.0 = 0x2 in every nibble;
    // rows 1..15: zero) and their scale atom (row 0, every key group: 2^0; everything else zero)
    for (int i = threadIdx.x; i < kStages * 2 * (L::ONES_BYTES / 4); i += kThreads) {
      const int blk = i / (L::ONES_BYTES / 4), off = i % (L::ONES_BYTES / 4);
      const int st = blk / 2, half = blk % 2;
      reinterpret_cast<uint32_t*>(smem + L::STAGE0 + st * L::STAGE_BYTES + L::K_BYTES + half * L::VH_STRIDE +
                                  L::VH_BYTES)[off] = off < 32 / 4 ? 0x22222222u : 0u;
    }
    for (int i = threadIdx.x; i < 512 / 4; i += kThreads)
      reinterpret_cast<uint32_t*>(smem + L::SF_ONES)[i] = i == 0 ? 0x7F7F7F7Fu : 0u;
    fence_proxy_async_smem();
  }
  for (int i = threadIdx.x; i < kBM; i += kThreads)  // no tile's index: nothing handed over yet
    reinterpret_cast<volatile unsigned long long*>(smem + L::MX)[i] = ~0ull;
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
      mbar_arrive_expect_tx(bar(L::B_Q), L::Q_BYTES + 512);
      bulk_g2s(sb + L::Q_CODES, a.q_codes + q_tile * (size_t)L::Q_BYTES, L::Q_BYTES, bar(L::B_Q));
      bulk_g2s(sb + L::SF_Q, a.q_scales + q_tile * 512, 512, bar(L::B_Q));
      for (int j = 0; j < TJ; j++) {
        const int s = j % kStages;
        if (j >= kStages) {
          ok = mbar_wait_sleep(bar(L::B_KV_EMPTY + s), ((j / kStages) - 1) & 1, abort_flag, a.wait_budget, kIssuerSleepNs);
          if (!ok) break;
        }
        // the second 64-key half of V^ exists in memory unless the keys end in the first one (its
        // P^ codes are then zero, so whatever the stage held there adds nothing)
        const bool second = 2 * j + 1 < v_halves;
        const uint32_t fb = bar(L::B_KV_FULL + s);
        const uint32_t st = sb + L::STAGE0 + s * L::STAGE_BYTES;
        mbar_arrive_expect_tx(fb, L::K_BYTES + (second ? 2 : 1) * L::VH_BYTES + 1024);
        bulk_g2s(st, a.k_codes + (k_tile0 + j) * (size_t)L::K_BYTES, L::K_BYTES, fb);
        bulk_g2s(sb + L::SF_K + s * 512, a.k_scales + (k_tile0 + j) * 512, 512, fb);
        bulk_g2s(st + L::K_BYTES, a.v_codes + (v_tile0 + 2 * j) * (size_t)L::VH_BYTES, L::VH_BYTES, fb);
        if (second)
          bulk_g2s(st + L::K_BYTES + L::VH_STRIDE, a.v_codes + (v_tile0 + 2 * j + 1) * (size_t)L::VH_BYTES,
                   L::VH_BYTES, fb);
        bulk_g2s(sb + L::SF_V + s * 512, a.v_scales + (k_tile0 + j) * 512, 512, fb);  // one atom per 128 keys
        issued = j + 1;
      }
      if (!ok) raise_abort(abort_flag, a.status, 1);
      // Let every copy issued land before the CTA can exit, whichever warp gave up.
      mbar_wait(bar(L::B_Q), 0, no_abort, kDrainBudgetCycles);
      for (int j = (issued > kStages ? issued - kStages : 0); j < issued; j++)
        mbar_wait(bar(L::B_KV_FULL + j % kStages), (j / kStages) & 1, no_abort, kDrainBudgetCycles);
    }
  } else if (warp == kQkWarp || warp == kQkWarp + 1) {
    // ------------------------------------------------------------------ QK issuers
    // Issuer g serves the tiles of softmax group g.  The warp runs the loop converged (waits and
    // descriptor arithmetic stay warp-uniform); lane 0 alone issues its tcgen05 operations, so that
    // each of its commits covers all of them.
    const int g = warp - kQkWarp;
    const bool leader = lane == 0;
    const uint32_t t_sfq = tmem + L::T_SFQ + 4 * g;  // this issuer's own copy of the Q scales
    bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_sleep(bar(L::B_Q), 0, abort_flag, a.wait_budget, kIssuerSleepNs));
    if (ok) {
      tc_fence_after();
      if (leader) tmem_cp_sf_atom(t_sfq, sb + L::SF_Q);
      __syncwarp();
      const uint64_t qdesc = smem_desc(sb + L::Q_CODES, 16, 8 * (D / 2), L::QK_LAYOUT);
      for (int j = g; j < TJ; j += 2) {
        const int s = j % kStages, f = 2 * g + ((j >> 1) & 1);
        ok = __all_sync(0xFFFFFFFFu, mbar_wait_sleep(bar(L::B_KV_FULL + s), (j / kStages) & 1, abort_flag, a.wait_budget, kIssuerSleepNs));
        if (!ok) break;
        tc_fence_after();
        // K scale slot f was last read by QK(j-4), complete since group g read that S before
        // releasing it, which this warp waited for before issuing QK(j-2)
        if (leader) tmem_cp_sf_atom(tmem + L::T_SFK + 4 * f, sb + L::SF_K + 512 * s);
        if (j >= 2) {  // S buffer g was last read by group g at tile j-2
          ok = __all_sync(0xFFFFFFFFu, mbar_wait_sleep(bar(L::B_S_FREE + g), ((j - 2) >> 1) & 1, abort_flag, a.wait_budget, kIssuerSleepNs));
          if (!ok) break;
          tc_fence_after();
        }
        const uint64_t kdesc = smem_desc(sb + L::STAGE0 + s * L::STAGE_BYTES, 16, 8 * (D / 2), L::QK_LAYOUT);
        if (leader) {
#pragma unroll
          for (int kb = 0; kb < D / 64; kb++)  // head dims 64kb..: 32 bytes along each row, scale bytes 2kb, 2kb+1
            mma_mxf4(tmem + L::T_S + 128 * g, qdesc + (uint64_t)(kb * 2), kdesc + (uint64_t)(kb * 2),
                     mxf4_idesc(kBM, kBN, 2 * kb, 2 * kb), t_sfq, tmem + L::T_SFK + 4 * f, kb > 0 ? 1u : 0u);
        }
        if (j >= kPBufs) {
          // S(j) also tells group g that P buffer j % 4 (last read by PV(j-4)) is free: see PV(j-4)
          // complete before committing S(j).  Each O_DONE barrier is at most one phase away here:
          // PV(j) needs S(j), and this issuer saw PV(j-8) complete before committing S(j-4).
          const int pb = j % kPBufs;
          ok = __all_sync(0xFFFFFFFFu, mbar_wait_sleep(bar(L::B_O_DONE + pb), ((j - kPBufs) / kPBufs) & 1, abort_flag,
                                                       a.wait_budget, kIssuerSleepNs));
          if (!ok) break;
          tc_fence_after();
        }
        // V scale atom of tile j into its slot (j % 5), for PV(j): the slot was last read by PV(j-5),
        // complete since this issuer saw PV(j-4) complete just above (or j < 5: never used).  The
        // copy sits here, not with the PV issuer, to even out the asynchronous instructions issued
        // per SM sub-partition; the commit below covers it, so S(j), and hence P(j), imply it.
        if (leader) {
          if (PNQ && D == 64)  // the ones row is B-operand row 64, inside the V atom: scale 1 for all key groups
            *reinterpret_cast<volatile uint32_t*>(smem + L::SF_V + 512 * s + 8) = 0x7F7F7F7Fu;
          if (PNQ && D == 64) fence_proxy_async_smem();
          tmem_cp_sf_atom(tmem + L::T_SFV + 8 * (j % L::V_SLOTS), sb + L::SF_V + 512 * s);
        }
        if (leader) mma_commit(bar(L::B_S_FULL + j % kSFullSlots));
        __syncwarp();
      }
    }
    if (!ok && leader) raise_abort(abort_flag, a.status, 2);
    // wait for every tcgen05 operation of the three issuers before TMEM is released
    if (leader) mma_commit(bar(L::B_DRAIN));
    __syncwarp();
    mbar_wait(bar(L::B_DRAIN), 0, no_abort, kDrainBudgetCycles);
  } else if (warp == kPvWarp) {
    // ------------------------------------------------------------------ PV issuer (same scheme)
    const bool leader = lane == 0;
    if (PNQ && leader)
      for (int f = 0; f < L::V_SLOTS; f++) tmem_cp_sf_atom(tmem + L::T_SFV + 8 * f + 4, sb + L::SF_ONES);
    __syncwarp();
    bool ok = true;
    for (int j = 0; j < TJ; j++) {
      const int s = j % kStages, f = j % L::V_SLOTS, pb = j % kPBufs;
      // V^(j) landed with K^(j), before S(j) and so before P(j); this warp also waits for the stage
      // itself (it cannot have been refilled: that needs this warp's commit below)
      ok = __all_sync(0xFFFFFFFFu, mbar_wait_sleep(bar(L::B_KV_FULL + s), (j / kStages) & 1, abort_flag, a.wait_budget, kIssuerSleepNs));
      if (!ok) break;
      // (the V scale atom of tile j is already in slot f: the QK issuer copied it before
      // committing S(j))
      ok = __all_sync(0xFFFFFFFFu, mbar_wait_sleep(bar(L::B_P_FULL + pb), (j / kPBufs) & 1, abort_flag, a.wait_budget, kIssuerSleepNs));
      if (!ok) break;
      tc_fence_after();
      if (leader) {
        // P scale slot pb was last read by PV(j-4), complete before S(j) was committed
        tmem_cp_sf_atom(tmem + L::T_SFP + 4 * pb, sb + L::SF_P + 512 * pb);
        const uint32_t pbase = sb + L::P_CODES + pb * L::P_BYTES;
        const uint32_t vbase = sb + L::STAGE0 + s * L::STAGE_BYTES + L::K_BYTES;
#pragma unroll
        for (int kb = 0; kb < 2; kb++) {  // keys 64kb..64kb+63: P bytes 32kb.. of each row, V half kb
          const uint64_t pdesc = smem_desc(pbase, 16, 8 * 64, kLayoutSW64) + (uint64_t)(kb * 2);
          const uint64_t vdesc = smem_desc(vbase + kb * L::VH_STRIDE, 16, 8 * 32, kLayoutSW32);
          mma_mxf4(tmem + L::T_O, pdesc, vdesc, mxf4_idesc(kBM, NV, 2 * kb, 2 * kb), tmem + L::T_SFP + 4 * pb,
                   tmem + L::T_SFV + 8 * f, (j > 0 || kb > 0) ? 1u : 0u);
        }
        mma_commit(bar(L::B_O_DONE + pb));
        // QK(j) read the stage too: complete, since the softmax saw S(j) before P(j)
        mma_commit(bar(L::B_KV_EMPTY + s));
      }
      __syncwarp();
    }
    if (!ok && leader) raise_abort(abort_flag, a.status, 4);
    if (leader) mma_commit(bar(L::B_DRAIN));
    __syncwarp();
    mbar_wait(bar(L::B_DRAIN), 0, no_abort, kDrainBudgetCycles);
  } else if (warp < kSoftWarps) {
    // ------------------------------------------------------------------ softmax (warps 0-7)
    const int grp = warp >> 2;             // softmax group: key tiles j with j % kGroups == grp
    const int quad = warp & 3;             // TMEM lane quadrant = the warp pair's 32 query rows
    const int row = quad * 32 + lane;      // TMEM lane and query row within the tile
    const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
    const float c = a.scale_log2;
    const bool dumping = DUMP && bh == a.dump_bh && qt == a.dump_qt;
    const DumpLayout dl(D, T, kBN);
    volatile unsigned long long* mx = reinterpret_cast<volatile unsigned long long*>(smem + L::MX);
    // keys this row sees: all Nk, or under causal masking those up to its own position
    const int kmax = causal ? (qt * kBM + row + 1 < Nk ? qt * kBM + row + 1 : Nk) : Nk;
    float sm = -INFINITY;   // running max of S (raw MMA units) after this group's latest tile
    float l = 0.f;          // direct placement: this group's share of l, in the frame of sm
    bool ok = true;
    bool s_ready = false;   // S(j) was seen complete by the early test during tile j-2
    // one key tile; FULL: all 128 keys are inside this row's range, so the body carries no masking
    const float tau = a.tau, log2q = a.rule.log2q;
    auto tile = [&](int j, auto full_tag, auto floor_tag) -> bool {
      constexpr bool FULL = decltype(full_tag)::value;
      constexpr bool FLOOR = decltype(floor_tag)::value;  // the OCP floor scale rule
      if (!__all_sync(0xFFFFFFFFu, s_ready)) {
        ok = mbar_wait(bar(L::B_S_FULL + j % kSFullSlots), (j / kSFullSlots) & 1, abort_flag, a.wait_budget);
        if (!__all_sync(0xFFFFFFFFu, ok)) return false;
      }
      tc_fence_after();
      const uint32_t sbuf = tl + L::T_S + 128 * (j & 1);
      uint32_t s[128];
      tmem_ld128_wait(sbuf, s);
      // S(j) is in registers: the QK MMA of tile j+2 may overwrite the buffer.  Each thread fences
      // its own load and arrives (no warp barrier on the way to the maxima).
      tc_fence_before();
      mbar_arrive(bar(L::B_S_FREE + (j & 1)));
      if (!FULL) {
        const int valid = kmax - j * kBN;  // this row's keys in the tile (may be <= 0)
#pragma unroll
        for (int i = 0; i < 128; i++)
          if (i >= valid) s[i] = __float_as_uint(-INFINITY);
      }
      if (dumping && j < 2) {
        float* ds = reinterpret_cast<float*>(a.dump + dl.s) + ((size_t)j * 128 + row) * kBN;
        for (int i = 0; i < 128; i++) ds[i] = __uint_as_float(s[i]);
      }
      // the hand-over slot is first read here, so that its latency overlaps the maxima (the value is
      // normally there long before; the check below reads again until it is)
      unsigned long long v0 = j > 0 ? mx[row] : 0ull;
      float gmax[4];
      group_maxima(s, gmax);
      const float mt_raw = fmaxf(fmaxf(gmax[0], gmax[1]), fmaxf(gmax[2], gmax[3]));
      // Lazy running max (threshold tau, log2 units): the max moves only when the tile's max
      // exceeds the running max before the tile by more than tau.
      // The codes depend on the running max after this tile (their frame).  A group's maximum is
      // taken as 2^((gmax - frame) * c): exactly 1 for the group that holds the running max, as
      // exp(0) is in the oracle.
      uint32_t eb[4], w[16] = {};  // (every word is set by codes() before its store)
      float psum[4];
      // P buffer j % 4 was last read by PV(j-4), which the QK issuer saw complete before it
      // committed S(j).  Codes in the MMA's 64-byte swizzled rows: group g (16 bytes) at chunk
      // g ^ ((row >> 1) & 3); the four scale bytes in the row's word of the scale atom.  Each
      // piece is stored as soon as it exists, so the stores overlap the rest of the code phase.
      const int pb = j % kPBufs;
      uint8_t* prow = smem + L::P_CODES + pb * L::P_BYTES + row * 64;
      const int sw = (row >> 1) & 3;
      auto codes = [&](float fr) {
        float ex[4];  // the groups' shared exponents e
#pragma unroll
        for (int g = 0; g < 4; g++) {
          ex[g] = shared_exponent_log2f_rule<FLOOR>((gmax[g] - fr) * c, log2q, eb[g]);
          psum[g] = 0.f;
        }
        *reinterpret_cast<uint32_t*>(smem + L::SF_P + pb * 512 + (row % 32) * 16 + (row / 32) * 4) =
            eb[0] | (eb[1] << 8) | (eb[2] << 16) | (eb[3] << 24);
        auto store = [&](int g) {
          *reinterpret_cast<uint4*>(prow + ((g ^ sw) * 16)) = make_uint4(w[4 * g], w[4 * g + 1], w[4 * g + 2], w[4 * g + 3]);
        };
        group_codes<0, PNQ>(s, fr, c, ex[0], w, psum[0]);
        store(0);
        group_codes<1, PNQ>(s, fr, c, ex[1], w + 4, psum[1]);
        store(1);
        group_codes<2, PNQ>(s, fr, c, ex[2], w + 8, psum[2]);
        store(2);
        group_codes<3, PNQ>(s, fr, c, ex[3], w + 12, psum[3]);
        store(3);
      };
      // The running max before this tile is the one after tile j-1, which the other group hands
      // over in the row's slot; the codes are formed in the frame after this tile, so they wait
      // for it.  The two threads of a row write the slot in turn, each only after reading the
      // other's value, so one slot suffices; a single 64-bit access carries the max together with
      // its tile index, so the reader needs no barrier.  The hand-over is published right after
      // the maxima, before this group's own codes, so it is normally there long before it is read.
      float sm_prev = -INFINITY;
      if (j > 0) {
        unsigned long long v = v0;
        if (!__all_sync(0xFFFFFFFFu, (uint32_t)(v >> 32) == (uint32_t)(j - 1))) {
          const long long t0 = clock64();
          while (true) {
            v = mx[row];
            if (__all_sync(0xFFFFFFFFu, (uint32_t)(v >> 32) == (uint32_t)(j - 1))) break;
            if (__any_sync(0xFFFFFFFFu, *abort_flag != 0 || clock64() - t0 > a.wait_budget)) return ok = false;
          }
        }
        sm_prev = __uint_as_float((uint32_t)v);
      }
      const bool move = j == 0 || (mt_raw * c > sm_prev * c + tau);
      const float sm_new = move ? mt_raw : sm_prev;
      if (j + 1 < TJ)  // hand the max on as early as possible: the other group waits for it
        mx[row] = ((unsigned long long)(uint32_t)j << 32) | __float_as_uint(sm_new);
      codes(sm_new);
      const float m2 = sm_new * c;
      // O~ and l are rescaled by alpha = 2^(m_old - m_new) only when some row of the warp moves
      // its max (alpha = 1 elsewhere); tile 0 starts both at zero
      const bool any_move = j > 0 && __any_sync(0xFFFFFFFFu, move);
      float alpha = 1.f;
      if (any_move && move) alpha = ex2_approx((sm_prev - sm_new) * c);
      if (!PNQ && sm != sm_new) l *= ex2_approx((sm - sm_new) * c);  // this group's l into the new frame
      sm = sm_new;
      if (dumping) {  // the unquantized tile, relative to this tile's running max
        float* dpt = reinterpret_cast<float*>(a.dump + dl.p_tilde) + ((size_t)j * 128 + row) * kBN;
        for (int i = 0; i < 128; i++) dpt[i] = ex2_approx((__uint_as_float(s[i]) - sm_new) * c);
      }
      // test S(j+2) now, so that the test's latency overlaps the stores below
      s_ready = j + kGroups < TJ &&
                mbar_test(bar(L::B_S_FULL + (j + kGroups) % kSFullSlots), ((j + kGroups) / kSFullSlots) & 1);
      if (!PNQ) {
#pragma unroll
        for (int g = 0; g < 4; g++) l += psum[g] * __uint_as_float(eb[g] << 23);  // byte 0: 2^-127 -> 0
      }
      // Rescaling O~ needs PV(j-1) complete; its O_DONE barrier is at most one phase away.
      if (any_move) {
        const int pb = (j - 1) % kPBufs;
        ok = mbar_wait(bar(L::B_O_DONE + pb), ((j - 1) / kPBufs) & 1, abort_flag, a.wait_budget);
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
      // the P codes and scales of this tile are in shared memory (stored by codes())
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::B_P_FULL + pb));
      if (dumping) {
        uint32_t* dp = reinterpret_cast<uint32_t*>(a.dump + dl.p_codes + ((size_t)j * 128 + row) * 64);
        for (int i = 0; i < 16; i++) dp[i] = w[i];
        uint8_t* dsf = a.dump + dl.p_scales + ((size_t)j * 128 + row) * 4;
        for (int g = 0; g < 4; g++) dsf[g] = (uint8_t)eb[g];
        // the unquantized tile, relative to this tile's running max (dump only)
        reinterpret_cast<float*>(a.dump + dl.m_tiles)[(size_t)j * 128 + row] = m2;
      }
      return true;
    };
    // tiles every row of the CTA sees in full, then the masked ones (the ragged last tile of the
    // keys; under causal masking the diagonal tile)
    int full_tiles = (Nk % kBN == 0) ? T : T - 1;
    if (causal && full_tiles > qt) full_tiles = qt;
    auto sweep = [&](auto floor_tag) {
      int j = grp;
      for (; ok && j < full_tiles; j += kGroups) ok = tile(j, std::true_type{}, floor_tag);
      for (; ok && j < TJ; j += kGroups) ok = tile(j, std::false_type{}, floor_tag);
    };
    if (a.rule.mq == 0xFFFFFFFFu) sweep(std::true_type{});
    else sweep(std::false_type{});

    // Epilogue.  The group that ran the last tile knows PV(TJ-5) complete (S(TJ-1) was committed
    // after it), so its wait on PV(TJ-1)'s barrier is unambiguous; it then lets the other group in.
    const int last_grp = (TJ - 1) % kGroups;
    if (ok && grp == last_grp) {
      const int pb = (TJ - 1) % kPBufs;
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar(L::B_O_DONE + pb), ((TJ - 1) / kPBufs) & 1, abort_flag, a.wait_budget));
    }
    if (ok) {
      {  // each group's l (direct placement) and the running max it is expressed against
        float* lx = reinterpret_cast<float*>(smem + L::LX);
        lx[grp * 256 + row] = l;
        lx[grp * 256 + 128 + row] = sm;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::B_EPI));
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar(L::B_EPI), 0, abort_flag, a.wait_budget));
    }
    if (ok) {
      tc_fence_after();
      // the final frame is the running max after the last tile, which its group holds
      const float* lx = reinterpret_cast<const float*>(smem + L::LX);
      const float sm_final = lx[last_grp * 256 + 128 + row];
      float lsum;
      if (PNQ) {
        uint32_t lv;
        tmem_ld1(tl + L::T_O + D, lv);
        tmem_wait_ld();
        pin1(lv);
        lsum = __uint_as_float(lv);
      } else {
        lsum = 0.f;
        for (int g = 0; g < kGroups; g++) {
          const float lg = lx[g * 256 + row];
          if (lg != 0.f) lsum += lg * ex2_approx((lx[g * 256 + 128 + row] - sm_final) * c);
        }
      }
      const float inv_l = 1.f / lsum;
      const int qrow = qt * kBM + row;
      const bool store = qrow < Nq;
      const size_t obase = out_row0 + (size_t)(store ? qrow : 0) * out_step;
      if (dumping && grp == 0) {
        reinterpret_cast<float*>(a.dump + dl.l)[row] = lsum;
        reinterpret_cast<float*>(a.dump + dl.m)[row] = sm_final * c;
      }
      // the groups share the row's D outputs, 32 columns at a time
#pragma unroll 1
      for (int cc = grp; cc < D / 32; cc += kGroups) {
        uint32_t o[32];
        tmem_ld32(tl + L::T_O + 32 * cc, o);
        tmem_wait_ld();
        pin32(o);
        if (dumping) {
          float* d_o = reinterpret_cast<float*>(a.dump + dl.o) + (size_t)row * D + 32 * cc;
          for (int i = 0; i < 32; i++) d_o[i] = __uint_as_float(o[i]);
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

template <int D, int DT, bool PNQ>
static cudaError_t launch_t(const AttnArgs& a, cudaStream_t s) {
  using L = Layout<D>;
  const bool masked = a.causal || a.vl.cu_seqlens != nullptr;
  if (masked && a.dump != nullptr) return cudaErrorNotSupported;
  auto kern = a.dump != nullptr ? mxattn_fwd_wide_kernel<D, DT, PNQ, kModeDump>
              : masked          ? mxattn_fwd_wide_kernel<D, DT, PNQ, kModeMasked>
                                : mxattn_fwd_wide_kernel<D, DT, PNQ, kModeFull>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::DYN_SMEM);
  if (err != cudaSuccess) return err;
  const unsigned qtiles = a.vl.cu_seqlens != nullptr ? (unsigned)a.vl.tiles_per_head : (unsigned)((a.N + kBM - 1) / kBM);
  dim3 grid(qtiles, (unsigned)a.BH);
  kern<<<grid, kThreads, L::DYN_SMEM, s>>>(a);
  return cudaGetLastError();
}

template <int D, int DT>
static cudaError_t launch_d(const AttnArgs& a, cudaStream_t s) {
  return a.pnq ? launch_t<D, DT, true>(a, s) : launch_t<D, DT, false>(a, s);
}

}  // namespace wide

cudaError_t launch_attention_wide(const AttnArgs& a, int D, int dtype, cudaStream_t s) {
  if (a.fmt != kFmtMXFP4) return cudaErrorNotSupported;
  if (D == 128) return dtype == kBF16 ? wide::launch_d<128, kBF16>(a, s) : wide::launch_d<128, kFP32>(a, s);
  return dtype == kBF16 ? wide::launch_d<64, kBF16>(a, s) : wide::launch_d<64, kFP32>(a, s);
}

}  // namespace mxattn

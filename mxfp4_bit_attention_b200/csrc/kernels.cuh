// kernels.cuh -- argument blocks and launchers shared by the C ABI (api.cu) and the kernels.
#pragma once
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"

namespace mxattn {

enum { kBF16 = 0, kFP32 = 1 };
// Element formats: the method's MXFP4 (32-element groups, E8M0 scale chosen by a ScaleRule) and
// the NVFP4 comparison format (16-element blocks, E4M3 scale = E4M3(amax / 6)).
enum { kFmtMXFP4 = 0, kFmtNVFP4 = 1 };

// A packed batch of variable-length sequences ("varlen"): inputs and outputs are token-major
// [T, H, d]; sequence s holds tokens cu_seqlens[s] .. cu_seqlens[s+1]-1 and is padded to whole
// 128-row tiles in the packed operands, where it starts at tile tile_off[s] of each head's
// tiles_per_head tiles.  cu_seqlens == nullptr: the fixed-length [B, H, N, d] layout.
struct Varlen {
  const int* cu_seqlens;  // [nseq + 1] device
  const int* tile_off;    // [nseq + 1] device, written by the tile-table kernel
  int nseq;
  int tiles_per_head;
};

// Sequence owning packed tile g (tile_off[nseq] > g): the last s with tile_off[s] <= g (empty
// sequences own no tile and are skipped).
__device__ __forceinline__ int varlen_sequence(const Varlen& v, int g) {
  int lo = 0, hi = v.nseq - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(v.tile_off + mid) <= g) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

struct QKQuantArgs {
  const void* q;
  const void* k;
  uint8_t* q_codes;
  uint8_t* q_scales;
  uint8_t* k_codes;
  uint8_t* k_scales;
  int BH, N;             // N: tokens of Q (varlen: BH = H, N = T)
  int Nk;                // tokens of K (= N for self-attention)
  int rotate;
  float hadamard_scale;  // fl32(1/sqrt(d))
  ScaleRule rule;
  Varlen vl;
  int fmt;
};

struct VQuantArgs {
  const void* v;
  uint8_t* v_codes;
  uint8_t* v_scales;
  int BH, N;             // varlen: BH = H, N = T
  ScaleRule rule;
  Varlen vl;
  int fmt;
};

struct PlainQuantArgs {
  const void* x;
  uint8_t* codes;
  uint8_t* scales;
  int64_t rows, cols;
  int axis;
  ScaleRule rule;
  int fmt;
};

// Per-block Qmax sweep (scale-rule diagnostic): boundaries q_k as ceiling rules.
constexpr int kSweepMaxQ = 64;
struct SweepArgs {
  const void* x;
  int64_t rows, cols;
  int rotate;                       // Hadamard-rotate each row first (cols = 64 or 128)
  float hadamard_scale;
  int nq;
  ScaleRule rules[kSweepMaxQ];
  unsigned long long* counts;       // [nq], accumulated
  double* sse_sums;                 // [nq], accumulated
};

struct AttnArgs {
  const uint8_t* q_codes;
  const uint8_t* q_scales;
  const uint8_t* k_codes;
  const uint8_t* k_scales;
  const uint8_t* v_codes;
  const uint8_t* v_scales;
  void* out;
  int* status;           // workspace status block (error word at [0], detail at [1..3])
  int BH, N;             // N: query rows per head
  int Nk;                // keys (and values) per head (= N for self-attention)
  int causal;            // self-attention only: query row i sees keys 0..i
  float scale_log2;      // softmax_scale * log2(e)
  float tau;             // lazy max threshold, log2 units
  int pnq;
  ScaleRule rule;
  long long wait_budget; // SM clock cycles a bounded wait may spin before giving up
  uint8_t* dump;         // optional diagnostic dump of one CTA (layout: see dump_layout below)
  int dump_bh, dump_qt;
  Varlen vl;             // varlen: BH = H, N = Nk = T
  int fmt;               // kFmtNVFP4: the comparison format (full attention only)
  int key_tile;          // 64 or 128 keys per online-softmax step
};

// Diagnostic dump of the CTA (dump_bh, dump_qt), byte offsets for head dim D, key tiles of KT keys
// (64 or 128) and T = ceil(N / KT) tiles:
//   [0, 8 KT * 128)        S of key tiles 0 and 1, fp32 [2][128][KT] (as read from TMEM)
//   P codes                [T][128][KT/2] bytes, logical key order (element 2i in the low nibble)
//   P scales               [T][128][KT/32] bytes (E8M0 of the tile's 32-key groups)
//   O accumulator          [128][D] fp32, before the division by l
//   l, m                   [128] fp32 each (m in log2 units: running max of S * scale * log2 e)
//   P~                     [T][128][KT] fp32: 2^(S * scale * log2 e - m) with the running max m
//                          of that tile (0 for keys past N), the unquantized exponential tile
//   m of every tile        [T][128] fp32, the running max (log2 units) after each tile's update
struct DumpLayout {
  size_t s, p_codes, p_scales, o, l, m, p_tilde, m_tiles, total;
  __host__ __device__ DumpLayout(int D, int T, int KT = 64) {
    s = 0;
    p_codes = (size_t)2 * 128 * KT * 4;
    p_scales = p_codes + (size_t)T * 128 * (KT / 2);
    o = (p_scales + (size_t)T * 128 * (KT / 32) + 15) / 16 * 16;
    l = o + (size_t)128 * D * 4;
    m = l + 128 * 4;
    p_tilde = m + 128 * 4;
    m_tiles = p_tilde + (size_t)T * 128 * KT * 4;
    total = m_tiles + (size_t)T * 128 * 4;
  }
};

// Status words: a kernel whose bounded wait expired; sequence offsets that are not a partition
// of the packed tokens.
enum { kStatusTimeout = 0x54494D45 /* 'TIME' */, kStatusBadSeqlens = 0x5345514C /* 'SEQL' */ };

cudaError_t launch_rotate_quant_qk(const QKQuantArgs& a, int D, int dtype, cudaStream_t s);
cudaError_t launch_quant_v(const VQuantArgs& a, int D, int dtype, cudaStream_t s);
cudaError_t launch_quant_plain(const PlainQuantArgs& a, int dtype, cudaStream_t s);
cudaError_t launch_qmax_sweep(const SweepArgs& a, int dtype, cudaStream_t s);
cudaError_t launch_attention(const AttnArgs& a, int D, int dtype, cudaStream_t s);
cudaError_t launch_attention_wide(const AttnArgs& a, int D, int dtype, cudaStream_t s);
cudaError_t launch_fp4_mma_probe(int ctas, int iters, int n, int* status, cudaStream_t s);
enum { kProbeExp2Poly = 0, kProbeExp2Mufu = 1, kProbeE2m1StandIn = 2, kProbeE2m1Mufu = 3, kProbeScaleExpLog2 = 4,
       kProbeScaleExp = 5 };
cudaError_t launch_arith_probe(int op, const float* in, int64_t n, const ScaleRule& rule, void* out, cudaStream_t s);
cudaError_t launch_varlen_tiles(const int* cu_seqlens, int nseq, int T, int* tile_off, int* status, cudaStream_t s);

}  // namespace mxattn

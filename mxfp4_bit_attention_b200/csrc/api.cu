// api.cu -- the C ABI declared in include/mxattn.h: argument validation, workspace carving and
// kernel launches.  No allocation, no synchronization (except mxattn_get_device_error).
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/mxattn.h"
#include "kernels.cuh"

using namespace mxattn;

namespace {

constexpr size_t kStatusBytes = 256;
constexpr long long kWaitBudgetCycles = 2000000000LL;  // ~1 s at the B200's clocks

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool sizes_ok(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1) return false;
  if (d != 64 && d != 128) return false;
  if ((int64_t)B * H > 65535) return false;  // grid.y of the attention launch
  return true;
}

int64_t t128(int N) { return ((int64_t)N + 127) / 128; }
int64_t t64(int N) { return ((int64_t)N + 63) / 64; }

// Scale bytes of the packed operands: MXFP4 one 512-byte atom per 128-row Q/K tile and per
// 128-key V tile; NVFP4 (16-element blocks) d/64 atoms per Q/K tile and one per 64-key V tile.
size_t qk_scale_bytes(int B, int H, int N, int d, int fmt) {
  return (size_t)B * H * t128(N) * 512 * (fmt == MXATTN_FMT_NVFP4 ? d / 64 : 1);
}
size_t v_scale_bytes(int B, int H, int N, int fmt) {
  return (size_t)B * H * (fmt == MXATTN_FMT_NVFP4 ? t64(N) : t128(N)) * 512;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Boundary q = mq * 2^eq of a ceiling rule, or the OCP floor rule.
bool make_rule(const mxattn_opts* o, ScaleRule* r) {
  float q;
  switch (o->scale_rule) {
    case MXATTN_SCALE_UOS: q = 7.25f; break;
    case MXATTN_SCALE_QMAX6: q = 6.0f; break;
    case MXATTN_SCALE_OCP: r->eq = 2; r->mq = 0xFFFFFFFFu; r->log2q = 2.0f; return true;
    case MXATTN_SCALE_CEIL_CUSTOM:
      q = o->qmax;
      if (!(q >= 4.0f && q <= 8.0f)) return false;  // keeps every exponent inside [-127, 126]
      break;
    default: return false;
  }
  uint32_t bits;
  std::memcpy(&bits, &q, 4);
  r->eq = (int)(bits >> 23) - 127;
  r->mq = bits & 0x007FFFFFu;
  r->log2q = (float)std::log2((double)q);
  return true;
}

mxattn_status check_opts(const mxattn_opts* o) {
  if (o == nullptr) return MXATTN_ERR_INVALID_ARG;
  ScaleRule r;
  if (!make_rule(o, &r)) return MXATTN_ERR_INVALID_ARG;
  if (o->dtype != MXATTN_BF16 && o->dtype != MXATTN_FP32) return MXATTN_ERR_INVALID_ARG;
  if (o->pnq != 0 && o->pnq != 1) return MXATTN_ERR_INVALID_ARG;
  if (o->rotate != 0 && o->rotate != 1) return MXATTN_ERR_INVALID_ARG;
  if (!(o->rescale_tau >= 0.f && std::isfinite(o->rescale_tau))) return MXATTN_ERR_INVALID_ARG;
  if (o->key_tile != 64 && o->key_tile != 128) return MXATTN_ERR_INVALID_ARG;
  if (o->key_tile == 128 && o->format == MXATTN_FMT_NVFP4) return MXATTN_ERR_UNSUPPORTED;
  if (o->wait_budget_cycles < 0) return MXATTN_ERR_INVALID_ARG;
  if (o->causal != 0 && o->causal != 1) return MXATTN_ERR_INVALID_ARG;
  if (o->format != MXATTN_FMT_MXFP4 && o->format != MXATTN_FMT_NVFP4) return MXATTN_ERR_INVALID_ARG;
  if (o->causal && o->format == MXATTN_FMT_NVFP4) return MXATTN_ERR_UNSUPPORTED;  // NVFP4: full attention only
  return MXATTN_OK;
}

struct Carve {
  size_t q_codes, q_scales, k_codes, k_scales, v_codes, v_scales, total;
};

// Workspace carve-up: status block, then the packed Q operands (Nq tokens) and K/V operands (Nk).
Carve carve(int B, int H, int Nq, int Nk, int d, int fmt) {
  Carve c;
  size_t off = kStatusBytes;
  c.q_codes = off; off = align256(off + mxattn_qk_codes_bytes(B, H, Nq, d));
  c.q_scales = off; off = align256(off + qk_scale_bytes(B, H, Nq, d, fmt));
  c.k_codes = off; off = align256(off + mxattn_qk_codes_bytes(B, H, Nk, d));
  c.k_scales = off; off = align256(off + qk_scale_bytes(B, H, Nk, d, fmt));
  c.v_codes = off; off = align256(off + mxattn_v_codes_bytes(B, H, Nk, d));
  c.v_scales = off; off = align256(off + v_scale_bytes(B, H, Nk, fmt));
  c.total = off;
  return c;
}

int fmt_of(const mxattn_opts* o) { return o != nullptr ? o->format : MXATTN_FMT_MXFP4; }

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

mxattn_status launched(cudaError_t e) { return e == cudaSuccess ? MXATTN_OK : MXATTN_ERR_CUDA; }

mxattn_status check_workspace(const mxattn_opts* o, size_t need) {
  if (o->workspace == nullptr || o->workspace_bytes < need) return MXATTN_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(o->workspace) & 255u) != 0) return MXATTN_ERR_WORKSPACE;
  return MXATTN_OK;
}

}  // namespace

extern "C" {

void mxattn_opts_default(mxattn_opts* o) {
  if (o == nullptr) return;
  o->scale_rule = MXATTN_SCALE_UOS;
  o->qmax = 7.25f;
  o->pnq = 1;
  o->rotate = 1;
  o->dtype = MXATTN_BF16;
  o->key_tile = 128;
  o->rescale_tau = 8.0f;
  o->workspace = nullptr;
  o->workspace_bytes = 0;
  o->wait_budget_cycles = 0;
  o->causal = 0;
  o->format = MXATTN_FMT_MXFP4;
}

size_t mxattn_qk_codes_bytes(int B, int H, int N, int d) {
  if (!sizes_ok(B, H, N, d)) return 0;
  return (size_t)B * H * t128(N) * 128 * (d / 2);
}
size_t mxattn_qk_scales_bytes(int B, int H, int N, int d) {
  if (!sizes_ok(B, H, N, d)) return 0;
  return (size_t)B * H * t128(N) * 512;
}
size_t mxattn_v_codes_bytes(int B, int H, int N, int d) {
  if (!sizes_ok(B, H, N, d)) return 0;
  return (size_t)B * H * t64(N) * d * 32;
}
size_t mxattn_v_scales_bytes(int B, int H, int N, int d) {
  if (!sizes_ok(B, H, N, d)) return 0;
  return (size_t)B * H * t128(N) * 512;
}

mxattn_status mxattn_operand_bytes(int B, int H, int N, int d, const mxattn_opts* opts, size_t* sizes) {
  if (sizes == nullptr || !sizes_ok(B, H, N, d) || opts == nullptr) return MXATTN_ERR_INVALID_ARG;
  if (opts->format != MXATTN_FMT_MXFP4 && opts->format != MXATTN_FMT_NVFP4) return MXATTN_ERR_INVALID_ARG;
  sizes[0] = sizes[2] = mxattn_qk_codes_bytes(B, H, N, d);
  sizes[1] = sizes[3] = qk_scale_bytes(B, H, N, d, opts->format);
  sizes[4] = mxattn_v_codes_bytes(B, H, N, d);
  sizes[5] = v_scale_bytes(B, H, N, opts->format);
  return MXATTN_OK;
}

size_t mxattn_workspace_bytes(int B, int H, int N, int d, const mxattn_opts* opts) {
  (void)opts;
  if (!sizes_ok(B, H, N, d)) return 0;
  return carve(B, H, N, N, d, fmt_of(opts)).total;
}

mxattn_status mxattn_workspace_init(const mxattn_opts* o, void* stream) {
  if (o == nullptr) return MXATTN_ERR_INVALID_ARG;
  if (check_workspace(o, kStatusBytes) != MXATTN_OK) return MXATTN_ERR_WORKSPACE;
  return launched(cudaMemsetAsync(o->workspace, 0, kStatusBytes, as_stream(stream)));
}

mxattn_status mxattn_quantize_mxfp4(const void* x, int64_t rows, int64_t cols, int group_axis,
                                    const mxattn_opts* o, uint8_t* codes, uint8_t* scales, void* stream) {
  if (x == nullptr || codes == nullptr || scales == nullptr || rows < 1 || cols < 1) return MXATTN_ERR_INVALID_ARG;
  if (group_axis != 0 && group_axis != 1) return MXATTN_ERR_INVALID_ARG;
  mxattn_status st = check_opts(o);
  if (st != MXATTN_OK) return st;
  if (!aligned16(codes)) return MXATTN_ERR_INVALID_ARG;
  const int64_t outer = group_axis == 0 ? rows : cols;
  const int64_t inner = group_axis == 0 ? cols : rows;
  if (outer * ((inner + 31) / 32) > ((int64_t)1 << 38)) return MXATTN_ERR_UNSUPPORTED;
  PlainQuantArgs a;
  a.x = x;
  a.codes = codes;
  a.scales = scales;
  a.rows = rows;
  a.cols = cols;
  a.axis = group_axis;
  make_rule(o, &a.rule);
  a.fmt = o->format;
  return launched(launch_quant_plain(a, o->dtype, as_stream(stream)));
}

}  // extern "C"

namespace {

// Q (Nq tokens) and K (Nk tokens) rotated and quantized in one launch.
mxattn_status quant_qk(const void* q, const void* k, int B, int H, int Nq, int Nk, int d, const mxattn_opts* o,
                       uint8_t* q_codes, uint8_t* q_scales, uint8_t* k_codes, uint8_t* k_scales, void* stream) {
  if (!sizes_ok(B, H, Nq, d) || !sizes_ok(B, H, Nk, d))
    return (B >= 1 && H >= 1 && Nq >= 1 && Nk >= 1 && (d == 64 || d == 128)) ? MXATTN_ERR_UNSUPPORTED
                                                                               : MXATTN_ERR_INVALID_ARG;
  if (!q || !k || !q_codes || !q_scales || !k_codes || !k_scales) return MXATTN_ERR_INVALID_ARG;
  mxattn_status st = check_opts(o);
  if (st != MXATTN_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_codes) || !aligned16(k_codes)) return MXATTN_ERR_INVALID_ARG;
  QKQuantArgs a{};
  a.q = q;
  a.k = k;
  a.q_codes = q_codes;
  a.q_scales = q_scales;
  a.k_codes = k_codes;
  a.k_scales = k_scales;
  a.BH = B * H;
  a.N = Nq;
  a.Nk = Nk;
  a.rotate = o->rotate;
  a.hadamard_scale = (float)(1.0 / std::sqrt((double)d));
  make_rule(o, &a.rule);
  a.fmt = o->format;
  return launched(launch_rotate_quant_qk(a, d, o->dtype, as_stream(stream)));
}

}  // namespace

extern "C" {

mxattn_status mxattn_hadamard_quant_qk(const void* q, const void* k, int B, int H, int N, int d,
                                       const mxattn_opts* o, uint8_t* q_codes, uint8_t* q_scales,
                                       uint8_t* k_codes, uint8_t* k_scales, void* stream) {
  return quant_qk(q, k, B, H, N, N, d, o, q_codes, q_scales, k_codes, k_scales, stream);
}

mxattn_status mxattn_quant_v(const void* v, int B, int H, int N, int d, const mxattn_opts* o, uint8_t* v_codes,
                             uint8_t* v_scales, void* stream) {
  if (!sizes_ok(B, H, N, d)) return MXATTN_ERR_INVALID_ARG;
  if (!v || !v_codes || !v_scales) return MXATTN_ERR_INVALID_ARG;
  mxattn_status st = check_opts(o);
  if (st != MXATTN_OK) return st;
  if (!aligned16(v) || !aligned16(v_codes)) return MXATTN_ERR_INVALID_ARG;
  VQuantArgs a{};
  a.v = v;
  a.v_codes = v_codes;
  a.v_scales = v_scales;
  a.BH = B * H;
  a.N = N;
  make_rule(o, &a.rule);
  a.fmt = o->format;
  return launched(launch_quant_v(a, d, o->dtype, as_stream(stream)));
}

}  // extern "C"

namespace {

// Arguments of one attention launch on packed operands (no dump, no varlen table); the callers
// set those fields themselves.
AttnArgs attn_args(const uint8_t* q_codes, const uint8_t* q_scales, const uint8_t* k_codes, const uint8_t* k_scales,
                   const uint8_t* v_codes, const uint8_t* v_scales, int BH, int Nq, int Nk, float softmax_scale,
                   const mxattn_opts* o, void* out, int* status) {
  AttnArgs a{};
  a.q_codes = q_codes;
  a.q_scales = q_scales;
  a.k_codes = k_codes;
  a.k_scales = k_scales;
  a.v_codes = v_codes;
  a.v_scales = v_scales;
  a.out = out;
  a.status = status;
  a.BH = BH;
  a.N = Nq;
  a.Nk = Nk;
  a.causal = o->causal;
  a.scale_log2 = (float)((double)softmax_scale * 1.4426950408889634);  // softmax_scale * log2(e)
  a.tau = o->rescale_tau;
  a.pnq = o->pnq;
  make_rule(o, &a.rule);
  a.fmt = o->format;
  a.wait_budget = o->wait_budget_cycles > 0 ? o->wait_budget_cycles : kWaitBudgetCycles;
  a.dump = nullptr;
  a.dump_bh = a.dump_qt = -1;
  a.key_tile = o->key_tile;
  return a;
}

// The attention kernel for the options' key tile width.
cudaError_t launch_attn(const AttnArgs& a, int d, int dtype, cudaStream_t s) {
  return a.key_tile == 128 ? launch_attention_wide(a, d, dtype, s) : launch_attention(a, d, dtype, s);
}

mxattn_status attention(const uint8_t* q_codes, const uint8_t* q_scales, const uint8_t* k_codes,
                        const uint8_t* k_scales, const uint8_t* v_codes, const uint8_t* v_scales, int B, int H,
                        int Nq, int Nk, int d, float softmax_scale, const mxattn_opts* o, void* out, void* stream) {
  if (!sizes_ok(B, H, Nq, d) || !sizes_ok(B, H, Nk, d)) return MXATTN_ERR_INVALID_ARG;
  if (!q_codes || !q_scales || !k_codes || !k_scales || !v_codes || !v_scales || !out) return MXATTN_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f && std::isfinite(softmax_scale))) return MXATTN_ERR_INVALID_ARG;
  mxattn_status st = check_opts(o);
  if (st != MXATTN_OK) return st;
  if (o->causal && Nq != Nk) return MXATTN_ERR_UNSUPPORTED;
  st = check_workspace(o, kStatusBytes);
  if (st != MXATTN_OK) return st;
  const void* ptrs[] = {q_codes, q_scales, k_codes, k_scales, v_codes, v_scales, out};
  for (const void* p : ptrs)
    if (!aligned16(p)) return MXATTN_ERR_INVALID_ARG;
  const AttnArgs a = attn_args(q_codes, q_scales, k_codes, k_scales, v_codes, v_scales, B * H, Nq, Nk, softmax_scale,
                               o, out, reinterpret_cast<int*>(o->workspace));
  return launched(launch_attn(a, d, o->dtype, as_stream(stream)));
}

}  // namespace

extern "C" {

mxattn_status mxattn_attention_mxfp4(const uint8_t* q_codes, const uint8_t* q_scales, const uint8_t* k_codes,
                                     const uint8_t* k_scales, const uint8_t* v_codes, const uint8_t* v_scales,
                                     int B, int H, int N, int d, float softmax_scale, const mxattn_opts* o,
                                     void* out, void* stream) {
  return attention(q_codes, q_scales, k_codes, k_scales, v_codes, v_scales, B, H, N, N, d, softmax_scale, o, out,
                   stream);
}

size_t mxattn_attention_dump_bytes(int N, int d) {
  if (!sizes_ok(1, 1, N, d)) return 0;
  // large enough for either key tile width
  const size_t n64 = DumpLayout(d, (int)t64(N), 64).total, n128 = DumpLayout(d, (int)t128(N), 128).total;
  return n64 > n128 ? n64 : n128;
}

mxattn_status mxattn_attention_mxfp4_dump(const uint8_t* q_codes, const uint8_t* q_scales, const uint8_t* k_codes,
                                          const uint8_t* k_scales, const uint8_t* v_codes, const uint8_t* v_scales,
                                          int B, int H, int N, int d, float softmax_scale, const mxattn_opts* o,
                                          void* out, int dump_bh, int dump_qt, uint8_t* dump, void* stream) {
  if (dump == nullptr || !aligned16(dump) || dump_bh < 0 || dump_qt < 0) return MXATTN_ERR_INVALID_ARG;
  if (!sizes_ok(B, H, N, d) || dump_bh >= B * H || dump_qt >= t128(N)) return MXATTN_ERR_INVALID_ARG;
  if (!q_codes || !q_scales || !k_codes || !k_scales || !v_codes || !v_scales || !out) return MXATTN_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f && std::isfinite(softmax_scale))) return MXATTN_ERR_INVALID_ARG;
  mxattn_status st = check_opts(o);
  if (st != MXATTN_OK) return st;
  if (o->format != MXATTN_FMT_MXFP4) return MXATTN_ERR_UNSUPPORTED;  // the dump reads MXFP4 tiles
  if (o->causal) return MXATTN_ERR_UNSUPPORTED;                      // ... of full attention
  st = check_workspace(o, kStatusBytes);
  if (st != MXATTN_OK) return st;
  AttnArgs a = attn_args(q_codes, q_scales, k_codes, k_scales, v_codes, v_scales, B * H, N, N, softmax_scale, o, out,
                         reinterpret_cast<int*>(o->workspace));
  a.dump = dump;
  a.dump_bh = dump_bh;
  a.dump_qt = dump_qt;
  return launched(launch_attn(a, d, o->dtype, as_stream(stream)));
}

mxattn_status mxattn_forward(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                             float softmax_scale, const mxattn_opts* o, void* out, void* stream) {
  if (!sizes_ok(B, H, N, d)) return MXATTN_ERR_INVALID_ARG;
  if (!q || !k || !v || !out) return MXATTN_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f && std::isfinite(softmax_scale))) return MXATTN_ERR_INVALID_ARG;
  mxattn_status st = check_opts(o);
  if (st != MXATTN_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return MXATTN_ERR_INVALID_ARG;
  const Carve c = carve(B, H, N, N, d, o->format);
  st = check_workspace(o, c.total);
  if (st != MXATTN_OK) return st;
  uint8_t* ws = reinterpret_cast<uint8_t*>(o->workspace);
  st = mxattn_hadamard_quant_qk(q, k, B, H, N, d, o, ws + c.q_codes, ws + c.q_scales, ws + c.k_codes,
                                ws + c.k_scales, stream);
  if (st != MXATTN_OK) return st;
  st = mxattn_quant_v(v, B, H, N, d, o, ws + c.v_codes, ws + c.v_scales, stream);
  if (st != MXATTN_OK) return st;
  return mxattn_attention_mxfp4(ws + c.q_codes, ws + c.q_scales, ws + c.k_codes, ws + c.k_scales, ws + c.v_codes,
                                ws + c.v_scales, B, H, N, d, softmax_scale, o, out, stream);
}

size_t mxattn_workspace_bytes_cross(int B, int H, int Nq, int Nk, int d, const mxattn_opts* opts) {
  (void)opts;
  if (!sizes_ok(B, H, Nq, d) || !sizes_ok(B, H, Nk, d)) return 0;
  return carve(B, H, Nq, Nk, d, fmt_of(opts)).total;
}

mxattn_status mxattn_forward_cross(const void* q, const void* k, const void* v, int B, int H, int Nq, int Nk, int d,
                                   float softmax_scale, const mxattn_opts* o, void* out, void* stream) {
  if (!sizes_ok(B, H, Nq, d) || !sizes_ok(B, H, Nk, d)) return MXATTN_ERR_INVALID_ARG;
  if (!q || !k || !v || !out) return MXATTN_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f && std::isfinite(softmax_scale))) return MXATTN_ERR_INVALID_ARG;
  mxattn_status st = check_opts(o);
  if (st != MXATTN_OK) return st;
  if (o->causal) return MXATTN_ERR_UNSUPPORTED;  // no query/key position correspondence
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return MXATTN_ERR_INVALID_ARG;
  const Carve c = carve(B, H, Nq, Nk, d, o->format);
  st = check_workspace(o, c.total);
  if (st != MXATTN_OK) return st;
  uint8_t* ws = reinterpret_cast<uint8_t*>(o->workspace);
  st = quant_qk(q, k, B, H, Nq, Nk, d, o, ws + c.q_codes, ws + c.q_scales, ws + c.k_codes, ws + c.k_scales, stream);
  if (st != MXATTN_OK) return st;
  st = mxattn_quant_v(v, B, H, Nk, d, o, ws + c.v_codes, ws + c.v_scales, stream);
  if (st != MXATTN_OK) return st;
  return attention(ws + c.q_codes, ws + c.q_scales, ws + c.k_codes, ws + c.k_scales, ws + c.v_codes, ws + c.v_scales,
                   B, H, Nq, Nk, d, softmax_scale, o, out, stream);
}

}  // extern "C"

namespace {

// Packed varlen batch: nseq sequences, T tokens, token-major [T, H, d].  Every sequence is padded
// to whole 128-row tiles in the packed operands; sum over s of ceil(len_s / 128) is at most
// (T + 127 nseq) / 128 tiles per head, the stride the packing reserves.
constexpr int kMaxVarlenSeqs = 1 << 24;

bool varlen_sizes_ok(int nseq, int H, int T, int d, int64_t* tiles_per_head) {
  if (nseq < 1 || nseq > kMaxVarlenSeqs || H < 1 || H > 65535 || T < 1 || (d != 64 && d != 128)) return false;
  const int64_t tph = ((int64_t)T + 127 * (int64_t)nseq) / 128;
  if ((int64_t)H * 2 * tph >= ((int64_t)1 << 31)) return false;  // blocks of the V quantizer
  *tiles_per_head = tph;
  return true;
}

struct VarlenCarve {
  size_t tile_off, q_codes, q_scales, k_codes, k_scales, v_codes, v_scales, total;
};

VarlenCarve carve_varlen(int nseq, int H, int64_t tph, int d) {
  VarlenCarve c;
  const size_t codes = (size_t)H * tph * 128 * (d / 2), scales = (size_t)H * tph * 512;
  size_t off = kStatusBytes;
  c.tile_off = off; off = align256(off + ((size_t)nseq + 1) * sizeof(int));
  c.q_codes = off; off = align256(off + codes);
  c.q_scales = off; off = align256(off + scales);
  c.k_codes = off; off = align256(off + codes);
  c.k_scales = off; off = align256(off + scales);
  c.v_codes = off; off = align256(off + codes);  // 2 tph tiles of 64 keys x d channels x 32 bytes
  c.v_scales = off; off = align256(off + scales);
  c.total = off;
  return c;
}

}  // namespace

extern "C" {

size_t mxattn_workspace_bytes_varlen(int nseq, int H, int T, int d, const mxattn_opts* opts) {
  (void)opts;
  int64_t tph;
  if (!varlen_sizes_ok(nseq, H, T, d, &tph)) return 0;
  return carve_varlen(nseq, H, tph, d).total;
}

mxattn_status mxattn_forward_varlen(const void* q, const void* k, const void* v, const int* cu_seqlens, int nseq,
                                    int H, int T, int d, float softmax_scale, const mxattn_opts* o, void* out,
                                    void* stream) {
  int64_t tph;
  if (!varlen_sizes_ok(nseq, H, T, d, &tph)) return MXATTN_ERR_INVALID_ARG;
  if (!q || !k || !v || !out || !cu_seqlens) return MXATTN_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f && std::isfinite(softmax_scale))) return MXATTN_ERR_INVALID_ARG;
  mxattn_status st = check_opts(o);
  if (st != MXATTN_OK) return st;
  if (o->format != MXATTN_FMT_MXFP4) return MXATTN_ERR_UNSUPPORTED;  // NVFP4: full attention only
  const VarlenCarve c = carve_varlen(nseq, H, tph, d);
  st = check_workspace(o, c.total);
  if (st != MXATTN_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return MXATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return MXATTN_ERR_INVALID_ARG;
  uint8_t* ws = reinterpret_cast<uint8_t*>(o->workspace);
  int* status = reinterpret_cast<int*>(ws);
  int* tile_off = reinterpret_cast<int*>(ws + c.tile_off);
  const cudaStream_t s = as_stream(stream);
  const Varlen vl{cu_seqlens, tile_off, nseq, (int)tph};
  st = launched(launch_varlen_tiles(cu_seqlens, nseq, T, tile_off, status, s));
  if (st != MXATTN_OK) return st;
  ScaleRule rule;
  make_rule(o, &rule);

  QKQuantArgs qa{};
  qa.q = q;
  qa.k = k;
  qa.q_codes = ws + c.q_codes;
  qa.q_scales = ws + c.q_scales;
  qa.k_codes = ws + c.k_codes;
  qa.k_scales = ws + c.k_scales;
  qa.BH = H;
  qa.N = qa.Nk = T;
  qa.rotate = o->rotate;
  qa.hadamard_scale = (float)(1.0 / std::sqrt((double)d));
  qa.rule = rule;
  qa.fmt = o->format;
  qa.vl = vl;
  st = launched(launch_rotate_quant_qk(qa, d, o->dtype, s));
  if (st != MXATTN_OK) return st;

  VQuantArgs va{};
  va.v = v;
  va.v_codes = ws + c.v_codes;
  va.v_scales = ws + c.v_scales;
  va.BH = H;
  va.N = T;
  va.rule = rule;
  va.fmt = o->format;
  va.vl = vl;
  st = launched(launch_quant_v(va, d, o->dtype, s));
  if (st != MXATTN_OK) return st;

  AttnArgs a = attn_args(ws + c.q_codes, ws + c.q_scales, ws + c.k_codes, ws + c.k_scales, ws + c.v_codes,
                         ws + c.v_scales, H, T, T, softmax_scale, o, out, status);
  a.vl = vl;
  return launched(launch_attn(a, d, o->dtype, s));
}

}  // extern "C"

namespace {

// Internal streams and events of the host-buffer forward, created once per device on first use and
// kept until the process exits.
struct HostStreams {
  std::mutex mutex;  // one call at a time enqueues on them
  cudaStream_t s_in = nullptr, s_out = nullptr, s_c1 = nullptr;
  cudaEvent_t ev_start = nullptr, ev_in[2] = {}, ev_comp[2] = {}, ev_out[2] = {};
};
constexpr int kMaxHostDevices = 64;
std::mutex g_host_mutex;
HostStreams* g_host_streams[kMaxHostDevices] = {};

mxattn_status host_streams(HostStreams** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxHostDevices) return MXATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_host_mutex);
  if (g_host_streams[dev] == nullptr) {
    HostStreams* h = new HostStreams();
    bool ok = cudaStreamCreateWithFlags(&h->s_in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&h->s_out, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&h->s_c1, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&h->ev_start, cudaEventDisableTiming) == cudaSuccess;
    for (int b = 0; ok && b < 2; b++)
      ok = cudaEventCreateWithFlags(&h->ev_in[b], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&h->ev_comp[b], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&h->ev_out[b], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {  // release what was made; the next call tries again
      for (int b = 0; b < 2; b++) {
        if (h->ev_in[b]) cudaEventDestroy(h->ev_in[b]);
        if (h->ev_comp[b]) cudaEventDestroy(h->ev_comp[b]);
        if (h->ev_out[b]) cudaEventDestroy(h->ev_out[b]);
      }
      if (h->ev_start) cudaEventDestroy(h->ev_start);
      if (h->s_in) cudaStreamDestroy(h->s_in);
      if (h->s_out) cudaStreamDestroy(h->s_out);
      if (h->s_c1) cudaStreamDestroy(h->s_c1);
      delete h;
      return MXATTN_ERR_CUDA;
    }
    g_host_streams[dev] = h;
  }
  *out = g_host_streams[dev];
  return MXATTN_OK;
}

// Host-buffer forward: the heads are processed in chunks, each chunk an independent problem.
#ifndef MXATTN_HOST_CHUNKS
#define MXATTN_HOST_CHUNKS 40
#endif
constexpr int kHostChunks = MXATTN_HOST_CHUNKS;

struct HostPlan {
  int BH, hc, nch;               // heads, heads per chunk, chunks
  size_t head_bytes;             // one head of q, k, v or out
  size_t in_off[2], out_off[2];  // double-buffered q|k|v and out staging
  size_t qc[2], qs[2], kc[2], ks[2], vc[2], vs[2];  // packed operands, one set per compute stream
  size_t total;
};

HostPlan host_plan(int B, int H, int N, int d, int dtype, int fmt) {
  HostPlan p;
  p.BH = B * H;
  int nch = p.BH < kHostChunks ? p.BH : kHostChunks;
  p.hc = (p.BH + nch - 1) / nch;
  p.nch = (p.BH + p.hc - 1) / p.hc;
  p.head_bytes = (size_t)N * d * (dtype == MXATTN_BF16 ? 2 : 4);
  size_t off = kStatusBytes;
  for (int b = 0; b < 2; b++) {
    p.in_off[b] = off;
    off = align256(off + 3 * (size_t)p.hc * p.head_bytes);
  }
  for (int b = 0; b < 2; b++) {
    p.out_off[b] = off;
    off = align256(off + (size_t)p.hc * p.head_bytes);
  }
  for (int b = 0; b < 2; b++) {
    p.qc[b] = off; off = align256(off + mxattn_qk_codes_bytes(1, p.hc, N, d));
    p.qs[b] = off; off = align256(off + qk_scale_bytes(1, p.hc, N, d, fmt));
    p.kc[b] = off; off = align256(off + mxattn_qk_codes_bytes(1, p.hc, N, d));
    p.ks[b] = off; off = align256(off + qk_scale_bytes(1, p.hc, N, d, fmt));
    p.vc[b] = off; off = align256(off + mxattn_v_codes_bytes(1, p.hc, N, d));
    p.vs[b] = off; off = align256(off + v_scale_bytes(1, p.hc, N, fmt));
  }
  p.total = off;
  return p;
}

}  // namespace

extern "C" {

size_t mxattn_workspace_bytes_host(int B, int H, int N, int d, const mxattn_opts* opts) {
  if (!sizes_ok(B, H, N, d)) return 0;
  return host_plan(B, H, N, d, opts != nullptr ? opts->dtype : MXATTN_BF16, fmt_of(opts)).total;
}

mxattn_status mxattn_forward_host(const void* q_host, const void* k_host, const void* v_host, int B, int H, int N,
                                  int d, float softmax_scale, const mxattn_opts* o, void* out_host, void* stream) {
  if (!sizes_ok(B, H, N, d)) return MXATTN_ERR_INVALID_ARG;
  if (!q_host || !k_host || !v_host || !out_host) return MXATTN_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f && std::isfinite(softmax_scale))) return MXATTN_ERR_INVALID_ARG;
  mxattn_status st = check_opts(o);
  if (st != MXATTN_OK) return st;
  const HostPlan p = host_plan(B, H, N, d, o->dtype, o->format);
  st = check_workspace(o, p.total);
  if (st != MXATTN_OK) return st;
  uint8_t* ws = reinterpret_cast<uint8_t*>(o->workspace);
  const uint8_t* qh = reinterpret_cast<const uint8_t*>(q_host);
  const uint8_t* kh = reinterpret_cast<const uint8_t*>(k_host);
  const uint8_t* vh = reinterpret_cast<const uint8_t*>(v_host);
  uint8_t* oh = reinterpret_cast<uint8_t*>(out_host);
  cudaStream_t s = as_stream(stream);

  // Copies in on s_in, copies out on s_out, and the chunks' kernels alternately on the caller's
  // stream and a second compute stream, each with its own operand buffers: a chunk's kernels start
  // on the SMs that the previous chunk's last wave of CTAs leaves idle instead of after it.  Every
  // cross-stream order is an event; the caller's stream finally waits for the last copies out.
  // The internal streams and events are created once per device and kept; calls on one device
  // enqueue one at a time (a host mutex), so two host threads never interleave their records.
  HostStreams* hs = nullptr;
  st = host_streams(&hs);
  if (st != MXATTN_OK) return st;
  std::lock_guard<std::mutex> lock(hs->mutex);
  const cudaStream_t s_in = hs->s_in, s_out = hs->s_out, s_c1 = hs->s_c1;
  cudaEvent_t const* ev_in = hs->ev_in;
  cudaEvent_t const* ev_comp = hs->ev_comp;
  cudaEvent_t const* ev_out = hs->ev_out;
  // work already on the caller's stream comes first
  bool ok = cudaEventRecord(hs->ev_start, s) == cudaSuccess && cudaStreamWaitEvent(s_in, hs->ev_start, 0) == cudaSuccess &&
            cudaStreamWaitEvent(s_out, hs->ev_start, 0) == cudaSuccess &&
            cudaStreamWaitEvent(s_c1, hs->ev_start, 0) == cudaSuccess;
  const cudaStream_t s_comp[2] = {s, s_c1};
  st = ok ? MXATTN_OK : MXATTN_ERR_CUDA;
  bool recorded_out[2] = {false, false};
  for (int c = 0; st == MXATTN_OK && c < p.nch; c++) {
    const int b = c & 1;
    const cudaStream_t cs = s_comp[b];  // chunk c-2 ran on it too, with the same buffers
    void* const csv = reinterpret_cast<void*>(cs);
    const int h0 = c * p.hc;
    const int hn = p.BH - h0 < p.hc ? p.BH - h0 : p.hc;
    const size_t bytes = (size_t)hn * p.head_bytes, src = (size_t)h0 * p.head_bytes;
    uint8_t* in = ws + p.in_off[b];
    uint8_t* qd = in;
    uint8_t* kd = in + (size_t)p.hc * p.head_bytes;
    uint8_t* vd = in + 2 * (size_t)p.hc * p.head_bytes;
    uint8_t* od = ws + p.out_off[b];
    // inputs of chunk c into buffer b once chunk c-2 has finished reading it
    if (c >= 2 && cudaStreamWaitEvent(s_in, ev_comp[b], 0) != cudaSuccess) { st = MXATTN_ERR_CUDA; break; }
    if (cudaMemcpyAsync(qd, qh + src, bytes, cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
        cudaMemcpyAsync(kd, kh + src, bytes, cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
        cudaMemcpyAsync(vd, vh + src, bytes, cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
        cudaEventRecord(ev_in[b], s_in) != cudaSuccess || cudaStreamWaitEvent(cs, ev_in[b], 0) != cudaSuccess) {
      st = MXATTN_ERR_CUDA;
      break;
    }
    // the output buffer b is free once chunk c-2's copy out has finished
    if (c >= 2 && cudaStreamWaitEvent(cs, ev_out[b], 0) != cudaSuccess) { st = MXATTN_ERR_CUDA; break; }
    st = quant_qk(qd, kd, 1, hn, N, N, d, o, ws + p.qc[b], ws + p.qs[b], ws + p.kc[b], ws + p.ks[b], csv);
    if (st == MXATTN_OK) st = mxattn_quant_v(vd, 1, hn, N, d, o, ws + p.vc[b], ws + p.vs[b], csv);
    if (st == MXATTN_OK)
      st = attention(ws + p.qc[b], ws + p.qs[b], ws + p.kc[b], ws + p.ks[b], ws + p.vc[b], ws + p.vs[b], 1, hn, N, N,
                     d, softmax_scale, o, od, csv);
    if (st != MXATTN_OK) break;
    if (cudaEventRecord(ev_comp[b], cs) != cudaSuccess || cudaStreamWaitEvent(s_out, ev_comp[b], 0) != cudaSuccess ||
        cudaMemcpyAsync(oh + src, od, bytes, cudaMemcpyDeviceToHost, s_out) != cudaSuccess ||
        cudaEventRecord(ev_out[b], s_out) != cudaSuccess) {
      st = MXATTN_ERR_CUDA;
      break;
    }
    recorded_out[b] = true;
  }
  // join: the caller's stream waits for every copy out of this call (and, through them, everything
  // else), and for the internal streams' starting point
  for (int b = 0; b < 2; b++)
    if (recorded_out[b] && cudaStreamWaitEvent(s, ev_out[b], 0) != cudaSuccess && st == MXATTN_OK) st = MXATTN_ERR_CUDA;
  if (cudaStreamWaitEvent(s, hs->ev_start, 0) != cudaSuccess && st == MXATTN_OK) st = MXATTN_ERR_CUDA;
  return st;
}

mxattn_status mxattn_qmax_sweep(const void* x, int64_t rows, int64_t cols, int dtype, int rotate,
                                const float* qs, int nq, unsigned long long* counts, double* sse_sums,
                                void* stream) {
  if (x == nullptr || qs == nullptr || counts == nullptr || sse_sums == nullptr) return MXATTN_ERR_INVALID_ARG;
  if (rows < 1 || cols < 1 || nq < 1 || nq > kSweepMaxQ) return MXATTN_ERR_INVALID_ARG;
  if (dtype != MXATTN_BF16 && dtype != MXATTN_FP32) return MXATTN_ERR_INVALID_ARG;
  if (rotate != 0 && rotate != 1) return MXATTN_ERR_INVALID_ARG;
  if (rotate && cols != 64 && cols != 128) return MXATTN_ERR_INVALID_ARG;
  if (rows * ((cols + 31) / 32) > ((int64_t)1 << 38)) return MXATTN_ERR_UNSUPPORTED;
  SweepArgs a;
  a.x = x;
  a.rows = rows;
  a.cols = cols;
  a.rotate = rotate;
  a.hadamard_scale = (float)(1.0 / std::sqrt((double)cols));
  a.nq = nq;
  mxattn_opts o;
  mxattn_opts_default(&o);
  o.scale_rule = MXATTN_SCALE_CEIL_CUSTOM;
  for (int k = 0; k < nq; k++) {
    if (k > 0 && !(qs[k] > qs[k - 1])) return MXATTN_ERR_INVALID_ARG;
    o.qmax = qs[k];
    if (!make_rule(&o, &a.rules[k])) return MXATTN_ERR_INVALID_ARG;  // q in [4, 8]
  }
  a.counts = counts;
  a.sse_sums = sse_sums;
  return launched(launch_qmax_sweep(a, dtype, as_stream(stream)));
}

mxattn_status mxattn_get_device_error(const mxattn_opts* o, void* stream) {
  if (o == nullptr) return MXATTN_ERR_INVALID_ARG;
  if (check_workspace(o, kStatusBytes) != MXATTN_OK) return MXATTN_ERR_WORKSPACE;
  int words[4] = {0, 0, 0, 0};
  cudaStream_t s = as_stream(stream);
  if (cudaMemcpyAsync(words, o->workspace, sizeof(words), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MXATTN_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MXATTN_ERR_CUDA;
  if (words[0] == 0) return MXATTN_OK;
  if (cudaMemsetAsync(o->workspace, 0, kStatusBytes, s) != cudaSuccess) return MXATTN_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MXATTN_ERR_CUDA;
  return words[0] == kStatusBadSeqlens ? MXATTN_ERR_INVALID_ARG : MXATTN_ERR_TIMEOUT;
}

const char* mxattn_status_string(mxattn_status s) {
  switch (s) {
    case MXATTN_OK: return "MXATTN_OK";
    case MXATTN_ERR_INVALID_ARG: return "MXATTN_ERR_INVALID_ARG";
    case MXATTN_ERR_UNSUPPORTED: return "MXATTN_ERR_UNSUPPORTED";
    case MXATTN_ERR_WORKSPACE: return "MXATTN_ERR_WORKSPACE";
    case MXATTN_ERR_CUDA: return "MXATTN_ERR_CUDA";
    case MXATTN_ERR_TIMEOUT: return "MXATTN_ERR_TIMEOUT";
  }
  return "unknown mxattn_status";
}

mxattn_status mxattn_arith_probe(int op, const float* in, int64_t n, const mxattn_opts* o, void* out, void* stream) {
  if (in == nullptr || out == nullptr || n < 1 || op < MXATTN_PROBE_EXP2_POLY || op > MXATTN_PROBE_SCALE_EXP)
    return MXATTN_ERR_INVALID_ARG;
  const mxattn_status st = check_opts(o);
  if (st != MXATTN_OK) return st;
  if ((reinterpret_cast<uintptr_t>(in) & 3u) != 0 || (op != MXATTN_PROBE_E2M1_OF_EXP2_STANDIN &&
                                                      op != MXATTN_PROBE_E2M1_OF_EXP2_MUFU &&
                                                      (reinterpret_cast<uintptr_t>(out) & 3u) != 0))
    return MXATTN_ERR_INVALID_ARG;
  ScaleRule r;
  make_rule(o, &r);
  return launched(launch_arith_probe(op, in, n, r, out, as_stream(stream)));
}

mxattn_status mxattn_fp4_mma_probe(int ctas, int iters, int n, void* stream) {
  if (ctas < 1 || ctas > 65535 || iters < 1 || (n != 64 && n != 128 && n != 256)) return MXATTN_ERR_INVALID_ARG;
  return launched(launch_fp4_mma_probe(ctas, iters, n, nullptr, as_stream(stream)));
}

}  // extern "C"

// quant.cu -- MXFP4 quantizers (rotation + quantization of Q/K, V along keys, and a plain
// generic quantizer).  Memory-bound: every byte is read once and written once, loads and
// stores are 16-byte vectors (inputs staged through shared memory by cp.async), and the FWHT
// butterflies of a row run in one thread's registers.
//
// Method: "MXAttention: Data-Free Optimal Scaling and Pre-Normalization Quantization for
// MXFP4 Attention" -- Pith review page (axioms ledger: 32-element E2M1 groups with one E8M0
// scale, round to nearest with saturation; Fig. 3: OCP floor [4,8), TFS (3,6], UOS
// (3.625,7.25]; Fig. 1: fixed Hadamard rotation on Q/K) and the 10100.com article.
//
// Every product here is x * 2^-e (exact) and every sum is an fp32 butterfly with explicit
// round-to-nearest intrinsics, so the codes are a deterministic function of the inputs.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace mxattn {

// One NVFP4 block of 16 values (the comparison format): the scale is the E4M3 rounding of
// fl32(amax / 6), each value is divided by it in fp32 (correctly rounded) and rounded to E2M1
// with saturation; a scale that rounds to zero gives zero codes.  Returns the scale byte.
// The quotients: with r = RN(1/s), y = RN(v r) is within an ulp of v/s, the remainder
// v - y s is exact in one fma, and RN(y + (v - y s) r) is RN(v/s) (Markstein's theorem); three
// FMA-pipe operations per value instead of a division (checked against RN(v/s) for every positive
// E4M3 scale on 25 million quotients, and bit-exact against the oracle's division in the tests).
__device__ __forceinline__ uint32_t nvfp4_block(const float* v, uint32_t* w) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; i++) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t byte = cvt_e4m3x2(__fdiv_rn(amax, 6.f), 0.f) & 0xFFu;
  const float s = e4m3x2_to_float2(byte).x;
  const float r = s > 0.f ? __frcp_rn(s) : 0.f;
  float y[16];
#pragma unroll
  for (int i = 0; i < 16; i++) {
    // on |v|, the sign copied back (RN is symmetric; -0 keeps its sign, as the division does)
    const float av = fabsf(v[i]);
    const float y0 = __fmul_rn(av, r);
    y[i] = s > 0.f ? copysignf(__fmaf_rn(__fmaf_rn(-y0, s, av), r, y0), v[i]) : 0.f;
  }
  w[0] = cvt_e2m1x8(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]);
  w[1] = cvt_e2m1x8(y[8], y[9], y[10], y[11], y[12], y[13], y[14], y[15]);
  return byte;
}

// ------------------------------------------------------------------------------------------------
// Q/K: Hadamard rotation + quantization along d into the packed QK operand layout.
// One thread per padded token row: the row's D values are staged through shared memory (16-byte
// cp.async copies of the block's rows, zeros for padding rows), then the thread runs every
// butterfly stage h = 1, 2, ..., D/2 of the fast Walsh-Hadamard transform in registers, scales by
// fl32(1/sqrt(D)), and quantizes its D/32 groups.  No value crosses threads, so the row needs no
// shuffles.  Grid: x over the 128-row packed tiles of the longer of Q and K (SPLIT blocks per
// tile), y = 0 for Q, 1 for K; varlen: over H * tiles_per_head tiles, each tile belonging to one
// sequence.
// ------------------------------------------------------------------------------------------------
// Where the rows of packed tile `tile` (bh * T128 + tile within the head) come from: rows r <
// nvalid are source rows src_row0 + r * stride of the [rows, D] input; the rest are padding.
struct QKTile {
  bool ok;  // the tile exists (varlen: tiles past the last sequence's are unused)
  int nvalid;
  int64_t src_row0, stride;
};

__device__ __forceinline__ QKTile qk_tile(const QKQuantArgs& a, uint32_t tile, uint32_t T128, int Nt) {
  QKTile q;
  const uint32_t bh = tile / T128;  // tile counts fit 32 bits (the grid is one-dimensional)
  const int tt = (int)(tile - bh * T128);
  q.ok = bh < (uint32_t)a.BH;
  if (a.vl.cu_seqlens != nullptr) {
    q.ok = q.ok && tt < __ldg(a.vl.tile_off + a.vl.nseq);
    const int sq = q.ok ? varlen_sequence(a.vl, tt) : 0;
    const int start = __ldg(a.vl.cu_seqlens + sq);
    const int n0 = (tt - __ldg(a.vl.tile_off + sq)) * 128;
    const int len = __ldg(a.vl.cu_seqlens + sq + 1) - start;
    q.nvalid = len - n0 < 0 ? 0 : (len - n0 > 128 ? 128 : len - n0);
    q.src_row0 = ((int64_t)start + n0) * a.BH + (int64_t)bh;  // token-major [T, H, d]
    q.stride = a.BH;
  } else {
    const int tok0 = tt * 128;
    q.nvalid = Nt - tok0 < 0 ? 0 : (Nt - tok0 > 128 ? 128 : Nt - tok0);
    q.src_row0 = (int64_t)bh * Nt + tok0;
    q.stride = 1;
  }
  return q;
}

// In-place fast Walsh-Hadamard transform of one row, stages h = 1, ..., D/2, each butterfly
// (x, y) -> (x + y, x - y) rounded once (x - y as fma(y, -1, x)); from h = 2 on, neighbours i,
// i+1 pair up into f32x2 operations with the same roundings.  The multiply by fl32(1/sqrt(D))
// that ends the rotation is left to the quantizer (rotate_quant_qk_kernel), which folds it into
// the group's scaling where that is exact.
template <int D>
__device__ __forceinline__ void fwht_row(float (&v)[D]) {
#pragma unroll
  for (int i = 0; i < D; i += 2) {
    const float x = v[i], y = v[i + 1];
    v[i] = __fadd_rn(x, y);
    v[i + 1] = __fsub_rn(x, y);
  }
  const float2 minus1 = make_float2(-1.f, -1.f);
#pragma unroll
  for (int h = 2; h < D; h <<= 1) {
#pragma unroll
    for (int i = 0; i < D; i += 2) {
      if ((i & h) == 0) {
        const float2 x = make_float2(v[i], v[i + 1]), y = make_float2(v[i + h], v[i + h + 1]);
        const float2 sum = __fadd2_rn(x, y), dif = __ffma2_rn(y, minus1, x);
        v[i] = sum.x; v[i + 1] = sum.y;
        v[i + h] = dif.x; v[i + h + 1] = dif.y;
      }
    }
  }
}

// Rows (threads) per block, and the blocks each SM must hold at D = 128 (the register cap that
// follows, 168 a thread, holds the row's 128 values without spilling).  Measured on the 720p
// shapes: 64-row blocks six to an SM beat 128-row blocks three to an SM by 5%, and either is
// a third faster than two 128-row blocks at the registers the compiler would otherwise take.
constexpr int kQKRows = 64;
constexpr int kQKBlocksPerSM128 = 6;
template <int D, int DT>
struct QKBlock {
  static constexpr int ES = DT == kBF16 ? 2 : 4;       // bytes per element
  static constexpr int ROWS = kQKRows;                 // rows per block (threads)
  static constexpr int SPLIT = 128 / ROWS;             // blocks per packed tile
  static constexpr int ROWB = D * ES;                  // source bytes per row
  static constexpr int PITCH = ROWB + 16;              // staged row pitch: rows 4 banks apart
};

// MXFP4 codes of one group of 32 rotated values x = fl(y * hs) (rotate) or x = y: with
// e = shared_exponent(max |x|), each code is E2M1(x * 2^-e).  max |x| = fl(max |y| * hs) as
// rounding is monotone, and fl(y * hs) * 2^-e = fl(y * (hs * 2^-e)) exactly whenever hs * 2^-e is
// a normal number and y * hs does not underflow; a y * hs that does underflow gives code 0 either
// way unless e is near -127, and those groups (max |x| below ~2^-97) take the two roundings as
// the definition states.
__device__ __forceinline__ int mx_group_codes(float* y, bool rotate, float hs, ScaleRule rule, uint32_t (&w)[4]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; i++) amax = fmaxf(amax, fabsf(y[i]));
  if (rotate) amax = __fmul_rn(amax, hs);
  const int e = shared_exponent(amax, rule);
  float mul = pow2_neg(e);
  if (rotate) {
    if (e > -100) {
      mul = __fmul_rn(hs, mul);  // exact
    } else {
#pragma unroll
      for (int i = 0; i < 32; i++) y[i] = __fmul_rn(y[i], hs);
    }
  }
  const float2 m2 = make_float2(mul, mul);
#pragma unroll
  for (int q = 0; q < 4; q++) {
    float2 p[4];
#pragma unroll
    for (int k = 0; k < 4; k++) p[k] = __fmul2_rn(make_float2(y[8 * q + 2 * k], y[8 * q + 2 * k + 1]), m2);
    w[q] = cvt_e2m1x8(p[0].x, p[0].y, p[1].x, p[1].y, p[2].x, p[2].y, p[3].x, p[3].y);
  }
  return e;
}

template <int D, int DT, bool NVF>
__global__ void __launch_bounds__(QKBlock<D, DT>::ROWS, kQKBlocksPerSM128) rotate_quant_qk_kernel(QKQuantArgs a) {
  using B = QKBlock<D, DT>;
  __shared__ __align__(16) uint8_t stage[B::ROWS * B::PITCH];
  const int t = threadIdx.x;
  const int Nt = blockIdx.y == 0 ? a.N : a.Nk;  // tokens of this tensor
  const uint32_t T128 = a.vl.cu_seqlens != nullptr ? (uint32_t)a.vl.tiles_per_head : (uint32_t)(Nt + 127) / 128;
  const uint32_t tile = blockIdx.x / B::SPLIT;
  const int row0 = (int)(blockIdx.x % B::SPLIT) * B::ROWS;  // first row of the tile this block takes
  const QKTile qt = qk_tile(a, tile, T128, Nt);
  if (!qt.ok) return;  // the whole block
  const uint8_t* src = reinterpret_cast<const uint8_t*>(blockIdx.y == 0 ? a.q : a.k);
  // stage: consecutive threads copy consecutive 16-byte chunks of a row (coalesced)
#pragma unroll
  for (int idx = t; idx < B::ROWS * (B::ROWB / 16); idx += B::ROWS) {
    const int rr = idx / (B::ROWB / 16), chunk = idx % (B::ROWB / 16);
    const int r = row0 + rr;
    const bool valid = r < qt.nvalid;
    const uint8_t* g = src + (qt.src_row0 + (int64_t)(valid ? r : 0) * qt.stride) * B::ROWB + chunk * 16;
    cp_async16(smem_u32(stage + rr * B::PITCH + chunk * 16), g, valid ? 16u : 0u);
  }
  cp_async_wait_all();
  __syncthreads();
  float v[D];
  const uint8_t* mine = stage + t * B::PITCH;
#pragma unroll
  for (int c = 0; c < B::ROWB / 16; c++) {
    const uint4 w = *reinterpret_cast<const uint4*>(mine + 16 * c);
    if (DT == kBF16) {
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int k = 0; k < 4; k++) {
        v[8 * c + 2 * k] = __uint_as_float(ww[k] << 16);
        v[8 * c + 2 * k + 1] = __uint_as_float(ww[k] & 0xFFFF0000u);
      }
    } else {
      v[4 * c] = __uint_as_float(w.x);
      v[4 * c + 1] = __uint_as_float(w.y);
      v[4 * c + 2] = __uint_as_float(w.z);
      v[4 * c + 3] = __uint_as_float(w.w);
    }
  }
  const bool rotate = a.rotate != 0;
  if (rotate) fwht_row<D>(v);
  const int r = row0 + t;  // row within the tile
  uint8_t* codes = blockIdx.y == 0 ? a.q_codes : a.k_codes;
  uint8_t* scales = blockIdx.y == 0 ? a.q_scales : a.k_scales;
  uint8_t* rowp = codes + ((int64_t)tile * 128 + r) * (D / 2);
  const int sw = (D == 128) ? ((r >> 1) & 3) : ((r >> 2) & 1);
  uint32_t sbytes = 0;  // MXFP4: the row's D/32 scale bytes; NVFP4: four block bytes per atom
#pragma unroll
  for (int g = 0; g < D / 32; g++) {
    float* x = v + 32 * g;
    uint32_t w[4];
    if (NVF) {
      if (rotate) {
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float2 r2 = __fmul2_rn(make_float2(x[i], x[i + 1]), make_float2(a.hadamard_scale, a.hadamard_scale));
          x[i] = r2.x; x[i + 1] = r2.y;
        }
      }
      const uint32_t b = nvfp4_block(x, w) | (nvfp4_block(x + 16, w + 2) << 8);
      sbytes |= b << (16 * (g % 2));
      if (g % 2 == 1) {
        // D/64 scale atoms per tile, one per 64 dims (one K = 64 MMA): blocks 4a..4a+3 in the
        // bytes of row r's word
        uint8_t* atom = scales + (int64_t)tile * (512 * (D / 64)) + (g / 2) * 512 + (r % 32) * 16 + (r / 32) * 4;
        *reinterpret_cast<uint32_t*>(atom) = sbytes;
        sbytes = 0;
      }
    } else {
      const int e = mx_group_codes(x, rotate, a.hadamard_scale, a.rule, w);
      sbytes |= (uint32_t)(e + 127) << (8 * g);  // D = 64: bytes 2, 3 (unused slots) stay 0
    }
    *reinterpret_cast<uint4*>(rowp + ((g ^ sw) * 16)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (!NVF) *reinterpret_cast<uint32_t*>(scales + (int64_t)tile * 512 + (r % 32) * 16 + (r / 32) * 4) = sbytes;
}

// ------------------------------------------------------------------------------------------------
// V: quantization along keys (32 consecutive tokens per channel) into the packed V operand
// layout.  One block of D threads per (head, 64-key tile): the tile's 64 key rows are copied into
// shared memory as they are (bf16 or fp32, 16-byte cp.async copies, zeros for keys past the
// sequence), then thread t quantizes channels 2p, 2p+1 (p = t mod D/2) over keys 32h..32h+31
// (h = t / (D/2)), reading both channels of a key in one 32- or 64-bit word.
// Varlen: items over (head, 64-key tile of the packed tiles); each sequence's groups start at its
// first token, and a sequence's tiles past its own keys are left unwritten.
// ------------------------------------------------------------------------------------------------
struct VTile {
  bool ok;                 // the item holds keys of a sequence
  int N, T64, j;           // keys of its sequence, their 64-key tiles, and this tile among them
  int64_t src_row0;        // source row of key 0
  int64_t src_stride;      // source rows per key
  int64_t vtile;           // packed 64-key code tile
  int64_t atom_tile;       // packed 128-key scale atom
};

__device__ __forceinline__ VTile v_tile(const VQuantArgs& a, int64_t item) {
  VTile t;
  t.ok = true;
  if (a.vl.cu_seqlens != nullptr) {
    const int per_head = 2 * a.vl.tiles_per_head;
    const int bh = (int)(item / per_head);
    const int jg = (int)(item % per_head);
    if (jg / 2 >= __ldg(a.vl.tile_off + a.vl.nseq)) {
      t.ok = false;
      return t;
    }
    const int sq = varlen_sequence(a.vl, jg / 2);
    const int start = __ldg(a.vl.cu_seqlens + sq);
    t.N = __ldg(a.vl.cu_seqlens + sq + 1) - start;
    t.T64 = (t.N + 63) / 64;
    t.j = jg - 2 * __ldg(a.vl.tile_off + sq);
    t.ok = t.j < t.T64;  // not the unused odd half of a sequence's last atom
    t.src_row0 = (int64_t)start * a.BH + bh;
    t.src_stride = a.BH;
    t.vtile = (int64_t)bh * per_head + jg;
    t.atom_tile = (int64_t)bh * a.vl.tiles_per_head + jg / 2;
  } else {
    t.N = a.N;
    t.T64 = (a.N + 63) / 64;
    const int bh = (int)(item / t.T64);
    t.j = (int)(item % t.T64);
    t.src_row0 = (int64_t)bh * a.N;
    t.src_stride = 1;
    t.vtile = item;
    t.atom_tile = (int64_t)bh * ((a.N + 127) / 128) + t.j / 2;
  }
  return t;
}

template <int D, int DT, bool NVF>
__global__ void __launch_bounds__(D) quant_v_kernel(VQuantArgs a) {
  constexpr int ES = DT == kBF16 ? 2 : 4;  // bytes per element
  constexpr int ROW = D * ES;              // bytes per key row
  __shared__ __align__(16) uint8_t tile[64 * ROW];
  const int t = threadIdx.x;
  const VTile vt = v_tile(a, blockIdx.x);
  if (!vt.ok) return;  // the whole block
  const int j = vt.j;
#pragma unroll
  for (int idx = t; idx < 64 * ROW / 16; idx += D) {
    const int row = idx / (ROW / 16), chunk = idx % (ROW / 16);
    const int tok = j * 64 + row;
    const bool valid = tok < vt.N;
    const uint8_t* src = reinterpret_cast<const uint8_t*>(a.v) +
                         (vt.src_row0 + (int64_t)(valid ? tok : 0) * vt.src_stride) * ROW + chunk * 16;
    cp_async16(smem_u32(tile + row * ROW + chunk * 16), src, valid ? 16u : 0u);
  }
  cp_async_wait_all();
  __syncthreads();
  const int p = t % (D / 2), h = t / (D / 2);
  float x[2][32];  // channels 2p, 2p+1 over keys 32h..32h+31
#pragma unroll
  for (int i = 0; i < 32; i++) {
    const uint8_t* r = tile + (32 * h + i) * ROW;
    if (DT == kBF16) {
      const uint32_t wv = *reinterpret_cast<const uint32_t*>(r + 4 * p);
      x[0][i] = __uint_as_float(wv << 16);
      x[1][i] = __uint_as_float(wv & 0xFFFF0000u);
    } else {
      const float2 f = *reinterpret_cast<const float2*>(r + 8 * p);
      x[0][i] = f.x;
      x[1][i] = f.y;
    }
  }
#pragma unroll
  for (int k = 0; k < 2; k++) {
    const int c = 2 * p + k;
    const float* v = x[k];
    uint8_t* dst = a.v_codes + (vt.vtile * D + c) * 32 + ((h ^ ((c >> 2) & 1)) * 16);
    uint32_t w[4];
    if (NVF) {
      // two blocks of 16 keys; one scale atom per 64-key tile, keys 16b..16b+15 in byte b of
      // channel c's word
      const uint32_t b = nvfp4_block(v, w) | (nvfp4_block(v + 16, w + 2) << 8);
      *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
      uint8_t* atom = a.v_scales + vt.vtile * 512;
      *reinterpret_cast<uint16_t*>(atom + (c % 32) * 16 + (c / 32) * 4 + 2 * h) = (uint16_t)b;
      if (D == 64) *reinterpret_cast<uint16_t*>(atom + ((c + 64) % 32) * 16 + ((c + 64) / 32) * 4 + 2 * h) = 0;
      continue;
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; i++) amax = fmaxf(amax, fabsf(v[i]));
    const int e = shared_exponent(amax, a.rule);
    const float inv = pow2_neg(e);
#pragma unroll
    for (int q = 0; q < 4; q++)
      w[q] = cvt_e2m1x8(__fmul_rn(v[8 * q + 0], inv), __fmul_rn(v[8 * q + 1], inv), __fmul_rn(v[8 * q + 2], inv),
                        __fmul_rn(v[8 * q + 3], inv), __fmul_rn(v[8 * q + 4], inv), __fmul_rn(v[8 * q + 5], inv),
                        __fmul_rn(v[8 * q + 6], inv), __fmul_rn(v[8 * q + 7], inv));
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
    uint8_t* atom = a.v_scales + vt.atom_tile * 512;
    atom[(c % 32) * 16 + (c / 32) * 4 + (j % 2) * 2 + h] = (uint8_t)(e + 127);
    if (D == 64) atom[((c + 64) % 32) * 16 + ((c + 64) / 32) * 4 + (j % 2) * 2 + h] = 0;
    // a ragged last 64-key tile that is the even half of its atom leaves the odd half unwritten
    if (j == vt.T64 - 1 && (j % 2) == 0) {
      atom[(c % 32) * 16 + (c / 32) * 4 + 2 + h] = 0;
      if (D == 64) atom[((c + 64) % 32) * 16 + ((c + 64) / 32) * 4 + 2 + h] = 0;
    }
  }
}

// ------------------------------------------------------------------------------------------------
// Generic quantizer, plain layout: one thread per group of 32.
// axis 0: groups along columns of a row; axis 1: groups along rows of a column (transposed out).
// ------------------------------------------------------------------------------------------------
template <int DT, bool NVF>
__global__ void __launch_bounds__(256) quant_plain_kernel(PlainQuantArgs a) {
  constexpr int G = NVF ? 16 : 32;  // elements per group / block
  const int64_t outer = a.axis == 0 ? a.rows : a.cols;
  const int64_t inner = a.axis == 0 ? a.cols : a.rows;
  const int64_t ng = (inner + G - 1) / G;
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= outer * ng) return;
  // axis 1: consecutive threads take consecutive columns (coalesced); axis 0: consecutive groups
  const int64_t o = a.axis == 0 ? gid / ng : gid % outer;
  const int64_t g = a.axis == 0 ? gid % ng : gid / outer;
  float v[32];
#pragma unroll
  for (int i = 0; i < G; i++) {
    const int64_t in = g * G + i;
    float x = 0.f;
    if (in < inner) {
      const int64_t idx = a.axis == 0 ? o * a.cols + in : in * a.cols + o;
      if (DT == kBF16)
        x = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(a.x)[idx]);
      else
        x = reinterpret_cast<const float*>(a.x)[idx];
    }
    v[i] = x;
  }
  if (NVF) {
    uint32_t w[2];
    const uint32_t b = nvfp4_block(v, w);
    *reinterpret_cast<uint2*>(a.codes + (o * ng + g) * 8) = make_uint2(w[0], w[1]);
    a.scales[o * ng + g] = (uint8_t)b;
    return;
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; i++) amax = fmaxf(amax, fabsf(v[i]));
  const int e = shared_exponent(amax, a.rule);
  const float inv = pow2_neg(e);
  uint32_t w[4];
#pragma unroll
  for (int q = 0; q < 4; q++)
    w[q] = cvt_e2m1x8(__fmul_rn(v[q * 8 + 0], inv), __fmul_rn(v[q * 8 + 1], inv), __fmul_rn(v[q * 8 + 2], inv),
                      __fmul_rn(v[q * 8 + 3], inv), __fmul_rn(v[q * 8 + 4], inv), __fmul_rn(v[q * 8 + 5], inv),
                      __fmul_rn(v[q * 8 + 6], inv), __fmul_rn(v[q * 8 + 7], inv));
  *reinterpret_cast<uint4*>(a.codes + (o * ng + g) * 16) = make_uint4(w[0], w[1], w[2], w[3]);
  a.scales[o * ng + g] = (uint8_t)(e + 127);
}

// ------------------------------------------------------------------------------------------------
// Launchers
// ------------------------------------------------------------------------------------------------
template <int D, int DT>
static void qk_launch(const QKQuantArgs& a, dim3 grid, cudaStream_t s) {
  constexpr int T = QKBlock<D, DT>::ROWS;
  if (a.fmt == kFmtNVFP4) rotate_quant_qk_kernel<D, DT, true><<<grid, T, 0, s>>>(a);
  else rotate_quant_qk_kernel<D, DT, false><<<grid, T, 0, s>>>(a);
}

cudaError_t launch_rotate_quant_qk(const QKQuantArgs& a, int D, int dtype, cudaStream_t s) {
  // one block per 128-row packed tile or part of one, over the longer of Q and K
  const int64_t tiles = a.vl.cu_seqlens != nullptr ? (int64_t)a.BH * a.vl.tiles_per_head
                                                   : (int64_t)a.BH * (((a.N > a.Nk ? a.N : a.Nk) + 127) / 128);
  const int split = dtype == kBF16 ? QKBlock<128, kBF16>::SPLIT : QKBlock<128, kFP32>::SPLIT;
  const dim3 grid((unsigned)(tiles * split), 2);
  if (D == 128 && dtype == kBF16) qk_launch<128, kBF16>(a, grid, s);
  else if (D == 128) qk_launch<128, kFP32>(a, grid, s);
  else if (dtype == kBF16) qk_launch<64, kBF16>(a, grid, s);
  else qk_launch<64, kFP32>(a, grid, s);
  return cudaGetLastError();
}

template <int D, int DT>
static void v_launch(const VQuantArgs& a, int64_t items, cudaStream_t s) {
  // one block of D threads per item (16 or 32 KB of shared memory at D = 128)
  if (a.fmt == kFmtNVFP4) quant_v_kernel<D, DT, true><<<(unsigned)items, D, 0, s>>>(a);
  else quant_v_kernel<D, DT, false><<<(unsigned)items, D, 0, s>>>(a);
}

cudaError_t launch_quant_v(const VQuantArgs& a, int D, int dtype, cudaStream_t s) {
  const int64_t blocks = (int64_t)a.BH * (a.vl.cu_seqlens != nullptr ? 2 * (int64_t)a.vl.tiles_per_head
                                                                     : (a.N + 63) / 64);
  if (D == 128 && dtype == kBF16) v_launch<128, kBF16>(a, blocks, s);
  else if (D == 128) v_launch<128, kFP32>(a, blocks, s);
  else if (dtype == kBF16) v_launch<64, kBF16>(a, blocks, s);
  else v_launch<64, kFP32>(a, blocks, s);
  return cudaGetLastError();
}

cudaError_t launch_quant_plain(const PlainQuantArgs& a, int dtype, cudaStream_t s) {
  const int64_t outer = a.axis == 0 ? a.rows : a.cols;
  const int64_t inner = a.axis == 0 ? a.cols : a.rows;
  const int G = a.fmt == kFmtNVFP4 ? 16 : 32;
  const int64_t groups = outer * ((inner + G - 1) / G);
  const unsigned blocks = (unsigned)((groups + 255) / 256);
  const bool nv = a.fmt == kFmtNVFP4;
  if (dtype == kBF16) {
    if (nv) quant_plain_kernel<kBF16, true><<<blocks, 256, 0, s>>>(a);
    else quant_plain_kernel<kBF16, false><<<blocks, 256, 0, s>>>(a);
  } else {
    if (nv) quant_plain_kernel<kFP32, true><<<blocks, 256, 0, s>>>(a);
    else quant_plain_kernel<kFP32, false><<<blocks, 256, 0, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace mxattn

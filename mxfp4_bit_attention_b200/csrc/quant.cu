// quant.cu -- MXFP4 quantizers (rotation + quantization of Q/K, V along keys, and a plain
// generic quantizer).  Memory-bound: every byte is read once and written once, loads and
// stores are 16-byte vectors, FWHT butterflies run in registers and warp shuffles.
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

template <int DT>
__device__ __forceinline__ void load8(const void* base, int64_t idx, bool valid, float (&v)[8]) {
  if (!valid) {
#pragma unroll
    for (int i = 0; i < 8; i++) v[i] = 0.f;
    return;
  }
  if (DT == kBF16) {
    const uint4 raw = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(base) + idx);
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; i++) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + idx);
    const float4 a = p[0], b = p[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

// One NVFP4 block of 16 values (the comparison format): the scale is the E4M3 rounding of
// fl32(amax / 6), each value is divided by it in fp32 (correctly rounded) and rounded to E2M1
// with saturation; a scale that rounds to zero gives zero codes.  Returns the scale byte.
__device__ __forceinline__ uint32_t nvfp4_block(const float* v, uint32_t* w) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; i++) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t byte = cvt_e4m3x2(__fdiv_rn(amax, 6.f), 0.f) & 0xFFu;
  const float s = e4m3x2_to_float2(byte).x;
  float y[16];
#pragma unroll
  for (int i = 0; i < 16; i++) y[i] = s > 0.f ? __fdiv_rn(v[i], s) : 0.f;
  w[0] = cvt_e2m1x8(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]);
  w[1] = cvt_e2m1x8(y[8], y[9], y[10], y[11], y[12], y[13], y[14], y[15]);
  return byte;
}

// ------------------------------------------------------------------------------------------------
// Q/K: Hadamard rotation + quantization along d into the packed QK operand layout.
// One thread per MX group (32 consecutive elements of a row, four 16-byte loads in flight), D/32
// threads per row: butterfly stages h = 1..16 run inside the thread, h = 32 and 64 across the
// row's threads by shuffles, in the order h = 1, 2, ..., D/2; the group max is the thread's own.
// Grid: x over (B*H*T128*128) padded token rows of the longer of Q and K, y = 0 for Q, 1 for K;
// varlen: over H * tiles_per_head * 128 padded rows, each tile belonging to one sequence.
// ------------------------------------------------------------------------------------------------
// Where padded row prow of the Q or K operand comes from: its row of the [rows, D] source (valid: a
// real token; a padding row is quantized from zeros) and its packed tile and row within the tile.
struct QKRow {
  bool ok, valid;
  int64_t src_row, tile;
  int r;
};

__device__ __forceinline__ QKRow qk_row(const QKQuantArgs& a, int64_t prow, int64_t total, int64_t T128, int Nt) {
  QKRow q;
  q.ok = prow < total;
  const int64_t bh = prow / (T128 * 128);
  q.r = (int)(prow % 128);
  q.tile = prow / 128;  // bh * T128 + tile within the head
  if (a.vl.cu_seqlens != nullptr) {
    // the tile's sequence and the row's token within it; tiles past the last sequence's are unused
    const int gt = (int)(q.tile - bh * T128);
    q.ok = q.ok && gt < __ldg(a.vl.tile_off + a.vl.nseq);
    const int sq = q.ok ? varlen_sequence(a.vl, gt) : 0;
    const int start = __ldg(a.vl.cu_seqlens + sq);
    const int n = (gt - __ldg(a.vl.tile_off + sq)) * 128 + q.r;
    q.valid = q.ok && n < __ldg(a.vl.cu_seqlens + sq + 1) - start;
    q.src_row = ((int64_t)start + n) * a.BH + bh;  // token-major [T, H, d]
  } else {
    const int tok = (int)(prow % (T128 * 128));
    q.valid = q.ok && tok < Nt;
    q.src_row = (int64_t)bh * Nt + tok;
  }
  return q;
}

// The 32 inputs of one thread's group as loaded (bf16: four 16-byte words; fp32: eight).
template <int DT>
struct GroupRaw {
  uint4 w[DT == kBF16 ? 4 : 8];
};

template <int DT>
__device__ __forceinline__ void load_group(const void* src, int64_t idx, bool valid, GroupRaw<DT>& raw) {
  constexpr int NW = DT == kBF16 ? 4 : 8;
  const uint4* p = DT == kBF16 ? reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(src) + idx)
                               : reinterpret_cast<const uint4*>(reinterpret_cast<const float*>(src) + idx);
#pragma unroll
  for (int i = 0; i < NW; i++) raw.w[i] = valid ? p[i] : make_uint4(0u, 0u, 0u, 0u);
}

template <int DT>
__device__ __forceinline__ void unpack_group(const GroupRaw<DT>& raw, float (&v)[32]) {
  if (DT == kBF16) {
#pragma unroll
    for (int i = 0; i < 4; i++) {
      const uint32_t w[4] = {raw.w[i].x, raw.w[i].y, raw.w[i].z, raw.w[i].w};
#pragma unroll
      for (int k = 0; k < 4; k++) {
        v[8 * i + 2 * k] = __uint_as_float(w[k] << 16);
        v[8 * i + 2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; i++) {
      v[4 * i] = __uint_as_float(raw.w[i].x);
      v[4 * i + 1] = __uint_as_float(raw.w[i].y);
      v[4 * i + 2] = __uint_as_float(raw.w[i].z);
      v[4 * i + 3] = __uint_as_float(raw.w[i].w);
    }
  }
}

// Hadamard rotation of one row held by its TPR = D/32 lanes, 32 values each, in place: butterfly
// stages h = 1..16 inside the thread, h = 32..D/2 across the row's lanes by shuffles, then the
// multiply by fl32(1/sqrt(D)).  Every lane of the warp must take part (the shuffles are full-warp).
template <int TPR>
__device__ __forceinline__ void rotate_group(float (&v)[32], int g, float hadamard_scale) {
  // Butterflies (x, y) -> (x + y, x - y), each result rounded once: x - y as fma(y, -1, x).
  // From h = 2 on, neighbours i, i+1 pair up into f32x2 operations with the same roundings.
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const float x = v[i], y = v[i + 1];
    v[i] = __fadd_rn(x, y);
    v[i + 1] = __fsub_rn(x, y);
  }
  const float2 minus1 = make_float2(-1.f, -1.f);
#pragma unroll
  for (int h = 2; h < 32; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      if ((i & h) == 0) {
        const float2 x = make_float2(v[i], v[i + 1]), y = make_float2(v[i + h], v[i + h + 1]);
        const float2 sum = __fadd2_rn(x, y), dif = __ffma2_rn(y, minus1, x);
        v[i] = sum.x; v[i + 1] = sum.y;
        v[i + h] = dif.x; v[i + h + 1] = dif.y;
      }
    }
  }
  // stages h = 32 .. D/2 across the TPR lanes of the row (lane bit = h / 32): the lower lane
  // keeps x + y, the upper one y' = x - y, both as fma(own, +-1, other)
#pragma unroll
  for (int hb = 1; hb < TPR; hb <<= 1) {
    const float sg = (g & hb) != 0 ? -1.f : 1.f;
    const float2 sg2 = make_float2(sg, sg);
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const float o0 = __shfl_xor_sync(0xFFFFFFFFu, v[i], hb);
      const float o1 = __shfl_xor_sync(0xFFFFFFFFu, v[i + 1], hb);
      const float2 r = __ffma2_rn(make_float2(v[i], v[i + 1]), sg2, make_float2(o0, o1));
      v[i] = r.x; v[i + 1] = r.y;
    }
  }
  const float2 hs = make_float2(hadamard_scale, hadamard_scale);
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const float2 r = __fmul2_rn(make_float2(v[i], v[i + 1]), hs);
    v[i] = r.x; v[i + 1] = r.y;
  }
}

template <int D, int DT, bool NVF>
__global__ void __launch_bounds__(256) rotate_quant_qk_kernel(QKQuantArgs a) {
  constexpr int TPR = D / 32;                // threads per row = groups per row
  constexpr int ROWS = 256 / TPR;            // rows per block and pass
  const int t = threadIdx.x;
  const int g = t % TPR;                     // group (and 16-byte code chunk) within the row
  const int Nt = blockIdx.y == 0 ? a.N : a.Nk;  // tokens of this tensor
  const int64_t T128 = a.vl.cu_seqlens != nullptr ? a.vl.tiles_per_head : (Nt + 127) / 128;
  const int64_t total = (int64_t)a.BH * T128 * 128;
  const void* src = blockIdx.y == 0 ? a.q : a.k;
  uint8_t* codes = blockIdx.y == 0 ? a.q_codes : a.k_codes;
  uint8_t* scales = blockIdx.y == 0 ? a.q_scales : a.k_scales;

  // Grid-stride over passes of ROWS rows (the pass count is the block's, so a row's lanes, which
  // exchange values by shuffles, always run together); the next pass's inputs are loaded before
  // this pass's rotation and quantization, so a load is in flight while the thread computes.
  const int64_t stride = (int64_t)gridDim.x * ROWS;
  int64_t prow = (int64_t)blockIdx.x * ROWS + t / TPR;
  QKRow row = qk_row(a, prow, total, T128, Nt);
  GroupRaw<DT> raw;
  load_group<DT>(src, (row.valid ? row.src_row : 0) * D + g * 32, row.valid, raw);
  for (int64_t pass = (int64_t)blockIdx.x * ROWS; pass < total; pass += stride, prow += stride) {
    const QKRow cur = row;
    float v[32];
    unpack_group<DT>(raw, v);
    if (pass + stride < total) {
      row = qk_row(a, prow + stride, total, T128, Nt);
      load_group<DT>(src, (row.valid ? row.src_row : 0) * D + g * 32, row.valid, raw);
    }
    if (a.rotate) rotate_group<TPR>(v, g, a.hadamard_scale);
    uint32_t w[4];
    int e = 0;
    uint32_t nvb = 0;  // NVFP4: the two E4M3 scale bytes of the thread's blocks of 16
    if (NVF) {
      nvb = nvfp4_block(v, w) | (nvfp4_block(v + 16, w + 2) << 8);
    } else {
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 32; i++) amax = fmaxf(amax, fabsf(v[i]));
      e = shared_exponent(amax, a.rule);
      const float inv = pow2_neg(e);
#pragma unroll
      for (int q = 0; q < 4; q++)
        w[q] = cvt_e2m1x8(__fmul_rn(v[8 * q + 0], inv), __fmul_rn(v[8 * q + 1], inv), __fmul_rn(v[8 * q + 2], inv),
                          __fmul_rn(v[8 * q + 3], inv), __fmul_rn(v[8 * q + 4], inv), __fmul_rn(v[8 * q + 5], inv),
                          __fmul_rn(v[8 * q + 6], inv), __fmul_rn(v[8 * q + 7], inv));
    }
    if (!cur.ok) continue;
    const int r = cur.r;
    const int sw = (D == 128) ? ((r >> 1) & 3) : ((r >> 2) & 1);
    uint8_t* rowp = codes + (cur.tile * 128 + r) * (D / 2);
    *reinterpret_cast<uint4*>(rowp + ((g ^ sw) * 16)) = make_uint4(w[0], w[1], w[2], w[3]);
    if (NVF) {
      // D/64 scale atoms per tile, one per 64 dims (one K = 64 MMA): blocks 4a..4a+3 in the bytes
      // of row r's word; this thread's blocks 2g, 2g+1 sit in atom g/2, bytes 2(g%2), 2(g%2)+1
      uint8_t* atom = scales + cur.tile * (512 * (D / 64)) + (g / 2) * 512 + (r % 32) * 16 + (r / 32) * 4;
      *reinterpret_cast<uint16_t*>(atom + 2 * (g % 2)) = (uint16_t)nvb;
    } else {
      uint8_t* atom = scales + cur.tile * 512 + (r % 32) * 16 + (r / 32) * 4;
      atom[g] = (uint8_t)(e + 127);
      if (D == 64) atom[g + 2] = 0;                         // unused scale slots
    }
  }
}

// ------------------------------------------------------------------------------------------------
// V: quantization along keys (32 consecutive tokens per channel) into the packed V operand
// layout.  Blocks stride over the (head, 64-key tile) items; each tile is staged through shared
// memory as fp32 [64][D+1], then thread (channel c, half h) quantizes keys 32h..32h+31 of channel
// c.  The next tile's inputs are loaded into registers before the current tile is quantized, so
// a load is always in flight while the block computes.
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
__global__ void __launch_bounds__(256) quant_v_kernel(VQuantArgs a, int64_t items) {
  __shared__ float tile[64][D + 1];
  constexpr int VEC_PER_ROW = D / 8;             // 8 values per load
  constexpr int NVEC = 64 * VEC_PER_ROW / 256;   // loads per thread and tile
  const int t = threadIdx.x;
  float nxt[NVEC][8];
  auto load_tile = [&](const VTile& vt) {
#pragma unroll
    for (int u = 0; u < NVEC; u++) {
      const int idx = t + 256 * u, row = idx / VEC_PER_ROW, cv = idx % VEC_PER_ROW;
      const int tok = vt.j * 64 + row;
      const bool valid = vt.ok && tok < vt.N;
      load8<DT>(a.v, (vt.src_row0 + (valid ? tok : 0) * vt.src_stride) * D + cv * 8, valid, nxt[u]);
    }
  };
  int64_t item = blockIdx.x;
  VTile next = v_tile(a, item);
  load_tile(next);
  for (; item < items; item += gridDim.x) {
    __syncthreads();  // the previous tile has been read out of shared memory
#pragma unroll
    for (int u = 0; u < NVEC; u++) {
      const int idx = t + 256 * u, row = idx / VEC_PER_ROW, cv = idx % VEC_PER_ROW;
#pragma unroll
      for (int i = 0; i < 8; i++) tile[row][cv * 8 + i] = nxt[u][i];
    }
    const VTile me = next;
    if (item + gridDim.x < items) {
      next = v_tile(a, item + gridDim.x);
      load_tile(next);  // in flight while this tile is quantized
    }
    __syncthreads();
    if (!me.ok) continue;
    const int j = me.j;
    for (int it = t; it < 2 * D; it += 256) {
      const int c = it % D, h = it / D;
      if (NVF) {
        // two blocks of 16 keys; one scale atom per 64-key tile, keys 16b..16b+15 in byte b of
        // channel c's word
        float x[32];
#pragma unroll
        for (int i = 0; i < 32; i++) x[i] = tile[h * 32 + i][c];
        uint32_t w[4];
        const uint32_t b = nvfp4_block(x, w) | (nvfp4_block(x + 16, w + 2) << 8);
        uint8_t* dst = a.v_codes + (me.vtile * D + c) * 32 + ((h ^ ((c >> 2) & 1)) * 16);
        *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
        uint8_t* atom = a.v_scales + me.vtile * 512;
        *reinterpret_cast<uint16_t*>(atom + (c % 32) * 16 + (c / 32) * 4 + 2 * h) = (uint16_t)b;
        if (D == 64) *reinterpret_cast<uint16_t*>(atom + ((c + 64) % 32) * 16 + ((c + 64) / 32) * 4 + 2 * h) = 0;
        continue;
      }
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 32; i++) amax = fmaxf(amax, fabsf(tile[h * 32 + i][c]));
      const int e = shared_exponent(amax, a.rule);
      const float inv = pow2_neg(e);
      uint32_t w[4];
#pragma unroll
      for (int q = 0; q < 4; q++) {
        const int b = h * 32 + q * 8;
        w[q] = cvt_e2m1x8(__fmul_rn(tile[b + 0][c], inv), __fmul_rn(tile[b + 1][c], inv),
                          __fmul_rn(tile[b + 2][c], inv), __fmul_rn(tile[b + 3][c], inv),
                          __fmul_rn(tile[b + 4][c], inv), __fmul_rn(tile[b + 5][c], inv),
                          __fmul_rn(tile[b + 6][c], inv), __fmul_rn(tile[b + 7][c], inv));
      }
      uint8_t* dst = a.v_codes + (me.vtile * D + c) * 32 + ((h ^ ((c >> 2) & 1)) * 16);
      *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
      uint8_t* atom = a.v_scales + me.atom_tile * 512;
      atom[(c % 32) * 16 + (c / 32) * 4 + (j % 2) * 2 + h] = (uint8_t)(e + 127);
      if (D == 64) atom[((c + 64) % 32) * 16 + ((c + 64) / 32) * 4 + (j % 2) * 2 + h] = 0;
      // a ragged last 64-key tile that is the even half of its atom leaves the odd half unwritten
      if (j == me.T64 - 1 && (j % 2) == 0) {
        atom[(c % 32) * 16 + (c / 32) * 4 + 2 + h] = 0;
        if (D == 64) atom[((c + 64) % 32) * 16 + ((c + 64) / 32) * 4 + 2 + h] = 0;
      }
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
  if (a.fmt == kFmtNVFP4) rotate_quant_qk_kernel<D, DT, true><<<grid, 256, 0, s>>>(a);
  else rotate_quant_qk_kernel<D, DT, false><<<grid, 256, 0, s>>>(a);
}

cudaError_t launch_rotate_quant_qk(const QKQuantArgs& a, int D, int dtype, cudaStream_t s) {
  const int64_t rows = a.vl.cu_seqlens != nullptr ? (int64_t)a.BH * a.vl.tiles_per_head * 128
                                                  : (int64_t)a.BH * (((a.N > a.Nk ? a.N : a.Nk) + 127) / 128) * 128;
  const int rows_per_block = 256 / (D / 32);
  // enough blocks for every SM to hold several at once; each loops over the rest of the rows
  const int64_t want = (rows + rows_per_block - 1) / rows_per_block;
  constexpr int64_t kMaxBlocks = 148 * 8;
  dim3 grid((unsigned)(want < kMaxBlocks ? want : kMaxBlocks), 2);
  if (D == 128 && dtype == kBF16) qk_launch<128, kBF16>(a, grid, s);
  else if (D == 128) qk_launch<128, kFP32>(a, grid, s);
  else if (dtype == kBF16) qk_launch<64, kBF16>(a, grid, s);
  else qk_launch<64, kFP32>(a, grid, s);
  return cudaGetLastError();
}

template <int D, int DT>
static void v_launch(const VQuantArgs& a, int64_t items, cudaStream_t s) {
  // several blocks per SM (33 KB of shared memory each at D = 128), each striding over the items
  constexpr int64_t kMaxBlocks = 148 * 6;
  const unsigned blocks = (unsigned)(items < kMaxBlocks ? items : kMaxBlocks);
  if (a.fmt == kFmtNVFP4) quant_v_kernel<D, DT, true><<<blocks, 256, 0, s>>>(a, items);
  else quant_v_kernel<D, DT, false><<<blocks, 256, 0, s>>>(a, items);
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

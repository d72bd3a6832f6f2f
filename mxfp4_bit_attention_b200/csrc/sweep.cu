// sweep.cu -- per-block Qmax sweep: the scale-rule diagnostic behind the pages' per-block
// MSE-optimal boundary study (Pith review page, Table 4; the 7.25 argument of Fig. 2 and
// Theorem 1), run on the GPU over whole tensors.
//
// For every group of 32 consecutive elements of a row (the tail zero-padded; rows optionally
// Hadamard-rotated first, in the Q/K quantizer's exact operation order) and every boundary q_k,
// the ceiling-rule exponent e_k, the E2M1 reconstruction xhat = E2M1(x 2^-e_k) 2^e_k and the squared
// error SSE_k = sum_i (x_i - xhat_i)^2, each difference and square rounded in fp64 and the sum
// taken in index order.  A group counts for every q_k whose SSE_k equals its smallest.  Over
// q in [4, 8] a group's exponent takes at most two values (amax / q spans less than one binade),
// so at most two errors are evaluated per group.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace mxattn {

namespace {

__device__ __forceinline__ float load1(const void* x, int64_t idx, int dtype) {
  if (dtype == kBF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(x)[idx]);
  return reinterpret_cast<const float*>(x)[idx];
}

// E2M1 code (4 bits: sign, magnitude index m) to its value: m = 0, 1 -> 0, 0.5 (subnormal);
// m >= 2 -> (1 + (m & 1) / 2) * 2^((m >> 1) - 1)
__device__ __forceinline__ double e2m1_value(uint32_t code) {
  const uint32_t m = code & 7u;
  const double mag = m < 2 ? 0.5 * (double)m : (1.0 + 0.5 * (double)(m & 1u)) * (double)(1u << ((m >> 1) - 1));
  return (code & 8u) ? -mag : mag;
}

// squared reconstruction error of a group under exponent e (fp64, index order)
__device__ __forceinline__ double group_sse(const float (&v)[32], int e) {
  const float inv = pow2_neg(e);
  const double scale = __longlong_as_double((long long)(e + 1023) << 52);  // 2^e, e in [-127, 127]
  double s = 0.0;
#pragma unroll
  for (int q = 0; q < 4; q++) {
    const uint32_t w = cvt_e2m1x8(__fmul_rn(v[8 * q + 0], inv), __fmul_rn(v[8 * q + 1], inv),
                                  __fmul_rn(v[8 * q + 2], inv), __fmul_rn(v[8 * q + 3], inv),
                                  __fmul_rn(v[8 * q + 4], inv), __fmul_rn(v[8 * q + 5], inv),
                                  __fmul_rn(v[8 * q + 6], inv), __fmul_rn(v[8 * q + 7], inv));
#pragma unroll
    for (int i = 0; i < 8; i++) {
      const double xh = __dmul_rn(e2m1_value(w >> (4 * i)), scale);
      const double d = __dsub_rn((double)v[8 * q + i], xh);
      s = __dadd_rn(s, __dmul_rn(d, d));
    }
  }
  return s;
}

}  // namespace

// One thread per group.  With rotation, the cols / 32 threads of a row are adjacent lanes and the
// butterfly stages h = 32, 64 cross them by shuffles, as in the Q/K quantizer.
template <int DT, int ROTD>
__global__ void __launch_bounds__(256) qmax_sweep_kernel(const SweepArgs a) {
  const int64_t ng = ROTD ? ROTD / 32 : (a.cols + 31) / 32;
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t total = a.rows * ng;
  const bool valid = gid < total;
  const int64_t r = valid ? gid / ng : 0;
  const int g = (int)(valid ? gid % ng : 0);
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; i++) {
    const int64_t c = (int64_t)g * 32 + i;
    v[i] = (valid && c < a.cols) ? load1(a.x, r * a.cols + c, DT) : 0.f;
  }
  if (ROTD) {
    // identical operations, in the same order, as the Q/K quantizer's rotation
#pragma unroll
    for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
      for (int i = 0; i < 32; i++) {
        if ((i & h) == 0) {
          const float x = v[i], y = v[i + h];
          v[i] = __fadd_rn(x, y);
          v[i + h] = __fsub_rn(x, y);
        }
      }
    }
#pragma unroll
    for (int hb = 1; hb < ROTD / 32; hb <<= 1) {
      const bool upper = (g & hb) != 0;
#pragma unroll
      for (int i = 0; i < 32; i++) {
        const float other = __shfl_xor_sync(0xFFFFFFFFu, v[i], hb);
        v[i] = upper ? __fsub_rn(other, v[i]) : __fadd_rn(v[i], other);
      }
    }
#pragma unroll
    for (int i = 0; i < 32; i++) v[i] = __fmul_rn(v[i], a.hadamard_scale);
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; i++) amax = fmaxf(amax, fabsf(v[i]));
  // the exponent is non-increasing in q: e_a at the first boundary, e_b (<= e_a) at the last
  const int e_a = shared_exponent(amax, a.rules[0]);
  const int e_b = shared_exponent(amax, a.rules[a.nq - 1]);
  const double sse_a = group_sse(v, e_a);
  const double sse_b = e_b == e_a ? sse_a : group_sse(v, e_b);
  const double best = fmin(sse_a, sse_b);
  const int lane = threadIdx.x & 31;
  for (int k = 0; k < a.nq; k++) {
    const double sse = valid ? (shared_exponent(amax, a.rules[k]) == e_a ? sse_a : sse_b) : 0.0;
    const unsigned opt = __ballot_sync(0xFFFFFFFFu, valid && sse == best);
    double sum = sse;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, off);
    if (lane == 0) {
      if (opt) atomicAdd(a.counts + k, (unsigned long long)__popc(opt));
      atomicAdd(a.sse_sums + k, sum);
    }
  }
}

cudaError_t launch_qmax_sweep(const SweepArgs& a, int dtype, cudaStream_t s) {
  const int64_t ng = a.rotate ? a.cols / 32 : (a.cols + 31) / 32;
  const int64_t total = a.rows * ng;
  const unsigned blocks = (unsigned)((total + 255) / 256);
  if (blocks == 0) return cudaSuccess;
  if (a.rotate) {
    if (a.cols == 128) {
      if (dtype == kBF16) qmax_sweep_kernel<kBF16, 128><<<blocks, 256, 0, s>>>(a);
      else qmax_sweep_kernel<kFP32, 128><<<blocks, 256, 0, s>>>(a);
    } else {
      if (dtype == kBF16) qmax_sweep_kernel<kBF16, 64><<<blocks, 256, 0, s>>>(a);
      else qmax_sweep_kernel<kFP32, 64><<<blocks, 256, 0, s>>>(a);
    }
  } else {
    if (dtype == kBF16) qmax_sweep_kernel<kBF16, 0><<<blocks, 256, 0, s>>>(a);
    else qmax_sweep_kernel<kFP32, 0><<<blocks, 256, 0, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace mxattn

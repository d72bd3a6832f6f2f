// probe.cu -- dense FP4 tensor-core throughput probe: back-to-back tcgen05 kind::mxf4
// block-scaled MMAs (M = 128, N = n, K = 64) from shared memory into tensor memory, one CTA per
// SM holding all 512 TMEM columns.  It measures the roofline denominator for the attention
// kernel; it is not part of the method.
#include <cuda_runtime.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace mxattn {

constexpr int kProbeDynSmem = 160 * 1024;  // > half the SM's shared memory: one CTA per SM

__global__ void __launch_bounds__(128, 1) fp4_mma_probe_kernel(int iters, int n, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  // A: 128 x 32 bytes, B: 256 x 32 bytes (32-byte swizzle, contents arbitrary but finite),
  // scale atoms: A (512 B), B (2 x 512 B), then an mbarrier and the TMEM address slot.
  constexpr int A_OFF = 0, B_OFF = 4096, SFA_OFF = 12288, SFB_OFF = 12800, BAR_OFF = 13824, SLOT_OFF = 13832;
  __shared__ int never;
  for (int i = threadIdx.x; i < 12288 / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(smem)[i] = 0x2A3B1C22u ^ (uint32_t)(i * 2654435761u & 0x77777777u);
  for (int i = threadIdx.x; i < 1536; i += blockDim.x) smem[SFA_OFF + i] = 127;
  if (threadIdx.x == 0) {
    never = 0;
    mbar_init(sb + BAR_OFF, 1);
    fence_mbar_init();
  }
  fence_proxy_async_smem();
  if (threadIdx.x < 32) {
    tmem_alloc(sb + SLOT_OFF, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + SLOT_OFF);
  if (threadIdx.x == 0) {
    const uint32_t t_sfa = tmem + 256, t_sfb = tmem + 260;
    tmem_cp_sf_atom(t_sfa, sb + SFA_OFF);
    tmem_cp_sf_atom(t_sfb, sb + SFB_OFF);
    tmem_cp_sf_atom(t_sfb + 4, sb + SFB_OFF + 512);
    const uint64_t adesc = smem_desc(sb + A_OFF, 16, 256, kLayoutSW32);
    const uint64_t bdesc = smem_desc(sb + B_OFF, 16, 256, kLayoutSW32);
    const uint32_t idesc = mxf4_idesc(128, (uint32_t)n, 0, 0);
    for (int i = 0; i < iters; i++) mma_mxf4(tmem, adesc, bdesc, idesc, t_sfa, t_sfb, i > 0 ? 1u : 0u);
    mma_commit(sb + BAR_OFF);
    if (!mbar_wait(sb + BAR_OFF, 0, &never, 4000000000LL) && status != nullptr)
      atomicCAS(status, 0, kStatusTimeout);
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

cudaError_t launch_fp4_mma_probe(int ctas, int iters, int n, int* status, cudaStream_t s) {
  cudaError_t err =
      cudaFuncSetAttribute(fp4_mma_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kProbeDynSmem);
  if (err != cudaSuccess) return err;
  fp4_mma_probe_kernel<<<ctas, 128, kProbeDynSmem, s>>>(iters, n, status);
  return cudaGetLastError();
}

// Element-wise evaluation of the attention kernels' arithmetic shortcuts (device functions of
// ptx.cuh), so that tests can hold each against its definition.  Not part of the method.
__global__ void arith_probe_kernel(int op, const float* in, int64_t n, ScaleRule rule, void* out) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const float x = in[i];
    switch (op) {
      case kProbeExp2Poly:
        reinterpret_cast<float*>(out)[i] = exp2_poly2(make_float2(x, x)).x;
        break;
      case kProbeExp2Mufu:
        reinterpret_cast<float*>(out)[i] = ex2_approx(x);
        break;
      case kProbeE2m1StandIn: {
        const float w = fma_sat(x, 0.125f, -kStandInLo * 0.125f);  // the clamped argument the 128-key kernel feeds it
        const float y = e2m1_exp2_stand_in(make_float2(w, w)).x;
        reinterpret_cast<uint8_t*>(out)[i] = (uint8_t)(cvt_e2m1x8(y, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f) & 0xFu);
        break;
      }
      case kProbeE2m1Mufu:
        reinterpret_cast<uint8_t*>(out)[i] =
            (uint8_t)(cvt_e2m1x8(ex2_approx(x), 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f) & 0xFu);
        break;
      case kProbeScaleExpLog2: {
        uint32_t byte;
        reinterpret_cast<int*>(out)[i] = (int)shared_exponent_log2f(x, rule, byte);
        break;
      }
      default:  // kProbeScaleExp
        reinterpret_cast<int*>(out)[i] = shared_exponent(x, rule);
        break;
    }
  }
}

cudaError_t launch_arith_probe(int op, const float* in, int64_t n, const ScaleRule& rule, void* out, cudaStream_t s) {
  const int64_t want = (n + 255) / 256;
  arith_probe_kernel<<<(unsigned)(want < 4096 ? want : 4096), 256, 0, s>>>(op, in, n, rule, out);
  return cudaGetLastError();
}

}  // namespace mxattn

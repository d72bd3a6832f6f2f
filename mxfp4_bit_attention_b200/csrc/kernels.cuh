// kernels.cuh -- argument blocks and launchers shared by the C ABI (api.cu) and the kernels.
#pragma once
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"

namespace mxattn {

enum { kBF16 = 0, kFP32 = 1 };

struct QKQuantArgs {
  const void* q;
  const void* k;
  uint8_t* q_codes;
  uint8_t* q_scales;
  uint8_t* k_codes;
  uint8_t* k_scales;
  int BH, N;
  int rotate;
  float hadamard_scale;  // fl32(1/sqrt(d))
  ScaleRule rule;
};

struct VQuantArgs {
  const void* v;
  uint8_t* v_codes;
  uint8_t* v_scales;
  int BH, N;
  ScaleRule rule;
};

struct PlainQuantArgs {
  const void* x;
  uint8_t* codes;
  uint8_t* scales;
  int64_t rows, cols;
  int axis;
  ScaleRule rule;
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
  int BH, N;
  float scale_log2;      // softmax_scale * log2(e)
  float tau;             // lazy max threshold, log2 units
  int pnq;
  ScaleRule rule;
  long long wait_budget; // SM clock cycles a bounded wait may spin before giving up
};

// Status words written by a kernel whose bounded wait expired.
enum { kStatusTimeout = 0x54494D45 /* 'TIME' */ };

cudaError_t launch_rotate_quant_qk(const QKQuantArgs& a, int D, int dtype, cudaStream_t s);
cudaError_t launch_quant_v(const VQuantArgs& a, int D, int dtype, cudaStream_t s);
cudaError_t launch_quant_plain(const PlainQuantArgs& a, int dtype, cudaStream_t s);
cudaError_t launch_attention(const AttnArgs& a, int D, int dtype, cudaStream_t s);
cudaError_t launch_fp4_mma_probe(int ctas, int iters, int n, int* status, cudaStream_t s);

}  // namespace mxattn

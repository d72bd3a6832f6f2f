// varlen.cu -- tile table of a packed batch of variable-length sequences.
//
// A packed batch holds nseq sequences back to back along the token axis; sequence s spans tokens
// cu_seqlens[s] .. cu_seqlens[s+1]-1 and is an attention problem of its own.  In the packed MXFP4
// operands every sequence is padded to whole 128-row tiles: tile_off[s] = sum over s' < s of
// ceil(len(s') / 128), tile_off[nseq] = the tiles in use.  The offsets live on the device (the
// caller's cu_seqlens is a device array), so the table is built here, on the stream, and every
// later kernel of the pass reads it.
#include <cuda_runtime.h>

#include "kernels.cuh"

namespace mxattn {

namespace {

constexpr int kScanThreads = 1024;

// One block.  Thread t takes a contiguous run of sequences, sums their tile counts, the block
// scans the 1024 partial sums, and each thread writes its run's offsets.  cu_seqlens must start
// at 0, never decrease and end at T; otherwise the whole table is zero (no tiles: every later
// kernel of the pass does nothing) and the status word records kStatusBadSeqlens.
__global__ void __launch_bounds__(kScanThreads) varlen_tiles_kernel(const int* cu, int nseq, int T, int* tile_off,
                                                                    int* status) {
  __shared__ long long sums[kScanThreads];  // 64-bit: lengths of an invalid table may be anything
  __shared__ int bad;
  const int t = threadIdx.x;
  if (t == 0) bad = (cu[0] != 0 || cu[nseq] != T) ? 1 : 0;
  __syncthreads();
  const int per = (nseq + kScanThreads - 1) / kScanThreads;
  const int lo = t * per < nseq ? t * per : nseq;
  const int hi = lo + per < nseq ? lo + per : nseq;
  long long sum = 0;
  bool ok = true;
  for (int s = lo; s < hi; s++) {
    const long long len = (long long)cu[s + 1] - cu[s];
    ok = ok && len >= 0;
    sum += len > 0 ? (len + 127) / 128 : 0;
  }
  if (!ok) atomicOr(&bad, 1);
  sums[t] = sum;
  __syncthreads();
  // inclusive Hillis-Steele scan of the partial sums
  for (int off = 1; off < kScanThreads; off <<= 1) {
    const long long add = t >= off ? sums[t - off] : 0;
    __syncthreads();
    sums[t] += add;
    __syncthreads();
  }
  const bool zero = bad != 0;
  long long run = t > 0 ? sums[t - 1] : 0;
  for (int s = lo; s < hi; s++) {
    tile_off[s] = zero ? 0 : (int)run;
    const long long len = (long long)cu[s + 1] - cu[s];
    run += len > 0 ? (len + 127) / 128 : 0;
  }
  if (t == kScanThreads - 1) tile_off[nseq] = zero ? 0 : (int)sums[t];
  if (t == 0 && zero) atomicCAS(status, 0, kStatusBadSeqlens);
}

}  // namespace

cudaError_t launch_varlen_tiles(const int* cu_seqlens, int nseq, int T, int* tile_off, int* status, cudaStream_t s) {
  varlen_tiles_kernel<<<1, kScanThreads, 0, s>>>(cu_seqlens, nseq, T, tile_off, status);
  return cudaGetLastError();
}

}  // namespace mxattn

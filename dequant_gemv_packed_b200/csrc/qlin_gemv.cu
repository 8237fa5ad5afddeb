// qlin_gemv: decode-regime quantised linear layer (1 <= M <= 16).
//
// Y[m][n] = sum_k rht(x)[m][k] * w[n][k], w dequantised in registers
// ("24B0978-Week01-Track2_20-Submission01", "How these techniques accelerate
// inference on CUDA": the fp16 weight is never written to memory).
#include "qlin_internal.cuh"

namespace qlin {

// One warp per weight row; the rotated activations come from the workspace.
__global__ void gemv_simple_kernel(PackedView v, const __half* __restrict__ scales,
                                   const __half* __restrict__ zeros,
                                   const __half* __restrict__ xr, __half* __restrict__ y, int M) {
  const int lane = threadIdx.x & 31;
  const int warp0 = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  const int G = v.K / kGroup;
  for (int n = warp0; n < v.N; n += nwarps) {
    int b;
    const uint32_t* row = row_of(v, n, b);
    float acc[16];
#pragma unroll
    for (int m = 0; m < 16; ++m) acc[m] = 0.f;
    for (int k = lane; k < v.K; k += 32) {
      const int g = k / kGroup;
      const float s = __half2float(scales[(size_t)n * G + g]);
      const float z = __half2float(zeros[(size_t)n * G + g]);
      const float w = __half2float(dequant_exact(code_at(row, b, k), s, z));
#pragma unroll
      for (int m = 0; m < 16; ++m)
        if (m < M) acc[m] = fmaf(w, __half2float(xr[(size_t)m * v.K + k]), acc[m]);
    }
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      if (m >= M) break;
      float a = acc[m];
#pragma unroll
      for (int o = 16; o; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      if (lane == 0) y[(size_t)m * v.N + n] = __float2half_rn(a);
    }
  }
}

size_t gemv_workspace_bytes(int M, int K) { return ((size_t)M * K * 2 + 255) & ~(size_t)255; }

qlin_status launch_gemv(const PackedView& v, const __half* scales, const __half* zeros,
                        const uint32_t* sign_bits, const __half* x, __half* y, int M,
                        void* workspace, cudaStream_t s) {
  __half* xr = static_cast<__half*>(workspace);
  qlin_status r = launch_rht(x, xr, sign_bits, M, v.K, s);
  if (r != QLIN_OK) return r;
  const int threads = 256;
  int blocks = (v.N * 32 + threads - 1) / threads;
  if (blocks > 148 * 8) blocks = 148 * 8;
  gemv_simple_kernel<<<blocks, threads, 0, s>>>(v, scales, zeros, xr, y, M);
  return record_cuda(cudaGetLastError());
}

}  // namespace qlin

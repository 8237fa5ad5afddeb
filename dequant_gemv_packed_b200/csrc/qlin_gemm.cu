// qlin_gemm: prefill-regime quantised linear layer.
//
// The activations are rotated into the workspace, the weight is dequantised
// exactly (fp16, as qlin_dequant) into shared memory tile by tile, and the
// tiles are multiplied with fp32 accumulation.
#include "qlin_internal.cuh"

namespace qlin {

namespace simt {
constexpr int BM = 64, BN = 64, BK = 32;
}

// 64x64 output tile per CTA, 256 threads, 4x4 outputs per thread.
__global__ void __launch_bounds__(256) gemm_simt_kernel(PackedView v, const __half* __restrict__ scales,
                                                        const __half* __restrict__ zeros,
                                                        const __half* __restrict__ xr,
                                                        __half* __restrict__ y, int M) {
  using namespace simt;
  __shared__ float xs[BK][BM + 1];
  __shared__ float ws[BK][BN + 1];
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const int G = v.K / kGroup;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < v.K; k0 += BK) {
    for (int i = tid; i < BM * BK; i += 256) {
      const int r = i / BK, c = i % BK;
      const int m = m0 + r;
      xs[c][r] = m < M ? __half2float(xr[(size_t)m * v.K + k0 + c]) : 0.f;
    }
    for (int i = tid; i < BN * BK; i += 256) {
      const int r = i / BK, c = i % BK;
      const int n = n0 + r;
      float w = 0.f;
      if (n < v.N) {
        int b;
        const uint32_t* row = row_of(v, n, b);
        const int k = k0 + c, g = k / kGroup;
        w = __half2float(dequant_exact(code_at(row, b, k), __half2float(scales[(size_t)n * G + g]),
                                       __half2float(zeros[(size_t)n * G + g])));
      }
      ws[c][r] = w;
    }
    __syncthreads();
#pragma unroll 4
    for (int c = 0; c < BK; ++c) {
      float a[4], bb[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = xs[c][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bb[j] = ws[c][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < v.N) y[(size_t)m * v.N + n] = __float2half_rn(acc[i][j]);
    }
  }
}

size_t gemm_workspace_bytes(int M, int K) { return ((size_t)M * K * 2 + 255) & ~(size_t)255; }

qlin_status launch_gemm(const PackedView& v, const __half* scales, const __half* zeros,
                        const uint32_t* sign_bits, const __half* x, __half* y, int M,
                        void* workspace, cudaStream_t s) {
  __half* xr = static_cast<__half*>(workspace);
  qlin_status r = launch_rht(x, xr, sign_bits, M, v.K, s);
  if (r != QLIN_OK) return r;
  dim3 grid((v.N + simt::BN - 1) / simt::BN, (M + simt::BM - 1) / simt::BM);
  if (grid.y > 65535) return QLIN_ERR_SHAPE;
  gemm_simt_kernel<<<grid, 256, 0, s>>>(v, scales, zeros, xr, y, M);
  return record_cuda(cudaGetLastError());
}

}  // namespace qlin

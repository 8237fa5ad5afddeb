// qlin_pack / qlin_unpack / qlin_dequant kernels.
//
// Layout: per row, code k at stream bits [b*k, b*k+b), little-endian 32-bit
// words ("24B0978-Week01-Track2_20-Submission01", "How these techniques
// accelerate inference on CUDA": integer codes with one scale and zero per 128
// along K).  These run once per weight (pack) or only for checks (unpack,
// dequant), so they favour simplicity over speed.
#include "qlin_internal.cuh"

namespace qlin {

// One CTA per row (grid-stride); each thread assembles whole 32-bit words.
__global__ void pack_kernel(PackedView v, const uint8_t* __restrict__ codes,
                            uint8_t* __restrict__ packed) {
  for (int n = blockIdx.x; n < v.N; n += gridDim.x) {
    int b;
    const uint32_t* row_c = row_of(v, n, b);
    uint32_t* row = reinterpret_cast<uint32_t*>(packed + (reinterpret_cast<const uint8_t*>(row_c) - v.codes));
    const uint8_t* src = codes + (size_t)n * v.K;
    const uint32_t mask = (1u << b) - 1u;
    const int words = v.K * b / 32;
    for (int w = threadIdx.x; w < words; w += blockDim.x) {
      const int bit0 = 32 * w;
      const int k0 = bit0 / b, k1 = (bit0 + 31) / b;
      uint32_t word = 0;
      for (int k = k0; k <= k1; ++k) {
        const int pos = b * k - bit0;  // -b < pos < 32
        const uint32_t q = src[k] & mask;
        word |= pos >= 0 ? (q << pos) : (q >> (-pos));
      }
      row[w] = word;
    }
  }
}

// One CTA per row; thread per code.
__global__ void unpack_kernel(PackedView v, uint8_t* __restrict__ codes) {
  for (int n = blockIdx.x; n < v.N; n += gridDim.x) {
    int b;
    const uint32_t* row = row_of(v, n, b);
    for (int k = threadIdx.x; k < v.K; k += blockDim.x)
      codes[(size_t)n * v.K + k] = (uint8_t)code_at(row, b, k);
  }
}

__global__ void dequant_kernel(PackedView v, const __half* __restrict__ scales,
                               const __half* __restrict__ zeros, __half* __restrict__ w) {
  const int G = v.K / kGroup;
  for (int n = blockIdx.x; n < v.N; n += gridDim.x) {
    int b;
    const uint32_t* row = row_of(v, n, b);
    for (int k = threadIdx.x; k < v.K; k += blockDim.x) {
      const int g = k / kGroup;
      const float s = __half2float(scales[(size_t)n * G + g]);
      const float z = __half2float(zeros[(size_t)n * G + g]);
      w[(size_t)n * v.K + k] = dequant_exact(code_at(row, b, k), s, z);
    }
  }
}

static int rows_grid(int N) { return N < 65535 * 8 ? N : 65535 * 8; }

qlin_status launch_pack(const PackedView& v, const uint8_t* codes, uint8_t* packed, cudaStream_t s) {
  pack_kernel<<<rows_grid(v.N), 256, 0, s>>>(v, codes, packed);
  return record_cuda(cudaGetLastError());
}

qlin_status launch_unpack(const PackedView& v, uint8_t* codes, cudaStream_t s) {
  unpack_kernel<<<rows_grid(v.N), 256, 0, s>>>(v, codes);
  return record_cuda(cudaGetLastError());
}

qlin_status launch_dequant(const PackedView& v, const __half* scales, const __half* zeros, __half* w,
                           cudaStream_t s) {
  dequant_kernel<<<rows_grid(v.N), 256, 0, s>>>(v, scales, zeros, w);
  return record_cuda(cudaGetLastError());
}

}  // namespace qlin

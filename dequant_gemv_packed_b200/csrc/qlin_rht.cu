// qlin_rht: random Hadamard transform of the activations.
//
// Per block of 128 along K: negate x[k] where sign bit k is set, run the 7
// add/subtract stages of the Walsh-Hadamard butterfly in fp32 registers and
// warp shuffles, scale by 1/sqrt(128), round once to fp16
// ("24B0978-Week01-Track2_20-Submission01", "How these techniques accelerate
// inference on CUDA", paragraph "Random Hadamard transform").  One warp per
// (row, block); the transform is tiny next to the matmul it feeds.
#include "qlin_internal.cuh"
#include "qlin_sm100.cuh"

namespace qlin {

__global__ void rht_kernel(const __half* __restrict__ x, __half* __restrict__ xr,
                           const uint32_t* __restrict__ sign_bits, int M, int K, uint32_t* clear, int nclear,
                           float* xsum) {
  const int lane = threadIdx.x & 31;
  // A kernel launched after this one as a programmatic dependent (the GEMM)
  // may start now: it reads what this kernel writes only after its own
  // dependency wait.
  if (threadIdx.x == 0) grid_launch_dependents();
  // Words the kernel that follows expects to find zero (its completion flags).
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < nclear; i += blockDim.x) clear[i] = 0u;
  const int blocks_per_row = K / kHadamard;
  const long long total = (long long)M * blocks_per_row;
  const long long warp0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long t = warp0; t < total; t += nwarps) {
    const int m = (int)(t / blocks_per_row);
    const int blk = (int)(t % blocks_per_row);
    const size_t base = (size_t)m * K + (size_t)blk * kHadamard + 4 * lane;
    const uint2 raw = *reinterpret_cast<const uint2*>(x + base);
    const uint32_t sw = sign_bits[blk * 4 + (lane >> 3)] >> (4 * (lane & 7));
    __half2 h01 = *reinterpret_cast<const __half2*>(&raw.x);
    __half2 h23 = *reinterpret_cast<const __half2*>(&raw.y);
    float v[4] = {__low2float(h01), __high2float(h01), __low2float(h23), __high2float(h23)};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if ((sw >> i) & 1u) v[i] = -v[i];
    fwht128_warp(v, lane);
    h01 = __floats2half2_rn(v[0] * kInvSqrt128, v[1] * kInvSqrt128);
    h23 = __floats2half2_rn(v[2] * kInvSqrt128, v[3] * kInvSqrt128);
    uint2 out;
    out.x = *reinterpret_cast<uint32_t*>(&h01);
    out.y = *reinterpret_cast<uint32_t*>(&h23);
    *reinterpret_cast<uint2*>(xr + base) = out;
    if (xsum) {  // sum of the block's rounded values (one group of 128 along K)
      float sum = (__low2float(h01) + __high2float(h01)) + (__low2float(h23) + __high2float(h23));
#pragma unroll
      for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) xsum[t] = sum;
    }
  }
}

qlin_status launch_rht(const __half* x, __half* xr, const uint32_t* sign_bits, int M, int K,
                       cudaStream_t s, uint32_t* clear, int nclear, float* xsum) {
  const long long warps = (long long)M * (K / kHadamard);
  const int threads = 256;
  long long blocks = (warps * 32 + threads - 1) / threads;
  if (blocks > 148 * 16) blocks = 148 * 16;
  rht_kernel<<<(int)blocks, threads, 0, s>>>(x, xr, sign_bits, M, K, clear, nclear, xsum);
  return record_cuda(cudaGetLastError());
}

}  // namespace qlin

// qlin_quantize_rtn: the offline weight side of the layer on the GPU.
//
// Each weight row is rotated along K with the activations' signs and block-128
// Hadamard ("24B0978-Week01-Track2_20-Submission01", paragraph "Random
// Hadamard transform": the weight side of the rotation is folded in offline),
//   w~ = (1/sqrt(128)) H diag(d) w   per block of 128,
// then quantised per group of 128 by asymmetric round-to-nearest
// ("24B0978-Week02-Track2-40-Submission01", recipe op "quant_rtn", bits and
// group 128; the affine form w = s (q - z) of "Group-wise affine integer
// quantisation" on the first page):
//   s = fp16((max - min) / (2^b - 1))  (1 if that is 0),
//   z = fp16(-min / s),  q = clamp(rint(w~ / s + z), 0, 2^b - 1).
//
// Exactness: the input is fp16, so every value is an integer multiple of 2^-24
// below 2^16 in magnitude; a sum of 128 of them (any order) is a multiple of
// 2^-24 below 2^23, exact in fp64.  The butterflies are therefore exact, the
// scaling is one fp64 multiply by 1/sqrt(128) (sqrt and division each rounded
// to nearest), then one rounding to fp32; the quantiser is IEEE fp32 (no
// contraction).  The codes are a function of the input, independent of the
// order of the butterflies.
//
// One warp per (row, group): lane l holds elements 4l .. 4l + 3 of the block;
// butterfly strides 1 and 2 stay in the lane, strides 4 .. 64 are fp64
// shuffles with lane distance 1 .. 16.
#include "qlin_internal.cuh"

namespace qlin {
namespace {

constexpr int kWarpsPerBlock = 8;

// Rows [0, N) of the arguments (already offset to the first row), all of width b.
__global__ void __launch_bounds__(kWarpsPerBlock * 32) quantize_rtn_kernel(
    const __half* __restrict__ w, const uint32_t* __restrict__ sign_bits, int b, int N, int K,
    uint8_t* __restrict__ codes, __half* __restrict__ scales, __half* __restrict__ zeros) {
  const int G = K / kGroup;
  const long long item = (long long)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  if (item >= (long long)N * G) return;  // warp-uniform
  const int lane = threadIdx.x & 31;
  const int n = (int)(item / G), g = (int)(item % G);
  const float qmax = (float)((1 << b) - 1);

  // load 4 fp16 and their signs (bit e of the block's 128 sign bits: 1 -> -1)
  const size_t base = (size_t)n * K + (size_t)g * kGroup + 4 * lane;
  const uint2 raw = *reinterpret_cast<const uint2*>(w + base);
  const uint32_t sw = sign_bits[g * 4 + (lane >> 3)] >> (4 * (lane & 7));
  const __half2 h01 = *reinterpret_cast<const __half2*>(&raw.x);
  const __half2 h23 = *reinterpret_cast<const __half2*>(&raw.y);
  double v[4] = {(double)__low2float(h01), (double)__high2float(h01), (double)__low2float(h23),
                 (double)__high2float(h23)};
#pragma unroll
  for (int j = 0; j < 4; ++j)
    if ((sw >> j) & 1u) v[j] = -v[j];

  // block FWHT (natural order), exact in fp64
  {
    const double a0 = v[0] + v[1], a1 = v[0] - v[1], a2 = v[2] + v[3], a3 = v[2] - v[3];
    v[0] = a0 + a2;
    v[1] = a1 + a3;
    v[2] = a0 - a2;
    v[3] = a1 - a3;
  }
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const double p = __shfl_xor_sync(0xffffffffu, v[j], o);
      v[j] = upper ? p - v[j] : v[j] + p;
    }
  }
  const double inv_sqrt = __ddiv_rn(1.0, __dsqrt_rn(128.0));
  float f[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) f[j] = __double2float_rn(__dmul_rn(v[j], inv_sqrt));

  // group minimum and maximum (exact)
  float mn = fminf(fminf(f[0], f[1]), fminf(f[2], f[3]));
  float mx = fmaxf(fmaxf(f[0], f[1]), fmaxf(f[2], f[3]));
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  mn = __fadd_rn(mn, 0.f);  // a zero minimum is +0 whichever zero the reduction kept
  __half s16 = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), qmax));
  if (!(__half2float(s16) > 0.f)) s16 = __float2half_rn(1.f);
  const float s32 = __half2float(s16);
  const __half z16 = __float2half_rn(__fdiv_rn(-mn, s32));
  const float z32 = __half2float(z16);

  uint32_t packed = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float q = fminf(fmaxf(rintf(__fadd_rn(__fdiv_rn(f[j], s32), z32)), 0.f), qmax);
    packed |= (uint32_t)q << (8 * j);
  }
  *reinterpret_cast<uint32_t*>(codes + base) = packed;
  if (lane == 0) {
    scales[(size_t)n * G + g] = s16;
    zeros[(size_t)n * G + g] = z16;
  }
}

}  // namespace

// One launch per run of rows of one width (the whole matrix for uniform
// widths; runs of equal 64-row blocks, from the host width table, for mixed).
qlin_status launch_quantize_rtn(const __half* w, const uint32_t* sign_bits, const uint8_t* block_bits, int bits,
                                int N, int K, uint8_t* codes, __half* scales, __half* zeros, cudaStream_t s) {
  const int G = K / kGroup;
  for (int r0 = 0; r0 < N;) {
    int r1 = N, b = bits;
    if (!bits) {
      b = block_bits[r0 / kBlockRows];
      r1 = r0 + kBlockRows;
      while (r1 < N && block_bits[r1 / kBlockRows] == b) r1 += kBlockRows;
    }
    const long long items = (long long)(r1 - r0) * G;
    const long long grid = (items + kWarpsPerBlock - 1) / kWarpsPerBlock;
    if (grid > 0x7fffffffLL) return QLIN_ERR_SHAPE;
    quantize_rtn_kernel<<<(unsigned)grid, kWarpsPerBlock * 32, 0, s>>>(
        w + (size_t)r0 * K, sign_bits, b, r1 - r0, K, codes + (size_t)r0 * K, scales + (size_t)r0 * G,
        zeros + (size_t)r0 * G);
    const qlin_status st = record_cuda(cudaGetLastError());
    if (st != QLIN_OK) return st;
    r0 = r1;
  }
  return QLIN_OK;
}

}  // namespace qlin

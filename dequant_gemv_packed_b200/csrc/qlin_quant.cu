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
// Eight lanes per (row, group), four groups a warp: lane t = lane % 8 of the
// eight holds elements 16t .. 16t + 15 of the block.  Butterfly strides 1 .. 8
// stay in the lane, strides 16, 32, 64 are fp64 shuffles with lane distance
// 1, 2, 4; the group's min and max take three shuffle steps.
#include "qlin_internal.cuh"

namespace qlin {
namespace {

constexpr int kWarpsPerBlock = 8;
constexpr int kGroupsPerWarp = 4;

// Rows [0, N) of the arguments (already offset to the first row), all of width b.
// kRotateOnly: write the rotated rows (fp32) to `rotated` and stop there (the
// input of the error-compensated quantiser).
template <bool kRotateOnly>
__global__ void __launch_bounds__(kWarpsPerBlock * 32) quantize_rtn_kernel(
    const __half* __restrict__ w, const uint32_t* __restrict__ sign_bits, int b, int N, int K,
    uint8_t* __restrict__ codes, __half* __restrict__ scales, __half* __restrict__ zeros,
    float* __restrict__ rotated) {
  const int G = K / kGroup;
  const long long total = (long long)N * G;
  const int lane = threadIdx.x & 31, t = lane & 7;
  const long long item = ((long long)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5)) * kGroupsPerWarp + (lane >> 3);
  if (item - (lane >> 3) >= total) return;  // the warp's first item: warp-uniform
  const bool live = item < total;          // lanes past the last item shuffle along on a valid one
  const long long it = live ? item : total - 1;
  const int n = (int)(it / G), g = (int)(it % G);
  const float qmax = (float)((1 << b) - 1);

  // load 16 fp16 and their signs (bit e of the block's 128 sign bits: 1 -> -1)
  const size_t base = (size_t)n * K + (size_t)g * kGroup + 16 * t;
  const uint4 r0 = reinterpret_cast<const uint4*>(w + base)[0];
  const uint4 r1 = reinterpret_cast<const uint4*>(w + base)[1];
  const uint32_t sw = sign_bits[g * 4 + (t >> 1)] >> (16 * (t & 1));
  const uint32_t raw[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
  double v[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const __half2 h = *reinterpret_cast<const __half2*>(&raw[i]);
    v[2 * i] = (double)__low2float(h);
    v[2 * i + 1] = (double)__high2float(h);
  }
#pragma unroll
  for (int j = 0; j < 16; ++j)
    if ((sw >> j) & 1u) v[j] = -v[j];

  // block FWHT (natural order), exact in fp64: strides 1 .. 8 in the lane
#pragma unroll
  for (int h = 1; h < 16; h <<= 1)
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (!(j & h)) {
        const double u = v[j], x = v[j + h];
        v[j] = u + x;
        v[j + h] = u - x;
      }
  // strides 16, 32, 64 across the group's eight lanes
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) {
    const bool upper = (t & o) != 0;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const double p = __shfl_xor_sync(0xffffffffu, v[j], o);
      v[j] = upper ? p - v[j] : v[j] + p;
    }
  }
  const double inv_sqrt = __ddiv_rn(1.0, __dsqrt_rn(128.0));
  float f[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) f[j] = __double2float_rn(__dmul_rn(v[j], inv_sqrt));
  if constexpr (kRotateOnly) {
    if (live) {
      float4* out = reinterpret_cast<float4*>(rotated + base);
#pragma unroll
      for (int j = 0; j < 4; ++j) out[j] = make_float4(f[4 * j], f[4 * j + 1], f[4 * j + 2], f[4 * j + 3]);
    }
    return;
  }

  // group minimum and maximum (exact)
  float mn = f[0], mx = f[0];
#pragma unroll
  for (int j = 1; j < 16; ++j) {
    mn = fminf(mn, f[j]);
    mx = fmaxf(mx, f[j]);
  }
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  mn = __fadd_rn(mn, 0.f);  // a zero minimum is +0 whichever zero the reduction kept
  __half s16 = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), qmax));
  if (!(__half2float(s16) > 0.f)) s16 = __float2half_rn(1.f);
  const float s32 = __half2float(s16);
  const __half z16 = __float2half_rn(__fdiv_rn(-mn, s32));
  const float z32 = __half2float(z16);

  uint32_t packed[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float q = fminf(fmaxf(rintf(__fadd_rn(__fdiv_rn(f[j], s32), z32)), 0.f), qmax);
    packed[j >> 2] |= (uint32_t)q << (8 * (j & 3));
  }
  if (!live) return;
  *reinterpret_cast<uint4*>(codes + base) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  if (t == 0) {
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
    const long long per_block = (long long)kWarpsPerBlock * kGroupsPerWarp;
    const long long grid = (items + per_block - 1) / per_block;
    if (grid > 0x7fffffffLL) return QLIN_ERR_SHAPE;
    quantize_rtn_kernel<false><<<(unsigned)grid, kWarpsPerBlock * 32, 0, s>>>(
        w + (size_t)r0 * K, sign_bits, b, r1 - r0, K, codes + (size_t)r0 * K, scales + (size_t)r0 * G,
        zeros + (size_t)r0 * G, nullptr);
    const qlin_status st = record_cuda(cudaGetLastError());
    if (st != QLIN_OK) return st;
    r0 = r1;
  }
  return QLIN_OK;
}

// The rotated rows alone, fp32 [N][K]: w~ = fp32(fp64(1/sqrt(128)) (H diag(d) w))
// per block of 128, the same values the quantiser above works on.
qlin_status launch_rotate_weight(const __half* w, const uint32_t* sign_bits, int N, int K, float* rotated,
                                 cudaStream_t s) {
  const long long items = (long long)N * (K / kGroup);
  const long long per_block = (long long)kWarpsPerBlock * kGroupsPerWarp;
  const long long grid = (items + per_block - 1) / per_block;
  if (grid > 0x7fffffffLL) return QLIN_ERR_SHAPE;
  quantize_rtn_kernel<true><<<(unsigned)grid, kWarpsPerBlock * 32, 0, s>>>(w, sign_bits, 8, N, K, nullptr, nullptr,
                                                                           nullptr, rotated);
  return record_cuda(cudaGetLastError());
}

}  // namespace qlin

// Block-128 random Hadamard transform of one block of x by one warp, as a
// tensor-core product, for the decode kernels' prologues.
//
// The order-128 Sylvester matrix factors as H16 (x) H8: with element index
// e = i + 16 j (bits 0-3 and 4-6 of e), popcount(e & e') splits over the two
// bit fields, so for X[i][j] = d_e x_e the transform is H16 X H8.  One
// m16n8k16 product (A = H16, +-1 exact in fp16; B = X; fp32 accumulation)
// does the H16 side, three butterfly stages along j (one in registers, two
// across lanes t ^ 1 and t ^ 2) the H8 side; then x 1/sqrt(128) in fp32 and
// one rounding to fp16 ("24B0978-Week01-Track2_20-Submission01", paragraph
// "Random Hadamard transform": random signs, then the Walsh-Hadamard
// transform; orthonormal scaling).
//
// Lane (g, t) = (lane / 4, lane % 4) supplies X[2t, 2t+1][g] and X[2t+8, 2t+9][g],
// i.e. the fp16 pairs of x at 16g + 2t (b0) and 16g + 2t + 8 (b1) with their
// sign bits, and ends with the rotated elements g + 32t + rot_off(i).
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "qlin_internal.cuh"

namespace qlin {

// Offset of the lane's i-th rotated element: 0, 16, 8, 24.
__host__ __device__ __forceinline__ constexpr int rot_off(int i) { return ((i & 1) << 4) | ((i & 2) << 2); }

// (H[r][c], H[r][c+1]) of the Sylvester matrix of order 16 as two fp16 (+-1).
__device__ __forceinline__ uint32_t h16_pair(int r, int c) {
  const uint32_t lo = (__popc(r & c) & 1) ? 0xBC00u : 0x3C00u;
  const uint32_t hi = (__popc(r & (c + 1)) & 1) ? 0xBC00u : 0x3C00u;
  return lo | (hi << 16);
}

// The A fragment of H16 held by `lane` in an m16n8k16 product.
__device__ __forceinline__ void h16_fragment(int lane, uint32_t (&h)[4]) {
  const int g = lane >> 2, t = lane & 3;
  h[0] = h16_pair(g, 2 * t);
  h[1] = h16_pair(g + 8, 2 * t);
  h[2] = h16_pair(g, 2 * t + 8);
  h[3] = h16_pair(g + 8, 2 * t + 8);
}

// Sign bits of the lane's four x values, from sign word (block * 4 + g / 2)
// shifted right by 16 (g & 1) + 2t: bits 0, 1 (b0's pair) and 8, 9 (b1's).
__device__ __forceinline__ uint32_t rot_sign_bits(const uint32_t* sign_bits, int blk, int lane) {
  const int g = lane >> 2, t = lane & 3;
  return sign_bits[blk * 4 + (g >> 1)] >> (16 * (g & 1) + 2 * t);
}

// Rotates one block: hv[i] = fp16 of the rotated element g + 32t + rot_off(i),
// f[i] the same value as fp32.
__device__ __forceinline__ void rotate_block16x8(uint32_t b0, uint32_t b1, uint32_t sw, const uint32_t (&h)[4],
                                                 int lane, __half (&hv)[4], float (&f)[4]) {
  const int t = lane & 3;
  b0 ^= ((sw & 1u) << 15) | ((sw & 2u) << 30);
  b1 ^= (((sw >> 8) & 1u) << 15) | (((sw >> 8) & 2u) << 30);
  float c0, c1, c2, c3;
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
      : "=f"(c0), "=f"(c1), "=f"(c2), "=f"(c3)
      : "r"(h[0]), "r"(h[1]), "r"(h[2]), "r"(h[3]), "r"(b0), "r"(b1), "f"(0.f));
  // columns 2t, 2t+1 (stride 1 in j), then partners t^1 and t^2 (strides 2, 4)
  float v[4] = {c0 + c1, c0 - c1, c2 + c3, c2 - c3};
#pragma unroll
  for (int o = 1; o <= 2; o <<= 1) {
    const bool up = (t & o) != 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float q = __shfl_xor_sync(0xffffffffu, v[i], o);
      v[i] = up ? q - v[i] : v[i] + q;
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    hv[i] = __float2half_rn(v[i] * kInvSqrt128);
    f[i] = __half2float(hv[i]);
  }
}

}  // namespace qlin

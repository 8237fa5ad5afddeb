// Internal declarations and device routines shared by the qlin kernels.
//
// Every kernel that reads packed codes goes through the decode routines here
// (code_at / dequant_exact / row_of), so qlin_unpack and qlin_dequant exercise
// exactly the arithmetic that qlin_gemv and qlin_gemm use.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "qlin.h"

namespace qlin {

constexpr int kGroup = 128;      // codes per scale/zero group along K
constexpr int kBlockRows = 64;   // rows per width block in the mixed format
constexpr int kHadamard = 128;   // block of the activation rotation
// 1/sqrt(128) = 2^-3.5, rounded to fp32 (0x3DB504F3).
constexpr float kInvSqrt128 = 0.0883883476483184405f;

// Device view of a packed weight.
struct PackedView {
  const uint8_t* codes;      // code stream
  const uint32_t* start16;   // mixed: block start in 16-byte units [N/64 + 1]
  const uint8_t* widths;     // mixed: block widths [N/64]
  int64_t row_bytes_uniform; // uniform: K * bits / 8
  int32_t N, K;
  int32_t bits;              // uniform width, 0 = mixed
};

// Host-side helpers (qlin_api.cu).
size_t code_bytes(const qlin_desc* d);
size_t table_offset(const qlin_desc* d);
PackedView make_view(const qlin_desc* d, const void* packed);
qlin_status record_cuda(cudaError_t e);
bool overlap_enabled();

// Launchers (each returns QLIN_OK or QLIN_ERR_CUDA).
qlin_status launch_pack(const PackedView& v, const uint8_t* codes, uint8_t* packed,
                        cudaStream_t s);
qlin_status launch_unpack(const PackedView& v, uint8_t* codes, cudaStream_t s);
qlin_status launch_dequant(const PackedView& v, const __half* scales, const __half* zeros,
                           __half* w, cudaStream_t s);
// Rotation of M rows of x into xr; also zeroes clear[0, nclear) (completion
// flags of the kernel that follows on the stream) and, if xsum is given,
// writes the sum of each row's 128-value blocks of xr: xsum[m * K/128 + block].
qlin_status launch_rht(const __half* x, __half* xr, const uint32_t* sign_bits, int M, int K,
                       cudaStream_t s, uint32_t* clear = nullptr, int nclear = 0, float* xsum = nullptr);
size_t gemv_workspace_bytes(int bits, int N, int K, int M);
void gemv_plan_info(int bits, int N, int K, int M, qlin_gemv_plan_info* info);
unsigned take_gemv_error();
unsigned take_gemm_error();
qlin_status launch_gemv(const PackedView& v, const __half* scales, const __half* zeros,
                        const uint32_t* sign_bits, const __half* x, __half* y, int M,
                        void* workspace, cudaStream_t s);
// The M = 1 integer-tensor-core GEMV (4- and 8-bit codes, a CTA's rows resident
// in shared memory): whether it takes this shape, and its launch.
bool gemv_imma_fits(int bits, int N, int K, int M);
qlin_status launch_gemv_imma(const PackedView& v, const __half* scales, const __half* zeros,
                             const uint32_t* sign_bits, const __half* x, __half* y, cudaStream_t s);
void gemv_imma_plan_info(int bits, int N, int K, qlin_gemv_plan_info* info);
unsigned take_imma_error();
// The split-K tensor-core GEMV for M = 1..16 and one code width (x rotated in
// the kernel; workspace: per-tile counters and slice partial sums).
bool gemv_tc_fits(int bits, int N, int K, int M);
size_t gemv_tc_workspace_bytes(int bits, int N, int K, int M);
qlin_status launch_gemv_tc(const PackedView& v, const __half* scales, const __half* zeros, const uint32_t* sign_bits,
                           const __half* x, __half* y, int M, void* workspace, cudaStream_t s);
void gemv_tc_plan_info(int bits, int N, int K, int M, qlin_gemv_plan_info* info);
unsigned take_tc_error();
// Rotation and round-to-nearest quantisation of fp16 weight rows (offline tool).
qlin_status launch_quantize_rtn(const __half* w, const uint32_t* sign_bits, const uint8_t* block_bits, int bits,
                                int N, int K, uint8_t* codes, __half* scales, __half* zeros, cudaStream_t s);
// Rotation of fp16 weight rows into fp32 (the offline tools' first step).
qlin_status launch_rotate_weight(const __half* w, const uint32_t* sign_bits, int N, int K, float* rotated,
                                 cudaStream_t s);
// Rotation and error-compensated quantisation (GPTQ) of fp16 weight rows.
size_t gptq_workspace_bytes(int N, int K);
qlin_status launch_quantize_gptq(const __half* w, const uint32_t* sign_bits, const float* U, const uint8_t* block_bits,
                                 int bits, int N, int K, uint8_t* codes, __half* scales, __half* zeros,
                                 void* workspace, cudaStream_t s);
size_t gemm_workspace_bytes(int M, int K);
qlin_status launch_gemm(const PackedView& v, const __half* scales, const __half* zeros,
                        const uint32_t* sign_bits, const __half* x, __half* y, int M,
                        void* workspace, cudaStream_t s);

// ---------------------------------------------------------------------------
// Device decode routines
// ---------------------------------------------------------------------------

// Width of row n and the first 32-bit word of its bit stream.
__device__ __forceinline__ const uint32_t* row_of(const PackedView& v, int n, int& b) {
  if (v.bits) {
    b = v.bits;
    return reinterpret_cast<const uint32_t*>(v.codes + (size_t)n * (size_t)v.row_bytes_uniform);
  }
  const int j = n >> 6;
  b = v.widths[j];
  const size_t off = (size_t)v.start16[j] * 16u + (size_t)(n & 63) * (size_t)v.K * b / 8u;
  return reinterpret_cast<const uint32_t*>(v.codes + off);
}

// Code k of a row stream of width b: stream bits [b*k, b*k + b).
__device__ __forceinline__ uint32_t code_at(const uint32_t* row, int b, int k) {
  const uint32_t bit = (uint32_t)b * (uint32_t)k;
  const uint32_t w = bit >> 5, sh = bit & 31u;
  uint32_t q = row[w] >> sh;
  if (sh + (uint32_t)b > 32u) q |= row[w + 1] << (32u - sh);
  return q & ((1u << b) - 1u);
}

// fp32(a * b + c) with one rounding: a and b fp16 (bit patterns), c fp32.
__device__ __forceinline__ float fma_f16_f32(uint16_t a, uint16_t b, float c) {
  float d;
  asm("fma.rn.f32.f16 %0, %1, %2, %3;" : "=f"(d) : "h"(a), "h"(b), "f"(c));
  return d;
}

// The two fp16 halves of x times b_lo and b_hi, plus c, each rounded once to fp32.
__device__ __forceinline__ void fma_f16x2_f32(uint32_t x, uint16_t b_lo, uint16_t b_hi, float c, float& d_lo,
                                              float& d_hi) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "fma.rn.f32.f16 %0, l, %3, %5;\n\tfma.rn.f32.f16 %1, h, %4, %5;\n\t}"
      : "=f"(d_lo), "=f"(d_hi)
      : "r"(x), "h"(b_lo), "h"(b_hi), "f"(c));
}

// Subtraction of the zero point rounded exactly as fp32(q) - z, scaled by 2^-9:
//   fma_f16_f32(m q, 2^15 / m, -z 2^-9) = fp32(q - z) * 2^-9.
// The 16-bit pattern m q (< 2048) is the fp16 number m q 2^-24 (subnormal, or
// exponent field 1, where the value still grows by 2^-24 per step); times the
// fp16 multiplier 2^15 / m it is q 2^-9 exactly, and the fused add rounds
// q 2^-9 - z 2^-9 once.  Scaling by a power of two commutes with rounding while
// the result stays normal, which it does: |q - z| >= 2^-24 unless it is 0.
constexpr uint16_t kMul15 = 0x7800, kMul13 = 0x7000, kMul11 = 0x6800, kMul7 = 0x5800;  // 2^15, 2^13, 2^11, 2^7

// fp16 weight: t = fp32(q) - z, p = s * t (each rounded to nearest in fp32),
// then one round-to-nearest-even to fp16.  t comes from the form above and p from
// (s 2^9) * (t 2^-9): both scalings are exact, so p is the same fp32 number.
__device__ __forceinline__ __half dequant_exact(uint32_t q, float s, float z) {
  const float t9 = fma_f16_f32((uint16_t)q, kMul15, -z * 0x1p-9f);
  const float p = __fmul_rn(s * 512.0f, t9);
  return __float2half_rn(p);
}

// Unnormalised 128-point Walsh-Hadamard transform of one block held by a warp:
// lane l holds elements 4l..4l+3 in v[0..3].  Stages on index bits 0 and 1 run
// in registers, stages on bits 2..6 exchange with lane l ^ 1, ..., l ^ 16.
__device__ __forceinline__ void fwht128_warp(float v[4], int lane) {
  float a0 = v[0] + v[1], a1 = v[0] - v[1];
  float a2 = v[2] + v[3], a3 = v[2] - v[3];
  v[0] = a0 + a2; v[2] = a0 - a2;
  v[1] = a1 + a3; v[3] = a1 - a3;
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float p = __shfl_xor_sync(0xffffffffu, v[i], m);
      v[i] = upper ? (p - v[i]) : (v[i] + p);
    }
  }
}

}  // namespace qlin

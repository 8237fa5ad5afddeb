// qlin_quantize_gptq: the offline weight side with error compensation (GPTQ).
//
// The weight rows are rotated exactly as qlin_quantize_rtn rotates them (the
// compensation runs in the rotated basis, "24B0978-Week02-Track2-40-
// Submission01", section "Recipe": RHT + GPTQ, 6-bit, group 128), then
// quantised column by column against the calibration Hessian, through the
// upper Cholesky factor U of its damped inverse (U^T U = (H + damp I)^-1, given
// by the caller):
//
//   for each column i in order:
//     at the first column of a group: its grid (s, z) by round-to-nearest from
//         the group's weights as they stand now (qlin_quantize_rtn's formulas);
//     q_i = clamp(rint(w_i / s + z), 0, 2^b - 1);   e_i = (w_i - s (q_i - z)) / U[i][i];
//     w_j -= e_i U[i][j]  for every later column j.
//
// Every operation is an IEEE fp32 operation rounded to nearest, products and
// differences rounded separately (no fused multiply-add), and every weight
// receives its updates one source column at a time, in column order; the
// codes, scales and zeros are therefore a function of (w, U) alone,
// independent of the launch configuration.
//
// Block b of 128 columns (one group) takes two launches:
//   * gptq_block_kernel: one warp per row holds the row's 128 values in
//     registers (4 per lane); the group grid by warp reductions; then the 128
//     columns in order: the owning lane quantises, the error is broadcast by a
//     shuffle, every lane updates its later columns of the block with U's
//     diagonal block (shared memory).  Codes, scale, zero and the 128 errors
//     of the row go out.
//   * gptq_trailing_kernel: every later column of every row, in 32-row x
//     128-column tiles: the tile of w in registers (4 x 4 per thread), the
//     rows' errors and U's rows of the block in shared memory, 128 update
//     steps in order.
#include <atomic>

#include "qlin_internal.cuh"

namespace qlin {
namespace {

constexpr int kBlk = 128;             // columns per step: one group
constexpr int kRowsA = 16;            // rows (warps) per CTA of the block kernel
constexpr int kTR = 32, kTC = 128;    // trailing tile: rows x columns
constexpr int kTrailThreads = 256;    // 8 x 32 threads, 4 x 4 elements each
constexpr int kUBytes = kBlk * kBlk * 4;
constexpr int kETStride = kTR + 4;    // floats per row of the transposed error tile
constexpr int kTrailSmem = kUBytes + kBlk * kETStride * 4;

__device__ __forceinline__ float sel4(const float (&v)[4], int k) {
  return k == 0 ? v[0] : (k == 1 ? v[1] : (k == 2 ? v[2] : v[3]));
}

// Block b of every row: grid, codes and errors of columns [128 b, 128 b + 128),
// with the updates inside the block.  `widths`: per 64-row block (device), or
// null with `bits` uniform.
__global__ void __launch_bounds__(kRowsA * 32) gptq_block_kernel(
    const float* __restrict__ W, const float* __restrict__ U, int N, int K, int b, int bits,
    const uint8_t* __restrict__ widths, uint8_t* __restrict__ codes, __half* __restrict__ scales,
    __half* __restrict__ zeros, float* __restrict__ E) {
  extern __shared__ __align__(16) float us[];  // U[128 b + i][128 b + j], i, j < 128
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const size_t c0 = (size_t)b * kBlk;
  for (int q = threadIdx.x; q < kBlk * kBlk / 4; q += blockDim.x) {
    const int i = q / (kBlk / 4), j4 = q % (kBlk / 4);
    reinterpret_cast<float4*>(us)[q] = *reinterpret_cast<const float4*>(U + (c0 + i) * (size_t)K + c0 + 4 * j4);
  }
  __syncthreads();
  const int r = blockIdx.x * kRowsA + warp;
  if (r >= N) return;
  const int G = K / kBlk;
  const float4 w4 = *reinterpret_cast<const float4*>(W + (size_t)r * K + c0 + 4 * lane);
  float w[4] = {w4.x, w4.y, w4.z, w4.w};
  float mn = fminf(fminf(w[0], w[1]), fminf(w[2], w[3]));
  float mx = fmaxf(fmaxf(w[0], w[1]), fmaxf(w[2], w[3]));
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  mn = __fadd_rn(mn, 0.f);  // a zero minimum is +0 whichever zero the reduction kept
  const int width = widths ? widths[r / kBlockRows] : bits;
  const float qmax = (float)((1 << width) - 1);
  __half s16 = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), qmax));
  if (!(__half2float(s16) > 0.f)) s16 = __float2half_rn(1.f);
  const float s32 = __half2float(s16);
  const __half z16 = __float2half_rn(__fdiv_rn(-mn, s32));
  const float z32 = __half2float(z16);
  uint32_t qpack = 0u;
  float ev[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
  for (int i = 0; i < kBlk; ++i) {
    const int o = i >> 2, k = i & 3;
    float e = 0.f;
    if (lane == o) {
      const float wi = sel4(w, k);
      const float q = fminf(fmaxf(rintf(__fadd_rn(__fdiv_rn(wi, s32), z32)), 0.f), qmax);
      const float wq = __fmul_rn(s32, __fsub_rn(q, z32));
      e = __fdiv_rn(__fsub_rn(wi, wq), us[i * kBlk + i]);
      qpack |= (uint32_t)q << (8 * k);
      ev[0] = k == 0 ? e : ev[0];
      ev[1] = k == 1 ? e : ev[1];
      ev[2] = k == 2 ? e : ev[2];
      ev[3] = k == 3 ? e : ev[3];
    }
    e = __shfl_sync(0xffffffffu, e, o);
    const float4 u = reinterpret_cast<const float4*>(us + i * kBlk)[lane];
    const int j0 = 4 * lane;
    if (j0 > i) w[0] = __fsub_rn(w[0], __fmul_rn(e, u.x));
    if (j0 + 1 > i) w[1] = __fsub_rn(w[1], __fmul_rn(e, u.y));
    if (j0 + 2 > i) w[2] = __fsub_rn(w[2], __fmul_rn(e, u.z));
    if (j0 + 3 > i) w[3] = __fsub_rn(w[3], __fmul_rn(e, u.w));
  }
  *reinterpret_cast<uint32_t*>(codes + (size_t)r * K + c0 + 4 * lane) = qpack;
  *reinterpret_cast<float4*>(E + (size_t)r * kBlk + 4 * lane) = make_float4(ev[0], ev[1], ev[2], ev[3]);
  if (lane == 0) {
    scales[(size_t)r * G + b] = s16;
    zeros[(size_t)r * G + b] = z16;
  }
}

// The later columns [128 (b + 1), K) of every row: w[r][j] -= E[r][i] U[128 b + i][j]
// for i = 0 .. 127 in order.
__global__ void __launch_bounds__(kTrailThreads) gptq_trailing_kernel(float* __restrict__ W,
                                                                      const float* __restrict__ U,
                                                                      const float* __restrict__ E, int N, int K,
                                                                      int b) {
  extern __shared__ __align__(16) float sm[];
  float* ut = sm;                    // [128 i][128 j]
  float* et = sm + kBlk * kBlk;      // [128 i][kETStride]: E transposed, rows of the tile
  const int t = threadIdx.x, tr = t >> 5, tc = t & 31;
  const int r0 = blockIdx.x * kTR;
  const size_t j0 = (size_t)(b + 1) * kBlk + (size_t)blockIdx.y * kTC;
  const size_t ib = (size_t)b * kBlk;
  for (int q = t; q < kBlk * kTC / 4; q += kTrailThreads) {
    const int i = q / (kTC / 4), j4 = q % (kTC / 4);
    reinterpret_cast<float4*>(ut)[q] = *reinterpret_cast<const float4*>(U + (ib + i) * (size_t)K + j0 + 4 * j4);
  }
  for (int q = t; q < kTR * kBlk; q += kTrailThreads) {
    const int rr = q / kBlk, i = q % kBlk;
    et[i * kETStride + rr] = r0 + rr < N ? E[(size_t)(r0 + rr) * kBlk + i] : 0.f;
  }
  float w[4][4];
#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    const int r = r0 + 4 * tr + rr;
    const float4 v = r < N ? *reinterpret_cast<const float4*>(W + (size_t)r * K + j0 + 4 * tc)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
    w[rr][0] = v.x;
    w[rr][1] = v.y;
    w[rr][2] = v.z;
    w[rr][3] = v.w;
  }
  __syncthreads();
#pragma unroll 4
  for (int i = 0; i < kBlk; ++i) {
    const float4 e = *reinterpret_cast<const float4*>(et + i * kETStride + 4 * tr);
    const float4 u = *reinterpret_cast<const float4*>(ut + i * kTC + 4 * tc);
    const float ea[4] = {e.x, e.y, e.z, e.w}, ua[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int rr = 0; rr < 4; ++rr)
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) w[rr][cc] = __fsub_rn(w[rr][cc], __fmul_rn(ea[rr], ua[cc]));
  }
#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    const int r = r0 + 4 * tr + rr;
    if (r < N)
      *reinterpret_cast<float4*>(W + (size_t)r * K + j0 + 4 * tc) = make_float4(w[rr][0], w[rr][1], w[rr][2], w[rr][3]);
  }
}

// Workspace: the rotated rows (fp32 [N][K]), one block's errors (fp32
// [N][128]) and, for mixed widths, the width of each 64-row block.
struct GptqWorkspace {
  size_t e_off, widths_off, total;
  GptqWorkspace(int N, int K) {
    e_off = ((size_t)N * K * 4 + 255) & ~(size_t)255;
    widths_off = e_off + (((size_t)N * kBlk * 4 + 255) & ~(size_t)255);
    total = widths_off + (((size_t)(N / kBlockRows + 1) + 255) & ~(size_t)255);
  }
};

}  // namespace

size_t gptq_workspace_bytes(int N, int K) { return GptqWorkspace(N, K).total; }

qlin_status launch_quantize_gptq(const __half* w, const uint32_t* sign_bits, const float* U, const uint8_t* block_bits,
                                 int bits, int N, int K, uint8_t* codes, __half* scales, __half* zeros,
                                 void* workspace, cudaStream_t s) {
  const GptqWorkspace ws(N, K);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  float* W = reinterpret_cast<float*>(base);
  float* E = reinterpret_cast<float*>(base + ws.e_off);
  uint8_t* widths = nullptr;
  if (!bits) {
    widths = base + ws.widths_off;
    qlin_status r = record_cuda(cudaMemcpyAsync(widths, block_bits, (size_t)N / kBlockRows, cudaMemcpyHostToDevice, s));
    if (r != QLIN_OK) return r;
  }
  qlin_status r = launch_rotate_weight(w, sign_bits, N, K, W, s);
  if (r != QLIN_OK) return r;
  static std::atomic<unsigned long long> configured{0};  // per-device attributes, set once
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda(e);
  if (dev >= 64 || !((configured.load(std::memory_order_acquire) >> dev) & 1ull)) {
    e = cudaFuncSetAttribute(gptq_block_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kUBytes);
    if (e != cudaSuccess) return record_cuda(e);
    e = cudaFuncSetAttribute(gptq_trailing_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTrailSmem);
    if (e != cudaSuccess) return record_cuda(e);
    if (dev < 64) configured.fetch_or(1ull << dev, std::memory_order_release);
  }
  const int G = K / kBlk;
  const unsigned grid_a = (unsigned)((N + kRowsA - 1) / kRowsA);
  const unsigned rows_b = (unsigned)((N + kTR - 1) / kTR);
  for (int b = 0; b < G; ++b) {
    gptq_block_kernel<<<grid_a, kRowsA * 32, kUBytes, s>>>(W, U, N, K, b, bits, widths, codes, scales, zeros, E);
    if (b + 1 < G) {
      const dim3 grid_b(rows_b, (unsigned)((K - (b + 1) * kBlk) / kTC));
      gptq_trailing_kernel<<<grid_b, kTrailThreads, kTrailSmem, s>>>(W, U, E, N, K, b);
    }
    r = record_cuda(cudaGetLastError());
    if (r != QLIN_OK) return r;
  }
  return QLIN_OK;
}

}  // namespace qlin

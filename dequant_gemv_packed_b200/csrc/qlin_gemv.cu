// qlin_gemv: decode-regime quantised linear layer (1 <= M <= 16).
//
// Y[m][n] = sum_k rht(x)[m][k] * w[n][k].  The weight is dequantised in
// registers and never written to memory; the per-group scale and zero are
// applied once to the partial sum of each run of codes that shares them
// ("24B0978-Week01-Track2_20-Submission01", "How these techniques accelerate
// inference on CUDA", paragraph "Group-wise affine integer quantisation"), and
// the random Hadamard rotation of x is fused as the kernel's prologue
// (paragraph "Random Hadamard transform").
//
// M = 1, uniform widths: gemv1_kernel.
//   * One CTA per SM owns a contiguous range of weight rows.  A producer thread
//     streams the rows (one bulk asynchronous copy per row, padded row stride
//     in shared memory so that reads are bank-conflict free) and the group
//     scales/zeros of each chunk of rows into a ring of shared-memory stages.
//     All stages are issued before the prologue, so the whole HBM latency is
//     overlapped with the rotation.
//   * The consumer warps first rotate x (sign flip, 7 butterfly stages in
//     registers and shuffles, x 1/sqrt(128), fp16 rounding) into shared memory.
//   * Each consumer lane then owns one fixed "unit" of K (64 codes for int4 and
//     int6, 128 for int3, 32 for int8) and keeps its slice of rotated x in
//     registers for the whole kernel, walking down the rows of each chunk.
//   * 4- and 8-bit codes: the lane converts its rotated x to 16-bit integers
//     with one power-of-two scale per unit (exact for values within 2^4 of the
//     unit's largest magnitude, else rounded at 2^-14 of it) and takes
//     sum_k q_k x_k exactly in int32 with dp2a (two 16x8-bit products per
//     instruction); nibbles are spread to byte lanes with one mask each.
//   * 3- and 6-bit codes are turned into fp16 without conversions: masking a
//     code into the mantissa of the fp16 constant 1024 (0x6400) gives exactly
//     1024 + c*q, where c is a power of two fixed by the code's bit position;
//     one lop3 produces two such values.  They are multiplied with x in fp16 x
//     fp16 -> fp32 fused multiply-adds, one accumulator per position scale c,
//     and the constant part 1024*sum(x/c) is removed afterwards with a
//     correction computed once per lane from its x registers.
//   * Per (row, unit) the lane stores s*(sum q x - z*sum x) to shared memory;
//     rows are summed over units in a fixed order (deterministic results).
//   * With qlin_set_overlap(1) the kernel is launched as a programmatic
//     dependent: it lets the next kernel start launching at once, streams its
//     weight before waiting on the previous kernel, and waits only before it
//     reads x (so back-to-back calls overlap their ramp and drain).
// Other cases (M > 1, mixed widths): the activation rotation runs as its own
// kernel into the workspace, then gemv_simple_kernel.
#include <algorithm>

#include "qlin_internal.cuh"
#include "qlin_sm100.cuh"

namespace qlin {

__device__ unsigned int g_gemv_error;  // nonzero: a bounded wait gave up

namespace {

constexpr uint32_t kMagic = 0x64006400u;  // fp16 1024.0 in both halves
constexpr int kMaxConsumerWarps = 16;
constexpr int kMaxThreads = (kMaxConsumerWarps + 1) * 32;
// Two CTAs per SM: at most 10 consumer warps each, so registers stay <= 93.
constexpr int kMaxConsumerWarps2 = 10;
constexpr int kMaxThreads2 = (kMaxConsumerWarps2 + 1) * 32;
constexpr int kSmemLimit = 227 * 1024;      // one CTA per SM
constexpr int kSmemLimit2 = 113 * 1024;     // two CTAs per SM
constexpr int kChunkTarget = 24 * 1024;
constexpr int kPartialBudget = 48 * 1024;
constexpr int kMaxStages = 16;
constexpr int kSms = 148;

template <int N> struct int_ {};

template <int B> struct UnitT;
template <> struct UnitT<3> { static constexpr int kBytes = 48, kCodes = 128; };
template <> struct UnitT<4> { static constexpr int kBytes = 32, kCodes = 64; };
template <> struct UnitT<6> { static constexpr int kBytes = 48, kCodes = 64; };
template <> struct UnitT<8> { static constexpr int kBytes = 32, kCodes = 32; };

struct Plan {
  int U;               // units per row
  int UW, RS, NW;      // units per warp, row slots per warp, consumer warps
  int rows_per_cta, grid;
  int row_bytes, row_stride;  // row_stride == row_bytes: a chunk is one contiguous copy
  int swap_odd;        // 32-byte units: lanes on odd row slots read their two halves swapped
  int ctas_per_sm;
  int rows_per_chunk;  // R_c, a multiple of RS
  int stages;
  int chunks_per_window;
  int G;               // groups per row
  int sz_halves;       // halves per stage for each of s and z
  int stage_bytes;
  int off_x, off_part, off_bar;
  int smem_bytes;
};

struct Args {
  const uint8_t* codes;
  const __half* scales;
  const __half* zeros;
  const uint32_t* sign_bits;
  const __half* x;
  __half* y;
  int N, K;
  Plan p;
};

// ---------------------------------------------------------------- decoders --
// Each returns sum_k (1024/c_k + q_k) * x_k over the unit, where c_k is the
// position scale of code k; the lane subtracts corr = sum_k 1024/c_k * x_k.

// Integer decoders (4- and 8-bit codes): dp2a multiplies two signed 16-bit
// activations by two unsigned 8-bit codes and adds to an int32, exactly.
// The lane's x registers hold 16-bit integer pairs ordered to match the byte
// lanes below.
__device__ __forceinline__ int dp2a_lo(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int dp2a_hi(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// int4: word i holds codes 8i..8i+7.  x pairs: (x0,x2) (x4,x6) (x1,x3) (x5,x7).
__device__ __forceinline__ int dot_unit_int(const uint32_t (&w)[8], const uint32_t (&x)[32], int_<4>) {
  int a0 = 0, a1 = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t lo = w[i] & 0x0F0F0F0Fu;         // q0 q2 q4 q6
    const uint32_t hi = (w[i] >> 4) & 0x0F0F0F0Fu;  // q1 q3 q5 q7
    int& A = (i & 1) ? a1 : a0;
    A = dp2a_lo(x[4 * i], lo, A);
    A = dp2a_hi(x[4 * i + 1], lo, A);
    A = dp2a_lo(x[4 * i + 2], hi, A);
    A = dp2a_hi(x[4 * i + 3], hi, A);
  }
  return a0 + a1;
}

// int8: word i holds codes 4i..4i+3.  x pairs: (x0,x1) (x2,x3).
__device__ __forceinline__ int dot_unit_int(const uint32_t (&w)[8], const uint32_t (&x)[16], int_<8>) {
  int a0 = 0, a1 = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int& A = (i & 1) ? a1 : a0;
    A = dp2a_lo(x[2 * i], w[i], A);
    A = dp2a_hi(x[2 * i + 1], w[i], A);
  }
  return a0 + a1;
}

// Position of code c (0-based within the unit) in the lane's int16 x layout.
template <int B>
__device__ __forceinline__ int int_slot(int c) {
  if (B == 8) return c;  // natural order
  // int4: word i = c/8, code j = c%8 -> pair order (0,2) (4,6) (1,3) (5,7)
  const int i = c >> 3, j = c & 7;
  const int pair = ((j & 1) << 1) | (j >> 2);  // j=0,2 ->0; 4,6 ->1; 1,3 ->2; 5,7 ->3
  return 8 * i + 2 * pair + ((j >> 1) & 1);
}

// 48 bits of a 48-byte unit starting at bit 48*p: A = bits [0, 32), B = bits [32, 48) (+ junk above).
__device__ __forceinline__ void piece48(const uint32_t (&w)[12], int p, uint32_t& A, uint32_t& B) {
  const int m = p >> 1;
  if ((p & 1) == 0) {
    A = w[3 * m];
    B = w[3 * m + 1];
  } else {
    A = __funnelshift_r(w[3 * m + 1], w[3 * m + 2], 16);
    B = w[3 * m + 2] >> 16;
  }
}

__device__ __forceinline__ float dot_unit(const uint32_t (&w)[12], const uint32_t (&x)[32],
                                          int_<6>) {
  float a1a = 0.f, a1b = 0.f, a4a = 0.f, a4b = 0.f;
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    uint32_t A, B;
    piece48(w, p, A, B);
    const uint32_t T0 = (A & 0x00FC003Fu) | kMagic;                             // (q0, 4 q3)
    const uint32_t T1 = ((A >> 6) & 0x00FC003Fu) | kMagic;                      // (q1, 4 q4)
    const uint32_t T2 = (__funnelshift_r(A, B, 12) & 0x00FC003Fu) | kMagic;     // (q2, 4 q5)
    const uint32_t R = ((B >> 4) & 0x3Fu) | (B << 8);
    const uint32_t T3 = (R & 0x00FC003Fu) | kMagic;                             // (q6, 4 q7)
    const uint32_t x01 = x[4 * p], x23 = x[4 * p + 1], x45 = x[4 * p + 2], x67 = x[4 * p + 3];
    float& A1 = (p & 1) ? a1b : a1a;
    float& A4 = (p & 1) ? a4b : a4a;
    A1 = fma_f16f32(lo16(T0), lo16(x01), A1);
    A4 = fma_f16f32(hi16(T0), hi16(x23), A4);
    A1 = fma_f16f32(lo16(T1), hi16(x01), A1);
    A4 = fma_f16f32(hi16(T1), lo16(x45), A4);
    A1 = fma_f16f32(lo16(T2), lo16(x23), A1);
    A4 = fma_f16f32(hi16(T2), hi16(x45), A4);
    A1 = fma_f16f32(lo16(T3), lo16(x67), A1);
    A4 = fma_f16f32(hi16(T3), hi16(x67), A4);
  }
  return (a1a + a1b) + 0.25f * (a4a + a4b);
}

__device__ __forceinline__ float dot_unit(const uint32_t (&w)[12], const uint32_t (&x)[64],
                                          int_<3>) {
  float a1 = 0.f, a2 = 0.f, a8 = 0.f, a16 = 0.f, a64 = 0.f, a128 = 0.f;
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    uint32_t A, B;
    piece48(w, p, A, B);
    const uint32_t u0 = A << 1;
    const uint32_t u1 = __funnelshift_r(A, B, 23);
    const uint32_t T0 = (u0 & 0x0007000Eu) | kMagic;  // (2 q0, q5)
    const uint32_t T1 = (u0 & 0x00380070u) | kMagic;  // (16 q1, 8 q6)
    const uint32_t T2 = (u0 & 0x01C00380u) | kMagic;  // (128 q2, 64 q7)
    const uint32_t T3 = (u1 & 0x0007000Eu) | kMagic;  // (2 q8, q13)
    const uint32_t T4 = (u1 & 0x00380070u) | kMagic;  // (16 q9, 8 q14)
    const uint32_t T5 = (u1 & 0x01C00380u) | kMagic;  // (128 q10, 64 q15)
    const uint32_t R = ((A >> 9) & 0x3Fu) | (B << 15);
    const uint32_t T6 = (R & 0x00070007u) | kMagic;   // (q3, q11)
    const uint32_t T7 = (R & 0x00380038u) | kMagic;   // (8 q4, 8 q12)
    const uint32_t* xp = x + 8 * p;  // xp[i] = (x_{2i}, x_{2i+1}) of this pair of pieces
    a2 = fma_f16f32(lo16(T0), lo16(xp[0]), a2);
    a1 = fma_f16f32(hi16(T0), hi16(xp[2]), a1);
    a16 = fma_f16f32(lo16(T1), hi16(xp[0]), a16);
    a8 = fma_f16f32(hi16(T1), lo16(xp[3]), a8);
    a128 = fma_f16f32(lo16(T2), lo16(xp[1]), a128);
    a64 = fma_f16f32(hi16(T2), hi16(xp[3]), a64);
    a2 = fma_f16f32(lo16(T3), lo16(xp[4]), a2);
    a1 = fma_f16f32(hi16(T3), hi16(xp[6]), a1);
    a16 = fma_f16f32(lo16(T4), hi16(xp[4]), a16);
    a8 = fma_f16f32(hi16(T4), lo16(xp[7]), a8);
    a128 = fma_f16f32(lo16(T5), lo16(xp[5]), a128);
    a64 = fma_f16f32(hi16(T5), hi16(xp[7]), a64);
    a1 = fma_f16f32(lo16(T6), hi16(xp[1]), a1);
    a1 = fma_f16f32(hi16(T6), hi16(xp[5]), a1);
    a8 = fma_f16f32(lo16(T7), lo16(xp[2]), a8);
    a8 = fma_f16f32(hi16(T7), lo16(xp[6]), a8);
  }
  return a1 + 0.5f * a2 + 0.125f * a8 + 0.0625f * a16 + 0.015625f * a64 + 0.0078125f * a128;
}

// 1024 / c for code position i of a unit (see the decoders above).
template <int B>
__device__ __forceinline__ float corr_weight(int i) {
  if (B == 8) return 1024.f;
  if (B == 4) return (i & 1) ? 64.f : 1024.f;
  if (B == 6) {
    const int r = i & 7;
    return (r == 3 || r == 4 || r == 5 || r == 7) ? 256.f : 1024.f;
  }
  // B == 3, period 16
  const int r = i & 15;
  switch (r & 7) {
    case 0: return 512.f;
    case 1: return 64.f;
    case 2: return 8.f;
    case 3: return 1024.f;
    case 4: return 128.f;
    case 5: return 1024.f;
    case 6: return 128.f;
    default: return 16.f;
  }
}

__device__ __forceinline__ void gemv_fail(unsigned code) { atomicOr(&g_gemv_error, code); }

// sum_k q_k x_k over one unit: exact integer dot (scaled back) or the fp16
// mantissa-code path minus its constant part.
template <int B, bool kInt, int kWords, int kXw>
__device__ __forceinline__ float unit_dot(const uint32_t (&w)[kWords], const uint32_t (&x)[kXw], float corr,
                                          float xinv) {
  if constexpr (kInt) {
    return (float)dot_unit_int(w, x, int_<B>()) * xinv;
  } else {
    return dot_unit(w, x, int_<B>()) - corr;
  }
}

template <int kWords>
__device__ __forceinline__ void load_unit(const uint8_t* src, uint32_t (&w)[kWords], int half_first = 0) {
  const uint4* cp = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int i = 0; i < kWords / 4; ++i) {
    const uint4 v = cp[kWords == 8 ? (i ^ half_first) : i];
    w[4 * i] = v.x;
    w[4 * i + 1] = v.y;
    w[4 * i + 2] = v.z;
    w[4 * i + 3] = v.w;
  }
}

// ------------------------------------------------------------------ kernel --

template <int B>
__global__ void __launch_bounds__(B == 3 ? kMaxThreads : kMaxThreads2, B == 3 ? 1 : 2)
    gemv1_kernel(const __grid_constant__ Args a) {
  using UT = UnitT<B>;
  constexpr int kWords = UT::kBytes / 4;
  constexpr int kXw = UT::kCodes / 2;  // half2 registers of x per lane
  extern __shared__ __align__(128) uint8_t smem[];
  const Plan& p = a.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ncons = p.NW * 32;
  const int n0 = blockIdx.x * p.rows_per_cta;
  const int rows = min(p.rows_per_cta, a.N - n0);
  if (rows <= 0) return;
  const int Rc = p.rows_per_chunk;
  const int nchunks = (rows + Rc - 1) / Rc;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  uint64_t* empty = full + kMaxStages;
  __half* xs = reinterpret_cast<__half*>(smem + p.off_x);
  float* part = reinterpret_cast<float*>(smem + p.off_part);

  if (tid == ncons) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], p.NW);
    }
    mbar_fence_init();
  }
  __syncthreads();
  // Programmatic dependent launch: the next kernel on the stream may start
  // launching now; this kernel's own weight stream does not depend on the
  // previous kernel, x and y do (grid_dependency_wait below).
  if (tid == 0) grid_launch_dependents();

  if (warp == p.NW) {
    // ------------------------------------------------------- producer ----
    if (lane != 0) return;
    for (int t = 0; t < nchunks; ++t) {
      const int s = t % p.stages;
      if (t >= p.stages && !mbar_wait(&empty[s], ((t / p.stages) - 1) & 1, &g_gemv_error)) gemv_fail(1u);
      uint8_t* st = smem + (size_t)s * p.stage_bytes;
      __half* ssm = reinterpret_cast<__half*>(st + (size_t)Rc * p.row_stride);
      __half* zsm = ssm + p.sz_halves;
      const int cr0 = t * Rc, cr = min(Rc, rows - cr0);
      const size_t h0 = (size_t)(n0 + cr0) * p.G, h1 = h0 + (size_t)cr * p.G;
      const size_t al = h0 & ~(size_t)7, bl = h1 & ~(size_t)7;
      for (size_t h = (bl > h0 ? bl : h0); h < h1; ++h) {  // unaligned tail: plain copies
        ssm[h - al] = a.scales[h];
        zsm[h - al] = a.zeros[h];
      }
      const uint32_t szb = bl > al ? (uint32_t)(bl - al) * 2u : 0u;
      mbar_arrive_expect_tx(&full[s], (uint32_t)cr * p.row_bytes + 2u * szb);
      bulk_g2s(st, a.codes + (size_t)(n0 + cr0) * p.row_bytes, (uint32_t)cr * p.row_bytes, &full[s]);
      if (szb) {
        bulk_g2s(ssm, a.scales + al, szb, &full[s]);
        bulk_g2s(zsm, a.zeros + al, szb, &full[s]);
      }
    }
    return;
  }

  // --------------------------------------------------------- prologue ----
  // Rotate x into shared memory: warp per block of 128, lane holds 4 values.
  // All of a warp's x loads are issued before any is used (one memory latency).
  grid_dependency_wait();
  const int nblk = a.K / kHadamard;
  for (int blk0 = warp; blk0 < nblk; blk0 += 8 * p.NW) {
    uint2 raw[8];
    uint32_t sw[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int blk = blk0 + j * p.NW;
      if (blk < nblk) {
        raw[j] = *reinterpret_cast<const uint2*>(a.x + blk * kHadamard + 4 * lane);
        sw[j] = a.sign_bits[blk * 4 + (lane >> 3)] >> (4 * (lane & 7));
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int blk = blk0 + j * p.NW;
      if (blk >= nblk) break;
      const __half2 h01 = *reinterpret_cast<const __half2*>(&raw[j].x);
      const __half2 h23 = *reinterpret_cast<const __half2*>(&raw[j].y);
      float v[4] = {__low2float(h01), __high2float(h01), __low2float(h23), __high2float(h23)};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if ((sw[j] >> i) & 1u) v[i] = -v[i];
      fwht128_warp(v, lane);
      __half2 o01 = __floats2half2_rn(v[0] * kInvSqrt128, v[1] * kInvSqrt128);
      __half2 o23 = __floats2half2_rn(v[2] * kInvSqrt128, v[3] * kInvSqrt128);
      uint2 out;
      out.x = *reinterpret_cast<uint32_t*>(&o01);
      out.y = *reinterpret_cast<uint32_t*>(&o23);
      *reinterpret_cast<uint2*>(xs + blk * kHadamard + 4 * lane) = out;
    }
  }
  named_barrier(1, ncons);

  // Fixed unit of this lane, its x slice in registers, and its corrections.
  const int u = warp * p.UW + (lane % p.UW);
  const int row_sub = lane / p.UW;
  const bool active = row_sub < p.RS && u < p.U;
  constexpr bool kIntPath = (B == 4 || B == 8);
  uint32_t xr[kXw];
  float corr = 0.f, sx = 0.f, xinv = 1.f;
  if (active) {
    const uint4* xp = reinterpret_cast<const uint4*>(xs + (size_t)u * UT::kCodes);
#pragma unroll
    for (int i = 0; i < kXw / 4; ++i) {
      const uint4 v = xp[i];
      xr[4 * i] = v.x;
      xr[4 * i + 1] = v.y;
      xr[4 * i + 2] = v.z;
      xr[4 * i + 3] = v.w;
    }
    if constexpr (kIntPath) {
      // 16-bit integers with one power-of-two scale per unit: x_int = rne(x * 2^(13-E)),
      // E the exponent of the unit's largest |x| (|x_int| < 2^14, exact for values
      // within 2^4 of that maximum, else rounded at 2^(E-14)).
      float m = 0.f;
#pragma unroll
      for (int i = 0; i < kXw; ++i) {
        const __half2 h = *reinterpret_cast<const __half2*>(&xr[i]);
        m = fmaxf(m, fmaxf(fabsf(__low2float(h)), fabsf(__high2float(h))));
      }
      const int E = m > 0.f ? (int)((__float_as_uint(m) >> 23) & 0xFF) - 127 : 0;
      const float up = __uint_as_float((uint32_t)(127 + 13 - E) << 23);
      xinv = __uint_as_float((uint32_t)(127 - 13 + E) << 23);
      uint32_t xi[kXw];
      int isum = 0;
#pragma unroll
      for (int i = 0; i < kXw; ++i) {
        const __half2 h = *reinterpret_cast<const __half2*>(&xr[i]);
        const int v0 = __float2int_rn(__low2float(h) * up), v1 = __float2int_rn(__high2float(h) * up);
        isum += v0 + v1;
        const int s0 = int_slot<B>(2 * i), s1 = int_slot<B>(2 * i + 1);
        reinterpret_cast<uint16_t*>(xi)[s0] = (uint16_t)v0;
        reinterpret_cast<uint16_t*>(xi)[s1] = (uint16_t)v1;
      }
#pragma unroll
      for (int i = 0; i < kXw; ++i) xr[i] = xi[i];
      sx = (float)isum * xinv;
    } else {
#pragma unroll
      for (int i = 0; i < kXw; ++i) {
        const __half2 h = *reinterpret_cast<const __half2*>(&xr[i]);
        const float f0 = __low2float(h), f1 = __high2float(h);
        sx += f0 + f1;
        corr = fmaf(corr_weight<B>(2 * i), f0, corr);
        corr = fmaf(corr_weight<B>(2 * i + 1), f1, corr);
      }
    }
  }
  // Lanes on odd row slots read their unit's two 16-byte halves in the other
  // order (bank-conflict-free unpadded rows); their x registers are swapped to match.
  const int half_first = (UT::kBytes == 32 && p.swap_odd && (row_sub & 1)) ? 1 : 0;
  if (half_first) {
#pragma unroll
    for (int i = 0; i < kXw / 2; ++i) {
      const uint32_t t = xr[i];
      xr[i] = xr[i + kXw / 2];
      xr[i + kXw / 2] = t;
    }
  }
  const int g = (u * UT::kCodes) / kGroup;
  const int win_rows = p.chunks_per_window * Rc;

  // -------------------------------------------------------- main loop ----
  for (int t = 0; t < nchunks; ++t) {
    const int s = t % p.stages;
    if (!mbar_wait(&full[s], (t / p.stages) & 1, &g_gemv_error)) gemv_fail(2u);
    const uint8_t* st = smem + (size_t)s * p.stage_bytes;
    const __half* ssm = reinterpret_cast<const __half*>(st + (size_t)Rc * p.row_stride);
    const __half* zsm = ssm + p.sz_halves;
    const int cr0 = t * Rc, cr = min(Rc, rows - cr0);
    const int aoff = (int)(((size_t)(n0 + cr0) * p.G) & 7);
    // partial-sum rows of this chunk inside the window buffer
    float* pchunk = part + (size_t)((t % p.chunks_per_window) * Rc) * p.U + u;
    if (active) {
      const uint8_t* cbase = st + u * UT::kBytes;
      int r = row_sub;
      // two rows per iteration: independent accumulator chains
      for (; r + p.RS < cr; r += 2 * p.RS) {
        const int r2 = r + p.RS;
        uint32_t w[kWords], w2[kWords];
        load_unit<kWords>(cbase + (size_t)r * p.row_stride, w, half_first);
        load_unit<kWords>(cbase + (size_t)r2 * p.row_stride, w2, half_first);
        const float d = unit_dot<B, kIntPath>(w, xr, corr, xinv);
        const float d2 = unit_dot<B, kIntPath>(w2, xr, corr, xinv);
        const float sc = __half2float(ssm[aoff + r * p.G + g]), zc = __half2float(zsm[aoff + r * p.G + g]);
        const float sc2 = __half2float(ssm[aoff + r2 * p.G + g]), zc2 = __half2float(zsm[aoff + r2 * p.G + g]);
        pchunk[(size_t)r * p.U] = sc * fmaf(-zc, sx, d);
        pchunk[(size_t)r2 * p.U] = sc2 * fmaf(-zc2, sx, d2);
      }
      if (r < cr) {
        uint32_t w[kWords];
        load_unit<kWords>(cbase + (size_t)r * p.row_stride, w, half_first);
        const float d = unit_dot<B, kIntPath>(w, xr, corr, xinv);
        const float sc = __half2float(ssm[aoff + r * p.G + g]), zc = __half2float(zsm[aoff + r * p.G + g]);
        pchunk[(size_t)r * p.U] = sc * fmaf(-zc, sx, d);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    if ((t + 1) % p.chunks_per_window == 0 || t + 1 == nchunks) {
      named_barrier(1, ncons);
      const int wr0 = (t / p.chunks_per_window) * win_rows;
      const int wrows = min(win_rows, rows - wr0);
      for (int rr = tid; rr < wrows; rr += ncons) {
        const float* pr = part + (size_t)rr * p.U;
        float acc = 0.f;
        for (int uu = 0; uu < p.U; ++uu) acc += pr[uu];
        a.y[n0 + wr0 + rr] = __float2half_rn(acc);
      }
      named_barrier(1, ncons);
    }
  }
}

// ------------------------------------------------------------- host plan --

int unit_bytes(int b) { return (b == 3 || b == 6) ? 48 : 32; }
int unit_codes(int b) { return b == 3 ? 128 : (b == 8 ? 32 : 64); }

// Worst bank-conflict degree of one 16-byte shared load by a warp whose lane l
// reads row (l / UW) at unit (l % UW) (two-piece units on odd rows swapped if asked).
int conflict_degree(int UW, int RS, int ub, int stride, int swap_odd) {
  int worst = 1;
  for (int piece = 0; piece < ub / 16; ++piece)
    for (int ph = 0; ph < 4; ++ph) {
      int count[8] = {0};
      for (int l = ph * 8; l < ph * 8 + 8; ++l) {
        const int row = l / UW;
        if (row >= RS) continue;
        const int pc = (ub == 32 && swap_odd && (row & 1)) ? (piece ^ 1) : piece;
        const long addr = (long)row * stride + (long)(l % UW) * ub + 16 * pc;
        worst = std::max(worst, ++count[(addr / 16) % 8]);
      }
    }
  return worst;
}

int gemv1_ctas_per_sm(int b) { return b == 3 ? 1 : 2; }  // int3 lanes hold 64 registers of x

bool make_plan(int b, int N, int K, Plan& p) {
  const int c = unit_codes(b), ub = unit_bytes(b);
  const int max_warps = gemv1_ctas_per_sm(b) == 1 ? kMaxConsumerWarps : kMaxConsumerWarps2;
  p.U = K / c;
  if (p.U < 1 || p.U > max_warps * 32) return false;
  // Units per warp: most busy lanes, then most warps.
  double best = -1.0;
  for (int UW = (p.U + max_warps - 1) / max_warps; UW <= 32 && UW <= p.U; ++UW) {
    const int RS = 32 / UW, NW = (p.U + UW - 1) / UW;
    const double eff = (double)RS * p.U / (NW * 32.0) + 1e-3 * NW;
    if (eff > best) {
      best = eff;
      p.UW = UW;
      p.RS = RS;
      p.NW = NW;
    }
  }
  p.row_bytes = K * b / 8;
  p.row_stride = p.row_bytes;
  p.swap_odd = (ub == 32 && conflict_degree(p.UW, p.RS, ub, p.row_stride, 1) <
                                conflict_degree(p.UW, p.RS, ub, p.row_stride, 0)) ? 1 : 0;
  p.G = K / kGroup;
  p.ctas_per_sm = gemv1_ctas_per_sm(b);
  const int smem_limit = p.ctas_per_sm == 1 ? kSmemLimit : kSmemLimit2;
  p.grid = std::min(kSms * p.ctas_per_sm, N);
  p.rows_per_cta = (N + p.grid - 1) / p.grid;
  p.grid = (N + p.rows_per_cta - 1) / p.rows_per_cta;
  const int k = std::max(1, kChunkTarget / (p.RS * p.row_stride));
  p.rows_per_chunk = std::min(p.RS * k, ((p.rows_per_cta + p.RS - 1) / p.RS) * p.RS);
  const int nchunks = (p.rows_per_cta + p.rows_per_chunk - 1) / p.rows_per_chunk;
  p.sz_halves = ((p.rows_per_chunk * p.G + 8) + 7) & ~7;
  p.stage_bytes = (p.rows_per_chunk * p.row_stride + 4 * p.sz_halves + 127) & ~127;
  const int max_win_chunks = std::max(1, kPartialBudget / p.ctas_per_sm / (p.rows_per_chunk * p.U * 4));
  p.chunks_per_window = std::min(max_win_chunks, nchunks);
  const int part_bytes = (p.chunks_per_window * p.rows_per_chunk * p.U * 4 + 127) & ~127;
  const int x_bytes = (K * 2 + 127) & ~127;
  const int fixed = x_bytes + part_bytes + 2 * kMaxStages * 8;
  const int room = (smem_limit - fixed) / p.stage_bytes;
  p.stages = std::min(std::min(room, kMaxStages), nchunks);
  if (p.stages < 1) return false;
  p.off_x = p.stages * p.stage_bytes;
  p.off_part = p.off_x + x_bytes;
  p.off_bar = p.off_part + part_bytes;
  p.smem_bytes = p.off_bar + 2 * kMaxStages * 8;
  return p.smem_bytes <= smem_limit;
}

template <int B>
qlin_status launch_gemv1(const Args& a, cudaStream_t s) {
  static unsigned long long configured = 0;  // one bit per device (the attribute is per device)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda(e);
  if (dev >= 64 || !((configured >> dev) & 1ull)) {
    e = cudaFuncSetAttribute(gemv1_kernel<B>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             gemv1_ctas_per_sm(B) == 1 ? kSmemLimit : kSmemLimit2);
    if (e != cudaSuccess) return record_cuda(e);
    if (dev < 64) configured |= 1ull << dev;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.p.grid);
  cfg.blockDim = dim3((a.p.NW + 1) * 32);
  cfg.dynamicSmemBytes = a.p.smem_bytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = overlap_enabled() ? 1 : 0;
  return record_cuda(cudaLaunchKernelEx(&cfg, gemv1_kernel<B>, a));
}

// ----------------------------------------------------- general fallback --

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

}  // namespace

static bool gemv_fused_path(int bits, int N, int K, int M) {
  Plan p;
  return M == 1 && bits != 0 && make_plan(bits, N, K, p);
}

size_t gemv_workspace_bytes(int bits, int N, int K, int M) {
  // The fused M = 1 kernel rotates x in its prologue and needs no workspace;
  // the other cases rotate x into the workspace first.
  if (gemv_fused_path(bits, N, K, M)) return 0;
  return ((size_t)M * K * 2 + 255) & ~(size_t)255;
}

qlin_status launch_gemv(const PackedView& v, const __half* scales, const __half* zeros,
                        const uint32_t* sign_bits, const __half* x, __half* y, int M,
                        void* workspace, cudaStream_t s) {
  if (gemv_fused_path(v.bits, v.N, v.K, M)) {
    Args a;
    if (make_plan(v.bits, v.N, v.K, a.p)) {
      a.codes = v.codes;
      a.scales = scales;
      a.zeros = zeros;
      a.sign_bits = sign_bits;
      a.x = x;
      a.y = y;
      a.N = v.N;
      a.K = v.K;
      switch (v.bits) {
        case 3: return launch_gemv1<3>(a, s);
        case 4: return launch_gemv1<4>(a, s);
        case 6: return launch_gemv1<6>(a, s);
        default: return launch_gemv1<8>(a, s);
      }
    }
  }
  __half* xr = static_cast<__half*>(workspace);
  qlin_status r = launch_rht(x, xr, sign_bits, M, v.K, s);
  if (r != QLIN_OK) return r;
  const int threads = 256;
  int blocks = (v.N * 32 + threads - 1) / threads;
  if (blocks > 148 * 8) blocks = 148 * 8;
  gemv_simple_kernel<<<blocks, threads, 0, s>>>(v, scales, zeros, xr, y, M);
  return record_cuda(cudaGetLastError());
}

unsigned take_gemv_error() {
  unsigned v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_gemv_error, sizeof(v)) != cudaSuccess) return ~0u;
  if (v) cudaMemcpyToSymbol(g_gemv_error, &zero, sizeof(zero));
  return v;
}

}  // namespace qlin

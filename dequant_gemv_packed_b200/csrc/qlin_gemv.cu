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
//     streams the rows (one bulk asynchronous copy per chunk of rows, laid out
//     in shared memory exactly as in global memory) and the group scales/zeros
//     of each chunk into a ring of shared-memory stages; when the CTA's whole
//     share fits (the common decode shapes), every chunk has its own stage and
//     all copies are in flight before the first x value is read.
//   * The consumer warps rotate x (sign flip, 7 butterfly stages in registers
//     and shuffles, x 1/sqrt(128), fp16 rounding) and, in the same pass, put
//     each "unit" of K (64 codes; 32 for int8) into the form its decoder
//     reads, with the unit's scalars (below).
//   * Each consumer lane then owns one fixed unit, keeps that unit's x in
//     registers for the whole kernel, and walks down the rows of each chunk;
//     the UW lanes that share a row (UW a power of two) add their per-unit
//     results with shuffles, and rows are summed over warps in a fixed order
//     (deterministic results).
//   * 4- and 8-bit codes: x becomes 16-bit integers with one power-of-two scale
//     per unit (exact for values within 2^4 of the unit's largest magnitude,
//     else rounded at 2^-14 of it) and sum_k q_k x_k is taken exactly in int32
//     with dp2a (two 16x8-bit products per instruction); nibbles are spread to
//     byte lanes with one mask each.
//   * 3- and 6-bit codes are turned into fp16 without conversions: masking a
//     code into the mantissa of the fp16 constant 1024 (0x6400) gives exactly
//     1024 + c*q, where c is a power of two fixed by the code's bit position;
//     one lop3 produces two such values.  They are multiplied with x in fp16 x
//     fp16 -> fp32 fused multiply-adds, one accumulator per position scale c,
//     and the constant part 1024*sum(x/c) is removed with the unit's
//     correction.
//   * With qlin_set_overlap(1) the kernel is launched as a programmatic
//     dependent: it lets the next kernel start launching at once, streams its
//     weight before waiting on the previous kernel, and waits only before it
//     reads x; two CTAs fit on an SM, so the next call's weight stream runs
//     under this call's arithmetic.
// Other cases (M > 1, mixed widths, very long K): gemv_mma_kernel below.
#include <algorithm>
#include <atomic>

#include "qlin_internal.cuh"
#include "qlin_rot16.cuh"
#include "qlin_sm100.cuh"

namespace qlin {

__device__ unsigned int g_gemv_error;  // nonzero: a bounded wait gave up

namespace {

constexpr uint32_t kMagic = 0x64006400u;  // fp16 1024.0 in both halves
// Two CTAs fit on one SM (registers and shared memory), so that with
// programmatic dependent launch the next call's CTA is resident, and streams
// its weight, while this call's CTA finishes.
constexpr int kMaxConsumerWarps = 10;
constexpr int kMaxThreads = (kMaxConsumerWarps + 1) * 32;
constexpr int kSmemLimit = 113 * 1024;
constexpr int kMinSmem = 80 * 1024;
constexpr int kChunkTarget = 16 * 1024;
constexpr int kInflightBytes = 64 * 1024;
constexpr int kPartialBudget = 24 * 1024;
constexpr int kMaxStages = 16;
constexpr int kSms = 148;

template <int N> struct int_ {};
template <int N> struct rows_ { static constexpr int value = N; };  // rows a lane takes in one pass

// A unit is the run of codes one lane multiplies with its x registers.
template <int B> struct UnitT;
template <> struct UnitT<3> { static constexpr int kBytes = 24, kCodes = 64; };
template <> struct UnitT<4> { static constexpr int kBytes = 32, kCodes = 64; };
template <> struct UnitT<6> { static constexpr int kBytes = 48, kCodes = 64; };
template <> struct UnitT<8> { static constexpr int kBytes = 32, kCodes = 32; };

struct Plan {
  int U;               // units per row
  int UW, RS, NW;      // units per warp (a power of two), row slots per warp (32 / UW), consumer warps
  int rows_per_cta, grid;  // rows_per_cta: the most rows one CTA owns
  int row_bytes;       // rows are contiguous in shared memory as in global memory
  int swap_bit;        // 32-byte units: lanes with this lane-index bit set read their halves swapped (-1: none)
  int rows_per_chunk;  // R_c, a multiple of the rows one consumer iteration covers
  int inflight;        // chunks of one CTA in flight at once
  int stages;
  int chunks_per_window;
  int G;               // groups per row
  int sz_halves;       // halves per stage for each of s and z
  int off_sz, off_x, off_unit, off_part, off_bar;
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
  int weights_first;  // dependent launch: stream the weight before waiting for x
  Plan p;
};

// ---------------------------------------------------------------- decoders --

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
// The odd codes are used in place (16 q in the high nibble of each byte), so
// their sums carry a factor 16 that is shifted out at the end (exactly: the sum
// is a multiple of 16).
__device__ __forceinline__ int dot_unit_int(const uint32_t (&w)[8], const uint32_t (&x)[32], int_<4>) {
  int lo0 = 0, lo1 = 0, hi0 = 0, hi1 = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t lo = w[i] & 0x0F0F0F0Fu;  // q0 q2 q4 q6
    const uint32_t hi = w[i] & 0xF0F0F0F0u;  // 16 q1, 16 q3, 16 q5, 16 q7
    int& L = (i & 1) ? lo1 : lo0;
    int& H = (i & 1) ? hi1 : hi0;
    L = dp2a_lo(x[4 * i], lo, L);
    L = dp2a_hi(x[4 * i + 1], lo, L);
    H = dp2a_lo(x[4 * i + 2], hi, H);
    H = dp2a_hi(x[4 * i + 3], hi, H);
  }
  return (lo0 + lo1) + ((hi0 + hi1) >> 4);
}

// int8: word i holds codes 4i..4i+3.  x pairs: (x0,x1) (x2,x3).
__device__ __forceinline__ int dot_unit_int(const uint32_t (&w)[8], const uint32_t (&x)[16], int_<8>) {
  int acc[4] = {0, 0, 0, 0};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int& A = acc[i & 3];
    A = dp2a_lo(x[2 * i], w[i], A);
    A = dp2a_hi(x[2 * i + 1], w[i], A);
  }
  return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

// 48 bits of a unit starting at bit 48*p: A = bits [0, 32), B = bits [32, 48) (+ junk above).
template <int kWords>
__device__ __forceinline__ void piece48(const uint32_t (&w)[kWords], int p, uint32_t& A, uint32_t& B) {
  const int m = p >> 1;
  if ((p & 1) == 0) {
    A = w[3 * m];
    B = w[3 * m + 1];
  } else {
    A = __funnelshift_r(w[3 * m + 1], w[3 * m + 2], 16);
    B = w[3 * m + 2] >> 16;
  }
}

// The fp16 decoders (3- and 6-bit codes) return sum_k (1024/c_k + q_k) * x_k
// over the unit, where c_k is the position scale of code k; the caller
// subtracts corr = sum_k 1024/c_k * x_k.
__device__ __forceinline__ float dot_unit(const uint32_t (&w)[12], const uint32_t (&x)[32], int_<6>) {
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
    A1 = fma_f16_f32(lo16(T0), lo16(x01), A1);
    A4 = fma_f16_f32(hi16(T0), hi16(x23), A4);
    A1 = fma_f16_f32(lo16(T1), hi16(x01), A1);
    A4 = fma_f16_f32(hi16(T1), lo16(x45), A4);
    A1 = fma_f16_f32(lo16(T2), lo16(x23), A1);
    A4 = fma_f16_f32(hi16(T2), hi16(x45), A4);
    A1 = fma_f16_f32(lo16(T3), lo16(x67), A1);
    A4 = fma_f16_f32(hi16(T3), hi16(x67), A4);
  }
  return (a1a + a1b) + 0.25f * (a4a + a4b);
}

// int3: a 64-code unit is four 48-bit pieces of 16 codes.
__device__ __forceinline__ float dot_unit(const uint32_t (&w)[6], const uint32_t (&x)[32], int_<3>) {
  float a1 = 0.f, a2 = 0.f, a8 = 0.f, a16 = 0.f, a64 = 0.f, a128 = 0.f;
#pragma unroll
  for (int p = 0; p < 4; ++p) {
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
    const uint32_t* xp = x + 8 * p;  // xp[i] = (x_{2i}, x_{2i+1}) of this piece
    a2 = fma_f16_f32(lo16(T0), lo16(xp[0]), a2);
    a1 = fma_f16_f32(hi16(T0), hi16(xp[2]), a1);
    a16 = fma_f16_f32(lo16(T1), hi16(xp[0]), a16);
    a8 = fma_f16_f32(hi16(T1), lo16(xp[3]), a8);
    a128 = fma_f16_f32(lo16(T2), lo16(xp[1]), a128);
    a64 = fma_f16_f32(hi16(T2), hi16(xp[3]), a64);
    a2 = fma_f16_f32(lo16(T3), lo16(xp[4]), a2);
    a1 = fma_f16_f32(hi16(T3), hi16(xp[6]), a1);
    a16 = fma_f16_f32(lo16(T4), hi16(xp[4]), a16);
    a8 = fma_f16_f32(hi16(T4), lo16(xp[7]), a8);
    a128 = fma_f16_f32(lo16(T5), lo16(xp[5]), a128);
    a64 = fma_f16_f32(hi16(T5), hi16(xp[7]), a64);
    a1 = fma_f16_f32(lo16(T6), hi16(xp[1]), a1);
    a1 = fma_f16_f32(hi16(T6), hi16(xp[5]), a1);
    a8 = fma_f16_f32(lo16(T7), lo16(xp[2]), a8);
    a8 = fma_f16_f32(hi16(T7), lo16(xp[6]), a8);
  }
  return a1 + 0.5f * a2 + 0.125f * a8 + 0.0625f * a16 + 0.015625f * a64 + 0.0078125f * a128;
}

// 1024 / c for code position i of a unit (see the fp16 decoders above): a
// power of two whose exponent, for i mod 8, is a nibble of a constant (no
// branches: lanes ask for different positions).
template <int B>
__device__ __forceinline__ float corr_weight(int i) {
  // int6: 1024 except 256 at positions 3, 4, 5, 7; int3: 512 64 8 1024 128 1024 128 16
  constexpr uint32_t kExp = B == 6 ? 0x8A888AAAu : 0x47A7A369u;
  const uint32_t e = (kExp >> (4 * (i & 7))) & 0xFu;
  return __uint_as_float((127u + e) << 23);
}

__device__ __forceinline__ void gemv_fail(unsigned code) { atomicOr(&g_gemv_error, code); }

// sum_k q_k x_k over one unit: exact integer dot (scaled back) or the fp16
// mantissa-code path minus its constant part.  `c` is the unit's scale
// 2^(E-13) (integer path) or its correction (fp16 path).
template <int B, bool kInt, int kWords, int kXw>
__device__ __forceinline__ float unit_dot(const uint32_t (&w)[kWords], const uint32_t (&x)[kXw], float c) {
  if constexpr (kInt) {
    return (float)dot_unit_int(w, x, int_<B>()) * c;
  } else {
    return dot_unit(w, x, int_<B>()) - c;
  }
}

// One unit of codes from shared memory (16-byte pieces, or 8-byte pieces for
// 24-byte units); `half_first` swaps the two 16-byte halves of a 32-byte unit.
template <int kWords>
__device__ __forceinline__ void load_unit(const uint8_t* src, uint32_t (&w)[kWords], int half_first) {
  if constexpr (kWords % 4 == 0) {
    const uint4* cp = reinterpret_cast<const uint4*>(src);
#pragma unroll
    for (int i = 0; i < kWords / 4; ++i) {
      const uint4 v = cp[kWords == 8 ? (i ^ half_first) : i];
      w[4 * i] = v.x;
      w[4 * i + 1] = v.y;
      w[4 * i + 2] = v.z;
      w[4 * i + 3] = v.w;
    }
  } else {
    const uint2* cp = reinterpret_cast<const uint2*>(src);
#pragma unroll
    for (int i = 0; i < kWords / 2; ++i) {
      const uint2 v = cp[i];
      w[2 * i] = v.x;
      w[2 * i + 1] = v.y;
    }
  }
}

// Rows per consumer iteration: four for int4; two for int3 and int6 (registers) and
// int8 (long rows: smaller chunks keep more ring stages).
template <int B> struct RowsPerIter { static constexpr int value = B == 4 ? 4 : 2; };

// The UW lanes of a row group hold per-unit partials v[k] of the R rows
// rb + k RS (k < R).  A reduce-scatter butterfly leaves the full sum of row
// k = (lane & (min(R, UW) - 1)) in each lane (log2(R) exchange steps that halve
// the values a lane carries, then a plain butterfly over the remaining lane
// bits); the lanes of the group's first min(R, UW) holding distinct rows store
// them.  Every lane of the warp executes it.
template <int UW, int R>
__device__ __forceinline__ void reduce_store_rows(float (&v)[R], int lane, float* pchunk, int r0, int RS, int cr,
                                                  int NW) {
  if constexpr (UW == 1) {
#pragma unroll
    for (int k = 0; k < R; ++k)
      if (r0 + k * RS < cr) pchunk[(r0 + k * RS) * NW] = v[k];
  } else {
    constexpr int kSplit = UW < R ? UW : R;  // lanes that end up with distinct rows
    float c[R];
#pragma unroll
    for (int k = 0; k < R; ++k) c[k] = v[k];
    int n = R;  // values still carried
#pragma unroll
    for (int o = kSplit / 2; o >= 1; o /= 2) {
      // keep the upper or lower half of the carried values, add the partner's copy
      const bool upper = (lane & o) != 0;
      n /= 2;
#pragma unroll
      for (int k = 0; k < R / 2; ++k) {
        if (k < n) {
          const float keep = upper ? c[k + n] : c[k];
          const float send = upper ? c[k] : c[k + n];
          c[k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
    }
    // c[0 .. n) now hold rows (lane & (kSplit-1)) * n + j; finish over the other lane bits
#pragma unroll
    for (int o = kSplit; o < UW; o *= 2)
#pragma unroll
      for (int k = 0; k < R; ++k)
        if (k < n) c[k] += __shfl_xor_sync(0xffffffffu, c[k], o);
    if ((lane & (UW - 1)) < kSplit) {
      const int kb = (lane & (kSplit - 1)) * n;
#pragma unroll
      for (int j = 0; j < R; ++j)
        if (j < n && r0 + (kb + j) * RS < cr) pchunk[(r0 + (kb + j) * RS) * NW] = c[j];
    }
  }
}

// ------------------------------------------------------------------ kernel --

// Maximum (of non-negative values) and sum over the lanes of this lane's group
// (grp in [0, kGroups)): one warp-wide redux per group.
template <int kGroups>
__device__ __forceinline__ uint32_t group_max(uint32_t m, int grp) {
  uint32_t r = 0;
#pragma unroll
  for (int q = 0; q < kGroups; ++q) {
    const uint32_t mq = __reduce_max_sync(0xffffffffu, grp == q ? m : 0u);
    if (grp == q) r = mq;
  }
  return r;
}
template <int kGroups>
__device__ __forceinline__ int group_add(int v, int grp) {
  int r = 0;
#pragma unroll
  for (int q = 0; q < kGroups; ++q) {
    const int sq = __reduce_add_sync(0xffffffffu, grp == q ? v : 0);
    if (grp == q) r = sq;
  }
  return r;
}

// Position in dp2a order of code c of a 64-code int4 unit (pairs (0,2) (4,6)
// (1,3) (5,7) of each word of 8 codes; see dot_unit_int).
__device__ __forceinline__ int int4_slot(int c) {
  const int j = c & 7;
  return 8 * (c >> 3) + 2 * (((j & 1) << 1) | (j >> 2)) + ((j >> 1) & 1);
}

// Unit u's x occupies kXw words of shared memory as 16-byte pieces; logical
// piece i is stored at piece i ^ (u mod P), P pieces a unit, so that the lanes
// of a load phase, which read the same piece of different units, hit distinct
// banks.  x_half maps a 16-bit position of the unit to its place.
__device__ __forceinline__ int x_half(int p, int u, int P) { return (((p >> 3) ^ (u & (P - 1))) << 3) | (p & 7); }

// Sign flip, block-128 FWHT, x 1/sqrt(128) and fp16 rounding of one block
// (rotate_block16x8: one tensor-core product with H16, butterflies along H8),
// then the unit preparation described at the top of the file.  Lane (g, t)
// ends with elements g + 32t + {0, 16, 8, 24}.
template <int B>
__device__ __forceinline__ void rotate_prepare(uint32_t b0, uint32_t b1, uint32_t sw, int blk, bool store,
                                               const uint32_t (&h)[4], uint32_t* xs, float2* ust, int lane) {
  using UT = UnitT<B>;
  constexpr int kXw = UT::kCodes / 2;
  const int g = lane >> 2, t = lane & 3;
  __half hv[4];
  float f[4];
  rotate_block16x8(b0, b1, sw, h, lane, hv, f);
  constexpr int kOff[4] = {rot_off(0), rot_off(1), rot_off(2), rot_off(3)};  // element of f[i]: g + 32 t + kOff[i]
  // units: 64 codes = elements [0, 64) or [64, 128) of the block (t < 2 or t >= 2);
  // 32 codes (int8) = the 32 elements of one t
  constexpr int kGroups = UT::kCodes == 64 ? 2 : 4;
  const int grp = UT::kCodes == 64 ? (t >> 1) : t;
  const int u = blk * (kHadamard / UT::kCodes) + grp;
  const bool leader = g == 0 && (UT::kCodes == 32 || (t & 1) == 0);
  uint16_t* xu = reinterpret_cast<uint16_t*>(xs + (size_t)u * kXw);
  if constexpr (B == 4 || B == 8) {
    // x_int = rne(x * 2^(13-E)), E the exponent of the unit's largest |x|:
    // |x_int| < 2^14, exact for values within 2^4 of that maximum.
    const uint32_t m = group_max<kGroups>(
        __float_as_uint(fmaxf(fmaxf(fabsf(f[0]), fabsf(f[1])), fmaxf(fabsf(f[2]), fabsf(f[3])))), grp);
    const int E = m ? (int)((m >> 23) & 0xFF) - 127 : 0;
    const float up = __uint_as_float((uint32_t)(127 + 13 - E) << 23);
    const float xinv = __uint_as_float((uint32_t)(127 - 13 + E) << 23);
    int vi[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) vi[i] = __float2int_rn(f[i] * up);
    const int isum = group_add<kGroups>((vi[0] + vi[1]) + (vi[2] + vi[3]), grp);
    if (store) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c = (B == 4) ? g + 32 * (t & 1) + kOff[i] : g + kOff[i];  // position in the unit
        xu[x_half(B == 4 ? int4_slot(c) : c, u, kXw / 4)] = (uint16_t)vi[i];
      }
      if (leader) ust[u] = make_float2(xinv, (float)isum * xinv);
    }
  } else {
    float corr = 0.f, sx = (f[0] + f[1]) + (f[2] + f[3]);
#pragma unroll
    for (int i = 0; i < 4; ++i) corr = fmaf(corr_weight<B>(g + 32 * (t & 1) + kOff[i]), f[i], corr);
#pragma unroll
    for (int o = 1; o <= 16; o <<= 1) {
      if (o == 2) continue;  // lane bit 1 selects the unit
      corr += __shfl_xor_sync(0xffffffffu, corr, o);
      sx += __shfl_xor_sync(0xffffffffu, sx, o);
    }
    if (store) {
      __half* xh = reinterpret_cast<__half*>(xu);
#pragma unroll
      for (int i = 0; i < 4; ++i) xh[x_half(g + 32 * (t & 1) + kOff[i], u, kXw / 4)] = hv[i];
      if (leader) ust[u] = make_float2(corr, sx);
    }
  }
}

template <int B, int UW>
__global__ void __launch_bounds__(kMaxThreads, 2) gemv1_kernel(const __grid_constant__ Args a) {
  using UT = UnitT<B>;
  constexpr int R = RowsPerIter<B>::value;
  constexpr int kWords = UT::kBytes / 4;
  constexpr int kXw = UT::kCodes / 2;  // 32-bit registers of x per lane
  constexpr bool kIntPath = (B == 4 || B == 8);
  extern __shared__ __align__(128) uint8_t smem[];
  const Plan& p = a.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ncons = p.NW * 32;
  // CTA i owns rows [i N / grid, (i + 1) N / grid): every SM gets work.
  const int n0 = (int)(((long long)blockIdx.x * a.N) / gridDim.x);
  const int rows = (int)(((long long)(blockIdx.x + 1) * a.N) / gridDim.x) - n0;
  if (rows <= 0) return;
  const int Rc = p.rows_per_chunk;
  const int nchunks = (rows + Rc - 1) / Rc;
  const size_t stage_bytes = (size_t)Rc * p.row_bytes;
  uint8_t* codes_ring = smem;  // stage s holds rows [0, Rc) of its chunk at s * Rc * row_bytes
  __half* s_ring = reinterpret_cast<__half*>(smem + p.off_sz);
  __half* z_ring = s_ring + p.stages * p.sz_halves;
  uint32_t* xs = reinterpret_cast<uint32_t*>(smem + p.off_x);
  float2* ust = reinterpret_cast<float2*>(smem + p.off_unit);
  float* part = reinterpret_cast<float*>(smem + p.off_part);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  uint64_t* empty = full + kMaxStages;
  uint64_t* x_issued = empty + kMaxStages;

  if (tid == ncons) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], p.NW);
    }
    mbar_init(x_issued, p.NW);
    mbar_fence_init();
  }
  __syncthreads();
  // Programmatic dependent launch: the next kernel on the stream may start
  // launching now; this kernel's weight stream does not depend on the
  // previous kernel, x and y do (grid_dependency_wait below).
  if (tid == 0) grid_launch_dependents();

  if (warp == p.NW) {
    // ------------------------------------------------------- producer ----
    if (lane != 0) return;
    // Stand-alone launches let the x loads go first (the weight stream would
    // otherwise queue ahead of them); dependent launches stream at once.
    if (!a.weights_first && !mbar_wait(x_issued, 0, &g_gemv_error)) gemv_fail(4u);
    const size_t total_h = (size_t)a.N * p.G;
    int s = 0, sd = 0;
    uint32_t ph = 0, phd = 0;
    for (int t = 0; t < nchunks; ++t) {
      if (t >= p.stages && !mbar_wait(&empty[s], ph ^ 1u, &g_gemv_error)) gemv_fail(1u);
      // Pace the stream: at most p.inflight chunks of this CTA in flight, so
      // that the first chunks land early instead of all together.
      if (t >= p.inflight) {
        if (!mbar_wait(&full[sd], phd, &g_gemv_error)) gemv_fail(8u);
        if (++sd == p.stages) {
          sd = 0;
          phd ^= 1u;
        }
      }
      uint8_t* dst = codes_ring + (size_t)s * stage_bytes;
      __half* ssm = s_ring + (size_t)s * p.sz_halves;
      __half* zsm = z_ring + (size_t)s * p.sz_halves;
      const int cr0 = t * Rc, cr = min(Rc, rows - cr0);
      const size_t h0 = (size_t)(n0 + cr0) * p.G, h1 = h0 + (size_t)cr * p.G;
      const size_t al = h0 & ~(size_t)7;
      size_t bh = (h1 + 7) & ~(size_t)7;  // whole 16-byte pieces, reading a little past the chunk
      if (bh > total_h) {                 // ... except at the end of the arrays: plain copies
        bh = h1 & ~(size_t)7;
        for (size_t h = (bh > h0 ? bh : h0); h < h1; ++h) {
          ssm[h - al] = a.scales[h];
          zsm[h - al] = a.zeros[h];
        }
      }
      const uint32_t szb = bh > al ? (uint32_t)(bh - al) * 2u : 0u;
      mbar_arrive_expect_tx(&full[s], (uint32_t)cr * p.row_bytes + 2u * szb);
      bulk_g2s(dst, a.codes + (size_t)(n0 + cr0) * p.row_bytes, (uint32_t)cr * p.row_bytes, &full[s]);
      if (szb) {
        bulk_g2s(ssm, a.scales + al, szb, &full[s]);
        bulk_g2s(zsm, a.zeros + al, szb, &full[s]);
      }
      if (++s == p.stages) {
        s = 0;
        ph ^= 1u;
      }
    }
    return;
  }

  // --------------------------------------------------------- prologue ----
  // Rotate x and prepare each unit in shared memory in the form the decoders
  // read (rotate_prepare): warp per block of 128, two blocks per pass.  All of
  // a warp's x loads are issued before any is used (one memory latency).
  grid_dependency_wait();
  const int nblk = a.K / kHadamard;
  constexpr int kBatch = 8;
  if (warp >= nblk && lane == 0) mbar_arrive(x_issued);  // a warp with no block has nothing to load
  {
    const int g = lane >> 2, t = lane & 3;
    const uint32_t h[4] = {h16_pair(g, 2 * t), h16_pair(g + 8, 2 * t), h16_pair(g, 2 * t + 8),
                           h16_pair(g + 8, 2 * t + 8)};
    const int xo = 16 * g + 2 * t;                 // x offset of this lane's b0 (b1: + 8)
    const int so = (g >> 1), sb = 16 * (g & 1) + 2 * t;  // its sign word and bit
    for (int blk0 = warp; blk0 < nblk; blk0 += kBatch * p.NW) {
      uint32_t xb0[kBatch], xb1[kBatch], sw[kBatch];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int blk = min(blk0 + j * p.NW, nblk - 1);
        const __half* xp = a.x + blk * kHadamard + xo;
        xb0[j] = *reinterpret_cast<const uint32_t*>(xp);
        xb1[j] = *reinterpret_cast<const uint32_t*>(xp + 8);
        sw[j] = a.sign_bits[blk * 4 + so] >> sb;
      }
      if (blk0 == warp) {
        __syncwarp();
        if (lane == 0) mbar_arrive(x_issued);
      }
#pragma unroll
      for (int j = 0; j < kBatch; j += 2) {
        const int b0 = blk0 + j * p.NW, b1 = b0 + p.NW;
        if (b0 >= nblk) break;  // warp-uniform
        rotate_prepare<B>(xb0[j], xb1[j], sw[j], b0, true, h, xs, ust, lane);
        rotate_prepare<B>(xb0[j + 1], xb1[j + 1], sw[j + 1], min(b1, nblk - 1), b1 < nblk, h, xs, ust, lane);
      }
    }
  }
  named_barrier(1, ncons);

  // Fixed unit of this lane: x slice in registers, unit scalars.
  const int u = warp * UW + (lane & (UW - 1));
  const int row_sub = lane / UW;
  const bool unit_ok = u < p.U;
  const int uc = unit_ok ? u : p.U - 1;  // lanes past the last unit read a valid unit, contribute 0
  const int half_first = (UT::kBytes == 32 && p.swap_bit >= 0) ? ((lane >> p.swap_bit) & 1) : 0;
  uint32_t xr[kXw];
  {
    const uint4* xp = reinterpret_cast<const uint4*>(xs + (size_t)uc * kXw);
#pragma unroll
    for (int i = 0; i < kXw / 4; ++i) {
      const uint4 v = xp[(i ^ (half_first * (kXw / 8))) ^ (uc & (kXw / 4 - 1))];
      xr[4 * i] = v.x;
      xr[4 * i + 1] = v.y;
      xr[4 * i + 2] = v.z;
      xr[4 * i + 3] = v.w;
    }
  }
  const float2 us = ust[uc];
  const float uscale = us.x, sx = us.y;
  const int g = (uc * UT::kCodes) / kGroup;
  const uint8_t* lane_codes = codes_ring + uc * UT::kBytes;
  const int G = p.G, RS = p.RS, NW = p.NW, row_bytes = p.row_bytes;
  const bool ring = p.stages < nchunks;  // stages are reused: release each one when done

  // -------------------------------------------------------- main loop ----
  int s = 0, wt = 0, wr0 = 0, cr0 = 0;
  uint32_t ph = 0;
  int aoff = (int)(((size_t)n0 * G) & 7);  // offset of the chunk's first scale in its 16-byte-aligned copy
  const int aoff_step = (Rc * G) & 7;
  for (int t = 0; t < nchunks; ++t) {
    if (!mbar_wait_poll(&full[s], ph, &g_gemv_error)) gemv_fail(2u);
    const int cr = min(Rc, rows - cr0);
    const uint8_t* cbase = lane_codes + (size_t)s * stage_bytes;
    const __half* sp = s_ring + (size_t)s * p.sz_halves + aoff + g;
    const __half* zp = z_ring + (size_t)s * p.sz_halves + aoff + g;
    float* pchunk = part + (size_t)(wt * Rc) * NW + warp;
    // One pass: RR rows a lane (independent accumulator chains), RR * RS rows
    // a warp.  Every lane runs every pass (the row sums are warp shuffles);
    // lanes whose row is at or past `cr` read the chunk's last row instead and
    // store nothing.
    const auto pass = [&](int rb, auto rows_tag) {
      constexpr int RR = decltype(rows_tag)::value;
      const int r0 = rb + row_sub;
      uint32_t w[RR][kWords];
      float sc[RR], zc[RR], v[RR];
#pragma unroll
      for (int k = 0; k < RR; ++k) {
        const int rl = min(r0 + k * RS, cr - 1);
        load_unit<kWords>(cbase + rl * row_bytes, w[k], half_first);
        sc[k] = __half2float(sp[rl * G]);
        zc[k] = __half2float(zp[rl * G]);
      }
#pragma unroll
      for (int k = 0; k < RR; ++k) {
        const float d = unit_dot<B, kIntPath>(w[k], xr, uscale);
        v[k] = unit_ok ? sc[k] * fmaf(-zc[k], sx, d) : 0.f;
      }
      reduce_store_rows<UW, RR>(v, lane, pchunk, r0, RS, cr, NW);
    };
    // Full passes while more than (R - 1) RS rows remain; a short remainder
    // (the last rows of a CTA's share) goes RS rows at a time.  8-bit codes
    // keep full passes (measured: the one-row pass made them slower).
    for (int rb = 0; rb < cr;) {
      if constexpr (B != 8) {
        if (cr - rb <= (R - 1) * RS) {
          pass(rb, rows_<1>{});
          rb += RS;
          continue;
        }
      }
      pass(rb, rows_<R>{});
      rb += R * RS;
    }
    if (ring) {
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (++s == p.stages) {
      s = 0;
      ph ^= 1u;
    }
    aoff = (aoff + aoff_step) & 7;
    cr0 += Rc;
    if (++wt == p.chunks_per_window || t + 1 == nchunks) {
      named_barrier(1, ncons);
      const int wrows = min(wt * Rc, rows - wr0);
      for (int rr = tid; rr < wrows; rr += ncons) {
        const float* pr = part + (size_t)rr * NW;
        float acc = 0.f;
        for (int ww = 0; ww < NW; ++ww) acc += pr[ww];
        a.y[n0 + wr0 + rr] = __float2half_rn(acc);
      }
      named_barrier(1, ncons);
      wr0 += wt * Rc;
      wt = 0;
    }
  }
}

// ------------------------------------------------------------- host plan --

int unit_bytes(int b) { return b == 3 ? 24 : (b == 6 ? 48 : 32); }
int unit_codes(int b) { return b == 8 ? 32 : 64; }

// Worst bank-conflict degree of one shared load (16-byte pieces, 8-byte pieces
// for 24-byte units) by a warp whose lane l reads row (l / UW) at unit (l % UW);
// 32-byte units of lanes with bit `swap_bit` set are read second half first.
int conflict_degree(int UW, int ub, int stride, int swap_bit) {
  const int aw = ub % 16 ? 8 : 16, per_phase = 128 / aw, groups = 128 / aw;
  int worst = 1;
  for (int piece = 0; piece < ub / aw; ++piece)
    for (int ph = 0; ph < 32 / per_phase; ++ph) {
      int count[16] = {0};
      for (int l = ph * per_phase; l < (ph + 1) * per_phase; ++l) {
        const int row = l / UW;
        const int pc = (ub == 32 && swap_bit >= 0 && ((l >> swap_bit) & 1)) ? (piece ^ 1) : piece;
        const long addr = (long)row * stride + (long)(l % UW) * ub + (long)aw * pc;
        worst = std::max(worst, ++count[(addr / aw) % groups]);
      }
    }
  return worst;
}

bool make_plan(int b, int N, int K, Plan& p) {
  const int c = unit_codes(b), ub = unit_bytes(b);
  if (K % c) return false;
  p.U = K / c;
  if (p.U < 1 || p.U > kMaxConsumerWarps * 32) return false;
  // Units per warp (a power of two): most busy lanes, then most warps.
  // Row slots beyond the rows a CTA owns would idle.
  const int rows_est = (N + std::min(kSms, N) - 1) / std::min(kSms, N);
  double best = -1.0;
  for (int UW = 1; UW <= 32; UW *= 2) {
    const int RS = 32 / UW, NW = (p.U + UW - 1) / UW;
    if (NW > kMaxConsumerWarps) continue;
    const double eff = (double)std::min(RS, rows_est) * p.U / (NW * 32.0) + 1e-3 * NW;
    if (eff > best) {
      best = eff;
      p.UW = UW;
      p.RS = RS;
      p.NW = NW;
    }
  }
  if (best < 0) return false;
  p.row_bytes = K * b / 8;
  p.swap_bit = -1;
  if (ub == 32) {
    int worst = conflict_degree(p.UW, ub, p.row_bytes, -1);
    for (int bit = 0; bit < 5; ++bit) {
      const int d = conflict_degree(p.UW, ub, p.row_bytes, bit);
      if (d < worst) {
        worst = d;
        p.swap_bit = bit;
      }
    }
  }
  p.G = K / kGroup;
  p.grid = std::min(kSms, N);
  p.rows_per_cta = (N + p.grid - 1) / p.grid;  // the most rows a CTA owns
  const int step = (b == 4 ? 4 : 2) * p.RS;  // rows per consumer iteration (RowsPerIter)
  const int k = std::max(1, (kChunkTarget + step * p.row_bytes / 2) / (step * p.row_bytes));
  p.rows_per_chunk = std::min(step * k, ((p.rows_per_cta + step - 1) / step) * step);
  const int nchunks = (p.rows_per_cta + p.rows_per_chunk - 1) / p.rows_per_chunk;
  p.sz_halves = (p.rows_per_chunk * p.G + 16 + 7) & ~7;
  const int x_bytes = (K * 2 + 127) & ~127;
  const int unit_scalars = (p.U * 8 + 127) & ~127;
  const int sz_stage = 4 * p.sz_halves;
  const auto part_bytes = [&](int cpw) { return (cpw * p.rows_per_chunk * p.NW * 4 + 127) & ~127; };
  const int bars = (2 * kMaxStages + 1) * 8;
  // The whole share in shared memory at once (each chunk its own stage)?
  const int codes_all = (p.rows_per_cta * p.row_bytes + 127) & ~127;
  const int single = codes_all + ((nchunks * sz_stage + 127) & ~127) + x_bytes + unit_scalars +
                     part_bytes(nchunks) + bars;
  if (nchunks <= kMaxStages && single <= kSmemLimit) {
    p.stages = nchunks;
    p.chunks_per_window = nchunks;
    p.off_sz = codes_all;
  } else {
    const int max_win_chunks = std::max(1, kPartialBudget / (p.rows_per_chunk * p.NW * 4));
    p.chunks_per_window = std::min(max_win_chunks, nchunks);
    const int fixed = x_bytes + unit_scalars + part_bytes(p.chunks_per_window) + bars;
    const int stage_cost = p.rows_per_chunk * p.row_bytes + sz_stage;
    p.stages = std::min(std::min((kSmemLimit - fixed - 256) / stage_cost, kMaxStages), nchunks);
    if (p.stages < 1) return false;
    p.off_sz = (p.stages * p.rows_per_chunk * p.row_bytes + 127) & ~127;
  }
  // About 64 KB of one CTA's stream in flight (148 CTAs: ~9.5 MB, enough to cover
  // the memory latency at full bandwidth).
  p.inflight = std::max(1, std::min(p.stages, (kInflightBytes + p.rows_per_chunk * p.row_bytes - 1) /
                                                  (p.rows_per_chunk * p.row_bytes)));
  p.off_x = (p.off_sz + p.stages * sz_stage + 127) & ~127;
  p.off_unit = p.off_x + x_bytes;
  p.off_part = p.off_unit + unit_scalars;
  p.off_bar = p.off_part + part_bytes(p.chunks_per_window);
  // At least kMinSmem per CTA, so that no more than two calls' CTAs share an SM
  // (the one running and the next, prefetching), whatever their shapes.
  p.smem_bytes = std::max(p.off_bar + bars, kMinSmem);
  return p.off_bar + bars <= kSmemLimit;
}

template <int B, int UW>
qlin_status launch_gemv1_uw(const Args& a, cudaStream_t s) {
  // One bit per device (the attributes are per device), atomic: host threads
  // making their first call together may both set the attributes (harmless).
  static std::atomic<unsigned long long> configured{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda(e);
  if (dev >= 64 || !((configured.load(std::memory_order_acquire) >> dev) & 1ull)) {
    e = cudaFuncSetAttribute(gemv1_kernel<B, UW>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
    if (e != cudaSuccess) return record_cuda(e);
    // Every instance asks for the largest shared-memory carveout, so that
    // consecutive calls of different shapes find the SM configured alike and
    // the next call's CTA fits beside the running one.
    e = cudaFuncSetAttribute(gemv1_kernel<B, UW>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return record_cuda(e);
    if (dev < 64) configured.fetch_or(1ull << dev, std::memory_order_release);
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
  return record_cuda(cudaLaunchKernelEx(&cfg, gemv1_kernel<B, UW>, a));
}

template <int B>
qlin_status launch_gemv1(const Args& a, cudaStream_t s) {
  switch (a.p.UW) {
    case 1: return launch_gemv1_uw<B, 1>(a, s);
    case 2: return launch_gemv1_uw<B, 2>(a, s);
    case 4: return launch_gemv1_uw<B, 4>(a, s);
    case 8: return launch_gemv1_uw<B, 8>(a, s);
    case 16: return launch_gemv1_uw<B, 16>(a, s);
    default: return launch_gemv1_uw<B, 32>(a, s);
  }
}

// ------------------------------------------- M up to 16: tensor cores ----
//
// gemv_mma_kernel: rotation of x by the stand-alone kernel into the workspace
// (with each 128-value group's sum), then one warp per share of the (16-row
// tile, 128-code group) items.  Per item the codes become the A operand of
// m16n8k16 products (q exact in fp16: the code in the mantissa of 1024.0, minus
// 1024), the rotated x the B operand (n8 = 8 rows of x per product), fp32
// accumulation; the group's scale and zero then apply to the accumulator,
// y += s (sum q x - z sum x).  Thread (g, t) = (lane / 4, lane % 4) takes codes
// [32t, 32t + 32) of the group for weight rows g and g + 8 (k-step j: codes
// 32t + 4j .. 32t + 4j + 3 in k slots 2t, 2t+1, 2t+8, 2t+9), and the same
// codes' x for x row g: both operands use one permutation of k, so the sum is
// unchanged.  Partial sums of a row tile split between warps go to the
// workspace; the last warp to finish the tile adds them in warp order
// (deterministic) and writes y.

struct MmaArgs {
  PackedView v;
  const __half* scales;
  const __half* zeros;
  const __half* xr;     // [M][K] rotated x
  const float* xsum;    // [M][G] group sums of xr
  __half* y;            // [M][N]
  float* part;          // [W * max_seg][16][16]
  uint32_t* counters;   // [tiles], zero on entry, zero on exit
  int M, G, tiles, max_seg;
  long long T;          // tiles * G items
};

// Code i (0..31) of a 32-code run held in words w (b bits each, little-endian).
template <int B>
__device__ __forceinline__ uint32_t run_code(const uint32_t (&w)[B], int i) {
  const int bit = B * i;
  const int wi = bit >> 5, sh = bit & 31;
  uint32_t v = w[wi] >> sh;
  if (sh + B > 32) v |= w[wi + 1 < B ? wi + 1 : wi] << (32 - sh);
  return v & ((1u << B) - 1u);
}

// (q_i, q_{i+1}) as two exact fp16 values.
template <int B>
__device__ __forceinline__ uint32_t code_pair(const uint32_t (&w)[B], int i) {
  const uint32_t h = (run_code<B>(w, i) | (run_code<B>(w, i + 1) << 16)) | kMagic;
  const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&h), __halves2half2(__ushort_as_half(0x6400), __ushort_as_half(0x6400)));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// The 32-code run [32t, 32t + 32) of group g of a row: 4b bytes.
template <int B>
__device__ __forceinline__ void load_run(const uint32_t* row, int g, int t, uint32_t (&w)[B]) {
  const uint32_t* p = row + (size_t)g * 4 * B + t * B;  // 16b bytes per group, 4b per run
  if constexpr (B == 4) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if constexpr (B == 8) {
    const uint4 v0 = __ldg(reinterpret_cast<const uint4*>(p)), v1 = __ldg(reinterpret_cast<const uint4*>(p) + 1);
    w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w; w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
  } else if constexpr (B == 6) {
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(p) + i);
      w[2 * i] = v.x; w[2 * i + 1] = v.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < B; ++i) w[i] = __ldg(p + i);
  }
}

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
               "{%0,%1,%2,%3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// sum_k q x over one group for rows ra, rb of width B and x rows 8 nt + g:
// d[nt][0..3] = (ra, 2t), (ra, 2t+1), (rb, 2t), (rb, 2t+1) of column tile nt.
template <int B, int NT>
__device__ __forceinline__ void group_products(const uint32_t (&wa)[B], const uint32_t (&wb)[B],
                                               const uint2* const (&xp)[NT], float (&d)[NT][4]) {
  // all of the group's x fragments first (x of codes 32t + 4j .. 32t + 4j + 3), so
  // that their loads overlap one another and the decoding
  uint2 xv[NT][8];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int j = 0; j < 8; ++j) xv[nt][j] = __ldg(xp[nt] + j);
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) d[nt][i] = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t a0 = code_pair<B>(wa, 4 * j), a2 = code_pair<B>(wa, 4 * j + 2);
    const uint32_t a1 = code_pair<B>(wb, 4 * j), a3 = code_pair<B>(wb, 4 * j + 2);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) mma16816(d[nt], a0, a1, a2, a3, xv[nt][j].x, xv[nt][j].y);
  }
}

template <int B, int NT>
__global__ void __launch_bounds__(256) gemv_mma_kernel(const __grid_constant__ MmaArgs a) {
  const int lane = threadIdx.x & 31;
  const int gq = lane >> 2, t = lane & 3;
  const long long W = (long long)gridDim.x * (blockDim.x >> 5);
  const long long w = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const long long i0 = a.T * w / W, i1 = a.T * (w + 1) / W;
  if (i0 >= i1) return;
  const int N = a.v.N, K = a.v.K, G = a.G, M = a.M;
  const int rt_first = (int)(i0 / G);
  // x rows of this lane's B fragments (zero beyond M)
  const int xm[2] = {gq, 8 + gq};
  float acc[NT][4];
  int cur = -1;
  auto flush = [&](int rt) {
    // this warp's partial of row tile rt: rows 16 rt + {gq, gq + 8}, x rows 8 nt + {2t, 2t + 1}
    const int seg = rt - rt_first;
    float* slot = a.part + ((size_t)w * a.max_seg + seg) * 256;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      slot[gq * 16 + 8 * nt + 2 * t] = acc[nt][0];
      slot[gq * 16 + 8 * nt + 2 * t + 1] = acc[nt][1];
      slot[(gq + 8) * 16 + 8 * nt + 2 * t] = acc[nt][2];
      slot[(gq + 8) * 16 + 8 * nt + 2 * t + 1] = acc[nt][3];
    }
    __threadfence();
    __syncwarp();
    // warps covering tile rt: the ones holding its first and last items
    const long long f = (long long)rt * G, l = f + G - 1;
    // warp of item i: the largest w' with floor(T w' / W) <= i, i.e. T w' < (i + 1) W
    auto warp_of = [&](long long i) { return ((i + 1) * W - 1) / a.T; };
    const long long w_first = warp_of(f), w_last = warp_of(l);
    unsigned prev = 0;
    if (lane == 0) prev = atomicAdd(a.counters + rt, 1u);
    prev = __shfl_sync(0xffffffffu, prev, 0);
    if (prev != (unsigned)(w_last - w_first)) return;  // not the last contributor
    __threadfence();
    // sum the contributors' partials in warp order and write y
    float sum[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) sum[e] = 0.f;
    for (long long ww = w_first; ww <= w_last; ++ww) {
      const int sg = rt - (int)(a.T * ww / W / G);
      const float* sl = a.part + ((size_t)ww * a.max_seg + sg) * 256;
#pragma unroll
      for (int e = 0; e < 8; ++e) sum[e] += __ldcg(sl + lane * 8 + e);
    }
    // element lane * 8 + e of the 16 x 16 tile: weight row r = (lane*8+e) / 16, x row m = (lane*8+e) % 16
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int idx = lane * 8 + e, r = 16 * rt + idx / 16, m = idx % 16;
      if (r < N && m < M) a.y[(size_t)m * N + r] = __float2half_rn(sum[e]);
    }
    if (lane == 0) a.counters[rt] = 0u;  // ready for the next call
  };
  // The next item's code runs, scales and zeros are loaded while the current
  // item is multiplied (one item of prefetch).
  constexpr int kW = B ? B : 8;  // words of a 32-code run (mixed widths: up to 8)
  uint32_t nwa[kW], nwb[kW];
  int nb = B;
  float nsa = 0.f, nza = 0.f, nsb = 0.f, nzb = 0.f;
  auto fetch = [&](long long i) {
    const int rt = (int)(i / G), grp = (int)(i % G);
    const int ra = min(16 * rt + gq, N - 1), rb = min(16 * rt + gq + 8, N - 1);
    const uint32_t* row_a = row_of(a.v, ra, nb);
    const uint32_t* row_b = row_of(a.v, rb, nb);  // same 64-row block: same width
    if constexpr (B != 0) {
      load_run<B>(row_a, grp, t, nwa);
      load_run<B>(row_b, grp, t, nwb);
    } else {
      switch (nb) {
        case 3:
          load_run<3>(row_a, grp, t, reinterpret_cast<uint32_t(&)[3]>(nwa));
          load_run<3>(row_b, grp, t, reinterpret_cast<uint32_t(&)[3]>(nwb));
          break;
        case 4:
          load_run<4>(row_a, grp, t, reinterpret_cast<uint32_t(&)[4]>(nwa));
          load_run<4>(row_b, grp, t, reinterpret_cast<uint32_t(&)[4]>(nwb));
          break;
        case 6:
          load_run<6>(row_a, grp, t, reinterpret_cast<uint32_t(&)[6]>(nwa));
          load_run<6>(row_b, grp, t, reinterpret_cast<uint32_t(&)[6]>(nwb));
          break;
        default:
          load_run<8>(row_a, grp, t, nwa);
          load_run<8>(row_b, grp, t, nwb);
          break;
      }
    }
    nsa = __half2float(a.scales[(size_t)ra * G + grp]);
    nza = __half2float(a.zeros[(size_t)ra * G + grp]);
    nsb = __half2float(a.scales[(size_t)rb * G + grp]);
    nzb = __half2float(a.zeros[(size_t)rb * G + grp]);
  };
  fetch(i0);
  int rt = (int)(i0 / G), grp = (int)(i0 % G);  // item i = rt * G + grp, advanced incrementally
  for (long long i = i0; i < i1; ++i) {
    if (rt != cur) {
      if (cur >= 0) flush(cur);
      cur = rt;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
    }
    uint32_t wa[kW], wb[kW];
#pragma unroll
    for (int e = 0; e < kW; ++e) {
      wa[e] = nwa[e];
      wb[e] = nwb[e];
    }
    const int bw = nb;
    const float sa = nsa, za = nza, sb = nsb, zb = nzb;
    if (i + 1 < i1) fetch(i + 1);
    const uint2* xp[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int m = min(xm[nt], M - 1);
      xp[nt] = reinterpret_cast<const uint2*>(a.xr + (size_t)m * K + (size_t)grp * kGroup + 32 * t);
    }
    float d[NT][4];
    if constexpr (B != 0) {
      group_products<B, NT>(wa, wb, xp, d);
    } else {
      switch (bw) {
        case 3:
          group_products<3, NT>(reinterpret_cast<uint32_t(&)[3]>(wa), reinterpret_cast<uint32_t(&)[3]>(wb), xp, d);
          break;
        case 4:
          group_products<4, NT>(reinterpret_cast<uint32_t(&)[4]>(wa), reinterpret_cast<uint32_t(&)[4]>(wb), xp, d);
          break;
        case 6:
          group_products<6, NT>(reinterpret_cast<uint32_t(&)[6]>(wa), reinterpret_cast<uint32_t(&)[6]>(wb), xp, d);
          break;
        default:
          group_products<8, NT>(wa, wb, xp, d);
          break;
      }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int m0 = 8 * nt + 2 * t;
      const float x0 = m0 < M ? a.xsum[(size_t)m0 * G + grp] : 0.f;
      const float x1 = m0 + 1 < M ? a.xsum[(size_t)(m0 + 1) * G + grp] : 0.f;
      acc[nt][0] += sa * fmaf(-za, x0, d[nt][0]);
      acc[nt][1] += sa * fmaf(-za, x1, d[nt][1]);
      acc[nt][2] += sb * fmaf(-zb, x0, d[nt][2]);
      acc[nt][3] += sb * fmaf(-zb, x1, d[nt][3]);
    }
    if (++grp == G) {
      grp = 0;
      ++rt;
    }
  }
  flush(cur);
}

template <int B>
void launch_mma(const MmaArgs& a, int grid, int threads, int M, cudaStream_t s) {
  if (M <= 8)
    gemv_mma_kernel<B, 1><<<grid, threads, 0, s>>>(a);
  else
    gemv_mma_kernel<B, 2><<<grid, threads, 0, s>>>(a);
}

void gemv_mma_mixed(const MmaArgs& a, int grid, int threads, int M, cudaStream_t s) {
  launch_mma<0>(a, grid, threads, M, s);
}

}  // namespace

static bool gemv_fused_path(int bits, int N, int K, int M) {
  Plan p;
  return M == 1 && bits != 0 && (gemv_imma_fits(bits, N, K, M) || make_plan(bits, N, K, p));
}

// M = 2..16 with one code width: the split-K tensor-core kernel (qlin_gemv_tc.cu).
static bool gemv_tc_path(int bits, int N, int K, int M) {
  return bits != 0 && M >= 2 && gemv_tc_fits(bits, N, K, M);
}

// Workspace of the tensor-core path: rotated x, its group sums, the row-tile
// counters and the warps' partial sums.
struct MmaWorkspace {
  size_t xsum_off, cnt_off, part_off, total;
  int tiles, warps, max_seg, grid, warps_per_block;
  MmaWorkspace(int N, int K, int M) {
    const int G = K / kGroup;
    tiles = (N + 15) / 16;
    const long long T = (long long)tiles * G;
    // no more warps than items: every warp then owns at least one item (and
    // reports to each row tile it touches)
    warps_per_block = (int)std::min<long long>(8, T);
    grid = (int)std::max<long long>(1, std::min<long long>(kSms, T / warps_per_block));
    warps = grid * warps_per_block;
    const long long per = (T + warps - 1) / warps;
    max_seg = (int)((per + G - 1) / G) + 1;
    xsum_off = ((size_t)M * K * 2 + 255) & ~(size_t)255;
    cnt_off = xsum_off + (((size_t)M * G * 4 + 255) & ~(size_t)255);
    part_off = cnt_off + (((size_t)tiles * 4 + 255) & ~(size_t)255);
    total = part_off + (size_t)warps * max_seg * 256 * 4;
  }
};

size_t gemv_workspace_bytes(int bits, int N, int K, int M) {
  // The fused M = 1 kernel rotates x in its prologue and needs no workspace.
  if (gemv_fused_path(bits, N, K, M)) return 0;
  if (gemv_tc_path(bits, N, K, M)) return gemv_tc_workspace_bytes(bits, N, K, M);
  return MmaWorkspace(N, K, M).total;
}

qlin_status launch_gemv(const PackedView& v, const __half* scales, const __half* zeros,
                        const uint32_t* sign_bits, const __half* x, __half* y, int M,
                        void* workspace, cudaStream_t s) {
  if (gemv_imma_fits(v.bits, v.N, v.K, M)) return launch_gemv_imma(v, scales, zeros, sign_bits, x, y, s);
  if (gemv_tc_path(v.bits, v.N, v.K, M)) return launch_gemv_tc(v, scales, zeros, sign_bits, x, y, M, workspace, s);
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
      a.weights_first = overlap_enabled() ? 1 : 0;
      switch (v.bits) {
        case 3: return launch_gemv1<3>(a, s);
        case 4: return launch_gemv1<4>(a, s);
        case 6: return launch_gemv1<6>(a, s);
        default: return launch_gemv1<8>(a, s);
      }
    }
  }
  const MmaWorkspace ws(v.N, v.K, M);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  MmaArgs a;
  a.v = v;
  a.scales = scales;
  a.zeros = zeros;
  a.xr = reinterpret_cast<const __half*>(base);
  a.xsum = reinterpret_cast<const float*>(base + ws.xsum_off);
  a.y = y;
  a.counters = reinterpret_cast<uint32_t*>(base + ws.cnt_off);
  a.part = reinterpret_cast<float*>(base + ws.part_off);
  a.M = M;
  a.G = v.K / kGroup;
  a.tiles = ws.tiles;
  a.max_seg = ws.max_seg;
  a.T = (long long)ws.tiles * a.G;
  qlin_status r = launch_rht(x, reinterpret_cast<__half*>(base), sign_bits, M, v.K, s, a.counters, ws.tiles,
                             reinterpret_cast<float*>(base + ws.xsum_off));
  if (r != QLIN_OK) return r;
  if (v.bits == 0) {
    gemv_mma_mixed(a, ws.grid, 32 * ws.warps_per_block, M, s);
  } else {
    switch (v.bits) {
      case 3: launch_mma<3>(a, ws.grid, 32 * ws.warps_per_block, M, s); break;
      case 4: launch_mma<4>(a, ws.grid, 32 * ws.warps_per_block, M, s); break;
      case 6: launch_mma<6>(a, ws.grid, 32 * ws.warps_per_block, M, s); break;
      default: launch_mma<8>(a, ws.grid, 32 * ws.warps_per_block, M, s); break;
    }
  }
  return record_cuda(cudaGetLastError());
}

void gemv_plan_info(int bits, int N, int K, int M, qlin_gemv_plan_info* info) {
  *info = qlin_gemv_plan_info{};
  if (gemv_imma_fits(bits, N, K, M)) {
    gemv_imma_plan_info(bits, N, K, info);
    return;
  }
  if (gemv_tc_path(bits, N, K, M)) {
    gemv_tc_plan_info(bits, N, K, M, info);
    return;
  }
  Plan p;
  if (M == 1 && bits != 0 && make_plan(bits, N, K, p)) {
    info->kernel = 1;
    info->grid = p.grid;
    info->threads = (p.NW + 1) * 32;
    info->smem_bytes = p.smem_bytes;
    info->consumer_warps = p.NW;
    info->units_per_warp = p.UW;
    info->rows_per_cta = p.rows_per_cta;
    info->rows_per_chunk = p.rows_per_chunk;
    info->stages = p.stages;
    info->chunks_in_flight = p.inflight;
    return;
  }
  const MmaWorkspace ws(N, K, M);
  info->kernel = 2;
  info->grid = ws.grid;
  info->threads = 32 * ws.warps_per_block;
  info->workspace_bytes = ws.total;
}

unsigned take_gemv_error() {
  unsigned v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_gemv_error, sizeof(v)) != cudaSuccess) return ~0u;
  if (v) cudaMemcpyToSymbol(g_gemv_error, &zero, sizeof(zero));
  return v;
}

}  // namespace qlin

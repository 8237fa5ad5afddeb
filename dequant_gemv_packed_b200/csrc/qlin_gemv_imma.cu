// qlin_gemv for M = 1 on the integer tensor cores: 4- and 8-bit codes.
//
// y[n] = sum_k rht(x)[k] * s[n][k/128] * (q[n][k] - z[n][k/128]), computed as
// y[n] = sum_g s[n][g] * xs[g] * (S[n][g] - z[n][g] * X[g]), where per group g
// of 128 codes the rotated x is taken as 16-bit integers xi = rint(x~ / xs)
// with one power-of-two scale xs (exact for values within a factor 8 of the
// group's largest magnitude, others rounded at 2^-14 of it), X[g] = sum xi and
// S[n][g] = sum_k q[n][k] xi[k] exactly in int32.  The scale and zero act on
// each group's sum, never on single weights ("24B0978-Week01-Track2_20-
// Submission01", "How these techniques accelerate inference on CUDA",
// paragraph "Group-wise affine integer quantisation": all 128 weights sharing
// a scale feed one dot product, so the scale is applied once to it).
//
// S is a matrix product: A = codes (16 weight rows x 32 codes, unsigned bytes)
// times B = xi split into two signed-byte digits, xi = 256 hi + lo (hi in
// [-64, 64], lo in [-128, 127]), on mma.sync.m16n8k32 (u8 x s8 -> s32).
// The packed words are the A fragments almost as stored: an 8-bit code word
// is four bytes as is; a 4-bit word becomes two by masking (even codes in the
// low nibbles; odd codes left in the high nibbles, i.e. times 16, in an MMA
// and accumulator of their own, shifted back exactly).  The B columns hold
// (group slot, digit): two groups per work item, so one MMA sequence
// computes 16 rows x 2 groups.  The order of codes along the MMA's k differs
// from the stored order; the digit planes of x are stored in the same order.
//
// CTA layout (one CTA per SM, rows split evenly; all of a CTA's rows resident
// in shared memory):
//   * producer warp: two bulk asynchronous copies per 16-row tile, one per
//     8-row chunk (completing on the tile's barrier), and two for the CTA's
//     scales and zeros.  The tile's second chunk starts 64 bytes (4-bit) or 16
//     bytes (8-bit) past a 128-byte boundary, and MMA row m takes row m / 2 of
//     chunk m % 2: the lanes of one fragment-load phase read rows of both
//     chunks, whose pieces then fall in distinct banks;
//   * 16 consumer warps: rotate x (one block of 128 per warp at a time, on the
//     tensor cores: qlin_rot16.cuh), write each group's digit planes and
//     (xs, xs X) to shared memory, then take (16-row tile, group pair) items
//     in tile-major order, one contiguous range per warp; over its run of
//     items of one tile a lane keeps its rows' partial sums in registers and
//     writes them once to a shared [warp][row] array, which is summed over
//     the warps in a fixed order at the end (deterministic results).
// With qlin_set_overlap(1) the kernel is a programmatic dependent, like the
// other M = 1 kernel: the weight stream starts before the previous kernel
// ends; x is read, and y written, after it.
#include <algorithm>
#include <atomic>

#include "qlin_internal.cuh"
#include "qlin_rot16.cuh"
#include "qlin_sm100.cuh"

namespace qlin {

__device__ unsigned int g_imma_error;  // nonzero: a bounded wait gave up

namespace {

constexpr int kNW = 16;                       // consumer warps
constexpr int kThreads = (kNW + 1) * 32;      // + one producer warp
constexpr int kSmemLimit = 113 * 1024;        // two CTAs (this call's and the next) per SM
constexpr int kMinSmem = 80 * 1024;           // never three
constexpr int kMaxTiles = 64;                 // 16-row tiles per CTA
constexpr int kSms = 148;
constexpr int kPlaneLo = 144;                 // the low-digit plane, 16 bytes past 128: the two planes'
                                              // fragment loads (lanes gl = 0 and 1) fall in distinct banks
constexpr int kGroupXB = 288;                 // bytes of a group's two planes
constexpr int kXBatch = 8;                    // x blocks a warp loads before rotating
constexpr int kInflightTiles = 64;            // producer pacing: tiles in flight per CTA

struct ImmaPlan {
  int G, GP;           // groups per row, group pairs (items per tile)
  int grid, rows_max, T;
  int row_bytes;
  int chunk_b;         // offset of a tile's second 8-row chunk from its first
  int tile_bytes;      // stride of the tiles in shared memory (a multiple of 128)
  int sz_halves;       // halves per array (scales, zeros) in shared memory
  int inflight;        // tiles whose copies the producer has in flight at once
  int off_sz, off_xb, off_xc, off_part, off_x, off_bar;
  int smem_bytes;
};

struct ImmaArgs {
  const uint8_t* codes;
  const __half* scales;
  const __half* zeros;
  const uint32_t* sign_bits;
  const __half* x;
  __half* y;
  int N, K;
  int weights_first;
  ImmaPlan p;
};

__device__ __forceinline__ void imma_fail(unsigned code) { atomicOr(&g_imma_error, code); }

// D += A . B, A 16x32 unsigned bytes, B 32x8 signed bytes (fragments of lane
// (g, t) = (lane / 4, lane % 4): a0 = A[g][4t..4t+3], a1 = A[g+8][4t..],
// a2 = A[g][16+4t..], a3 = A[g+8][16+4t..]; b0 = B[4t..4t+3][g],
// b1 = B[16+4t..16+4t+3][g]; d = D[g][2t, 2t+1], D[g+8][2t, 2t+1]).
__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ldsu128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ float ldsh2f(uint32_t addr) {
  uint16_t h;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(h) : "r"(addr));
  return __half2float(__ushort_as_half(h));
}

// Where code c (0..127) of a group sits in a digit plane.  Lane t's 32 bytes
// [32t, 32t + 32) are its B fragments in MMA order.
//   8-bit: lane t's codes are 32t..32t+31, words in MMA order: as stored.
//   4-bit: lane t holds stored words 4t..4t+3 (codes 32t..32t+31); the MMA
//   (half o: even/odd codes, j: words 2j and 2j+1, h: b0/b1) takes byte i of
//   word 2j+h, i.e. code 32t + 16j + 8h + 2i + o, at plane byte
//   32t + 4(4o + 2j + h) + i.
template <int B>
__device__ __forceinline__ int digit_pos(int c) {
  if constexpr (B == 8) {
    return c;
  } else {
    const int rem = c & 31;
    const int j = rem >> 4, h = (rem >> 3) & 1, i = (rem >> 1) & 3, o = rem & 1;
    return (c & ~31) + 4 * (4 * o + 2 * j + h) + i;
  }
}

// Rotation of one block of x (= one group), its power-of-two scale and the
// two digit planes of xi; (xs, xs * sum xi) to xc.
template <int B>
__device__ __forceinline__ void prepare_group(uint32_t b0, uint32_t b1, uint32_t sw, const uint32_t (&h)[4],
                                              int lane, uint8_t* plane, float2* xc) {
  __half hv[4];
  float f[4];
  rotate_block16x8(b0, b1, sw, h, lane, hv, f);
  const uint32_t m = __reduce_max_sync(
      0xffffffffu, __float_as_uint(fmaxf(fmaxf(fabsf(f[0]), fabsf(f[1])), fmaxf(fabsf(f[2]), fabsf(f[3])))));
  // xi = rint(x~ 2^(13-E)), E the exponent of the group's largest |x~|: |xi| <= 2^14
  const int E = m ? (int)((m >> 23) & 0xFF) - 127 : 0;
  const float up = __uint_as_float((uint32_t)(127 + 13 - E) << 23);
  const float xs = __uint_as_float((uint32_t)(127 - 13 + E) << 23);
  int xi[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) xi[i] = __float2int_rn(f[i] * up);
  const int xsum = __reduce_add_sync(0xffffffffu, (xi[0] + xi[1]) + (xi[2] + xi[3]));
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int pos = digit_pos<B>(g + 32 * t + rot_off(i));
    const int hi = (xi[i] + 128) >> 8;  // arithmetic shift: round(xi / 256) in [-64, 64]
    const int lo = xi[i] - (hi << 8);   // in [-128, 127]
    plane[pos] = (uint8_t)hi;
    plane[kPlaneLo + pos] = (uint8_t)lo;
  }
  if (lane == 0) *xc = make_float2(xs, xs * (float)xsum);
}

template <int B>
__global__ void __launch_bounds__(kThreads, 2) gemv_imma_kernel(const __grid_constant__ ImmaArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int kGroupBytes = 16 * B;  // bytes of one group of one row
  const ImmaPlan& p = a.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gl = lane >> 2, t = lane & 3;
  const int n0 = (int)(((long long)blockIdx.x * a.N) / gridDim.x);
  const int R = (int)(((long long)(blockIdx.x + 1) * a.N) / gridDim.x) - n0;
  if (R <= 0) return;
  const int T = (R + 15) >> 4, G = p.G, GP = p.GP, Rp = 16 * T;
  uint8_t* codes_s = smem;
  __half* s_raw = reinterpret_cast<__half*>(smem + p.off_sz);
  __half* z_raw = s_raw + p.sz_halves;
  uint8_t* xb = smem + p.off_xb;            // [G][288]: digit planes (high at 0, low at 144), then 32 zero bytes
  uint8_t* zero32 = xb + (size_t)G * kGroupXB;
  float2* xc = reinterpret_cast<float2*>(smem + p.off_xc);
  float* part = reinterpret_cast<float*>(smem + p.off_part);  // [kNW][Rp]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  uint64_t* sz_full = full + kMaxTiles;
  uint64_t* x_issued = sz_full + 1;
  uint64_t* x_full = x_issued + 1;
  const __half* xs = reinterpret_cast<const __half*>(smem + p.off_x);  // x, copied in once

  if (tid == kNW * 32) {
    for (int r = 0; r < T; ++r) mbar_init(&full[r], 1);
    mbar_init(sz_full, 1);
    mbar_init(x_issued, 1);
    mbar_init(x_full, 1);
    mbar_fence_init();
  }
  if (tid < 8) reinterpret_cast<uint32_t*>(zero32)[tid] = 0u;
  __syncthreads();
  if (tid == 0) grid_launch_dependents();

  if (warp == kNW) {
    // ----------------------------------------------------------- producer --
    if (lane != 0) return;
    if (!a.weights_first && !mbar_wait(x_issued, 0, &g_imma_error)) imma_fail(0x40u);
    // scales and zeros of rows [n0, n0 + R): aligned 16-byte pieces (a little
    // past the range), plain copies where that would pass the end of the arrays
    const size_t total_h = (size_t)a.N * G;
    const size_t h0 = (size_t)n0 * G, h1 = h0 + (size_t)R * G;
    const size_t al = h0 & ~(size_t)7;
    size_t bh = (h1 + 7) & ~(size_t)7;
    if (bh > total_h) {
      bh = h1 & ~(size_t)7;
      for (size_t q = (bh > h0 ? bh : h0); q < h1; ++q) {
        s_raw[q - al] = a.scales[q];
        z_raw[q - al] = a.zeros[q];
      }
    }
    const uint32_t szb = bh > al ? (uint32_t)(bh - al) * 2u : 0u;
    mbar_arrive_expect_tx(sz_full, 2u * szb);
    if (szb) {
      bulk_g2s(s_raw, a.scales + al, szb, sz_full);
      bulk_g2s(z_raw, a.zeros + al, szb, sz_full);
    }
    for (int r = 0; r < T; ++r) {
      // Pace the stream: at most p.inflight tiles in flight, so that this
      // CTA's copies do not flood the memory system while the kernel before
      // it (whose x loads are on the critical path) is still running.
      if (r >= p.inflight && !mbar_wait(&full[r - p.inflight], 0, &g_imma_error)) imma_fail(0x80u);
      const int rows = min(16, R - 16 * r), ra = min(8, rows), rb = rows - ra;
      uint8_t* dst = codes_s + (size_t)r * p.tile_bytes;
      const uint8_t* src = a.codes + (size_t)(n0 + 16 * r) * p.row_bytes;
      mbar_arrive_expect_tx(&full[r], (uint32_t)rows * (uint32_t)p.row_bytes);
      bulk_g2s(dst, src, (uint32_t)(ra * p.row_bytes), &full[r]);
      if (rb > 0) bulk_g2s(dst + p.chunk_b, src + (size_t)8 * p.row_bytes, (uint32_t)(rb * p.row_bytes), &full[r]);
    }
    return;
  }

  // ------------------------------------------------------------- prologue --
  // x arrives in one bulk copy, issued by thread 0 right after the dependency
  // wait (one request per CTA for the vector every CTA reads, instead of one
  // per warp and block); the sign bits (weights side) are read before it.
  // Blocks g = warp, warp + 16, ... are then rotated from shared memory.
  {
    uint32_t h[4];
    h16_fragment(lane, h);
    const int xo = 16 * gl + 2 * t;
    for (int blk0 = warp; blk0 < G; blk0 += kXBatch * kNW) {
      uint32_t xb0[kXBatch], xb1[kXBatch], sw[kXBatch];
#pragma unroll
      for (int j = 0; j < kXBatch; ++j) {
        const int blk = min(blk0 + j * kNW, G - 1);
        sw[j] = rot_sign_bits(a.sign_bits, blk, lane);
      }
      if (blk0 == warp) {
        if (tid == 0) {
          grid_dependency_wait();
          mbar_arrive_expect_tx(x_full, 2u * (uint32_t)a.K);
          bulk_g2s(const_cast<__half*>(xs), a.x, 2u * (uint32_t)a.K, x_full);
          mbar_arrive(x_issued);
        }
        if (!mbar_wait(x_full, 0, &g_imma_error)) imma_fail(0x40u);
      }
#pragma unroll
      for (int j = 0; j < kXBatch; ++j) {
        const int blk = min(blk0 + j * kNW, G - 1);
        const __half* xp = xs + (size_t)blk * kHadamard + xo;
        xb0[j] = *reinterpret_cast<const uint32_t*>(xp);
        xb1[j] = *reinterpret_cast<const uint32_t*>(xp + 8);
      }
#pragma unroll
      for (int j = 0; j < kXBatch; ++j) {
        const int blk = blk0 + j * kNW;
        if (blk >= G) break;  // warp-uniform
        prepare_group<B>(xb0[j], xb1[j], sw[j], h, lane, xb + (size_t)blk * kGroupXB, xc + blk);
      }
    }
  }
  named_barrier(1, kNW * 32);  // digit planes and (xs, xs X) of every group written
  if (!mbar_wait(sz_full, 0, &g_imma_error)) imma_fail(0x20u);

  // ------------------------------------------------------------ main loop --
  // Items (16-row tile r, group pair pp) in tile-major order, item = r GP + pp;
  // warp w takes the contiguous range [w I / 16, (w + 1) I / 16).  Over a run
  // of items of one tile each lane keeps its two rows' partial sums in
  // registers (lanes t = 0, 1: groups 2 pp + t), so an item is one chain of
  // loads, MMAs and two multiply-adds; at the end of the run the two lanes'
  // sums are added and written once, to part[w][row].  A tile's barrier is
  // tested once per run.  Shared memory is addressed with 32-bit offsets.
  const int I = T * GP;
  const int i0 = (int)(((long long)warp * I) / kNW), i1 = (int)(((long long)(warp + 1) * I) / kNW);
  const int slot = gl >> 1;  // this lane's B column: (slot, digit) = (gl / 2, gl % 2)
  const uint32_t xb_lane = smem_addr(xb) + (uint32_t)((gl & 1) * kPlaneLo + 32 * t);
  const uint32_t zero_u = smem_addr(zero32);
  const uint32_t code0 = smem_addr(codes_s) + (uint32_t)((kGroupBytes / 4) * t);
  // MMA rows gl and gl + 8 are rows la and la + 4 of chunk gl % 2 of a tile
  const int la = 8 * (gl & 1) + (gl >> 1);
  const uint32_t lane_row = (uint32_t)((gl & 1) * p.chunk_b + (gl >> 1) * p.row_bytes);
  const uint32_t row4 = 4u * (uint32_t)p.row_bytes;
  const uint32_t s_u = smem_addr(s_raw), z_u = smem_addr(z_raw);
  const int sz_off = (int)(((size_t)n0 * G) & 7);  // the CTA's first scale in its aligned copy
  int r = i0 / GP, pp = i0 - r * GP;
  bool at_run_start = true;
  uint32_t ra_u = 0, rb_u = 0;
  int ra = 0, rb = 0;
  float acc_a = 0.f, acc_b = 0.f;
  for (int it = i0; it < i1; ++it) {
    if (at_run_start) {  // warp-uniform: this warp's first item of tile r
      at_run_start = false;
      if (!mbar_wait_poll(&full[r], 0, &g_imma_error)) imma_fail(0x10u);
      // this lane's two rows (in the last tile, rows past the share read the last row)
      const uint32_t tile_u = code0 + (uint32_t)r * (uint32_t)p.tile_bytes;
      ra_u = tile_u + lane_row;
      rb_u = ra_u + row4;
      ra = 16 * r + la;
      rb = ra + 4;
      if (rb > R - 1) {
        const int lr = R - 1 - 16 * r;
        const uint32_t last = tile_u + (uint32_t)((lr >> 3) * p.chunk_b + (lr & 7) * p.row_bytes);
        if (ra > R - 1) {
          ra = R - 1;
          ra_u = last;
        }
        rb = R - 1;
        rb_u = last;
      }
    }
    const int g0 = 2 * pp;
    const bool has1 = g0 + 1 < G;
    const int gq = (t == 1 && has1) ? g0 + 1 : g0;  // lanes t = 0, 1: group g0 + t
    const uint32_t b0 = slot == 0 ? xb_lane + (uint32_t)(g0 * kGroupXB) : zero_u;
    const uint32_t b1 = (slot == 1 && has1) ? xb_lane + (uint32_t)((g0 + 1) * kGroupXB) : zero_u;
    const uint4 b0A = ldsu128(b0), b0B = ldsu128(b0 + 16);
    const uint4 b1A = ldsu128(b1), b1B = ldsu128(b1 + 16);
    const float sa = ldsh2f(s_u + 2u * (uint32_t)(sz_off + ra * G + gq));
    const float za = ldsh2f(z_u + 2u * (uint32_t)(sz_off + ra * G + gq));
    const float sb = ldsh2f(s_u + 2u * (uint32_t)(sz_off + rb * G + gq));
    const float zb = ldsh2f(z_u + 2u * (uint32_t)(sz_off + rb * G + gq));
    const float2 xv = xc[gq];
    const uint32_t g0b = (uint32_t)(g0 * kGroupBytes);
    int dl[4] = {0, 0, 0, 0}, dh[4] = {0, 0, 0, 0};
    int Sa, Sb;
    if constexpr (B == 4) {
      const uint4 wa0 = ldsu128(ra_u + g0b), wb0 = ldsu128(rb_u + g0b);
      uint4 wa1 = {}, wb1 = {};
      if (has1) {
        wa1 = ldsu128(ra_u + g0b + kGroupBytes);
        wb1 = ldsu128(rb_u + g0b + kGroupBytes);
      }
      constexpr uint32_t kLo = 0x0F0F0F0Fu, kHi = 0xF0F0F0F0u;
      mma_u8s8(dl, wa0.x & kLo, wb0.x & kLo, wa0.y & kLo, wb0.y & kLo, b0A.x, b0A.y);
      mma_u8s8(dh, wa0.x & kHi, wb0.x & kHi, wa0.y & kHi, wb0.y & kHi, b0B.x, b0B.y);
      mma_u8s8(dl, wa0.z & kLo, wb0.z & kLo, wa0.w & kLo, wb0.w & kLo, b0A.z, b0A.w);
      mma_u8s8(dh, wa0.z & kHi, wb0.z & kHi, wa0.w & kHi, wb0.w & kHi, b0B.z, b0B.w);
      if (has1) {
        mma_u8s8(dl, wa1.x & kLo, wb1.x & kLo, wa1.y & kLo, wb1.y & kLo, b1A.x, b1A.y);
        mma_u8s8(dh, wa1.x & kHi, wb1.x & kHi, wa1.y & kHi, wb1.y & kHi, b1B.x, b1B.y);
        mma_u8s8(dl, wa1.z & kLo, wb1.z & kLo, wa1.w & kLo, wb1.w & kLo, b1A.z, b1A.w);
        mma_u8s8(dh, wa1.z & kHi, wb1.z & kHi, wa1.w & kHi, wb1.w & kHi, b1B.z, b1B.w);
      }
      // lane (gl, t < 2): rows ra, rb of group g0 + t; columns 2t (high digit), 2t + 1 (low digit)
      Sa = ((dl[0] + (dh[0] >> 4)) << 8) + (dl[1] + (dh[1] >> 4));
      Sb = ((dl[2] + (dh[2] >> 4)) << 8) + (dl[3] + (dh[3] >> 4));
    } else {
      {
        const uint4 wa0 = ldsu128(ra_u + g0b), wa1 = ldsu128(ra_u + g0b + 16);
        const uint4 wb0 = ldsu128(rb_u + g0b), wb1 = ldsu128(rb_u + g0b + 16);
        mma_u8s8(dl, wa0.x, wb0.x, wa0.y, wb0.y, b0A.x, b0A.y);
        mma_u8s8(dh, wa0.z, wb0.z, wa0.w, wb0.w, b0A.z, b0A.w);
        mma_u8s8(dl, wa1.x, wb1.x, wa1.y, wb1.y, b0B.x, b0B.y);
        mma_u8s8(dh, wa1.z, wb1.z, wa1.w, wb1.w, b0B.z, b0B.w);
      }
      if (has1) {
        const uint4 wa2 = ldsu128(ra_u + g0b + kGroupBytes), wa3 = ldsu128(ra_u + g0b + kGroupBytes + 16);
        const uint4 wb2 = ldsu128(rb_u + g0b + kGroupBytes), wb3 = ldsu128(rb_u + g0b + kGroupBytes + 16);
        mma_u8s8(dl, wa2.x, wb2.x, wa2.y, wb2.y, b1A.x, b1A.y);
        mma_u8s8(dh, wa2.z, wb2.z, wa2.w, wb2.w, b1A.z, b1A.w);
        mma_u8s8(dl, wa3.x, wb3.x, wa3.y, wb3.y, b1B.x, b1B.y);
        mma_u8s8(dh, wa3.z, wb3.z, wa3.w, wb3.w, b1B.z, b1B.w);
      }
      // two accumulators for latency only: both hold plain sums
      Sa = ((dl[0] + dh[0]) << 8) + (dl[1] + dh[1]);
      Sb = ((dl[2] + dh[2]) << 8) + (dl[3] + dh[3]);
    }
    if (t == 0 || (t == 1 && has1)) {
      acc_a += sa * fmaf(-za, xv.y, xv.x * (float)Sa);
      acc_b += sb * fmaf(-zb, xv.y, xv.x * (float)Sb);
    }
    if (++pp == GP || it + 1 == i1) {  // warp-uniform: the end of this warp's run of tile r
      acc_a += __shfl_xor_sync(0xffffffffu, acc_a, 1);
      acc_b += __shfl_xor_sync(0xffffffffu, acc_b, 1);
      if (t == 0) {
        part[warp * Rp + 16 * r + la] = acc_a;
        part[warp * Rp + 16 * r + la + 4] = acc_b;
      }
      acc_a = acc_b = 0.f;
      if (pp == GP) {
        pp = 0;
        ++r;
        at_run_start = true;
      }
    }
  }
  named_barrier(1, kNW * 32);

  // ---------------------------------------------------------- row sums ----
  // Row n0 + row of tile r: the sum of part[w][row] over the warps w whose
  // item ranges meet the tile's items [r GP, (r + 1) GP), in warp order.
  // Item x lies in the range of warp (16 x + 15) / I.
  for (int row = tid; row < R; row += kNW * 32) {
    const int rt = row >> 4;
    const int w_lo = (kNW * rt * GP + kNW - 1) / I;
    const int w_hi = (kNW * ((rt + 1) * GP - 1) + kNW - 1) / I;
    float acc = 0.f;
    for (int w = w_lo; w <= w_hi; ++w)
      if ((long long)w * I / kNW < (long long)(w + 1) * I / kNW) acc += part[w * Rp + row];
    a.y[n0 + row] = __float2half_rn(acc);
  }
}

// ------------------------------------------------------------- host plan --

bool make_imma_plan(int b, int N, int K, ImmaPlan& p) {
  if (b != 4 && b != 8) return false;
  if (K % kGroup || N < 1) return false;
  p.G = K / kGroup;
  p.GP = (p.G + 1) / 2;
  p.grid = std::min(kSms, N);
  p.rows_max = (N + p.grid - 1) / p.grid;
  p.T = (p.rows_max + 15) / 16;
  if (p.T > kMaxTiles) return false;
  p.row_bytes = K * b / 8;
  // A tile: chunk A (8 rows) at a 128-byte boundary, chunk B (8 rows) at 64
  // (4-bit) or 16 (8-bit) bytes mod 128 after it.
  const int want = b == 4 ? 64 : 16;
  const int a_bytes = 8 * p.row_bytes;
  p.chunk_b = a_bytes + ((want - a_bytes % 128) % 128 + 128) % 128;
  p.tile_bytes = (p.chunk_b + 8 * p.row_bytes + 127) & ~127;
  // the last tile holds only the rows left (at most rows_max - 16 (T - 1))
  const int last = p.rows_max - 16 * (p.T - 1);
  const int last_bytes = last <= 8 ? last * p.row_bytes : p.chunk_b + (last - 8) * p.row_bytes;
  const int codes = ((p.T - 1) * p.tile_bytes + last_bytes + 127) & ~127;
  p.sz_halves = (p.rows_max * p.G + 16 + 7) & ~7;
  p.off_sz = codes;
  p.off_xb = (p.off_sz + 4 * p.sz_halves + 127) & ~127;
  p.off_xc = (p.off_xb + p.G * kGroupXB + 32 + 15) & ~15;
  p.off_part = (p.off_xc + p.G * 8 + 127) & ~127;
  p.off_x = (p.off_part + kNW * 16 * p.T * 4 + 127) & ~127;
  p.off_bar = (p.off_x + 2 * K + 127) & ~127;
  p.inflight = kInflightTiles;
  const int end = p.off_bar + (kMaxTiles + 2) * 8 + 16;
  p.smem_bytes = std::max(end, kMinSmem);
  return end <= kSmemLimit;
}

template <int B>
qlin_status launch_imma(const ImmaArgs& a, cudaStream_t s) {
  // One bit per device (the attributes are per device), atomic: host threads
  // making their first call together may both set the attributes (harmless).
  static std::atomic<unsigned long long> configured{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda(e);
  if (dev >= 64 || !((configured.load(std::memory_order_acquire) >> dev) & 1ull)) {
    e = cudaFuncSetAttribute(gemv_imma_kernel<B>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
    if (e != cudaSuccess) return record_cuda(e);
    e = cudaFuncSetAttribute(gemv_imma_kernel<B>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return record_cuda(e);
    if (dev < 64) configured.fetch_or(1ull << dev, std::memory_order_release);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.p.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = a.p.smem_bytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = overlap_enabled() ? 1 : 0;
  return record_cuda(cudaLaunchKernelEx(&cfg, gemv_imma_kernel<B>, a));
}

}  // namespace

bool gemv_imma_fits(int bits, int N, int K, int M) {
  ImmaPlan p;
  return M == 1 && make_imma_plan(bits, N, K, p);
}

qlin_status launch_gemv_imma(const PackedView& v, const __half* scales, const __half* zeros,
                             const uint32_t* sign_bits, const __half* x, __half* y, cudaStream_t s) {
  ImmaArgs a;
  if (!make_imma_plan(v.bits, v.N, v.K, a.p)) return QLIN_ERR_UNSUPPORTED;
  a.codes = v.codes;
  a.scales = scales;
  a.zeros = zeros;
  a.sign_bits = sign_bits;
  a.x = x;
  a.y = y;
  a.N = v.N;
  a.K = v.K;
  a.weights_first = overlap_enabled() ? 1 : 0;
  return v.bits == 4 ? launch_imma<4>(a, s) : launch_imma<8>(a, s);
}

void gemv_imma_plan_info(int bits, int N, int K, qlin_gemv_plan_info* info) {
  ImmaPlan p;
  *info = qlin_gemv_plan_info{};
  if (!make_imma_plan(bits, N, K, p)) return;
  info->kernel = 3;
  info->grid = p.grid;
  info->threads = kThreads;
  info->smem_bytes = p.smem_bytes;
  info->consumer_warps = kNW;
  info->rows_per_cta = p.rows_max;
  info->rows_per_chunk = 16;
  info->stages = p.T;
  info->chunks_in_flight = p.T;
}

unsigned take_imma_error() {
  unsigned v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_imma_error, sizeof(v)) != cudaSuccess) return ~0u;
  if (v) cudaMemcpyToSymbol(g_imma_error, &zero, sizeof(zero));
  return v;
}

}  // namespace qlin

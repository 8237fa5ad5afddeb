// qlin_gemv for M = 1..16 rows of x on the tensor cores, any uniform code width.
//
// y[m][n] = sum_g s[n][g] * (sum_k q[n][k] x~[m][k] - z[n][g] * X[m][g]) over
// the groups g of 128 codes, x~ = rht(x) rounded to fp16 and X[m][g] the sum of
// group g of x~[m] ("24B0978-Week01-Track2_20-Submission01", "How these
// techniques accelerate inference on CUDA", paragraph "Group-wise affine
// integer quantisation": the scale and zero act once per group's dot product;
// the fp16 weight is never formed).
//
// Work split.  The weight is cut into 32-row tiles and groups; CTA (p, s) takes
// the rectangle of row part p and K slice s (grid = P x S <= 148, one CTA per
// SM).  Slice lengths are odd for 3-, 4- and 6-bit codes: a shared-memory row
// of an odd number of groups puts the eight rows a fragment load touches in
// eight distinct bank positions.  Inside a CTA the (tile, group) units, in
// tile-major order, are split into eight contiguous ranges, one per warp.
//
// Data path of a CTA:
//   * thread 0 loads each tile of the rectangle with one TMA 2-D box (32 rows x
//     the slice's bytes) into shared memory; rectangles too large for shared
//     memory go in rounds through two buffers;
//   * x~ in the order the B fragments of the MMA take it (ldmatrix, 16-byte
//     chunks XOR-swizzled by row), with each group's sum X: for M >= 2 a small
//     kernel (rot_tc_kernel) rotates x once per call into the workspace in
//     exactly that layout and each CTA bulk-copies its slice; for M = 1 the
//     CTA's warps rotate their slice themselves (qlin_rot16.cuh);
//   * per unit: the codes of the lane's four rows become exact fp16 pairs (the
//     code in the mantissa of 1024, then one fused multiply-add that removes
//     the offset and the bit position), A operands of m16n8k16 MMAs against x~
//     (n8 = eight rows of x per product; two products for M > 8), fp32
//     accumulation; then acc += s (D - z X).  Which codes of a group form a
//     pair, and which MMA k slot each pair takes, is a fixed permutation per
//     width; x~ is stored in the same permutation, so the sums are those of
//     the definition.
//   * reduction in a fixed order: a warp that covers a whole tile's units of
//     the slice writes its sums out directly; tiles shared by several warps
//     are added in warp order; with S > 1 the S slices of a row part run as
//     one thread-block cluster, each CTA keeps its tile sums in its shared
//     memory, and after a cluster barrier each adds all slices' sums for its
//     share of the outputs, in slice order, reading the others' shared memory
//     (distributed shared memory), and writes y (fp16).  No global partial
//     sums, counters or atomics; results do not depend on timing.
// With qlin_set_overlap(1) the kernel is a programmatic dependent: codes,
// scales, zeros and signs are fetched before the wait for the previous
// kernel; x, the workspace and y are touched after it.
#include <cuda.h>

#include <algorithm>
#include <atomic>

#include "qlin_internal.cuh"
#include "qlin_rot16.cuh"
#include "qlin_sm100.cuh"

namespace qlin {

__device__ unsigned int g_tc_error;  // nonzero: a bounded wait gave up

namespace {

constexpr int kW = 8;                 // warps per CTA
constexpr int kThreads = kW * 32;
constexpr int kTileRows = 32;
constexpr int kSmemMax = 227 * 1024;
constexpr int kSzBatch = 8;           // (scale, zero) pairs a thread loads ahead of the dependency wait
constexpr int kXBatch = 8;            // x blocks a warp loads before rotating
constexpr int kMaxCluster = 8;        // K slices of a row part: one portable thread-block cluster
// Clusters of S CTAs that fit on the GPU at once with one CTA per SM (B200, 148
// SMs in GPCs of 18 or 20; cudaOccupancyMaxActiveClusters at 160 KB and more
// of shared memory): the grid never exceeds one wave of clusters.
constexpr int kClustersAtOnce[kMaxCluster + 1] = {0, 148, 74, 45, 33, 26, 22, 15, 15};
constexpr uint32_t kMagic = 0x64006400u;  // fp16 1024.0 in both halves

struct TcPlan {
  int T, G;            // 32-row tiles of N, groups of K
  int S, P;            // K slices, row parts: grid = P * S
  int L, d, nhi;       // slice lengths: the first nhi slices L groups, the rest L - d
  int Tc;              // most tiles of a part
  int RT, nbuf;        // tiles per round, code buffers (1: one round)
  int NT;              // n8 tiles of x rows (1: M <= 8, 2: M <= 16)
  int off_xsum, off_sz, off_red, off_cp, off_codes, off_bar;
  int buf_bytes;       // one code buffer
  int smem_bytes;
  int xrot;            // 1: x rotated once per call by rot_tc_kernel into the workspace
  // workspace (xrot plans only): x~ in the shared-memory layout
  // [G][NT][8][256 B] at ws_xs and the group sums [G][16] at ws_xsum
  size_t ws_xs, ws_xsum, ws_total;
};

struct TcArgs {
  CUtensorMap map_hi;  // box: L groups x 32 rows
  CUtensorMap map_lo;  // box: L - d groups x 32 rows
  const __half* scales;
  const __half* zeros;
  const uint32_t* sign_bits;
  const __half* x;
  __half* y;
  const uint8_t* xrot; // xrot plans: x~ of every group in the shared-memory layout
  const float* xsum_g; // xrot plans: [G][16] group sums
  int N, K, M;
  TcPlan p;
};

struct RotArgs {
  const __half* x;
  const uint32_t* sign_bits;
  uint8_t* xrot;       // [G][NT][8][256 B]
  float* xsum_g;       // [G][16]
  int M, K, G;
  // the layer's weight arrays (codes, scales, zeros) and their sizes in bytes,
  // prefetched into L2 for the GEMV that follows
  const void* pf[3];
  size_t pf_bytes[3];
};

__device__ __forceinline__ void tc_fail(unsigned code) { atomicOr(&g_tc_error, code); }

// Hint: bring [p, p + bytes) into L2 (p and bytes multiples of 16).
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Lane `lane` of one warp per CTA prefetches its share of the CTA's slice
// [n b / nb, n (b + 1) / nb) of an array of n bytes (16-byte aligned), in
// pieces of at most 32 KB, ending on 16-byte boundaries.
__device__ __forceinline__ void prefetch_l2_share(const void* base, size_t n, int b, int nb, int lane) {
  if (base == nullptr || n < 16) return;
  const size_t lo = (n * (size_t)b / (size_t)nb) & ~(size_t)15, hi = (n * (size_t)(b + 1) / (size_t)nb) & ~(size_t)15;
  constexpr size_t kPiece = 32768;
  for (size_t o = lo + (size_t)lane * kPiece; o < hi; o += 32 * kPiece) {
    const size_t len = hi - o < kPiece ? hi - o : kPiece;
    prefetch_l2(static_cast<const uint8_t*>(base) + o, (uint32_t)len);
  }
}

// Barrier of every thread of every CTA of the cluster; shared-memory writes
// before it are visible to the cluster's loads after it.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// fp32 at this CTA's shared address `addr`, read from the same address in the
// shared memory of cluster CTA `rank`.
__device__ __forceinline__ float ld_cluster_f32(uint32_t addr, uint32_t rank) {
  uint32_t remote;
  float v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(addr), "r"(rank));
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
               "{%0,%1,%2,%3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint4 lds128u(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// ----------------------------------------------------------- code pairs --
//
// A lane's run: 32 consecutive codes of one row in one group (codes
// 32t..32t+31 for lane t), B words.  Pair p (0..15) is two codes of the run as
// an fp16 pair, exact: (lo, hi) = codes (pair_code(p, 0), pair_code(p, 1)).
// The MMA at k-step j takes pairs 2j (slots 2t, 2t+1) and 2j + 1 (slots
// 2t+8, 2t+9).

// Code (0..31 within the run) of half e of pair p.  3 and 6 bits: codes c and
// c + 16 (96 bits apart, so at the same offset of words three (6-bit) or
// halves three (3-bit) apart), c in the order the decoder extracts them (the
// nibbles of kOrder3 / kOrder6, pair 0 lowest); 4 bits: nibbles i and i + 4 of
// a word; 8 bits: bytes i and i + 2 of a word.
constexpr uint64_t kOrder3 = 0xA5FEDCB987643210ull;
constexpr uint64_t kOrder6 = 0xDA52FECB98764310ull;
__host__ __device__ constexpr int pair_code(int B, int p, int e) {
  return B == 3   ? (int)((kOrder3 >> (4 * p)) & 15) + 16 * e
         : B == 6 ? (int)((kOrder6 >> (4 * p)) & 15) + 16 * e
         : B == 4 ? 8 * (p >> 2) + (p & 3) + 4 * e
                  : 4 * (p >> 1) + (p & 1) + 2 * e;
}
static_assert(pair_code(3, 14, 0) == 5 && pair_code(3, 15, 1) == 26 && pair_code(3, 9, 0) == 11, "3-bit pairs");
static_assert(pair_code(6, 12, 0) == 2 && pair_code(6, 11, 1) == 31 && pair_code(6, 2, 0) == 3, "6-bit pairs");
static_assert(pair_code(4, 5, 1) == 13 && pair_code(8, 3, 1) == 7, "4- and 8-bit pairs");
// The inverse: pair and half of code c of the run.
constexpr uint64_t kInv3 = 0xDCBA9F8765E43210ull;
constexpr uint64_t kInv6 = 0xBAF98E7654D32C10ull;
template <int B>
__device__ __forceinline__ void code_slot(int c, int& p, int& h) {
  if constexpr (B == 3 || B == 6) {
    h = c >> 4;
    p = (int)(((B == 3 ? kInv3 : kInv6) >> (4 * (c & 15))) & 15);
  } else if constexpr (B == 4) {
    h = (c >> 2) & 1;
    p = 4 * (c >> 3) + (c & 3);
  } else {
    h = (c >> 1) & 1;
    p = 2 * (c >> 2) + (c & 1);
  }
}

// fp16 pair (1024 + 2^o a, 1024 + 2^o b) -> (a, b), exactly.
template <int O>
__device__ __forceinline__ uint32_t unbias(uint32_t h) {
  constexpr uint32_t kScale = O == 0 ? 0x3C003C00u : O == 2 ? 0x34003400u : O == 3 ? 0x30003000u
                            : O == 4 ? 0x2C002C00u : 0x24002400u;  // 1, 1/4, 1/8, 1/16, 1/64
  constexpr uint32_t kBias = O == 0 ? 0xE400E400u : O == 2 ? 0xDC00DC00u : O == 3 ? 0xD800D800u
                           : O == 4 ? 0xD400D400u : 0xCC00CC00u;  // -1024, -256, -128, -64, -16
  uint32_t r;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(h), "r"(kScale), "r"(kBias));
  return r;
}

// (v & mask) | 1024 in both halves: one LOP3.
__device__ __forceinline__ uint32_t field(uint32_t v, uint32_t mask) { return (v & mask) | kMagic; }

template <int B, int P>
__device__ __forceinline__ uint32_t code_pair(const uint32_t (&w)[B]) {
  if constexpr (B == 4) {
    const uint32_t v = w[P >> 2];
    constexpr int r = P & 3;
    if constexpr (r == 0) return unbias<0>(field(v, 0x000F000Fu));
    else if constexpr (r == 1) return unbias<4>(field(v, 0x00F000F0u));
    else if constexpr (r == 2) return unbias<0>(field(v >> 8, 0x000F000Fu));
    else return unbias<4>(field(v >> 8, 0x00F000F0u));
  } else if constexpr (B == 8) {
    const uint32_t v = w[P >> 1];
    const uint32_t h = __byte_perm(v, 0x64u, (P & 1) ? 0x4341u : 0x4240u);
    return unbias<0>(h);
  } else if constexpr (B == 3) {
    // halves: P0 = (w0 lo, w1 hi), P1 = (w0 hi, w2 lo), P2 = (w1 lo, w2 hi)
    if constexpr (P <= 4) {
      const uint32_t q = __byte_perm(w[0], w[1], 0x7610u);
      if constexpr (P == 0) return unbias<0>(field(q, 0x00070007u));
      else if constexpr (P == 1) return unbias<3>(field(q, 0x00380038u));
      else if constexpr (P == 2) return unbias<6>(field(q, 0x01C001C0u));
      else if constexpr (P == 3) return unbias<0>(field(q >> 9, 0x00070007u));
      else return unbias<3>(field(q >> 9, 0x00380038u));
    } else if constexpr (P <= 8) {
      const uint32_t q = __byte_perm(w[0], w[2], 0x5432u);
      if constexpr (P == 5) return unbias<0>(field(q >> 2, 0x00070007u));
      else if constexpr (P == 6) return unbias<3>(field(q >> 2, 0x00380038u));
      else if constexpr (P == 7) return unbias<6>(field(q >> 2, 0x01C001C0u));
      else return unbias<0>(field(q >> 11, 0x00070007u));
    } else if constexpr (P <= 13) {
      const uint32_t q = __byte_perm(w[1], w[2], 0x7610u);
      if constexpr (P == 9) return unbias<0>(field(q >> 1, 0x00070007u));
      else if constexpr (P == 10) return unbias<3>(field(q >> 1, 0x00380038u));
      else if constexpr (P == 11) return unbias<6>(field(q >> 1, 0x01C001C0u));
      else if constexpr (P == 12) return unbias<0>(field(q >> 10, 0x00070007u));
      else return unbias<3>(field(q >> 10, 0x00380038u));
    } else if constexpr (P == 14) {  // codes 5 (stream bits 15..17) and 21 (63..65)
      return unbias<0>(field(__byte_perm(w[0] >> 15, __funnelshift_r(w[1], w[2], 31), 0x5410u), 0x00070007u));
    } else {  // codes 10 (30..32) and 26 (78..80)
      return unbias<0>(field(__byte_perm(__funnelshift_r(w[0], w[1], 30), w[2] >> 14, 0x5410u), 0x00070007u));
    }
  } else {  // B == 6: halves of words k and k + 3 side by side
    if constexpr (P <= 11) {
      constexpr int k = P / 4;                 // word pair (k, k + 3)
      constexpr bool high = (P / 2) % 2 == 1;  // high halves of the words
      const uint32_t q = __byte_perm(w[k], w[k + 3], high ? 0x7632u : 0x5410u);
      // offsets in the half: w0 lo 0, 6; w0 hi 2, 8; w1 lo 4, 10; w1 hi 0, 6; w2 lo 2, 8; w2 hi 4, 10
      constexpr int o = (2 * (P / 2)) % 6;
      constexpr uint32_t m = (0x3Fu << o) * 0x10001u;
      const uint32_t v = (P & 1) ? (q >> 6) : q;
      return unbias<o>(field(v, m));
    } else if constexpr (P == 12) {  // codes 2 (bits 12..17) and 18
      return unbias<0>(field(__byte_perm(w[0] >> 12, w[3] >> 12, 0x5410u), 0x003F003Fu));
    } else if constexpr (P == 13) {  // codes 5 (30..35) and 21
      return unbias<0>(field(__byte_perm(__funnelshift_r(w[0], w[1], 30), __funnelshift_r(w[3], w[4], 30), 0x5410u),
                             0x003F003Fu));
    } else if constexpr (P == 14) {  // codes 10 (60..65) and 26
      return unbias<0>(field(__byte_perm(__funnelshift_r(w[1], w[2], 28), __funnelshift_r(w[4], w[5], 28), 0x5410u),
                             0x003F003Fu));
    } else {  // codes 13 (78..83) and 29
      return unbias<0>(field(__byte_perm(w[2] >> 14, w[5] >> 14, 0x5410u), 0x003F003Fu));
    }
  }
}

// The lane's run of row `row_u` (shared address of the run's first byte).
template <int B>
__device__ __forceinline__ void load_run(uint32_t a, uint32_t (&w)[B], bool swap_halves) {
  if constexpr (B == 4) {
    const uint4 v = lds128u(a);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if constexpr (B == 8) {
    // odd rows read their second half first: the two rows of one load phase then
    // fall in different banks
    const uint32_t o0 = swap_halves ? 16u : 0u;
    const uint4 v0 = lds128u(a + o0), v1 = lds128u(a + (16u - o0));
    const uint4 lo = swap_halves ? v1 : v0, hi = swap_halves ? v0 : v1;
    w[0] = lo.x; w[1] = lo.y; w[2] = lo.z; w[3] = lo.w; w[4] = hi.x; w[5] = hi.y; w[6] = hi.z; w[7] = hi.w;
  } else if constexpr (B == 6) {
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      const uint2 v = lds64(a + 8u * i);
      w[2 * i] = v.x; w[2 * i + 1] = v.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < B; ++i) w[i] = lds32(a + 4u * i);
  }
}

// Where element e (0..127) of a group goes in the x~ layout: 16-byte chunk
// p (pair 2j is sub-slot 0 of k-step j, pair 2j + 1 sub-slot 1: chunk 2j + sub
// = p) and halfword 2t + h within it, t = e / 32 the lane of the run.
template <int B>
__device__ __forceinline__ void x_slot(int e, int& chunk, int& half) {
  int p, h;
  code_slot<B>(e & 31, p, h);
  chunk = p;
  half = 2 * (e >> 5) + h;
}

template <int B, int NT>
__global__ void __launch_bounds__(kThreads, 1) gemv_tc_kernel(const __grid_constant__ TcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const TcPlan& p = a.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int S = p.S, G = p.G, M = a.M, N = a.N;
  const int s = blockIdx.x % S, pidx = blockIdx.x / S;
  const int g0 = s * p.L - p.d * max(0, s - p.nhi);
  const int Gs = s < p.nhi ? p.L : p.L - p.d;
  const int t0 = (int)(((long long)pidx * p.T) / p.P), Ts = (int)(((long long)(pidx + 1) * p.T) / p.P) - t0;
  if (Ts <= 0 || Gs <= 0) return;
  const CUtensorMap* map = s < p.nhi ? &a.map_hi : &a.map_lo;
  constexpr int kRunBytes = 4 * B;            // bytes of a lane's run
  const uint32_t pitch = (uint32_t)Gs * 16u * B;  // bytes of one row of the slice in shared memory
  const uint32_t tile_bytes = (uint32_t)kTileRows * pitch;
  const int rounds = (Ts + p.RT - 1) / p.RT;

  uint8_t* xs = smem;                                         // [Gs][NT][8 rows][256 B]
  float* xsum = reinterpret_cast<float*>(smem + p.off_xsum);  // [Gs][16]
  uint32_t* sz = reinterpret_cast<uint32_t*>(smem + p.off_sz);  // [RT * 32][Gs] (s, z) fp16 pairs
  float* red = reinterpret_cast<float*>(smem + p.off_red);    // [kW][3][32][8 NT + 1]
  float* cpart = reinterpret_cast<float*>(smem + p.off_cp);   // S > 1: [RT][8 NT][32] this slice's tile sums
  uint8_t* codes = smem + p.off_codes;                        // [nbuf][RT][32][pitch]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.off_bar);

  uint64_t* xfull = full + 2;  // xrot plans: the slice of x~ and its sums
  if (tid == 0) {
    for (int i = 0; i < p.nbuf; ++i) mbar_init(&full[i], 1);
    mbar_init(xfull, 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (tid == 0) grid_launch_dependents();

  // Round r's tiles into buffer r % nbuf: one box per tile.
  auto issue_round = [&](int r) {
    const int ta = r * p.RT, tb = min(Ts, ta + p.RT);
    uint8_t* buf = codes + (size_t)(r % p.nbuf) * p.buf_bytes;
    uint64_t* bar = &full[r % p.nbuf];
    mbar_arrive_expect_tx(bar, (uint32_t)(tb - ta) * tile_bytes);
    for (int j = ta; j < tb; ++j)
      tma_load_2d(buf + (size_t)(j - ta) * tile_bytes, map, 2 * B * g0, (t0 + j) * kTileRows, bar);
  };
  if (tid == 0)
    for (int r = 0; r < min(rounds, p.nbuf); ++r) issue_round(r);

  // (scale, zero) of round r's rows: entry i = row * Gs + group of the slice.
  auto sz_count = [&](int r) { return (min(Ts, (r + 1) * p.RT) - r * p.RT) * kTileRows * Gs; };
  auto sz_fetch = [&](int r, int i) -> uint32_t {
    const int row = i / Gs, gl = i - row * Gs;
    const int n = (t0 + r * p.RT) * kTileRows + row;
    if (n >= N) return 0u;
    const size_t o = (size_t)n * G + g0 + gl;
    return (uint32_t)__half_as_ushort(a.scales[o]) | ((uint32_t)__half_as_ushort(a.zeros[o]) << 16);
  };
  // Round 0's first entries: the loads are issued now and their values used
  // only when stored after the x prologue (the warps do not wait for them).
  unsigned short sr[kSzBatch], zr[kSzBatch];
  {
    const int n0 = sz_count(0);
#pragma unroll
    for (int i = 0; i < kSzBatch; ++i) {
      const int e = tid + i * kThreads;
      const int row = e / Gs, gl = e - row * Gs;
      const int n = t0 * kTileRows + row;
      sr[i] = zr[i] = 0;
      if (e < n0 && n < N) {
        const size_t o = (size_t)n * G + g0 + gl;
        sr[i] = __ldg(reinterpret_cast<const unsigned short*>(a.scales) + o);
        zr[i] = __ldg(reinterpret_cast<const unsigned short*>(a.zeros) + o);
      }
    }
  }

  // ---------------------------------------------------------- x prologue --
  if (p.xrot) {
    // x~ of the slice, already in the shared-memory layout, and its sums: two
    // bulk copies after the wait for the rotation kernel
    grid_dependency_wait();
    if (tid == 0) {
      const uint32_t xb = (uint32_t)Gs * NT * 2048u, sb = (uint32_t)Gs * 64u;
      mbar_arrive_expect_tx(xfull, xb + sb);
      bulk_g2s(xs, a.xrot + (size_t)g0 * NT * 2048, xb, xfull);
      bulk_g2s(xsum, a.xsum_g + (size_t)g0 * 16, sb, xfull);
    }
  } else {
    // Rows m >= M of the layout are zero (their products land in columns that
    // are never read, but stay finite).
    for (int i = tid; i < Gs * NT * 8 * 16; i += kThreads) {
      const int row = (i >> 4) & (8 * NT - 1);
      if (row >= M) reinterpret_cast<uint4*>(xs)[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    for (int i = tid; i < Gs * 16; i += kThreads)
      if ((i & 15) >= M) xsum[i] = 0.f;
    {
      uint32_t h[4];
      h16_fragment(lane, h);
      int ch[4], hf[4];  // the lane's four rotated elements: chunk and halfword in the layout
#pragma unroll
      for (int i = 0; i < 4; ++i) x_slot<B>(g + 32 * t + rot_off(i), ch[i], hf[i]);
      const int nblk = M * Gs;
      const int xo = 16 * g + 2 * t;
      bool waited = false;
      for (int b0i = warp; b0i < nblk || !waited; b0i += kXBatch * kW) {
        uint32_t xb0[kXBatch], xb1[kXBatch], sw[kXBatch];
#pragma unroll
        for (int j = 0; j < kXBatch; ++j) {
          const int bi = min(b0i + j * kW, nblk - 1);
          sw[j] = rot_sign_bits(a.sign_bits, g0 + bi % Gs, lane);
        }
        if (!waited) {
          grid_dependency_wait();
          waited = true;
        }
        if (b0i >= nblk) break;
#pragma unroll
        for (int j = 0; j < kXBatch; ++j) {
          const int bi = min(b0i + j * kW, nblk - 1);
          const int m = bi / Gs, gl = bi - m * Gs;
          const __half* xp = a.x + (size_t)m * a.K + (size_t)(g0 + gl) * kHadamard + xo;
          xb0[j] = *reinterpret_cast<const uint32_t*>(xp);
          xb1[j] = *reinterpret_cast<const uint32_t*>(xp + 8);
        }
#pragma unroll
        for (int j = 0; j < kXBatch; ++j) {
          const int bi = b0i + j * kW;
          if (bi >= nblk) break;  // warp-uniform
          const int m = bi / Gs, gl = bi - m * Gs;
          __half hv[4];
          float f[4];
          rotate_block16x8(xb0[j], xb1[j], sw[j], h, lane, hv, f);
          uint8_t* xrow = xs + (size_t)gl * (NT * 2048) + (m >> 3) * 2048 + (m & 7) * 256;
#pragma unroll
          for (int i = 0; i < 4; ++i) reinterpret_cast<__half*>(xrow + ((ch[i] ^ (m & 7)) << 4))[hf[i]] = hv[i];
          float sum = (f[0] + f[1]) + (f[2] + f[3]);
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
          if (lane == 0) xsum[gl * 16 + m] = sum;
        }
      }
    }
  }
  // (scale, zero) of round 0 to shared memory (loaded before the wait)
  {
    const int n0 = sz_count(0);
#pragma unroll
    for (int i = 0; i < kSzBatch; ++i) {
      const int e = tid + i * kThreads;
      if (e < n0) sz[e] = (uint32_t)sr[i] | ((uint32_t)zr[i] << 16);
    }
    for (int e = tid + kSzBatch * kThreads; e < n0; e += kThreads) sz[e] = sz_fetch(0, e);
  }
  __syncthreads();
  if (p.xrot && !mbar_wait(xfull, 0, &g_tc_error)) tc_fail(0x2u);

  // ------------------------------------------------------------- rounds --
  const uint32_t xs_u = smem_addr(xs), sz_u = smem_addr(sz), xsum_u = smem_addr(xsum);
  // ldmatrix row address of this lane: matrix q = lane / 8, row rr = lane % 8
  const int q = lane >> 3, rr = lane & 7;
  constexpr int kC = 8 * NT;             // x rows (columns of D) per tile
  constexpr int kRS = kC + 1;            // row stride of a segment in shared memory (odd: no bank conflicts)
  float* my_red = red + (size_t)warp * 3 * kTileRows * kRS;

  // Emits the slice's sums of tile `tl` (local, round r); lane = row of the
  // tile, v[m] its sums for x rows m: to y (S = 1), else to this CTA's
  // shared-memory tile sums, which the cluster adds after the round.  Called
  // by one whole warp.
  auto emit_tile = [&](int r, int tl, const float (&v)[kC]) {
    if (S == 1) {
      const int n = (t0 + r * p.RT + tl) * kTileRows + lane;
      if (n < N)
#pragma unroll
        for (int m = 0; m < kC; ++m)
          if (m < M) a.y[(size_t)m * N + n] = __float2half_rn(v[m]);
      return;
    }
#pragma unroll
    for (int m = 0; m < kC; ++m) cpart[((size_t)tl * kC + m) * kTileRows + lane] = v[m];
  };

  for (int r = 0; r < rounds; ++r) {
    const int nt_r = min(Ts, (r + 1) * p.RT) - r * p.RT;
    if (r > 0) {
      // (scale, zero) of this round (the previous round's are no longer read)
      const int n = sz_count(r);
      for (int e = tid; e < n; e += kThreads) sz[e] = sz_fetch(r, e);
      __syncthreads();
    }
    if (!mbar_wait(&full[r % p.nbuf], (uint32_t)((r / p.nbuf) & 1), &g_tc_error)) tc_fail(0x1u);
    const uint32_t buf_u = smem_addr(codes) + (uint32_t)((r % p.nbuf) * p.buf_bytes);
    const int U = nt_r * Gs;
    const int u0 = (int)(((long long)warp * U) / kW), u1 = (int)(((long long)(warp + 1) * U) / kW);
    const int tf = u0 / Gs;
    float acc[2][NT][4];
    int cur = -1;
    // A segment (this warp's sums of one tile) to shared memory; a whole tile
    // is emitted at once.
    auto flush = [&](int tl) {
      const int seg0 = max(u0, tl * Gs), seg1 = min(u1, (tl + 1) * Gs);
      const bool whole = seg0 == tl * Gs && seg1 == (tl + 1) * Gs;
      const int slot = whole ? 2 : (tl == tf ? 0 : 1);
      float* dst = my_red + slot * kTileRows * kRS;
#pragma unroll
      for (int rb = 0; rb < 2; ++rb)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int row = 16 * rb + g + 8 * (e >> 1), col = 8 * nt + 2 * t + (e & 1);
            dst[row * kRS + col] = acc[rb][nt][e];
          }
      __syncwarp();
      if (whole) {
        float v[kC];
#pragma unroll
        for (int m = 0; m < kC; ++m) v[m] = dst[lane * kRS + m];
        __syncwarp();
        emit_tile(r, tl, v);
      }
    };
    for (int u = u0; u < u1; ++u) {
      const int tl = u / Gs, gl = u - tl * Gs;
      if (tl != cur) {
        if (cur >= 0) flush(cur);
        cur = tl;
#pragma unroll
        for (int rb = 0; rb < 2; ++rb)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[rb][nt][e] = 0.f;
      }
      // B fragments of group gl: bf[nt][j][0..1]
      uint32_t bf[NT][8][2];
      const uint32_t xg = xs_u + (uint32_t)(gl * NT * 2048 + rr * 256);
      if constexpr (NT == 1) {
#pragma unroll
        for (int jp = 0; jp < 4; ++jp)
          ldmatrix_x4(xg + (uint32_t)((((4 * jp + q) ^ rr)) << 4), bf[0][2 * jp][0], bf[0][2 * jp][1],
                      bf[0][2 * jp + 1][0], bf[0][2 * jp + 1][1]);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          ldmatrix_x4(xg + (uint32_t)((q >> 1) * 2048 + (((2 * j + (q & 1)) ^ rr) << 4)), bf[0][j][0], bf[0][j][1],
                      bf[1][j][0], bf[1][j][1]);
      }
      // the lane's runs: rows g, g + 8, g + 16, g + 24 of the tile
      uint32_t w[4][B];
      const uint32_t run0 = buf_u + (uint32_t)tl * tile_bytes + (uint32_t)g * pitch + (uint32_t)gl * (16u * B) +
                            (uint32_t)t * kRunBytes;
#pragma unroll
      for (int k = 0; k < 4; ++k) load_run<B>(run0 + (uint32_t)(8 * k) * pitch, w[k], (g & 1) != 0);
      float d[2][NT][4];
#pragma unroll
      for (int rb = 0; rb < 2; ++rb)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) d[rb][nt][e] = 0.f;
#define QLIN_TC_STEP(J)                                                                                  \
  {                                                                                                      \
    _Pragma("unroll") for (int rb = 0; rb < 2; ++rb) {                                                   \
      const uint32_t a0 = code_pair<B, 2 * (J)>(w[2 * rb]), a2 = code_pair<B, 2 * (J) + 1>(w[2 * rb]);   \
      const uint32_t a1 = code_pair<B, 2 * (J)>(w[2 * rb + 1]),                                          \
                     a3 = code_pair<B, 2 * (J) + 1>(w[2 * rb + 1]);                                      \
      _Pragma("unroll") for (int nt = 0; nt < NT; ++nt)                                                  \
          mma16816(d[rb][nt], a0, a1, a2, a3, bf[nt][J][0], bf[nt][J][1]);                               \
    }                                                                                                    \
  }
      QLIN_TC_STEP(0)
      QLIN_TC_STEP(1)
      QLIN_TC_STEP(2)
      QLIN_TC_STEP(3)
      QLIN_TC_STEP(4)
      QLIN_TC_STEP(5)
      QLIN_TC_STEP(6)
      QLIN_TC_STEP(7)
#undef QLIN_TC_STEP
      // acc += s (D - z X) per row and x row
      const uint32_t szrow = sz_u + 4u * (uint32_t)((tl * kTileRows + g) * Gs + gl);
#pragma unroll
      for (int rb = 0; rb < 2; ++rb) {
        const uint32_t va = lds32(szrow + 4u * (uint32_t)(16 * rb * Gs));
        const uint32_t vb = lds32(szrow + 4u * (uint32_t)((16 * rb + 8) * Gs));
        const float sa = __half2float(__ushort_as_half((uint16_t)(va & 0xFFFFu)));
        const float za = __half2float(__ushort_as_half((uint16_t)(va >> 16)));
        const float sb = __half2float(__ushort_as_half((uint16_t)(vb & 0xFFFFu)));
        const float zb = __half2float(__ushort_as_half((uint16_t)(vb >> 16)));
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const uint2 xv = lds64(xsum_u + 4u * (uint32_t)(gl * 16 + 8 * nt + 2 * t));
          const float x0 = __uint_as_float(xv.x), x1 = __uint_as_float(xv.y);
          acc[rb][nt][0] = fmaf(sa, fmaf(-za, x0, d[rb][nt][0]), acc[rb][nt][0]);
          acc[rb][nt][1] = fmaf(sa, fmaf(-za, x1, d[rb][nt][1]), acc[rb][nt][1]);
          acc[rb][nt][2] = fmaf(sb, fmaf(-zb, x0, d[rb][nt][2]), acc[rb][nt][2]);
          acc[rb][nt][3] = fmaf(sb, fmaf(-zb, x1, d[rb][nt][3]), acc[rb][nt][3]);
        }
      }
    }
    if (cur >= 0) flush(cur);
    __syncthreads();  // every warp's partial segments of this round are in shared memory

    // Tiles shared by several warps: the last of them adds the segments in warp
    // order and emits the tile.
    if (u0 < u1) {
      const int tl_last = (u1 - 1) / Gs;
      for (int tl = tf; tl <= tl_last; ++tl) {
        const int f = tl * Gs, l = f + Gs - 1;
        // warp of unit i: the largest w with floor(w U / kW) <= i
        const int w_first = (int)((((long long)f + 1) * kW - 1) / U), w_last = (int)((((long long)l + 1) * kW - 1) / U);
        if (w_last != warp || w_first == w_last) continue;
        float v[kC];
#pragma unroll
        for (int m = 0; m < kC; ++m) v[m] = 0.f;
        for (int ww = w_first; ww <= w_last; ++ww) {
          const int a0 = (int)(((long long)ww * U) / kW), a1 = (int)(((long long)(ww + 1) * U) / kW);
          if (a0 >= a1) continue;  // a warp with no units
          const int slot = (tl == a0 / Gs) ? 0 : 1;
          const float* seg = red + ((size_t)ww * 3 + slot) * kTileRows * kRS + lane * kRS;
#pragma unroll
          for (int m = 0; m < kC; ++m) v[m] += seg[m];
        }
        emit_tile(r, tl, v);
      }
    }
    if (S > 1) {
      // The K slices of this row part are the CTAs of one cluster: after the
      // barrier every slice's tile sums are visible; CTA s adds, in slice
      // order, the elements [s E / S, (s + 1) E / S) of the round's E = x rows
      // x tile rows outputs (m-major: consecutive threads, consecutive rows)
      // and writes them to y.  The second barrier keeps every CTA's sums in
      // place until all have been read.
      cluster_sync();
      const int Rr = nt_r * kTileRows, E = kC * Rr;
      const int e0 = (int)(((long long)s * E) / S), e1 = (int)(((long long)(s + 1) * E) / S);
      const uint32_t cp_u = smem_addr(cpart);
      for (int e = e0 + tid; e < e1; e += kThreads) {
        const int m = e / Rr, row = e - m * Rr;
        const int n = (t0 + r * p.RT) * kTileRows + row;
        if (m >= M || n >= N) continue;
        const int tl = row / kTileRows, lr = row - tl * kTileRows;
        const uint32_t addr = cp_u + 4u * (uint32_t)(((tl * kC) + m) * kTileRows + lr);
        float v = 0.f;
        for (int ss = 0; ss < S; ++ss) v += ld_cluster_f32(addr, (uint32_t)ss);
        a.y[(size_t)m * N + n] = __float2half_rn(v);
      }
      cluster_sync();
    }
    __syncthreads();  // the round's codes and segments are no longer read
    if (tid == 0 && r + p.nbuf < rounds) issue_round(r + p.nbuf);
  }
}

// Rotation of x for the xrot plans, once per call.  Warp task (g, m), m <
// 8 NT, writes group g of row m of x~ (rows m >= M: zeros) as one 256-byte
// row of gemv_tc_kernel's shared-memory layout (pairs in MMA order, chunks
// XOR-swizzled by row) and the group's sum; the GEMV's CTAs then copy their
// slices with one bulk copy each.  It writes the workspace only after the wait
// for the previous kernel (which may be a GEMV still reading it).
template <int B, int NT>
__global__ void __launch_bounds__(kThreads) rot_tc_kernel(const __grid_constant__ RotArgs r) {
  __shared__ __align__(16) uint8_t rowbuf[kW][256];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  if (tid == 0) grid_launch_dependents();
  // Launched as a programmatic dependent, this kernel starts while the kernel
  // before it still runs, and waits for it below; before that wait, warp 0
  // brings this CTA's share of the layer's weights into L2, so that the
  // GEMV's tensor loads after this kernel find them there.
  if (warp == 0)
    for (int i = 0; i < 3; ++i) prefetch_l2_share(r.pf[i], r.pf_bytes[i], blockIdx.x, gridDim.x, lane);
  const int task = blockIdx.x * kW + warp;
  const int grp = task / (8 * NT), m = task % (8 * NT);
  const bool live = task < r.G * 8 * NT;
  uint32_t sw = 0u;
  if (live && m < r.M) sw = rot_sign_bits(r.sign_bits, grp, lane);
  grid_dependency_wait();
  if (!live) return;  // warp-uniform
  uint8_t* row = rowbuf[warp];
  float sum = 0.f;
  if (m < r.M) {
    uint32_t h[4];
    h16_fragment(lane, h);
    const __half* xp = r.x + (size_t)m * r.K + (size_t)grp * kHadamard + 16 * g + 2 * t;
    const uint32_t b0 = *reinterpret_cast<const uint32_t*>(xp), b1 = *reinterpret_cast<const uint32_t*>(xp + 8);
    __half hv[4];
    float f[4];
    rotate_block16x8(b0, b1, sw, h, lane, hv, f);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int chunk, half;
      x_slot<B>(g + 32 * t + rot_off(i), chunk, half);
      reinterpret_cast<__half*>(row + ((chunk ^ (m & 7)) << 4))[half] = hv[i];
    }
    sum = (f[0] + f[1]) + (f[2] + f[3]);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  } else {
    reinterpret_cast<uint2*>(row)[lane] = make_uint2(0u, 0u);
  }
  __syncwarp();
  if (lane < 16)
    reinterpret_cast<uint4*>(r.xrot + (size_t)grp * NT * 2048 + (m >> 3) * 2048 + (m & 7) * 256)[lane] =
        reinterpret_cast<const uint4*>(row)[lane];
  if (lane == 0) r.xsum_g[grp * 16 + m] = sum;
}

// ------------------------------------------------------------- host plan --

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn lookup_encode() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<EncodeTiledFn>(fn);
  return nullptr;
}

EncodeTiledFn tc_encode_fn() {
  static const EncodeTiledFn fn = lookup_encode();
  return fn;
}

// Slice lengths for S slices of G groups: the first nhi of length L, the rest
// L - d; odd lengths when `odd` (then S must have the parity of G).
bool slice_lengths(int G, int S, bool odd, int& L, int& d, int& nhi) {
  const int c = (G + S - 1) / S;
  if (!odd) {
    L = c;
    d = 1;
    nhi = G - S * (c - 1);
    return true;
  }
  if ((G - S) % 2) return false;
  L = (c % 2) ? c : c + 1;
  d = 2;
  if (L == 1) {
    nhi = S;
    return G == S;
  }
  nhi = (G - S * (L - 2)) / 2;
  return nhi >= 0 && nhi <= S;
}

bool make_tc_plan(int B, int N, int K, int M, TcPlan& p) {
  if (B != 3 && B != 4 && B != 6 && B != 8) return false;
  if (M < 1 || M > 16 || N < 1 || K < kGroup || K % kGroup) return false;
  p = TcPlan{};
  p.T = (N + kTileRows - 1) / kTileRows;
  p.G = K / kGroup;
  p.NT = M <= 8 ? 1 : 2;
  const int xs_per_group = p.NT * 2048;
  const int red_bytes = kW * 3 * kTileRows * (8 * p.NT + 1) * 4;
  double best = -1.0;
  for (int S = 1; S <= std::min(p.G, kMaxCluster); ++S) {
    int L, d, nhi;
    if (!slice_lengths(p.G, S, B != 8, L, d, nhi)) continue;
    if (16 * B * L > 2048) continue;  // TMA box: at most 256 eight-byte elements per row
    const int P = std::min(p.T, kClustersAtOnce[S]);
    const int Tc = (p.T + P - 1) / P;
    const int U = Tc * L;
    const int uw = (U + kW - 1) / kW;
    // busiest CTA: code bytes of its busiest warp times the warps, plus (S > 1)
    // the cluster's sum: two cluster barriers, each worth about 4 KB of
    // streaming, and the slices' sums read from distributed shared memory
    const double cost = (double)uw * kW * kTileRows * 16 * B +
                        (S > 1 ? 8192.0 + (double)Tc * kTileRows * 8 * p.NT * 4 : 0.0);
    // shared memory
    const int tile_bytes = kTileRows * 16 * B * L;
    const int fixed = L * xs_per_group + ((L * 64 + 127) & ~127) + red_bytes + 64;
    // per round tile: scale/zero pairs, the slice's tile sums (S > 1), the codes
    auto per_tiles = [&](int k) {
      return ((k * kTileRows * L * 4 + 127) & ~127) + (S > 1 ? ((k * kTileRows * 8 * p.NT * 4 + 127) & ~127) : 0);
    };
    int RT, nbuf;
    if (fixed + per_tiles(Tc) + Tc * tile_bytes <= kSmemMax) {
      RT = Tc;
      nbuf = 1;
    } else {
      RT = 0;
      for (int k = Tc; k >= 1; --k) {
        if (fixed + per_tiles(k) + 2 * k * tile_bytes <= kSmemMax) {
          RT = k;
          break;
        }
      }
      if (RT == 0) continue;
      nbuf = 2;
    }
    if (best < 0.0 || cost < best) {
      best = cost;
      p.S = S;
      p.P = P;
      p.L = L;
      p.d = d;
      p.nhi = nhi;
      p.Tc = Tc;
      p.RT = RT;
      p.nbuf = nbuf;
    }
  }
  if (best < 0.0) return false;
  const int L = p.L;
  p.buf_bytes = p.RT * kTileRows * 16 * B * L;
  p.off_xsum = L * xs_per_group;
  p.off_sz = (p.off_xsum + L * 64 + 127) & ~127;
  p.off_red = (p.off_sz + p.RT * kTileRows * L * 4 + 127) & ~127;
  p.off_cp = (p.off_red + red_bytes + 127) & ~127;
  const int cp_bytes = p.S > 1 ? p.RT * kTileRows * 8 * p.NT * 4 : 0;
  p.off_codes = (p.off_cp + cp_bytes + 127) & ~127;
  p.off_bar = p.off_codes + p.nbuf * p.buf_bytes;
  p.smem_bytes = p.off_bar + 64;
  if (p.smem_bytes > kSmemMax) return false;
  // M >= 2: x rotated once per call (in-kernel rotation would repeat the
  // slice's M x L blocks in each of the P CTAs that share it)
  p.xrot = M >= 2 ? 1 : 0;
  p.ws_xs = 0;
  p.ws_xsum = (size_t)p.G * p.NT * 2048;
  p.ws_total = p.xrot ? p.ws_xsum + (size_t)p.G * 64 : 0;
  return true;
}

template <int B, int NT>
qlin_status launch_tc_kernel(const TcArgs& a, cudaStream_t st) {
  static std::atomic<unsigned long long> configured{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda(e);
  if (dev >= 64 || !((configured.load(std::memory_order_acquire) >> dev) & 1ull)) {
    e = cudaFuncSetAttribute(gemv_tc_kernel<B, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax);
    if (e != cudaSuccess) return record_cuda(e);
    if (dev < 64) configured.fetch_or(1ull << dev, std::memory_order_release);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.p.P * a.p.S);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = a.p.smem_bytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (a.p.S > 1) {  // the K slices of a row part (consecutive blocks) form one cluster
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = (unsigned)a.p.S;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (overlap_enabled()) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return record_cuda(cudaLaunchKernelEx(&cfg, gemv_tc_kernel<B, NT>, a));
}

template <int B, int NT>
qlin_status launch_rot_kernel(const RotArgs& r, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((r.G * 8 * NT + kW - 1) / kW);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = overlap_enabled() ? 1 : 0;
  return record_cuda(cudaLaunchKernelEx(&cfg, rot_tc_kernel<B, NT>, r));
}

template <int B, int NT>
qlin_status launch_tc_nt(const TcArgs& a, const RotArgs& r, cudaStream_t st) {
  if (a.p.xrot) {
    const qlin_status q = launch_rot_kernel<B, NT>(r, st);
    if (q != QLIN_OK) return q;
  }
  return launch_tc_kernel<B, NT>(a, st);
}

template <int B>
qlin_status launch_tc_bits(const TcArgs& a, const RotArgs& r, cudaStream_t st) {
  return a.p.NT == 1 ? launch_tc_nt<B, 1>(a, r, st) : launch_tc_nt<B, 2>(a, r, st);
}

}  // namespace

bool gemv_tc_fits(int bits, int N, int K, int M) {
  TcPlan p;
  return make_tc_plan(bits, N, K, M, p);
}

size_t gemv_tc_workspace_bytes(int bits, int N, int K, int M) {
  TcPlan p;
  return make_tc_plan(bits, N, K, M, p) ? p.ws_total : 0;
}

qlin_status launch_gemv_tc(const PackedView& v, const __half* scales, const __half* zeros, const uint32_t* sign_bits,
                           const __half* x, __half* y, int M, void* workspace, cudaStream_t st) {
  TcArgs a;
  if (!make_tc_plan(v.bits, v.N, v.K, M, a.p)) return QLIN_ERR_UNSUPPORTED;
  if (a.p.ws_total && workspace == nullptr) return QLIN_ERR_WORKSPACE;
  const int B = v.bits;
  EncodeTiledFn enc = tc_encode_fn();
  if (!enc) return record_cuda(cudaErrorNotSupported);
  // the codes as rows of 8-byte elements: 2 B elements per group
  const cuuint64_t dims[2] = {(cuuint64_t)(2 * B) * (cuuint64_t)a.p.G, (cuuint64_t)v.N};
  const cuuint64_t strides[1] = {(cuuint64_t)v.row_bytes_uniform};
  const cuuint32_t estr[2] = {1, 1};
  const int lens[2] = {a.p.L, std::max(1, a.p.L - a.p.d)};
  CUtensorMap* maps[2] = {&a.map_hi, &a.map_lo};
  for (int i = 0; i < 2; ++i) {
    const cuuint32_t box[2] = {(cuuint32_t)(2 * B * lens[i]), (cuuint32_t)kTileRows};
    const CUresult cr = enc(maps[i], CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<uint8_t*>(v.codes), dims, strides,
                            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return record_cuda(cudaErrorInvalidValue);
  }
  a.scales = scales;
  a.zeros = zeros;
  a.sign_bits = sign_bits;
  a.x = x;
  a.y = y;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.xrot = a.p.xrot ? ws + a.p.ws_xs : nullptr;
  a.xsum_g = a.p.xrot ? reinterpret_cast<const float*>(ws + a.p.ws_xsum) : nullptr;
  a.N = v.N;
  a.K = v.K;
  a.M = M;
  RotArgs r = {};
  if (a.p.xrot) {
    r.x = x;
    r.sign_bits = sign_bits;
    r.xrot = ws + a.p.ws_xs;
    r.xsum_g = reinterpret_cast<float*>(ws + a.p.ws_xsum);
    r.M = M;
    r.K = v.K;
    r.G = a.p.G;
    r.pf[0] = v.codes;
    r.pf_bytes[0] = (size_t)v.N * (size_t)v.row_bytes_uniform;
    r.pf[1] = scales;
    r.pf[2] = zeros;
    r.pf_bytes[1] = r.pf_bytes[2] = (size_t)v.N * (size_t)a.p.G * 2;
  }
  switch (B) {
    case 3: return launch_tc_bits<3>(a, r, st);
    case 4: return launch_tc_bits<4>(a, r, st);
    case 6: return launch_tc_bits<6>(a, r, st);
    default: return launch_tc_bits<8>(a, r, st);
  }
}

void gemv_tc_plan_info(int bits, int N, int K, int M, qlin_gemv_plan_info* info) {
  TcPlan p;
  *info = qlin_gemv_plan_info{};
  if (!make_tc_plan(bits, N, K, M, p)) return;
  info->kernel = 4;
  info->grid = p.P * p.S;
  info->threads = kThreads;
  info->smem_bytes = p.smem_bytes;
  info->consumer_warps = kW;
  info->rows_per_cta = p.Tc * kTileRows;
  info->rows_per_chunk = kTileRows;
  info->stages = p.nbuf;
  info->chunks_in_flight = p.RT;
  info->workspace_bytes = p.ws_total;
}

unsigned take_tc_error() {
  unsigned v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_tc_error, sizeof(v)) != cudaSuccess) return ~0u;
  if (v) cudaMemcpyToSymbol(g_tc_error, &zero, sizeof(zero));
  return v;
}

}  // namespace qlin

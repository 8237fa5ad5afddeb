// qlin_gemm: prefill-regime quantised linear layer on the 5th-generation tensor
// cores (tcgen05, operands and accumulators in tensor memory).
//
// Y = rht(X) . dequant(W)^T.  The activations are rotated into the workspace
// by the stand-alone rotation kernel; the weight is dequantised exactly as
// qlin_dequant does (fp32 subtract and multiply, one rounding to fp16) straight
// into tensor memory, inside the main loop, and never reaches global memory
// ("24B0978-Week01-Track2_20-Submission01", "How these techniques accelerate
// inference on CUDA").
//
// Tiling (one CTA per SM, persistent over output tiles):
//   MMA  D[128 weight rows][BN activation rows] += A[128][64] . B[BN][64]^T
//   A = dequantised weight rows in tensor memory (row m in lane m, two fp16
//       along K per 32-bit column), one 32-column slot per pipeline stage,
//       written by 8 dequantisation warps with tcgen05.st;
//   B = rotated activations in shared memory, K-major, 128-byte swizzle,
//       loaded by TMA;
//   D = fp32 in tensor memory, columns [0, BN).
// Warp roles: 0 TMA producer, 1 MMA issuer (one thread) and TMEM owner,
// 4..7 epilogue (TMEM lane quarters 0..3), 8..15 dequantisation.
// The epilogue converts the tile to fp16 into a whole-tile staging buffer,
// hands the accumulator back to the MMA, and stores the buffer with one TMA
// store while the MMA already runs the next tile (three B stages leave room
// for the buffer).
// Dequantisation warp 8 + j owns TMEM lane quarter q = j % 4 (weight rows
// 32q .. 32q+31 of the tile, one per thread) and the stages of parity h = j / 4
// (codes [64h, 64h + 64) of every 128-code group).  Each thread copies its own
// row's 64-code piece and the group's scale and zero kRing groups ahead
// (16-byte cp.async into a private ring slot), so the dequantisation warps
// never wait for one another; results go to tensor memory, which the MMA reads
// without a proxy fence.
// The weight tile is the MMA's M side because dequantisation costs ALU work
// per weight element per activation tile: with 256 activation rows per tile
// each weight element is dequantised once per 256 rows of X.
#include <cuda.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "qlin_internal.cuh"
#include "qlin_sm100.cuh"

namespace qlin {

__device__ unsigned int g_gemm_error;

namespace {

constexpr int kStages = 3;
constexpr int kBK = 64;        // k per stage: 64 fp16 = one 128-byte swizzle row of B
constexpr int kBMw = 128;      // weight rows per tile (MMA M)
constexpr int kBNmax = 256;    // activation rows per tile (MMA N)
constexpr int kBStage = kBNmax * kBK * 2;   // 32 KB
constexpr int kThreads = 512;
constexpr int kDeqWarp0 = 8, kDeqWarps = 8;
constexpr int kDeqThreads = kDeqWarps * 32;
constexpr int kEpiWarp0 = 4;
constexpr int kTmemCols = 512;
constexpr int kAccCol = 0;     // accumulator: columns [0, BN)
constexpr int kACol = 256;     // A of stage s: columns [kACol + 32 s, kACol + 32 s + 32)
constexpr int kRing = 3;       // 128-code groups in flight per dequantisation thread
constexpr int kSms = 148;
constexpr int kSlot = 80;      // bytes per thread per group: piece at 0, scale/zero pairs at 64/68 (stride 5 x 16 B: no bank conflicts)
constexpr int kRingBytes = kRing * kDeqThreads * kSlot;   // 80 KB
constexpr int kStageOut = kBNmax * kBMw * 2;             // Y staging: a whole tile, up to 256 activation rows x 128 weight rows, fp16
constexpr int kSmemBytes = kStages * kBStage + kRingBytes + kStageOut + 1024 /*barriers*/ + 1024 /*align*/;

struct GemmArgs {
  PackedView v;
  const __half* scales;
  const __half* zeros;
  __half* y;
  int M, BN, m_tiles, n_tiles, KB;
  // Stream-K schedule (stream_k != 0): CTA c takes the 128-code groups
  // [c T / P, (c+1) T / P) of the T = tiles * G (tile, group) pairs in tile
  // order, P = gridDim.x.  A tile split between CTAs is finished by the CTA
  // holding its first groups, which adds the other CTAs' fp32 partial sums
  // (partials[c]: [BN][128], flag[c] = 1 when written) in CTA order.
  int stream_k;
  uint32_t* flags;   // [P], zero on entry (cleared by the rotation kernel), zero on exit
  float* partials;   // [P][part_cols][128]
  int part_cols;     // BN rounded up to the 32 columns one TMEM load covers
  int tma_store;     // Y written by TMA tensor stores through shared memory (N % 8 == 0)
  int box_m;         // activation rows per store box: BN (one store per tile)
};

// The (tile, group range) segments one CTA works through, in order.
struct Segments {
  int G, tiles, stream_k;
  long long it, end;  // stream-K: group cursor and end
  int t;              // data-parallel: tile cursor
  __device__ void init(const GemmArgs& a) {
    G = a.v.K / kGroup;
    tiles = a.m_tiles * a.n_tiles;
    stream_k = a.stream_k;
    const long long T = (long long)tiles * G, P = gridDim.x;
    it = T * blockIdx.x / P;
    end = T * (blockIdx.x + 1) / P;
    t = blockIdx.x;
  }
  // Next segment: tile t, groups [g0, g1); false when done.
  __device__ bool next(int& tile, int& g0, int& g1) {
    if (!stream_k) {
      if (t >= tiles) return false;
      tile = t;
      g0 = 0;
      g1 = G;
      t += gridDim.x;
      return true;
    }
    if (it >= end) return false;
    tile = (int)(it / G);
    g0 = (int)(it % G);
    g1 = (int)min((long long)G, g0 + (end - it));
    it += g1 - g0;
    return true;
  }
};

__device__ __forceinline__ long long sk_start(long long T, int P, int c) { return T * c / P; }

__device__ __forceinline__ void gemm_fail(unsigned code) { atomicOr(&g_gemm_error, code); }

__device__ __forceinline__ void wait_or_fail(uint64_t* bar, uint32_t parity, unsigned code) {
  if (!mbar_wait(bar, parity, &g_gemm_error)) gemm_fail(code);
}

// ---- tcgen05 / TMA wrappers ----

__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
  // K-major, 128-byte swizzle: rows of 128 B, 8-row groups 1024 B apart (SBO),
  // LBO unused (encoded 1), descriptor version 1, layout type 2.
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

// D (tensor memory) += A (tensor memory) . B (shared memory descriptor)
__device__ __forceinline__ void umma_f16_ts(uint32_t dtmem, uint32_t atmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(dtmem),
      "r"(atmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_addr(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// This thread's lane of the warp's TMEM quarter, 32 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}

// Tensor store of a shared-memory box to global memory (out-of-range parts are
// not written), and the waits on such stores.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_addr(src)), "r"(x), "r"(y)
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void tma_store_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void tma_store_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_async_shared() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ---- cp.async (per-thread asynchronous copies into shared memory) ----
template <int kBytes>
__device__ __forceinline__ void cp_async(void* dst, const void* src) {
  if constexpr (kBytes == 16)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(smem_addr(dst)), "l"(src), "n"(kBytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// ---- packed fp32 pairs (each lane of the pair rounded as its scalar op) ----
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void upk2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// ---- one row's 128-code group: copy its 64-code piece of parity h ----
// The piece holds codes [64 h, 64 h + 64): 8b bytes at byte 8 b h of the group
// (16 b bytes per group from the row start); it lands at byte 0 of the
// thread's ring slot.  The 4-byte words holding the group's scale and zero
// (fp16 pairs, aligned) land at bytes 64 and 68.
template <int B>
__device__ __forceinline__ void copy_piece(uint8_t* slot, const uint8_t* grp, int h) {
  const uint8_t* src = grp + 8 * B * h;
  if constexpr (B == 3) {
#pragma unroll
    for (int i = 0; i < 3; ++i) cp_async<8>(slot + 8 * i, src + 8 * i);
  } else {
#pragma unroll
    for (int i = 0; i < B / 2; ++i) cp_async<16>(slot + 16 * i, src + 16 * i);
  }
}

__device__ __forceinline__ void copy_piece_any(int b, uint8_t* slot, const uint8_t* grp, int h) {
  switch (b) {
    case 3: copy_piece<3>(slot, grp, h); break;
    case 4: copy_piece<4>(slot, grp, h); break;
    case 6: copy_piece<6>(slot, grp, h); break;
    default: copy_piece<8>(slot, grp, h); break;
  }
}

// ---- exact dequantisation of one 64-code piece (from the thread's ring slot) ----
// Codes are cut out two at a time into the halves of a 32-bit word, each half
// the 16-bit pattern m q with m a power of two (m q < 2048); one mixed-precision
// fused multiply-add per code then gives fp32(q - z) 2^-9 and a packed multiply
// by s 2^9 gives fp32(s t): the same two roundings as dequant_exact (see
// fma_f16_f32 there), then fp16.  Which codes share a word depends on the
// width:
//   8 bits: bytes (4j + e, 4j + e + 1) of word j by one byte permute;
//   4 bits: nibbles (8j + i, 8j + i + 4) of word j by one AND with 0x000F000F or
//           0x00F000F0 (m = 1 or 16), half of them after a shift by 8;
//   3 bits: codes (i, i + 8) from 27 bits starting at code i, AND 0x07000007
//           (m = 1 and 256), for i = 16a + r, r < 8;
//   6 bits: codes (i, i + 3), AND 0x00FC003F (m = 1 and 4), for i = 6a + r,
//           r < 3, a < 10, and (60, 63); codes 61 and 62 by shifts.
template <int B>
__device__ __forceinline__ void dequant_piece(const uint8_t* piece, float s, float z, uint32_t (&out)[32]) {
  uint32_t w[2 * B + 1];
  if constexpr (B == 3) {
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      const uint2 v = *reinterpret_cast<const uint2*>(piece + 8 * i);
      w[2 * i] = v.x; w[2 * i + 1] = v.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < B / 2; ++i) {
      const uint4 v = *reinterpret_cast<const uint4*>(piece + 16 * i);
      w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
    }
  }
  w[2 * B] = 0;
  // bits [bit, bit + 32) of the piece (zeros past its end)
  auto bits_from = [&](int bit) -> uint32_t {
    return (bit & 31) == 0 ? w[bit >> 5] : __funnelshift_r(w[bit >> 5], w[(bit >> 5) + 1], bit & 31);
  };
  const float zq = -z * 0x1p-9f;
  float t[64];
  if constexpr (B == 8) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      fma_f16x2_f32(__byte_perm(w[j], 0u, 0x4140u), kMul15, kMul15, zq, t[4 * j], t[4 * j + 1]);
      fma_f16x2_f32(__byte_perm(w[j], 0u, 0x4342u), kMul15, kMul15, zq, t[4 * j + 2], t[4 * j + 3]);
    }
  } else if constexpr (B == 4) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t v = w[j] >> 8;
      fma_f16x2_f32(w[j] & 0x000F000Fu, kMul15, kMul15, zq, t[8 * j], t[8 * j + 4]);
      fma_f16x2_f32(w[j] & 0x00F000F0u, kMul11, kMul11, zq, t[8 * j + 1], t[8 * j + 5]);
      fma_f16x2_f32(v & 0x000F000Fu, kMul15, kMul15, zq, t[8 * j + 2], t[8 * j + 6]);
      fma_f16x2_f32(v & 0x00F000F0u, kMul11, kMul11, zq, t[8 * j + 3], t[8 * j + 7]);
    }
  } else if constexpr (B == 3) {
#pragma unroll
    for (int a = 0; a < 4; ++a) {
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int i = 16 * a + r;
        fma_f16x2_f32(bits_from(3 * i) & 0x07000007u, kMul15, kMul7, zq, t[i], t[i + 8]);
      }
    }
  } else {
#pragma unroll
    for (int a = 0; a < 10; ++a) {
#pragma unroll
      for (int r = 0; r < 3; ++r) {
        const int i = 6 * a + r;
        fma_f16x2_f32(bits_from(6 * i) & 0x00FC003Fu, kMul15, kMul13, zq, t[i], t[i + 3]);
      }
    }
    const uint32_t v = w[11] >> 8;  // codes 60..63
    fma_f16x2_f32(v & 0x00FC003Fu, kMul15, kMul13, zq, t[60], t[63]);
    fma_f16x2_f32(((v >> 6) & 0x3Fu) | ((v << 4) & 0x003F0000u), kMul15, kMul15, zq, t[61], t[62]);
  }
  const uint64_t ss = pk2(s * 512.0f, s * 512.0f);
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    float p0, p1;
    upk2(mul2(ss, pk2(t[2 * i], t[2 * i + 1])), p0, p1);
    __half2 h = __floats2half2_rn(p0, p1);
    out[i] = *reinterpret_cast<uint32_t*>(&h);
  }
}

__device__ __forceinline__ void dequant_piece_any(int b, const uint8_t* piece, float s, float z, uint32_t (&out)[32]) {
  switch (b) {
    case 3: dequant_piece<3>(piece, s, z, out); break;
    case 4: dequant_piece<4>(piece, s, z, out); break;
    case 6: dequant_piece<6>(piece, s, z, out); break;
    default: dequant_piece<8>(piece, s, z, out); break;
  }
}

// fp16 element `idx` of an array, from the aligned 4-byte word holding it.
__device__ __forceinline__ float half_of_pair(uint32_t word, int idx) {
  const uint16_t bits = (idx & 1) ? (uint16_t)(word >> 16) : (uint16_t)(word & 0xFFFFu);
  return __half2float(__ushort_as_half(bits));
}

__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ CUtensorMap xmap,
                                                              const __grid_constant__ CUtensorMap ymap,
                                                              const __grid_constant__ GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* Bs = smem;
  uint8_t* ring = Bs + kStages * kBStage;
  __half* ystage = reinterpret_cast<__half*>(ring + kRingBytes);  // [BN][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + kRingBytes + kStageOut);
  uint64_t* st_empty = bars;
  uint64_t* a_full = bars + kStages;
  uint64_t* b_full = bars + 2 * kStages;
  uint64_t* acc_full = bars + 3 * kStages;
  uint64_t* acc_empty = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles = a.m_tiles * a.n_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&st_empty[s], 1);
      mbar_init(&a_full[s], kDeqWarps / 2);  // one warp per lane quarter writes each stage
      mbar_init(&b_full[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 4);
    mbar_fence_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      grid_dependency_wait();  // the rotated activations are the rotation kernel's output
      int g = 0, t, g0, g1;
      Segments sg;
      sg.init(a);
      while (sg.next(t, g0, g1)) {
        const int m0 = (t % a.m_tiles) * a.BN;
        for (int kb = 2 * g0; kb < 2 * g1; ++kb, ++g) {
          const int s = g % kStages, u = g / kStages;
          if (u > 0) wait_or_fail(&st_empty[s], (u - 1) & 1, 1u);
          mbar_arrive_expect_tx(&b_full[s], (uint32_t)a.BN * kBK * 2);
          tma_load_2d(Bs + s * kBStage, &xmap, kb * kBK, m0, &b_full[s]);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      // kind::f16, fp32 accumulate, fp16 A and B, both K-major, M = 128, N = BN.
      const uint32_t idesc = (1u << 4) | ((uint32_t)(a.BN >> 3) << 17) | ((uint32_t)(kBMw >> 4) << 24);
      const uint32_t dtmem = tmem_base + kAccCol;
      int g = 0, i = 0, t, g0, g1;
      Segments sg;
      sg.init(a);
      for (; sg.next(t, g0, g1); ++i) {
        if (i > 0) wait_or_fail(acc_empty, (i - 1) & 1, 2u);
        tc_fence_after();
        for (int kb = 2 * g0; kb < 2 * g1; ++kb, ++g) {
          const int s = g % kStages, u = g / kStages;
          wait_or_fail(&a_full[s], u & 1, 4u);
          wait_or_fail(&b_full[s], u & 1, 8u);
          tc_fence_after();
          const uint32_t atmem = tmem_base + (uint32_t)(kACol + 32 * s);
          const uint64_t bd = umma_desc_sw128(smem_addr(Bs + s * kBStage));
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)  // 16 fp16 = 8 TMEM columns of A, 32 bytes = 2 descriptor units of B
            umma_f16_ts(dtmem, atmem + 8u * k, bd + 2u * k, idesc, (kb > 2 * g0 || k > 0) ? 1u : 0u);
          umma_commit(&st_empty[s]);
        }
        umma_commit(acc_full);
      }
    }
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 4) {
    // --------------------------------------------------------- epilogue --
    const int q = warp & 3;  // TMEM lanes 32q..32q+31 = weight rows of the tile
    const int row = 32 * q + lane;
    grid_dependency_wait();  // the completion flags are cleared by the rotation kernel
    const long long T = (long long)tiles * (a.v.K / kGroup);
    const int G = a.v.K / kGroup, P = gridDim.x, c = blockIdx.x;
    // The accumulator is handed back to the MMA as soon as this warp has
    // loaded its last columns: the rest of the epilogue (partial sums,
    // conversion, stores) overlaps the next tile's MMAs.
    auto release_acc = [&]() {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
    };
    int i = 0, t, g0, g1;
    Segments sg;
    sg.init(a);
    for (; sg.next(t, g0, g1); ++i) {
      const int m0 = (t % a.m_tiles) * a.BN;
      const int n0 = (t / a.m_tiles) * kBMw;
      const int n = n0 + row;
      wait_or_fail(acc_full, i & 1, 16u);
      tc_fence_after();
      if (g0 > 0) {
        // a later part of a split tile: hand the fp32 partial to the tile's owner
        float* dst = a.partials + (size_t)c * a.part_cols * kBMw + row;
        for (int c0 = 0; c0 < a.BN; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(kAccCol + c0), r);
          if (c0 + 32 >= a.BN) release_acc();
#pragma unroll
          for (int j = 0; j < 32; ++j) dst[(size_t)(c0 + j) * kBMw] = __uint_as_float(r[j]);
        }
        __threadfence();
        named_barrier(3, 128);
        if (q == 0 && lane == 0)
          asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(a.flags + c), "r"(1u) : "memory");
      } else {
        if (a.tma_store) {  // the staging buffer may still be read by the previous tile's store
          if (q == 0 && lane == 0) tma_store_wait_read();
          named_barrier(3, 128);
        }
        // the tile's contributors after this CTA (stream-K split): CTAs whose
        // groups overlap [g1, G) of this tile
        int c_last = c;
        if (g1 < G)
          while (c_last + 1 < P && sk_start(T, P, c_last + 1) < (long long)(t + 1) * G) ++c_last;
        for (int cc = c + 1; cc <= c_last; ++cc) {
          if (lane == 0) {
            uint32_t f = 0;
            const uint64_t t0 = globaltimer_ns();
            while (true) {
              asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(f) : "l"(a.flags + cc) : "memory");
              if (f || g_gemm_error) break;
              if (globaltimer_ns() - t0 > kWaitLimitNs) {
                gemm_fail(64u);
                break;
              }
            }
          }
          __syncwarp();
          // acquire in every lane before its loads of the partial
          asm volatile("{\n\t.reg .b32 f;\n\tld.acquire.gpu.global.u32 f, [%0];\n\t}" ::"l"(a.flags + cc) : "memory");
        }
        // The later contributors' partials, one (chunk, contributor) after the
        // other in that order, each loaded while the one before is added.
        const int ncon = c_last - c, nk = ncon * ((a.BN + 31) / 32);
        float nxt[32];
        auto load_part = [&](int k) {
          const float* src =
              a.partials + (size_t)(c + 1 + k % ncon) * a.part_cols * kBMw + (size_t)(32 * (k / ncon)) * kBMw + row;
#pragma unroll
          for (int j = 0; j < 32; ++j) nxt[j] = __ldcg(src + (size_t)j * kBMw);
        };
        if (nk > 0) load_part(0);
        for (int c0 = 0, k = 0; c0 < a.BN; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(kAccCol + c0), r);
          float acc[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) acc[j] = __uint_as_float(r[j]);
          for (int cc = 0; cc < ncon; ++cc, ++k) {
#pragma unroll
            for (int j = 0; j < 32; ++j) acc[j] += nxt[j];
            if (k + 1 < nk) load_part(k + 1);
          }
          if (a.tma_store) {
            // the whole tile is staged (fp16, [m][n]) and stored by one thread
            // after the last chunk, while the MMA already runs the next tile
#pragma unroll
            for (int j = 0; j < 32; ++j) ystage[(c0 + j) * kBMw + row] = __float2half_rn(acc[j]);
          } else if (n < a.v.N) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int m = m0 + c0 + j;
              if (m < a.M) a.y[(size_t)m * a.v.N + n] = __float2half_rn(acc[j]);
            }
          }
        }
        release_acc();  // every column of the accumulator has been loaded
        if (a.tma_store) {
          fence_async_shared();
          named_barrier(3, 128);
          if (q == 0 && lane == 0) tma_store_2d(&ymap, ystage, n0, m0);
        }
        if (c_last > c) {
          named_barrier(3, 128);  // every epilogue warp has read the partials
          if (q == 0 && lane == 0)
            for (int cc = c + 1; cc <= c_last; ++cc) a.flags[cc] = 0u;
        }
      }
    }
    if (a.tma_store && q == 0 && lane == 0) tma_store_wait_all();
  } else if (warp >= kDeqWarp0) {
    // ---------------------------------------------------- dequantisation --
    const int j = warp - kDeqWarp0;
    const int q = j & 3, h = j >> 2;    // TMEM lane quarter (warp % 4) and stage parity
    const int r = 32 * q + lane;        // this thread's weight row in the tile
    const int dt = threadIdx.x - kDeqWarp0 * 32;
    const int G = a.v.K / kGroup;
    const uint32_t tq = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)kACol;
    // copy cursor: the (tile, group) items of this CTA's segments, in order;
    // this thread's row in tile ct, its width and its scale/zero row
    Segments cs;
    cs.init(a);
    int ct = 0, cg = 0, cg1 = 0, cb = 4;
    bool cmore = cs.next(ct, cg, cg1);
    const uint8_t* crow = nullptr;
    size_t csz = 0;
    int ci = 0;
    auto set_copy_tile = [&]() {
      const int n = (ct / a.m_tiles) * kBMw + r;
      crow = nullptr;
      if (cmore && n < a.v.N) {
        crow = reinterpret_cast<const uint8_t*>(row_of(a.v, n, cb));
        csz = (size_t)n * G;
      }
    };
    auto issue = [&]() {  // copies of item ci into ring slot ci % kRing, one commit group
      if (cmore && crow != nullptr) {
        uint8_t* slot = ring + (size_t)(ci % kRing) * kDeqThreads * kSlot + dt * kSlot;
        copy_piece_any(cb, slot, crow + (size_t)cg * 16 * cb, h);
        const size_t e = (csz + cg) & ~(size_t)1;
        cp_async<4>(slot + 64, a.scales + e);
        cp_async<4>(slot + 68, a.zeros + e);
      }
      cp_async_commit();
      if (cmore) {
        ++ci;
        if (++cg == cg1) {
          cmore = cs.next(ct, cg, cg1);
          set_copy_tile();
        }
      }
    };
    set_copy_tile();
#pragma unroll 1
    for (int k = 0; k < kRing - 1; ++k) issue();
    int it = 0, t, g0, g1;
    Segments sg;
    sg.init(a);
    while (sg.next(t, g0, g1)) {
      const int n = (t / a.m_tiles) * kBMw + r;
      const bool valid = n < a.v.N;
      int b = 4;
      if (valid) (void)row_of(a.v, n, b);
      for (int gi = g0; gi < g1; ++gi, ++it) {
        issue();                     // item it + kRing - 1
        cp_async_wait<kRing - 1>();  // this thread's copies of item `it` have landed
        const uint8_t* slot = ring + (size_t)(it % kRing) * kDeqThreads * kSlot + dt * kSlot;
        const int g = 2 * it + h;    // pipeline stage of this piece
        const int s = g % kStages, u = g / kStages;
        uint32_t out[32];
        if (valid) {
          const int e = (int)(((size_t)n * G + gi) & 1);
          const float sc = half_of_pair(*reinterpret_cast<const uint32_t*>(slot + 64), e);
          const float zc = half_of_pair(*reinterpret_cast<const uint32_t*>(slot + 68), e);
          dequant_piece_any(b, slot, sc, zc, out);
        } else {
#pragma unroll
          for (int i2 = 0; i2 < 32; ++i2) out[i2] = 0u;
        }
        if (u > 0) wait_or_fail(&st_empty[s], (u - 1) & 1, 32u);
        tc_fence_after();
        tmem_st32(tq + (uint32_t)(32 * s), out);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[s]);
      }
    }
    cp_async_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                 : "memory");
}

// ---- host side ----

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn lookup_encode_fn() {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<EncodeTiledFn>(p);
  return nullptr;
}

// The driver's tensor-map encoder, looked up once (a function-local static is
// initialised exactly once even when several host threads call at once).
EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = lookup_encode_fn();
  return fn;
}

}  // namespace

// Workspace of qlin_gemm: the rotated activations, then the stream-K
// completion flags and partial sums.
struct GemmWorkspace {
  size_t xr_bytes, flags_off, part_off, total;
  GemmWorkspace(int M, int K) {
    const int BN = std::min(kBNmax, (M + 15) / 16 * 16);
    xr_bytes = ((size_t)M * K * 2 + 255) & ~(size_t)255;
    flags_off = xr_bytes;
    part_off = flags_off + 1024;
    total = part_off + (size_t)kSms * ((BN + 31) & ~31) * kBMw * 4;
  }
};

size_t gemm_workspace_bytes(int M, int K) { return GemmWorkspace(M, K).total; }

// The GEMM proper, on activations already rotated into xr (M x K fp16).
// flags/partials: the stream-K scratch (both null: one CTA per tile instead).
qlin_status launch_gemm_rotated(const PackedView& v, const __half* scales, const __half* zeros, const __half* xr,
                                __half* y, int M, cudaStream_t s, uint32_t* flags, float* partials) {
  GemmArgs a;
  a.v = v;
  a.scales = scales;
  a.zeros = zeros;
  a.y = y;
  a.M = M;
  a.BN = std::min(kBNmax, (M + 15) / 16 * 16);
  a.m_tiles = (M + a.BN - 1) / a.BN;
  a.n_tiles = (v.N + kBMw - 1) / kBMw;
  a.KB = v.K / kBK;
  // Stream-K unless the tiles alone already fill at least half of the SMs and
  // a split tile's partial sum would be large (BN >= 192: a split costs the
  // owner ~4 us of waiting for and adding 96-128 KB): then one CTA per tile
  // (prefill M = 256: 33.0 instead of 35.3 us; at M = 32 or 512 stream-K wins).
  {
    const long long tiles = (long long)a.m_tiles * a.n_tiles;
    const bool per_tile = a.BN >= 192 && tiles <= kSms && 2 * tiles >= kSms;
    a.stream_k = (flags != nullptr && !per_tile) ? 1 : 0;
  }
  a.part_cols = (a.BN + 31) & ~31;
  a.flags = flags;
  a.partials = partials;

  EncodeTiledFn enc = encode_fn();
  if (!enc) return record_cuda(cudaErrorNotSupported);
  CUtensorMap map;
  const cuuint64_t dims[2] = {(cuuint64_t)v.K, (cuuint64_t)M};
  const cuuint64_t strides[1] = {(cuuint64_t)v.K * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)a.BN};
  const cuuint32_t estr[2] = {1, 1};
  CUresult cr = enc(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<__half*>(xr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return record_cuda(cudaErrorInvalidValue);
  // Y [M][N] fp16: tensor stores need rows of a multiple of 16 bytes
  CUtensorMap ymap;
  a.box_m = a.BN;
  a.tma_store = (v.N % 8 == 0) ? 1 : 0;
  if (a.tma_store) {
    const cuuint64_t ydims[2] = {(cuuint64_t)v.N, (cuuint64_t)M};
    const cuuint64_t ystrides[1] = {(cuuint64_t)v.N * 2};
    const cuuint32_t ybox[2] = {(cuuint32_t)kBMw, (cuuint32_t)a.box_m};
    cr = enc(&ymap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, y, ydims, ystrides, ybox, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return record_cuda(cudaErrorInvalidValue);
  } else {
    ymap = map;  // unused
  }

  // One bit per device: the attribute is set once per device.  Host threads
  // making their first call together may both set it (harmless); the bits are
  // atomic, so there is no data race.
  static std::atomic<unsigned long long> configured{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda(e);
  if (dev >= 64 || !((configured.load(std::memory_order_acquire) >> dev) & 1ull)) {
    e = cudaFuncSetAttribute(gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return record_cuda(e);
    if (dev < 64) configured.fetch_or(1ull << dev, std::memory_order_release);
  }
  const long long tiles = (long long)a.m_tiles * a.n_tiles;
  const long long work = a.stream_k ? tiles * (v.K / kGroup) : tiles;
  const int grid = (int)std::min<long long>(work, kSms);
  // A programmatic dependent of the rotation kernel: set-up, tensor memory and
  // the first stages' dequantisation (weights only) overlap the rotation; the
  // TMA producer and the epilogue wait for it before they read its output.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return record_cuda(cudaLaunchKernelEx(&cfg, gemm_tc_kernel, map, ymap, a));
}

qlin_status launch_gemm(const PackedView& v, const __half* scales, const __half* zeros,
                        const uint32_t* sign_bits, const __half* x, __half* y, int M,
                        void* workspace, cudaStream_t s) {
  const GemmWorkspace ws(M, v.K);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  __half* xr = reinterpret_cast<__half*>(base);
  uint32_t* flags = reinterpret_cast<uint32_t*>(base + ws.flags_off);
  float* partials = reinterpret_cast<float*>(base + ws.part_off);
  qlin_status r = launch_rht(x, xr, sign_bits, M, v.K, s, flags, kSms);
  if (r != QLIN_OK) return r;
  return launch_gemm_rotated(v, scales, zeros, xr, y, M, s, flags, partials);
}

unsigned take_gemm_error() {
  unsigned v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_gemm_error, sizeof(v)) != cudaSuccess) return ~0u;
  if (v) cudaMemcpyToSymbol(g_gemm_error, &zero, sizeof(zero));
  return v;
}

}  // namespace qlin

// ---------------------------------------------------------------------------
// qlin_gemm_noalloc: qlin_gemm with a library-owned scratch buffer.
//
// qlin_gemm needs a caller-provided workspace for the rotated activations.
// Some callers cannot allocate device memory where they run the layer: a plugin
// hosted by another runtime that owns every device allocation, or a serving loop
// that forbids allocation once it is running (cudaMalloc may synchronise the
// device).  This entry point keeps the rotated activations in the file-scope
// array below instead, so the caller passes only inputs and outputs.
//
// * The array holds kNoallocMaxElems fp16 values (16 MiB); every GPU that loads
//   the library holds it until the process exits.  Calls with M*K above that
//   limit are rejected with QLIN_ERR_SHAPE before anything is enqueued.
// * Host code must not hand the array's name to a kernel: on the host it is a
//   stand-in, not a device address.  The first call on each device, with that
//   device current, looks up the array's device address once with
//   cudaGetSymbolAddress and remembers it; make that first call before any
//   stream capture.
// * Every call on a device uses the same array and leaves its rotated
//   activations there.  Each call overwrites the M*K values it reads before
//   reading them, so nothing needs clearing; calls that overlap on the GPU (two
//   streams, or two threads) race on the array and must be serialised by the
//   caller.
// ---------------------------------------------------------------------------

namespace qlin {
namespace {

constexpr size_t kNoallocMaxElems = (size_t)8 << 20;  // 8,388,608 fp16 = 16 MiB
constexpr int kNoallocMaxDevices = 64;

static __device__ __align__(256) uint16_t g_noalloc_rotated_x[kNoallocMaxElems];

std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kNoallocMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once).
qlin_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda(e);
  if (dev < 0 || dev >= kNoallocMaxDevices) return QLIN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_rotated_x);
    if (e != cudaSuccess) return record_cuda(e);
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return QLIN_OK;
}

bool noalloc_width_ok(int b) { return b == 3 || b == 4 || b == 6 || b == 8; }
bool noalloc_aligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace qlin

extern "C" qlin_status qlin_gemm_noalloc(const qlin_desc* d, const void* packed, const uint16_t* scales,
                                         const uint16_t* zeros, const uint32_t* sign_bits, const uint16_t* x,
                                         uint16_t* y, int32_t M, qlin_stream_t st) {
  using namespace qlin;
  if (!d) return QLIN_ERR_INVALID_ARG;
  if (d->N < 1 || d->K < kGroup || d->K % kGroup || M < 1) return QLIN_ERR_SHAPE;
  if (d->bits == 0) {
    if (d->N % kBlockRows) return QLIN_ERR_SHAPE;
    if (!d->block_bits) return QLIN_ERR_INVALID_ARG;
    for (int j = 0; j < d->N / kBlockRows; ++j)
      if (!noalloc_width_ok(d->block_bits[j])) return QLIN_ERR_UNSUPPORTED;
  } else if (!noalloc_width_ok(d->bits)) {
    return QLIN_ERR_UNSUPPORTED;
  }
  if (!packed || !scales || !zeros || !sign_bits || !x || !y) return QLIN_ERR_INVALID_ARG;
  if (!noalloc_aligned(packed) || !noalloc_aligned(scales) || !noalloc_aligned(zeros) ||
      !noalloc_aligned(sign_bits) || !noalloc_aligned(x) || !noalloc_aligned(y))
    return QLIN_ERR_ALIGNMENT;
  if ((size_t)M * (size_t)d->K > kNoallocMaxElems) return QLIN_ERR_SHAPE;
  void* scratch = nullptr;
  qlin_status r = noalloc_scratch(&scratch);
  if (r != QLIN_OK) return r;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(st);
  const PackedView v = make_view(d, packed);
  __half* xr = static_cast<__half*>(scratch);
  r = launch_rht(reinterpret_cast<const __half*>(x), xr, sign_bits, M, v.K, s);
  if (r != QLIN_OK) return r;

  return launch_gemm_rotated(v, reinterpret_cast<const __half*>(scales), reinterpret_cast<const __half*>(zeros),
                             xr, reinterpret_cast<__half*>(y), M, s, nullptr, nullptr);
}

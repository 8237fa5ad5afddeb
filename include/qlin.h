/*
 * qlin.h -- weight-only-quantised linear layer for NVIDIA B200 (sm_100a).
 *
 * Computes  Y = rht(X) . dequant(Wq)^T  with fp16 inputs, fp32 accumulation and
 * fp16 output, where
 *
 *   dequant:  w[n][k] = s[n][k/128] * (q[n][k] - z[n][k/128])
 *             integer codes q of 3, 4, 6 or 8 bits with one fp16 scale s and one
 *             fp16 zero point z per group of 128 codes along the reduction
 *             dimension K ("24B0978-Week01-Track2_20-Submission01", section
 *             "How these techniques accelerate inference on CUDA", paragraph
 *             "Group-wise affine integer quantisation"; 6- and 8-bit codes:
 *             "24B0978-Week02-Track2-40-Submission01", section "Recipe").
 *
 *   rht:      random Hadamard transform of the activations: per block of 128
 *             along K, flip the sign of x[k] where sign bit k is set, apply the
 *             Walsh-Hadamard transform (7 add/subtract butterfly stages) and
 *             multiply by 1/sqrt(128), so the transform is orthonormal
 *             ("24B0978-Week01-Track2_20-Submission01", same section, paragraph
 *             "Random Hadamard transform").
 *
 * ---------------------------------------------------------------------------
 * Packed code layout (the format written by qlin_pack and read by every other
 * entry point)
 * ---------------------------------------------------------------------------
 *   Rows are stored one after the other with no padding.  Row n holds K codes
 *   of b_n bits as a little-endian bit stream: code k occupies stream bits
 *   [b_n*k, b_n*k + b_n), least significant bit first, and stream bit j is bit
 *   (j mod 32) of the little-endian 32-bit word j/32 of the row.
 *   Example (b = 4): codes 0,1,...,7 form the word 0x76543210.
 *   A group of 128 codes occupies exactly 16*b bytes (4*b words), so with
 *   K % 128 == 0 every group, and every row, starts on a 16-byte boundary.
 *
 *   Uniform width (desc.bits in {3,4,6,8}): b_n = bits, row n starts at byte
 *   n*K*bits/8, and the buffer holds N*K*bits/8 bytes.
 *
 *   Mixed width (desc.bits == 0): rows come in blocks of 64; block j has width
 *   block_bits[j] (3, 4, 6 or 8) for all of its rows and all of K
 *   ("25M2111-Week02-Track2-40-Submission01", section "Method, selection, and
 *   reproduction": 64-row blocks with per-block byte selectors).  Block j starts
 *   at byte 8*K*sum_{i<j} block_bits[i]; its row r at 8*K*... + r*K*b_j/8.
 *   After the code bytes (C = 8*K*sum_j block_bits[j]) the buffer holds a block
 *   table used by the kernels:
 *       uint32  start16[N/64 + 1]  at byte C:   block j starts at byte 16*start16[j]
 *       uint8   width[N/64]        after it:    block_bits[j]
 *   qlin_packed_bytes() includes the table (rounded up to 16 bytes).
 *
 *   Scales and zeros are not repacked: they stay two separate fp16 arrays
 *   [N][K/128], row-major, passed to every call that dequantises.
 *
 *   Sign bits: uint32 [K/32]; bit (k mod 32) of word k/32 set means x[k] is
 *   negated before the Hadamard transform.
 *
 * ---------------------------------------------------------------------------
 * Conventions
 * ---------------------------------------------------------------------------
 *   * Every buffer argument is a DEVICE pointer, allocated and owned by the
 *     caller, 16-byte aligned, and not aliasing any other argument; the library
 *     never allocates device memory.  The descriptor (and desc->block_bits) is
 *     HOST memory, read during the call only.
 *   * fp16 buffers are passed as uint16_t (IEEE binary16 bit patterns).
 *   * Calls are asynchronous on `stream` (NULL = the legacy default stream) and
 *     never synchronise, except qlin_pack on a mixed-width descriptor, which
 *     copies the block table from pageable host memory (the CUDA runtime
 *     orders such a copy after the work already queued on the stream).
 *   * Errors: argument validation happens before any launch and returns a
 *     negative qlin_status with nothing enqueued; a failed launch returns
 *     QLIN_ERR_CUDA (the CUDA error is then available from
 *     qlin_last_cuda_error()).  No C++ exception crosses this interface.
 *   * Results do not depend on the stream or on previous calls, except that
 *     qlin_gemv and qlin_gemm overwrite their workspace.
 */
#ifndef QLIN_H
#define QLIN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* qlin_stream_t;

typedef enum {
  QLIN_OK = 0,
  QLIN_ERR_INVALID_ARG = -1, /* null pointer or inconsistent descriptor            */
  QLIN_ERR_UNSUPPORTED = -2, /* code width not in {3,4,6,8} (or 0 for mixed)       */
  QLIN_ERR_SHAPE = -3,       /* K % 128 != 0, N < 1, M out of range, N % 64 (mixed)*/
  QLIN_ERR_ALIGNMENT = -4,   /* a buffer is not 16-byte aligned                    */
  QLIN_ERR_CUDA = -5,        /* a CUDA runtime call or kernel launch failed        */
  QLIN_ERR_WORKSPACE = -6    /* workspace missing or smaller than required         */
} qlin_status;

/* Describes one packed weight matrix Wq of N output rows and K codes per row.
 * Plain data, owned by the caller. */
typedef struct {
  int32_t N;                  /* output features, >= 1 (mixed: multiple of 64)   */
  int32_t K;                  /* input features, multiple of 128                 */
  int32_t bits;               /* 3, 4, 6 or 8; 0 selects mixed widths            */
  const uint8_t* block_bits;  /* HOST [N/64] widths in {3,4,6,8} when bits == 0,
                                 else ignored (may be NULL)                       */
} qlin_desc;

/* Human-readable name of a status code (static storage). */
const char* qlin_status_string(qlin_status status);

/* The cudaError_t (as int) of the last failed CUDA call made by this library
 * on the calling thread, 0 if none. */
int qlin_last_cuda_error(void);

/* Lets qlin_gemv (M = 1, uniform widths) overlap the kernel that precedes it on
 * the stream (programmatic dependent launch): the call may start, and read its
 * packed weight, scales, zeros and sign bits, before that kernel has finished;
 * it waits for it before reading x or writing y.  This hides the launch and
 * ramp of back-to-back calls, as in a decode loop over layers.  Enable it only
 * if no kernel that writes the weight, scale, zero or sign buffers immediately
 * precedes a call on the same stream.  Process-wide; default off.  Returns the
 * previous setting. */
int qlin_set_overlap(int enable);

/* Bytes of the packed buffer for `desc` (codes, plus the block table for mixed
 * widths), a multiple of 16.  Returns 0 for an invalid descriptor.  Counts the
 * stored format: K*b/8 bytes per row of b-bit codes ("24B0978-Week01-Track2_20-
 * Submission01", paragraph "Group-wise affine integer quantisation"; mixed
 * widths per 64-row block: "25M2111-Week02-Track2-40-Submission01", section
 * "Method, selection, and reproduction"). */
size_t qlin_packed_bytes(const qlin_desc* desc);

/* Bytes of the code stream alone (the layout above without the block table):
 * the packed codes that one pass over the weight reads, the bulk of the weight
 * traffic that the pages' decode speed-up rests on ("24B0978-Week01-Track2_20-
 * Submission01", section "How these techniques accelerate inference on CUDA"). */
size_t qlin_code_bytes(const qlin_desc* desc);

/* Pack integer codes into the layout above.
 *   codes  : device uint8 [N][K], row-major; only the low b_n bits of each code
 *            of row n are used.
 *   packed : device, qlin_packed_bytes(desc) bytes, written entirely.
 * Definition: "24B0978-Week01-Track2_20-Submission01", "How these techniques
 * accelerate inference on CUDA" (codes stored per group of 128 along K). */
qlin_status qlin_pack(const qlin_desc* desc, const uint8_t* codes, void* packed,
                      qlin_stream_t stream);

/* Inverse of qlin_pack: codes (device uint8 [N][K]) from a packed buffer.
 * Uses the same device decode routines as qlin_gemv and qlin_gemm.
 * Definition: the layout above ("24B0978-Week01-Track2_20-Submission01",
 * paragraph "Group-wise affine integer quantisation": integer codes per group
 * of 128 along K). */
qlin_status qlin_unpack(const qlin_desc* desc, const void* packed, uint8_t* codes,
                        qlin_stream_t stream);

/* Dequantise to fp16: w[n][k] = fp16_rn( fp32(s) * (fp32(q) - fp32(z)) ), each
 * fp32 operation rounded to nearest, no fused multiply-add, one rounding to
 * fp16.  This is the exact fp16 weight qlin_gemm multiplies.
 *   scales, zeros : device fp16 [N][K/128];  w : device fp16 [N][K].
 * Definition: "24B0978-Week01-Track2_20-Submission01", paragraph "Group-wise
 * affine integer quantisation". */
qlin_status qlin_dequant(const qlin_desc* desc, const void* packed, const uint16_t* scales,
                         const uint16_t* zeros, uint16_t* w, qlin_stream_t stream);

/* Offline weight side: rotate each weight row along K with the activations'
 * signs and block-128 Hadamard, then quantise it by asymmetric round-to-nearest
 * per group of 128, ready for qlin_pack with the same descriptor:
 *   w~ = fp32( fp64(1/sqrt(128)) * (H_128 diag(d) w) )   per block of 128
 *        (the sum exact in fp64, one multiply, sqrt and division rounded to
 *        nearest, then one rounding to fp32),
 *   s  = fp16_rn( (max w~ - min w~) / (2^b - 1) ), replaced by 1 if not > 0,
 *   z  = fp16_rn( -min w~ / s ),
 *   q  = min(max(rint(w~ / s + z), 0), 2^b - 1)
 * with every fp32 operation rounded to nearest and nothing fused, so the
 * outputs are a function of the input alone (bit-exact, deterministic).  A zero
 * minimum counts as +0 (z is then -0).  Inputs beyond the fp16 range of s are
 * not guarded.
 *   w        : device fp16 [N][K], the unrotated weight;
 *   sign_bits: device uint32 [K/32] (bit k set: d_k = -1), the signs qlin_gemv
 *              applies to x;
 *   codes    : device uint8 [N][K];  scales, zeros : device fp16 [N][K/128].
 * Widths: desc->bits, or per 64-row block from desc->block_bits (one launch per
 * run of equal widths).  No buffer may alias another.
 * Definition: "24B0978-Week01-Track2_20-Submission01", paragraph "Random
 * Hadamard transform" (the weight side is rotated offline, before
 * quantisation); "24B0978-Week02-Track2-40-Submission01", recipe op
 * "quant_rtn" (bits, group 128). */
qlin_status qlin_quantize_rtn(const qlin_desc* desc, const uint16_t* w, const uint32_t* sign_bits,
                              uint8_t* codes, uint16_t* scales, uint16_t* zeros, qlin_stream_t stream);

/* Workspace bytes of qlin_quantize_gptq: the rotated rows (fp32 [N][K]), the
 * quantisation errors of one group of columns (fp32 [N][128]) and the width
 * table; 0 for an invalid descriptor. */
size_t qlin_gptq_workspace_bytes(const qlin_desc* desc);

/* Offline weight side with error compensation (GPTQ): rotate each weight row
 * exactly as qlin_quantize_rtn does, w~ (fp32), then quantise the rotated rows
 * column by column against a calibration Hessian H, through the upper
 * triangular factor U of its damped inverse (U^T U = (H + damp I)^-1, the
 * Hessian of the ROTATED activations; computing H and U is the caller's):
 *   for each column i in order:
 *     at the first column of a group of 128: the group's grid by
 *       round-to-nearest from its weights as they stand now:
 *       s = fp16_rn((max - min) / (2^b - 1)) (1 if not > 0), z = fp16_rn(-min / s);
 *     q_i = min(max(rint(w~_i / s + z), 0), 2^b - 1);
 *     e_i = (w~_i - s (q_i - z)) / U[i][i];
 *     w~_j = w~_j - e_i U[i][j] for every later column j,
 * every step an IEEE fp32 operation rounded to nearest (products and
 * differences rounded separately), each weight updated one source column at a
 * time in column order: the outputs are a function of (w, sign_bits, U),
 * bit-exact and deterministic.  With U diagonal nothing propagates and the
 * result is qlin_quantize_rtn's.
 *   w           : device fp16 [N][K], the unrotated weight;
 *   sign_bits   : device uint32 [K/32], the activations' signs;
 *   hinv_factor : device fp32 [K][K], row-major, upper triangular (only the
 *                 upper triangle is read), positive diagonal;
 *   codes       : device uint8 [N][K];  scales, zeros : device fp16 [N][K/128];
 *   workspace   : device, >= qlin_gptq_workspace_bytes(desc) bytes, overwritten.
 * Widths: desc->bits or desc->block_bits (copied to the workspace from host
 * memory, like qlin_pack's table).  No buffer may alias another.
 * Definition: "24B0978-Week02-Track2-40-Submission01", section "Recipe" (stage
 * quant_rht_gptq: bits 6, group 128; GPTQ's compensation run in the rotated
 * basis, calibration Hessian of 128 sequences); "24B0908-Week03-Track1-40-
 * Submission01" (GPTQ int3, group 128); H = 2 X^T X as written on
 * "24B0908-Week02-Track1-40-Submission01". */
qlin_status qlin_quantize_gptq(const qlin_desc* desc, const uint16_t* w, const uint32_t* sign_bits,
                               const float* hinv_factor, uint8_t* codes, uint16_t* scales, uint16_t* zeros,
                               void* workspace, size_t workspace_bytes, qlin_stream_t stream);

/* Random Hadamard transform of M rows of K activations.
 *   x  : device fp16 [M][K];  xr : device fp16 [M][K] (may not alias x);
 *   sign_bits : device uint32 [K/32].
 * xr = fp16_rn( (1/sqrt(128)) * H_128 * diag(d) * x ) per block of 128, the
 * butterflies evaluated in fp32 (so within one fp16 ulp of the exact value,
 * up to fp32 rounding of intermediate sums).  M >= 1, K % 128 == 0.
 * Definition: "24B0978-Week01-Track2_20-Submission01", paragraph "Random
 * Hadamard transform". */
qlin_status qlin_rht(const uint16_t* x, uint16_t* xr, const uint32_t* sign_bits, int32_t M,
                     int32_t K, qlin_stream_t stream);

/* Launch plan of qlin_gemv for this weight and M, computed on the host
 * without launching anything: which kernel runs and how it is laid out (for
 * capacity planning, e.g. whether consecutive calls' CTAs fit on an SM
 * together).  Fields a kernel does not have are 0. */
typedef struct {
  int32_t kernel;           /* 1: fused M = 1 kernel (uniform widths);
                               2: rotation kernel + tensor-core kernel (mixed
                                  widths);
                               3: M = 1 integer tensor-core kernel (4, 8 bits);
                               4: split-K tensor-core kernel, x rotated in the
                                  kernel (M = 2..16, one width)                 */
  int32_t grid;             /* CTAs of the main kernel                         */
  int32_t threads;          /* threads per CTA                                 */
  int32_t smem_bytes;       /* dynamic shared memory per CTA                   */
  int32_t consumer_warps;   /* kernel 1: warps that multiply (plus 1 producer) */
  int32_t units_per_warp;   /* kernel 1: runs of 64 codes (8-bit: 32) per warp */
  int32_t rows_per_cta;     /* kernels 1, 3, 4: the most rows one CTA owns      */
  int32_t rows_per_chunk;   /* kernels 1, 3, 4: rows one bulk copy brings in    */
  int32_t stages;           /* kernels 1, 3: shared-memory stages; 4: buffers   */
  int32_t chunks_in_flight; /* kernels 1, 3: copies of one CTA in flight at
                               once; 4: 32-row tiles per buffer                 */
  uint64_t workspace_bytes; /* = qlin_gemv_workspace_bytes(desc, M)            */
} qlin_gemv_plan_info;

/* Fills *info; QLIN_ERR_INVALID_ARG / _UNSUPPORTED / _SHAPE as qlin_gemv
 * (M outside 1..16). */
qlin_status qlin_gemv_plan(const qlin_desc* desc, int32_t M, qlin_gemv_plan_info* info);

/* Workspace bytes qlin_gemv needs for this weight and M; 0 means none (the
 * workspace may then be NULL).  Returns 0 for an invalid descriptor or M. */
size_t qlin_gemv_workspace_bytes(const qlin_desc* desc, int32_t M);

/* Decode-regime quantised linear layer, 1 <= M <= 16:
 *   y[m][n] = fp16_rn( sum_k rht(x)[m][k] * w[n][k] ), fp32 accumulation,
 * with rht(x) rounded once to fp16.  Weights are dequantised in registers and
 * never written to memory; the per-group scale and zero may be applied to the
 * group's partial sum, sum_k s(q - z)x = s(sum qx - z sum x).
 * The M = 1 kernel (uniform widths) rotates x itself, evaluating the block
 * transform as H16 (x) H8 with one tensor-core product per block (fp32
 * accumulation; a rotated value can differ from qlin_rht's by one fp16 ulp
 * where the exact value lies near a rounding boundary), and for 4- and 8-bit
 * codes multiplies the rotated x as 16-bit integers with one power-of-two
 * scale per 64 (int8: 32) consecutive values: exact for values within a
 * factor 16 of the largest magnitude of their run, others rounded at 2^-14 of
 * it.  These readings are judged by the output tolerance, like the factored
 * scale.  For 2 <= M <= 16 (and mixed widths) x is rotated into the workspace
 * and the codes, exact as fp16, are multiplied with it on the tensor cores.
 *   x : device fp16 [M][K] (not rotated);  y : device fp16 [M][N];
 *   workspace : device buffer of workspace_bytes >= qlin_gemv_workspace_bytes(M, K)
 *               bytes (may be NULL when that is 0); overwritten.
 * Definition: "24B0978-Week01-Track2_20-Submission01", section "How these
 * techniques accelerate inference on CUDA" (fused in-register dequantisation;
 * per-group scale on the accumulator; activation rotation at runtime). */
qlin_status qlin_gemv(const qlin_desc* desc, const void* packed, const uint16_t* scales,
                      const uint16_t* zeros, const uint32_t* sign_bits, const uint16_t* x,
                      uint16_t* y, int32_t M, void* workspace, size_t workspace_bytes,
                      qlin_stream_t stream);

/* Workspace bytes qlin_gemm needs for this weight and M: the rotated
 * activations (M*K fp16, rounded up to 256 bytes), the completion flags of the
 * work split between CTAs, and one fp32 partial tile per CTA.  The rotated
 * activations are the runtime half of the random Hadamard transform
 * ("24B0978-Week01-Track2_20-Submission01", paragraph "Random Hadamard
 * transform"), computed once per call and read by every CTA. */
size_t qlin_gemm_workspace_bytes(const qlin_desc* desc, int32_t M);

/* Prefill-regime quantised linear layer, any M >= 1 (built for M >= 64):
 *   y[m][n] = fp16_rn( sum_k rht(x)[m][k] * w[n][k] ), fp32 accumulation,
 * with rht(x) rounded once to fp16 and w the fp16 weight exactly as
 * qlin_dequant writes it, dequantised into tensor memory inside the main loop
 * and multiplied on the tensor cores (fp16 operands, fp32 accumulation); the
 * fp16 weight never reaches global memory.  Tiles split between CTAs are
 * summed in a fixed order, so the result is deterministic.
 * Definition: "24B0978-Week01-Track2_20-Submission01", section "How these
 * techniques accelerate inference on CUDA" (dequantisation fused into the
 * matmul; group-wise affine codes; activation rotation at runtime).
 *   workspace : device buffer of workspace_bytes >= qlin_gemm_workspace_bytes(M, K)
 *               bytes; overwritten. */
qlin_status qlin_gemm(const qlin_desc* desc, const void* packed, const uint16_t* scales,
                      const uint16_t* zeros, const uint32_t* sign_bits, const uint16_t* x,
                      uint16_t* y, int32_t M, void* workspace, size_t workspace_bytes,
                      qlin_stream_t stream);

/* qlin_gemm for callers that cannot allocate device memory: the pages have no
 * counterpart; this is a library convenience.  It has no room for the partial
 * sums of tiles split between CTAs, so it runs the one-CTA-per-tile schedule
 * (each output tile summed over all of K by one CTA): the same result
 * definition as qlin_gemm within the output tolerance, but a different
 * summation order (not bit-identical to qlin_gemm) and slower when there are
 * fewer tiles than SMs.  qlin_gemm needs a workspace for
 * the rotated activations, but some callers cannot allocate one where they run
 * the layer (for example a plugin inside another runtime that owns all device
 * allocations, or a serving loop that forbids allocation once running, since
 * cudaMalloc can synchronise the device).  This entry point allocates nothing:
 * it keeps the rotated activations in a fixed 16 MiB array inside the library
 * (every GPU that loads the library holds it until the process exits).
 *   Arguments, layout and result: as qlin_gemm, without the workspace.
 *   Limit: M * K <= 8,388,608; larger calls return QLIN_ERR_SHAPE and enqueue
 *   nothing.
 *   The first call on each device (with that device current) looks up the
 *   array's device address once; make that first call before any stream
 *   capture.  All calls on a device share the array and leave their rotated
 *   activations in it; each call overwrites what it reads, so nothing needs
 *   clearing, but calls that overlap on the GPU (several streams or threads)
 *   race on it and must be serialised by the caller. */
qlin_status qlin_gemm_noalloc(const qlin_desc* desc, const void* packed, const uint16_t* scales,
                              const uint16_t* zeros, const uint32_t* sign_bits, const uint16_t* x,
                              uint16_t* y, int32_t M, qlin_stream_t stream);

/* The layer for activations that live in host memory, in one call: copies x
 * in, runs qlin_gemv (M <= 16) or qlin_gemm (M > 16) on it, and copies y back,
 * all enqueued on `stream` in that order (three asynchronous operations, one
 * per copy and the layer's kernels).  The pages have no counterpart; this is
 * a library convenience for a caller whose activations are on the host.
 *   x_host : host fp16 [M][K];  y_host : host fp16 [M][N].  Both must stay
 *            valid until the stream has passed the copies; page-locked
 *            (pinned) memory keeps the copies asynchronous.
 *   x_dev, y_dev : device fp16 [M][K] and [M][N] staging buffers (16-byte
 *            aligned), overwritten;
 *   workspace : as qlin_gemv (M <= 16) or qlin_gemm (M > 16) need it.
 *   Result: y_host holds the same bits as the device call would write into
 *   y_dev.  Every argument is checked before the first copy is enqueued, so an
 *   error enqueues nothing. */
qlin_status qlin_linear_host(const qlin_desc* desc, const void* packed, const uint16_t* scales,
                             const uint16_t* zeros, const uint32_t* sign_bits, const uint16_t* x_host,
                             uint16_t* y_host, uint16_t* x_dev, uint16_t* y_dev, int32_t M, void* workspace,
                             size_t workspace_bytes, qlin_stream_t stream);

/* Reads and clears the device-side error word (0 = no error).  Kernels that
 * wait on shared-memory barriers bound every wait; a wait that gives up sets a
 * bit here instead of hanging (the call's output is then invalid): bits 0-7
 * the M = 1 GEMV kernels, 8-15 the GEMM, 16-23 the split-K GEMV.  Synchronous:
 * waits for all work already queued on the device. */
qlin_status qlin_device_error(uint32_t* code);

#ifdef __cplusplus
}
#endif

#endif /* QLIN_H */

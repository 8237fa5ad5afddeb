// C ABI of the qlin library: argument validation, status codes, dispatch.
// Nothing here computes the layer; it checks arguments and enqueues kernels.
#include <atomic>
#include <cstring>
#include <vector>

#include "qlin_internal.cuh"

namespace qlin {

static thread_local int g_last_cuda_error = 0;
static std::atomic<int> g_overlap{0};

bool overlap_enabled() { return g_overlap.load(std::memory_order_relaxed) != 0; }

qlin_status record_cuda(cudaError_t e) {
  if (e == cudaSuccess) return QLIN_OK;
  g_last_cuda_error = (int)e;
  return QLIN_ERR_CUDA;
}

static bool width_ok(int b) { return b == 3 || b == 4 || b == 6 || b == 8; }

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Validates a descriptor; QLIN_OK if it describes a packed matrix we can read.
static qlin_status check_desc(const qlin_desc* d) {
  if (!d) return QLIN_ERR_INVALID_ARG;
  if (d->N < 1 || d->K < kGroup || d->K % kGroup) return QLIN_ERR_SHAPE;
  if (d->bits == 0) {
    if (d->N % kBlockRows) return QLIN_ERR_SHAPE;
    if (!d->block_bits) return QLIN_ERR_INVALID_ARG;
    for (int j = 0; j < d->N / kBlockRows; ++j)
      if (!width_ok(d->block_bits[j])) return QLIN_ERR_UNSUPPORTED;
    return QLIN_OK;
  }
  return width_ok(d->bits) ? QLIN_OK : QLIN_ERR_UNSUPPORTED;
}

size_t code_bytes(const qlin_desc* d) {
  if (d->bits) return (size_t)d->N * (size_t)d->K * (size_t)d->bits / 8u;
  size_t sum_bits = 0;
  for (int j = 0; j < d->N / kBlockRows; ++j) sum_bits += d->block_bits[j];
  return 8u * (size_t)d->K * sum_bits;
}

size_t table_offset(const qlin_desc* d) { return (code_bytes(d) + 15u) & ~(size_t)15u; }

static size_t packed_bytes(const qlin_desc* d) {
  if (d->bits) return (code_bytes(d) + 15u) & ~(size_t)15u;
  const size_t nb = (size_t)d->N / kBlockRows;
  const size_t t = table_offset(d) + 4u * (nb + 1) + nb;
  return (t + 15u) & ~(size_t)15u;
}

PackedView make_view(const qlin_desc* d, const void* packed) {
  PackedView v;
  v.codes = static_cast<const uint8_t*>(packed);
  v.N = d->N;
  v.K = d->K;
  v.bits = d->bits;
  v.row_bytes_uniform = d->bits ? (int64_t)d->K * d->bits / 8 : 0;
  if (d->bits == 0) {
    const size_t t = table_offset(d);
    v.start16 = reinterpret_cast<const uint32_t*>(v.codes + t);
    v.widths = v.codes + t + 4u * ((size_t)d->N / kBlockRows + 1);
  } else {
    v.start16 = nullptr;
    v.widths = nullptr;
  }
  return v;
}

}  // namespace qlin

using namespace qlin;

extern "C" {

const char* qlin_status_string(qlin_status s) {
  switch (s) {
    case QLIN_OK: return "QLIN_OK";
    case QLIN_ERR_INVALID_ARG: return "QLIN_ERR_INVALID_ARG: null pointer or inconsistent descriptor";
    case QLIN_ERR_UNSUPPORTED: return "QLIN_ERR_UNSUPPORTED: code width must be 3, 4, 6 or 8";
    case QLIN_ERR_SHAPE: return "QLIN_ERR_SHAPE: K must be a positive multiple of 128, N >= 1 (mixed: N % 64 == 0), M in range";
    case QLIN_ERR_ALIGNMENT: return "QLIN_ERR_ALIGNMENT: buffers must be 16-byte aligned";
    case QLIN_ERR_CUDA: return "QLIN_ERR_CUDA: a CUDA call failed (see qlin_last_cuda_error)";
    case QLIN_ERR_WORKSPACE: return "QLIN_ERR_WORKSPACE: workspace missing or too small";
  }
  return "unknown qlin_status";
}

int qlin_last_cuda_error(void) { return g_last_cuda_error; }

int qlin_set_overlap(int enable) { return g_overlap.exchange(enable ? 1 : 0); }

size_t qlin_packed_bytes(const qlin_desc* d) {
  return check_desc(d) == QLIN_OK ? packed_bytes(d) : 0;
}

size_t qlin_code_bytes(const qlin_desc* d) {
  return check_desc(d) == QLIN_OK ? code_bytes(d) : 0;
}

qlin_status qlin_pack(const qlin_desc* d, const uint8_t* codes, void* packed, qlin_stream_t st) {
  qlin_status r = check_desc(d);
  if (r != QLIN_OK) return r;
  if (!codes || !packed) return QLIN_ERR_INVALID_ARG;
  if (!aligned16(packed)) return QLIN_ERR_ALIGNMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(st);
  PackedView v = make_view(d, packed);
  if (d->bits == 0) {
    // Block table: start of each block in 16-byte units, then the widths.
    const int nb = d->N / kBlockRows;
    const size_t tbytes = 4u * (size_t)(nb + 1) + (size_t)nb;
    std::vector<uint8_t> table(tbytes);
    uint32_t* start = reinterpret_cast<uint32_t*>(table.data());
    uint64_t acc16 = 0;  // a block holds 64 * K * b / 8 = 8*K*b bytes = K*b/2 sixteen-byte units
    for (int j = 0; j < nb; ++j) {
      start[j] = (uint32_t)acc16;
      acc16 += (uint64_t)d->K * d->block_bits[j] / 2;
    }
    if (acc16 > 0xFFFFFFFFull) return QLIN_ERR_SHAPE;
    start[nb] = (uint32_t)acc16;
    std::memcpy(table.data() + 4u * (nb + 1), d->block_bits, (size_t)nb);
    uint8_t* dst = static_cast<uint8_t*>(packed) + table_offset(d);
    r = record_cuda(cudaMemcpyAsync(dst, table.data(), tbytes, cudaMemcpyHostToDevice, s));
    if (r != QLIN_OK) return r;
  }
  return launch_pack(v, codes, static_cast<uint8_t*>(packed), s);
}

qlin_status qlin_unpack(const qlin_desc* d, const void* packed, uint8_t* codes, qlin_stream_t st) {
  qlin_status r = check_desc(d);
  if (r != QLIN_OK) return r;
  if (!codes || !packed) return QLIN_ERR_INVALID_ARG;
  if (!aligned16(packed)) return QLIN_ERR_ALIGNMENT;
  return launch_unpack(make_view(d, packed), codes, reinterpret_cast<cudaStream_t>(st));
}

qlin_status qlin_dequant(const qlin_desc* d, const void* packed, const uint16_t* scales,
                         const uint16_t* zeros, uint16_t* w, qlin_stream_t st) {
  qlin_status r = check_desc(d);
  if (r != QLIN_OK) return r;
  if (!packed || !scales || !zeros || !w) return QLIN_ERR_INVALID_ARG;
  if (!aligned16(packed) || !aligned16(scales) || !aligned16(zeros) || !aligned16(w))
    return QLIN_ERR_ALIGNMENT;
  return launch_dequant(make_view(d, packed), reinterpret_cast<const __half*>(scales),
                        reinterpret_cast<const __half*>(zeros), reinterpret_cast<__half*>(w),
                        reinterpret_cast<cudaStream_t>(st));
}

qlin_status qlin_quantize_rtn(const qlin_desc* d, const uint16_t* w, const uint32_t* sign_bits, uint8_t* codes,
                              uint16_t* scales, uint16_t* zeros, qlin_stream_t st) {
  qlin_status r = check_desc(d);
  if (r != QLIN_OK) return r;
  if (!w || !sign_bits || !codes || !scales || !zeros) return QLIN_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(sign_bits) || !aligned16(codes) || !aligned16(scales) || !aligned16(zeros))
    return QLIN_ERR_ALIGNMENT;
  return launch_quantize_rtn(reinterpret_cast<const __half*>(w), sign_bits, d->block_bits, d->bits, d->N, d->K,
                             codes, reinterpret_cast<__half*>(scales), reinterpret_cast<__half*>(zeros),
                             reinterpret_cast<cudaStream_t>(st));
}

size_t qlin_gptq_workspace_bytes(const qlin_desc* d) {
  return check_desc(d) == QLIN_OK ? gptq_workspace_bytes(d->N, d->K) : 0;
}

qlin_status qlin_quantize_gptq(const qlin_desc* d, const uint16_t* w, const uint32_t* sign_bits,
                               const float* hinv_factor, uint8_t* codes, uint16_t* scales, uint16_t* zeros,
                               void* workspace, size_t workspace_bytes, qlin_stream_t st) {
  qlin_status r = check_desc(d);
  if (r != QLIN_OK) return r;
  if (!w || !sign_bits || !hinv_factor || !codes || !scales || !zeros) return QLIN_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(sign_bits) || !aligned16(hinv_factor) || !aligned16(codes) ||
      !aligned16(scales) || !aligned16(zeros))
    return QLIN_ERR_ALIGNMENT;
  if (!workspace || workspace_bytes < gptq_workspace_bytes(d->N, d->K)) return QLIN_ERR_WORKSPACE;
  if (!aligned16(workspace)) return QLIN_ERR_ALIGNMENT;
  return launch_quantize_gptq(reinterpret_cast<const __half*>(w), sign_bits, hinv_factor, d->block_bits, d->bits,
                              d->N, d->K, codes, reinterpret_cast<__half*>(scales), reinterpret_cast<__half*>(zeros),
                              workspace, reinterpret_cast<cudaStream_t>(st));
}

qlin_status qlin_rht(const uint16_t* x, uint16_t* xr, const uint32_t* sign_bits, int32_t M,
                     int32_t K, qlin_stream_t st) {
  if (!x || !xr || !sign_bits) return QLIN_ERR_INVALID_ARG;
  if (M < 1 || K < kHadamard || K % kHadamard) return QLIN_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(xr) || !aligned16(sign_bits)) return QLIN_ERR_ALIGNMENT;
  if (x == xr) return QLIN_ERR_INVALID_ARG;
  return launch_rht(reinterpret_cast<const __half*>(x), reinterpret_cast<__half*>(xr), sign_bits,
                    M, K, reinterpret_cast<cudaStream_t>(st));
}

static qlin_status check_linear(const qlin_desc* d, const void* packed, const uint16_t* scales,
                                const uint16_t* zeros, const uint32_t* sign_bits,
                                const uint16_t* x, uint16_t* y) {
  qlin_status r = check_desc(d);
  if (r != QLIN_OK) return r;
  if (!packed || !scales || !zeros || !sign_bits || !x || !y) return QLIN_ERR_INVALID_ARG;
  if (!aligned16(packed) || !aligned16(scales) || !aligned16(zeros) || !aligned16(sign_bits) ||
      !aligned16(x) || !aligned16(y))
    return QLIN_ERR_ALIGNMENT;
  return QLIN_OK;
}

qlin_status qlin_gemv_plan(const qlin_desc* d, int32_t M, qlin_gemv_plan_info* info) {
  qlin_status r = check_desc(d);
  if (r != QLIN_OK) return r;
  if (!info) return QLIN_ERR_INVALID_ARG;
  if (M < 1 || M > 16) return QLIN_ERR_SHAPE;
  gemv_plan_info(d->bits, d->N, d->K, M, info);
  return QLIN_OK;
}

size_t qlin_gemv_workspace_bytes(const qlin_desc* d, int32_t M) {
  if (check_desc(d) != QLIN_OK || M < 1 || M > 16) return 0;
  return gemv_workspace_bytes(d->bits, d->N, d->K, M);
}

qlin_status qlin_gemv(const qlin_desc* d, const void* packed, const uint16_t* scales,
                      const uint16_t* zeros, const uint32_t* sign_bits, const uint16_t* x,
                      uint16_t* y, int32_t M, void* workspace, size_t workspace_bytes,
                      qlin_stream_t st) {
  qlin_status r = check_linear(d, packed, scales, zeros, sign_bits, x, y);
  if (r != QLIN_OK) return r;
  if (M < 1 || M > 16) return QLIN_ERR_SHAPE;
  const size_t ws = gemv_workspace_bytes(d->bits, d->N, d->K, M);
  if (ws && (!workspace || workspace_bytes < ws)) return QLIN_ERR_WORKSPACE;
  if (ws && !aligned16(workspace)) return QLIN_ERR_ALIGNMENT;
  return launch_gemv(make_view(d, packed), reinterpret_cast<const __half*>(scales),
                     reinterpret_cast<const __half*>(zeros), sign_bits,
                     reinterpret_cast<const __half*>(x), reinterpret_cast<__half*>(y), M,
                     workspace, reinterpret_cast<cudaStream_t>(st));
}

size_t qlin_gemm_workspace_bytes(const qlin_desc* d, int32_t M) {
  if (check_desc(d) != QLIN_OK || M < 1) return 0;
  return gemm_workspace_bytes(M, d->K);
}

qlin_status qlin_device_error(uint32_t* code) {
  if (!code) return QLIN_ERR_INVALID_ARG;
  const unsigned a = take_gemv_error(), b = take_gemm_error(), c = take_imma_error(), d = take_tc_error();
  if (a == ~0u || b == ~0u || c == ~0u || d == ~0u) return QLIN_ERR_CUDA;
  *code = a | c | (b << 8) | (d << 16);
  return QLIN_OK;
}

qlin_status qlin_gemm(const qlin_desc* d, const void* packed, const uint16_t* scales,
                      const uint16_t* zeros, const uint32_t* sign_bits, const uint16_t* x,
                      uint16_t* y, int32_t M, void* workspace, size_t workspace_bytes,
                      qlin_stream_t st) {
  qlin_status r = check_linear(d, packed, scales, zeros, sign_bits, x, y);
  if (r != QLIN_OK) return r;
  if (M < 1) return QLIN_ERR_SHAPE;
  if (!workspace || workspace_bytes < gemm_workspace_bytes(M, d->K)) return QLIN_ERR_WORKSPACE;
  if (!aligned16(workspace)) return QLIN_ERR_ALIGNMENT;
  return launch_gemm(make_view(d, packed), reinterpret_cast<const __half*>(scales),
                     reinterpret_cast<const __half*>(zeros), sign_bits,
                     reinterpret_cast<const __half*>(x), reinterpret_cast<__half*>(y), M,
                     workspace, reinterpret_cast<cudaStream_t>(st));
}

qlin_status qlin_linear_host(const qlin_desc* d, const void* packed, const uint16_t* scales,
                             const uint16_t* zeros, const uint32_t* sign_bits, const uint16_t* x_host,
                             uint16_t* y_host, uint16_t* x_dev, uint16_t* y_dev, int32_t M, void* workspace,
                             size_t workspace_bytes, qlin_stream_t st) {
  if (!x_host || !y_host) return QLIN_ERR_INVALID_ARG;
  qlin_status r = check_linear(d, packed, scales, zeros, sign_bits, x_dev, y_dev);
  if (r != QLIN_OK) return r;
  if (M < 1) return QLIN_ERR_SHAPE;
  // every check before the first enqueue: an error enqueues nothing
  const bool gemv = M <= 16;
  const size_t ws = gemv ? gemv_workspace_bytes(d->bits, d->N, d->K, M) : gemm_workspace_bytes(M, d->K);
  if (ws && (!workspace || workspace_bytes < ws)) return QLIN_ERR_WORKSPACE;
  if (ws && !aligned16(workspace)) return QLIN_ERR_ALIGNMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(st);
  cudaError_t e = cudaMemcpyAsync(x_dev, x_host, (size_t)M * (size_t)d->K * 2, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return record_cuda(e);
  const PackedView v = make_view(d, packed);
  const __half* xs = reinterpret_cast<const __half*>(x_dev);
  __half* ys = reinterpret_cast<__half*>(y_dev);
  r = gemv ? launch_gemv(v, reinterpret_cast<const __half*>(scales), reinterpret_cast<const __half*>(zeros),
                         sign_bits, xs, ys, M, workspace, s)
           : launch_gemm(v, reinterpret_cast<const __half*>(scales), reinterpret_cast<const __half*>(zeros),
                         sign_bits, xs, ys, M, workspace, s);
  if (r != QLIN_OK) return r;
  return record_cuda(cudaMemcpyAsync(y_host, y_dev, (size_t)M * (size_t)d->N * 2, cudaMemcpyDeviceToHost, s));
}

}  // extern "C"

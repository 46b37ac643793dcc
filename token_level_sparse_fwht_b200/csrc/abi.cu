// C ABI of the Adamas decode path: host-side argument checks, then dispatch.
// Every check runs before any launch; a rejected call launches nothing.
#include <cmath>
#include <cstring>

#include "adamas_internal.cuh"

namespace adamas {

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int current_device_sms(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  if (dev_out) *dev_out = dev;
  return sms;
}

}  // namespace adamas

using namespace adamas;

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool good_dtype(adamas_dtype dt) { return dt == ADAMAS_F32 || dt == ADAMAS_BF16; }
bool good_t(float t) { return std::isfinite(t) && t >= 0.0f; }
bool good_group(int Hq, int Hkv) {
  if (Hkv <= 0 || Hq <= 0 || Hq % Hkv) return false;
  const int G = Hq / Hkv;
  return G == 1 || G == 2 || G == 4 || G == 8;
}
adamas_status from_cuda(cudaError_t e) { return e == cudaSuccess ? ADAMAS_OK : ADAMAS_ERR_CUDA; }

CacheLayout contiguous(int64_t Lmax) {
  CacheLayout c;
  c.Lmax = Lmax;
  return c;
}

// Encoders with a fixed threshold t (ratio == 0) or per-vector absmax thresholds
// (0 < ratio <= 1; t unused).
bool good_threshold(float t, float ratio) {
  if (ratio == 0.0f) return good_t(t);
  return std::isfinite(ratio) && ratio > 0.0f && ratio <= 1.0f;
}

adamas_status encode_keys_common(const void* k_cache, adamas_dtype dt, int B, int Hkv, int d,
                                 int64_t Lmax, int64_t pos0, int64_t n_new, float t, float ratio,
                                 uint8_t* codes, cudaStream_t stream) {
  if (!k_cache || !codes || !good_dtype(dt) || !good_threshold(t, ratio))
    return ADAMAS_ERR_INVALID_ARG;
  if (B <= 0 || Hkv <= 0 || Lmax <= 0 || pos0 < 0 || n_new <= 0 || pos0 + n_new > Lmax)
    return ADAMAS_ERR_INVALID_ARG;
  if (d != kD) return ADAMAS_ERR_UNSUPPORTED;
  if (!aligned(k_cache, 16) || !aligned(codes, 16)) return ADAMAS_ERR_INVALID_ARG;
  return from_cuda(launch_encode_rows(k_cache, dt, codes, int64_t(B) * Hkv * n_new, n_new, Lmax,
                                      pos0, t, stream, nullptr, 0, ratio));
}

adamas_status encode_queries_common(const void* q, adamas_dtype dt, int B, int Hq, int d,
                                    float t, float ratio, uint8_t* qcodes, cudaStream_t stream) {
  if (!q || !qcodes || !good_dtype(dt) || !good_threshold(t, ratio) || B <= 0 || Hq <= 0)
    return ADAMAS_ERR_INVALID_ARG;
  if (d != kD) return ADAMAS_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(qcodes, 16)) return ADAMAS_ERR_INVALID_ARG;
  const int64_t n = int64_t(B) * Hq;
  return from_cuda(launch_encode_rows(q, dt, qcodes, n, n, 0, 0, t, stream, nullptr, 0, ratio));
}

adamas_status encode_pages_common(const void* k_pages, adamas_dtype dt, int Hkv, int d,
                                  int page_size, int64_t num_pages, const int32_t* page_ids,
                                  int64_t n_ids, float t, float ratio, uint8_t* code_pages,
                                  cudaStream_t stream) {
  if (!k_pages || !code_pages || !good_dtype(dt) || !good_threshold(t, ratio))
    return ADAMAS_ERR_INVALID_ARG;
  if (d != kD) return ADAMAS_ERR_UNSUPPORTED;
  if (Hkv <= 0 || page_size < 1 || num_pages < 1 || num_pages > INT32_MAX)
    return ADAMAS_ERR_INVALID_ARG;
  if (page_ids && (n_ids < 0 || !aligned(page_ids, 4))) return ADAMAS_ERR_INVALID_ARG;
  if (!aligned(k_pages, 16) || !aligned(code_pages, 16)) return ADAMAS_ERR_INVALID_ARG;
  const int64_t per = int64_t(Hkv) * page_size;           // rows per page
  const int64_t groups = page_ids ? n_ids : num_pages;
  return from_cuda(launch_encode_rows(k_pages, dt, code_pages, groups * per, per, per, 0, t,
                                      stream, page_ids, num_pages, ratio));
}

// Device address of a page-locked, device-mapped host buffer; nullptr for any
// other memory (pageable host memory, device memory, unknown pointers).
template <typename P>
P* mapped_device_pointer(P* host) {
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, host) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (attr.type != cudaMemoryTypeHost || attr.devicePointer == nullptr) return nullptr;
  return static_cast<P*>(attr.devicePointer);
}

// Shared checks of the decode / select entry points.
adamas_status check_decode_sizes(int B, int Hq, int Hkv, int d, int64_t Lmax, int64_t L,
                                 int k) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Lmax <= 0 || L <= 0 || k <= 0) return ADAMAS_ERR_INVALID_ARG;
  if (L > Lmax) return ADAMAS_ERR_INVALID_ARG;
  if (Hq % Hkv) return ADAMAS_ERR_INVALID_ARG;
  if (d != kD) return ADAMAS_ERR_UNSUPPORTED;
  if (!good_group(Hq, Hkv)) return ADAMAS_ERR_UNSUPPORTED;
  if (int64_t(B) * Hkv > (1 << 24) || Lmax > (int64_t(1) << 40)) return ADAMAS_ERR_UNSUPPORTED;
  return ADAMAS_OK;
}

}  // namespace

extern "C" {

const char* adamas_status_string(adamas_status s) {
  switch (s) {
    case ADAMAS_OK: return "ok";
    case ADAMAS_ERR_INVALID_ARG: return "invalid argument";
    case ADAMAS_ERR_UNSUPPORTED: return "unsupported configuration";
    case ADAMAS_ERR_CUDA: return "CUDA error";
    case ADAMAS_ERR_TIMEOUT: return "a bounded device wait timed out";
    case ADAMAS_ERR_INTERNAL: return "inconsistent top-k counts on the device";
  }
  return "unknown status";
}

int adamas_abi_version(void) { return 2; }

adamas_status adamas_test_set_copy_fault(int extra_tx_bytes) {
  if (extra_tx_bytes < 0 || extra_tx_bytes > (1 << 20) || (extra_tx_bytes % 16))
    return ADAMAS_ERR_INVALID_ARG;
  set_copy_fault(uint32_t(extra_tx_bytes));
  return ADAMAS_OK;
}

adamas_status adamas_set_decode_policy(int policy) {
  if (policy < 0 || policy > 2) return ADAMAS_ERR_INVALID_ARG;
  set_decode_policy(policy);
  return ADAMAS_OK;
}



adamas_status adamas_encode_keys(const void* k_cache, adamas_dtype dt, int B, int Hkv, int d,
                                 int64_t Lmax, int64_t pos0, int64_t n_new, float t,
                                 uint8_t* codes, cudaStream_t stream) {
  return encode_keys_common(k_cache, dt, B, Hkv, d, Lmax, pos0, n_new, t, 0.0f, codes, stream);
}

adamas_status adamas_encode_keys_absmax(const void* k_cache, adamas_dtype dt, int B, int Hkv,
                                        int d, int64_t Lmax, int64_t pos0, int64_t n_new,
                                        float ratio, uint8_t* codes, cudaStream_t stream) {
  if (!(ratio > 0.0f)) return ADAMAS_ERR_INVALID_ARG;
  return encode_keys_common(k_cache, dt, B, Hkv, d, Lmax, pos0, n_new, 0.0f, ratio, codes,
                            stream);
}

adamas_status adamas_encode_queries(const void* q, adamas_dtype dt, int B, int Hq, int d,
                                    float t, uint8_t* qcodes, cudaStream_t stream) {
  return encode_queries_common(q, dt, B, Hq, d, t, 0.0f, qcodes, stream);
}

adamas_status adamas_encode_queries_absmax(const void* q, adamas_dtype dt, int B, int Hq, int d,
                                           float ratio, uint8_t* qcodes, cudaStream_t stream) {
  if (!(ratio > 0.0f)) return ADAMAS_ERR_INVALID_ARG;
  return encode_queries_common(q, dt, B, Hq, d, 0.0f, ratio, qcodes, stream);
}

adamas_status adamas_encode_pages(const void* k_pages, adamas_dtype dt, int Hkv, int d,
                                  int page_size, int64_t num_pages, const int32_t* page_ids,
                                  int64_t n_ids, float t, uint8_t* code_pages,
                                  cudaStream_t stream) {
  return encode_pages_common(k_pages, dt, Hkv, d, page_size, num_pages, page_ids, n_ids, t, 0.0f,
                             code_pages, stream);
}

adamas_status adamas_encode_pages_absmax(const void* k_pages, adamas_dtype dt, int Hkv, int d,
                                         int page_size, int64_t num_pages,
                                         const int32_t* page_ids, int64_t n_ids, float ratio,
                                         uint8_t* code_pages, cudaStream_t stream) {
  if (!(ratio > 0.0f)) return ADAMAS_ERR_INVALID_ARG;
  return encode_pages_common(k_pages, dt, Hkv, d, page_size, num_pages, page_ids, n_ids, 0.0f,
                             ratio, code_pages, stream);
}

size_t adamas_decode_workspace_bytes(int B, int Hq, int Hkv, int d, int64_t L, int k) {
  if (check_decode_sizes(B, Hq, Hkv, d, L, L, k) != ADAMAS_OK) return 0;
  return decode_workspace_bytes(B, Hq, Hkv, L, k);
}

adamas_status adamas_workspace_init(void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!ws || ws_bytes == 0) return ADAMAS_ERR_INVALID_ARG;
  return from_cuda(cudaMemsetAsync(ws, 0, ws_bytes, stream));
}

adamas_status adamas_check_workspace(const void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!ws || ws_bytes < 256) return ADAMAS_ERR_INVALID_ARG;
  uint32_t word = 0;
  const uint8_t* p = static_cast<const uint8_t*>(ws) + decode_workspace_error_offset();
  if (cudaMemcpyAsync(&word, p, sizeof(word), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return ADAMAS_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return ADAMAS_ERR_CUDA;
  if (word & (kErrWait | kErrCopy)) return ADAMAS_ERR_TIMEOUT;
  if (word & kErrInput) return ADAMAS_ERR_INVALID_ARG;
  return word ? ADAMAS_ERR_INTERNAL : ADAMAS_OK;
}

}  // extern "C"

namespace {

// The per-head and the shared-selection flavours of the decode / select entry
// points differ only in the kernel instance and in the idx_out shape.
adamas_status plan_common(bool shared, int B, int Hq, int Hkv, int d, int64_t L, int k,
                          int* ctas, int* cluster, int64_t* tokens_per_cta, int* smem_bytes) {
  const adamas_status s = check_decode_sizes(B, Hq, Hkv, d, L, L, k);
  if (s != ADAMAS_OK) return s;
  Plan p;
  if (!decode_plan_for_current_device(B, Hq, Hkv, L, k, shared, -1, p, !shared))
    return ADAMAS_ERR_UNSUPPORTED;
  if (ctas) *ctas = p.grid;
  if (cluster) *cluster = p.cluster;
  if (tokens_per_cta) *tokens_per_cta = p.keys_per_cta;
  if (smem_bytes) *smem_bytes = int(p.smem);
  return ADAMAS_OK;
}

adamas_status decode_common(bool shared, const void* q, const void* k_cache,
                            const void* v_cache, const uint8_t* codes, adamas_dtype dt, int B,
                            int Hq, int Hkv, int d, int64_t Lmax, int64_t L, int k, float t,
                            void* workspace, size_t ws_bytes, int32_t* idx_out, float* out,
                            cudaStream_t stream) {
  if (!q || !k_cache || !v_cache || !codes || !workspace || !out) return ADAMAS_ERR_INVALID_ARG;
  if (!good_dtype(dt) || !good_t(t)) return ADAMAS_ERR_INVALID_ARG;
  const adamas_status s = check_decode_sizes(B, Hq, Hkv, d, Lmax, L, k);
  if (s != ADAMAS_OK) return s;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(codes, 16) ||
      !aligned(out, 16) || !aligned(workspace, 256) || (idx_out && !aligned(idx_out, 4)))
    return ADAMAS_ERR_INVALID_ARG;
  Plan p;
  if (!decode_plan_for_current_device(B, Hq, Hkv, L, k, shared, -1, p, !shared))
    return ADAMAS_ERR_UNSUPPORTED;
  if (ws_bytes < decode_workspace_bytes(B, Hq, Hkv, L, k)) return ADAMAS_ERR_INVALID_ARG;
  return from_cuda(launch_decode(q, nullptr, k_cache, v_cache, codes, dt, B, Hq, Hkv,
                                 contiguous(Lmax), L, k, t, workspace, idx_out, out, shared, p,
                                 stream));
}

adamas_status decode_host_common(bool shared, const void* q_host, void* q_dev,
                                 const void* k_cache, const void* v_cache, const uint8_t* codes,
                                 adamas_dtype dt, int B, int Hq, int Hkv, int d, int64_t Lmax,
                                 int64_t L, int k, float t, void* workspace, size_t ws_bytes,
                                 int32_t* idx_out, float* out_dev, float* out_host,
                                 cudaStream_t stream) {
  if (!q_host || !out_host) return ADAMAS_ERR_INVALID_ARG;
  // everything else is checked here before the copy is queued
  if (!q_dev || !k_cache || !v_cache || !codes || !workspace || !out_dev || !good_dtype(dt) ||
      !good_t(t))
    return ADAMAS_ERR_INVALID_ARG;
  const adamas_status s = check_decode_sizes(B, Hq, Hkv, d, Lmax, L, k);
  if (s != ADAMAS_OK) return s;
  if (!aligned(q_dev, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(codes, 16) || !aligned(out_dev, 16) || !aligned(workspace, 256) ||
      (idx_out && !aligned(idx_out, 4)))
    return ADAMAS_ERR_INVALID_ARG;
  Plan p;
  if (!decode_plan_for_current_device(B, Hq, Hkv, L, k, shared, -1, p, !shared))
    return ADAMAS_ERR_UNSUPPORTED;
  if (ws_bytes < decode_workspace_bytes(B, Hq, Hkv, L, k)) return ADAMAS_ERR_INVALID_ARG;
  // Page-locked host buffers are mapped into the device's address space: then the
  // kernel reads q from, and writes out to, host memory itself (no copy engines,
  // no extra stream operations).  Otherwise the copies go through q_dev / out_dev.
  const void* qh_dev = mapped_device_pointer(q_host);
  void* oh_dev = mapped_device_pointer(out_host);
  if (qh_dev && oh_dev && aligned(qh_dev, 16) && aligned(oh_dev, 16)) {
    return from_cuda(launch_decode(qh_dev, nullptr, k_cache, v_cache, codes, dt, B, Hq, Hkv,
                                   contiguous(Lmax), L, k, t, workspace, idx_out,
                                   static_cast<float*>(oh_dev), shared, p, stream));
  }
  const size_t elem = dt == ADAMAS_F32 ? 4 : 2;
  const size_t qbytes = size_t(B) * Hq * kD * elem;
  const size_t obytes = size_t(B) * Hq * kD * sizeof(float);
  if (cudaMemcpyAsync(q_dev, q_host, qbytes, cudaMemcpyHostToDevice, stream) != cudaSuccess)
    return ADAMAS_ERR_CUDA;
  const adamas_status r = from_cuda(launch_decode(q_dev, nullptr, k_cache, v_cache, codes, dt, B,
                                                  Hq, Hkv, contiguous(Lmax), L, k, t, workspace,
                                                  idx_out, out_dev, shared, p, stream));
  if (r != ADAMAS_OK) return r;
  return from_cuda(cudaMemcpyAsync(out_host, out_dev, obytes, cudaMemcpyDeviceToHost, stream));
}

adamas_status select_common(bool shared, const uint8_t* qcodes, const uint8_t* codes, int B,
                            int Hq, int Hkv, int64_t Lmax, int64_t L, int k, void* workspace,
                            size_t ws_bytes, int32_t* idx_out, cudaStream_t stream) {
  if (!qcodes || !codes || !workspace || !idx_out) return ADAMAS_ERR_INVALID_ARG;
  const adamas_status s = check_decode_sizes(B, Hq, Hkv, kD, Lmax, L, k);
  if (s != ADAMAS_OK) return s;
  if (!aligned(qcodes, 16) || !aligned(codes, 16) || !aligned(workspace, 256) ||
      !aligned(idx_out, 4))
    return ADAMAS_ERR_INVALID_ARG;
  Plan p;
  if (!decode_plan_for_current_device(B, Hq, Hkv, L, k, shared, -1, p, !shared))
    return ADAMAS_ERR_UNSUPPORTED;
  if (ws_bytes < decode_workspace_bytes(B, Hq, Hkv, L, k)) return ADAMAS_ERR_INVALID_ARG;
  return from_cuda(launch_decode(nullptr, qcodes, nullptr, nullptr, codes, ADAMAS_BF16, B, Hq,
                                 Hkv, contiguous(Lmax), L, k, 0.0f, workspace, idx_out, nullptr,
                                 shared, p, stream));
}

// Checks of the page-pool arguments shared by the paged entry points; fills `lay`.
adamas_status check_pages(int page_size, int64_t num_pages, const int32_t* block_table,
                          int max_blocks, const int32_t* seq_lens, int64_t max_seq_len,
                          CacheLayout& lay) {
  if (!block_table || !seq_lens) return ADAMAS_ERR_INVALID_ARG;
  if (page_size < 1 || page_size > (1 << 20) || (page_size & (page_size - 1)))
    return ADAMAS_ERR_INVALID_ARG;
  if (num_pages < 1 || num_pages > INT32_MAX || max_blocks < 1 || max_seq_len < 1)
    return ADAMAS_ERR_INVALID_ARG;
  if (int64_t(max_blocks) * page_size < max_seq_len) return ADAMAS_ERR_INVALID_ARG;
  if (!aligned(block_table, 4) || !aligned(seq_lens, 4)) return ADAMAS_ERR_INVALID_ARG;
  int shift = 0;
  while ((1 << shift) < page_size) ++shift;
  lay.block_table = block_table;
  lay.max_blocks = max_blocks;
  lay.page_shift = shift;
  lay.num_pages = num_pages;
  lay.seq_lens = seq_lens;
  return ADAMAS_OK;
}

// Decode or select (q == nullptr: from qcodes, no attention) over any cache layout.
adamas_status layout_common(bool shared, const void* q, const uint8_t* qcodes, const void* kc,
                            const void* vc, const uint8_t* codes, adamas_dtype dt, int B, int Hq,
                            int Hkv, int d, const CacheLayout& lay, int64_t L, int k, float t,
                            void* workspace, size_t ws_bytes, int32_t* idx_out, float* out,
                            cudaStream_t stream, bool check_only = false) {
  const bool select_only = q == nullptr;
  if (!codes || !workspace) return ADAMAS_ERR_INVALID_ARG;
  if (select_only ? (!qcodes || !idx_out) : (!kc || !vc || !out)) return ADAMAS_ERR_INVALID_ARG;
  if (!select_only && (!good_dtype(dt) || !good_t(t))) return ADAMAS_ERR_INVALID_ARG;
  const adamas_status s = check_decode_sizes(B, Hq, Hkv, d, L, L, k);
  if (s != ADAMAS_OK) return s;
  if (!aligned(codes, 16) || !aligned(workspace, 256) || (idx_out && !aligned(idx_out, 4)))
    return ADAMAS_ERR_INVALID_ARG;
  if (select_only ? !aligned(qcodes, 16)
                  : (!aligned(q, 16) || !aligned(kc, 16) || !aligned(vc, 16) || !aligned(out, 16)))
    return ADAMAS_ERR_INVALID_ARG;
  Plan p;
  const int page_shift = lay.block_table != nullptr ? lay.page_shift : -1;
  if (!decode_plan_for_current_device(B, Hq, Hkv, L, k, shared, page_shift, p,
                                      !shared && page_shift < 0))
    return ADAMAS_ERR_UNSUPPORTED;
  if (ws_bytes < decode_workspace_bytes(B, Hq, Hkv, L, k)) return ADAMAS_ERR_INVALID_ARG;
  if (check_only) return ADAMAS_OK;
  return from_cuda(launch_decode(q, qcodes, kc, vc, codes, select_only ? ADAMAS_BF16 : dt, B, Hq,
                                 Hkv, lay, L, k, t, workspace, idx_out, out, shared, p, stream));
}

// Host-buffer form of a decode call whose arguments have been checked: `run(q, out)`
// launches the device call.  Page-locked host buffers mapped into the device's
// address space are used in place (the kernel reads q and writes the output through
// the mapping, no copy-engine work); otherwise q is copied in through q_dev and the
// output back through out_dev, all asynchronous on `stream`.
template <typename Run>
adamas_status with_host_buffers(const void* q_host, void* q_dev, float* out_dev, float* out_host,
                                size_t qbytes, size_t obytes, cudaStream_t stream, Run run) {
  const void* qh_dev = mapped_device_pointer(q_host);
  void* oh_dev = mapped_device_pointer(out_host);
  if (qh_dev && oh_dev && aligned(qh_dev, 16) && aligned(oh_dev, 16))
    return run(qh_dev, static_cast<float*>(oh_dev));
  if (!q_dev || !out_dev || !aligned(q_dev, 16) || !aligned(out_dev, 16))
    return ADAMAS_ERR_INVALID_ARG;
  if (cudaMemcpyAsync(q_dev, q_host, qbytes, cudaMemcpyHostToDevice, stream) != cudaSuccess)
    return ADAMAS_ERR_CUDA;
  const adamas_status r = run(q_dev, out_dev);
  if (r != ADAMAS_OK) return r;
  return from_cuda(cudaMemcpyAsync(out_host, out_dev, obytes, cudaMemcpyDeviceToHost, stream));
}

// Per-vector absmax thresholds, contiguous caches (check_only: arguments only).
adamas_status absmax_common(const void* q, const void* k_cache, const void* v_cache,
                            const uint8_t* codes, adamas_dtype dt, int B, int Hq, int Hkv, int d,
                            int64_t Lmax, int64_t L, int k, float ratio, int shared,
                            void* workspace, size_t ws_bytes, int32_t* idx_out, float* out,
                            cudaStream_t stream, bool check_only) {
  if (!(ratio > 0.0f) || !good_threshold(0.0f, ratio) || (shared != 0 && shared != 1))
    return ADAMAS_ERR_INVALID_ARG;
  if (!q || !k_cache || !v_cache || !codes || !workspace || !out) return ADAMAS_ERR_INVALID_ARG;
  if (!good_dtype(dt)) return ADAMAS_ERR_INVALID_ARG;
  const adamas_status s = check_decode_sizes(B, Hq, Hkv, d, Lmax, L, k);
  if (s != ADAMAS_OK) return s;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(codes, 16) ||
      !aligned(out, 16) || !aligned(workspace, 256) || (idx_out && !aligned(idx_out, 4)))
    return ADAMAS_ERR_INVALID_ARG;
  Plan p;
  if (!decode_plan_for_current_device(B, Hq, Hkv, L, k, shared != 0, -1, p, shared == 0))
    return ADAMAS_ERR_UNSUPPORTED;
  if (ws_bytes < decode_workspace_bytes(B, Hq, Hkv, L, k)) return ADAMAS_ERR_INVALID_ARG;
  if (check_only) return ADAMAS_OK;
  return from_cuda(launch_decode(q, nullptr, k_cache, v_cache, codes, dt, B, Hq, Hkv,
                                 contiguous(Lmax), L, k, 0.0f, workspace, idx_out, out,
                                 shared != 0, p, stream, ratio));
}

}  // namespace

extern "C" {

adamas_status adamas_decode_plan(int B, int Hq, int Hkv, int d, int64_t L, int k, int* ctas,
                                 int* cluster, int64_t* tokens_per_cta, int* smem_bytes) {
  return plan_common(false, B, Hq, Hkv, d, L, k, ctas, cluster, tokens_per_cta, smem_bytes);
}

adamas_status adamas_decode_plan_shared(int B, int Hq, int Hkv, int d, int64_t L, int k,
                                        int* ctas, int* cluster, int64_t* tokens_per_cta,
                                        int* smem_bytes) {
  return plan_common(true, B, Hq, Hkv, d, L, k, ctas, cluster, tokens_per_cta, smem_bytes);
}

adamas_status adamas_decode_step(const void* q, const void* k_cache, const void* v_cache,
                                 const uint8_t* codes, adamas_dtype dt, int B, int Hq,
                                 int Hkv, int d, int64_t Lmax, int64_t L, int k, float t,
                                 void* workspace, size_t ws_bytes, int32_t* idx_out,
                                 float* out, cudaStream_t stream) {
  return decode_common(false, q, k_cache, v_cache, codes, dt, B, Hq, Hkv, d, Lmax, L, k, t,
                       workspace, ws_bytes, idx_out, out, stream);
}

adamas_status adamas_decode_step_shared(const void* q, const void* k_cache, const void* v_cache,
                                        const uint8_t* codes, adamas_dtype dt, int B, int Hq,
                                        int Hkv, int d, int64_t Lmax, int64_t L, int k, float t,
                                        void* workspace, size_t ws_bytes, int32_t* idx_out,
                                        float* out, cudaStream_t stream) {
  return decode_common(true, q, k_cache, v_cache, codes, dt, B, Hq, Hkv, d, Lmax, L, k, t,
                       workspace, ws_bytes, idx_out, out, stream);
}

adamas_status adamas_decode_step_host(const void* q_host, void* q_dev, const void* k_cache,
                                      const void* v_cache, const uint8_t* codes, adamas_dtype dt,
                                      int B, int Hq, int Hkv, int d, int64_t Lmax, int64_t L,
                                      int k, float t, void* workspace, size_t ws_bytes,
                                      int32_t* idx_out, float* out_dev, float* out_host,
                                      cudaStream_t stream) {
  return decode_host_common(false, q_host, q_dev, k_cache, v_cache, codes, dt, B, Hq, Hkv, d,
                            Lmax, L, k, t, workspace, ws_bytes, idx_out, out_dev, out_host,
                            stream);
}

adamas_status adamas_decode_step_shared_host(const void* q_host, void* q_dev,
                                             const void* k_cache, const void* v_cache,
                                             const uint8_t* codes, adamas_dtype dt, int B,
                                             int Hq, int Hkv, int d, int64_t Lmax, int64_t L,
                                             int k, float t, void* workspace, size_t ws_bytes,
                                             int32_t* idx_out, float* out_dev, float* out_host,
                                             cudaStream_t stream) {
  return decode_host_common(true, q_host, q_dev, k_cache, v_cache, codes, dt, B, Hq, Hkv, d,
                            Lmax, L, k, t, workspace, ws_bytes, idx_out, out_dev, out_host,
                            stream);
}

adamas_status adamas_select_topk(const uint8_t* qcodes, const uint8_t* codes, int B, int Hq,
                                 int Hkv, int64_t Lmax, int64_t L, int k, void* workspace,
                                 size_t ws_bytes, int32_t* idx_out, cudaStream_t stream) {
  return select_common(false, qcodes, codes, B, Hq, Hkv, Lmax, L, k, workspace, ws_bytes,
                       idx_out, stream);
}

adamas_status adamas_decode_step_varlen(const void* q, const void* k_cache, const void* v_cache,
                                        const uint8_t* codes, adamas_dtype dt, int B, int Hq,
                                        int Hkv, int d, int64_t Lmax, const int32_t* seq_lens,
                                        int k, float t, int shared, void* workspace,
                                        size_t ws_bytes, int32_t* idx_out, float* out,
                                        cudaStream_t stream) {
  if (!q || !seq_lens || !aligned(seq_lens, 4) || (shared != 0 && shared != 1))
    return ADAMAS_ERR_INVALID_ARG;
  CacheLayout lay = contiguous(Lmax);
  lay.seq_lens = seq_lens;
  return layout_common(shared != 0, q, nullptr, k_cache, v_cache, codes, dt, B, Hq, Hkv, d, lay,
                       Lmax, k, t, workspace, ws_bytes, idx_out, out, stream);
}

adamas_status adamas_decode_step_paged(const void* q, const void* k_pages, const void* v_pages,
                                       const uint8_t* code_pages, adamas_dtype dt, int B, int Hq,
                                       int Hkv, int d, int page_size, int64_t num_pages,
                                       const int32_t* block_table, int max_blocks_per_seq,
                                       const int32_t* seq_lens, int64_t max_seq_len, int k,
                                       float t, int shared, void* workspace, size_t ws_bytes,
                                       int32_t* idx_out, float* out, cudaStream_t stream) {
  if (!q || (shared != 0 && shared != 1)) return ADAMAS_ERR_INVALID_ARG;
  CacheLayout lay;
  const adamas_status s = check_pages(page_size, num_pages, block_table, max_blocks_per_seq,
                                      seq_lens, max_seq_len, lay);
  if (s != ADAMAS_OK) return s;
  return layout_common(shared != 0, q, nullptr, k_pages, v_pages, code_pages, dt, B, Hq, Hkv, d,
                       lay, max_seq_len, k, t, workspace, ws_bytes, idx_out, out, stream);
}

adamas_status adamas_decode_step_paged_host(const void* q_host, void* q_dev, const void* k_pages,
                                            const void* v_pages, const uint8_t* code_pages,
                                            adamas_dtype dt, int B, int Hq, int Hkv, int d,
                                            int page_size, int64_t num_pages,
                                            const int32_t* block_table, int max_blocks_per_seq,
                                            const int32_t* seq_lens, int64_t max_seq_len, int k,
                                            float t, int shared, void* workspace,
                                            size_t ws_bytes, int32_t* idx_out, float* out_dev,
                                            float* out_host, cudaStream_t stream) {
  if (!q_host || !out_host || (shared != 0 && shared != 1)) return ADAMAS_ERR_INVALID_ARG;
  CacheLayout lay;
  const adamas_status s = check_pages(page_size, num_pages, block_table, max_blocks_per_seq,
                                      seq_lens, max_seq_len, lay);
  if (s != ADAMAS_OK) return s;
  // every argument of the device call is checked before anything is queued (the
  // aligned workspace pointer stands in for the q / out buffer the mapping decides)
  void* probe = workspace;
  const adamas_status c = layout_common(shared != 0, probe, nullptr, k_pages, v_pages, code_pages,
                                        dt, B, Hq, Hkv, d, lay, max_seq_len, k, t, workspace,
                                        ws_bytes, idx_out, static_cast<float*>(probe), stream,
                                        true);
  if (c != ADAMAS_OK) return c;
  const size_t qbytes = size_t(B) * Hq * kD * (dt == ADAMAS_F32 ? 4 : 2);
  const size_t obytes = size_t(B) * Hq * kD * sizeof(float);
  return with_host_buffers(q_host, q_dev, out_dev, out_host, qbytes, obytes, stream,
                           [&](const void* qd, float* od) {
                             return layout_common(shared != 0, qd, nullptr, k_pages, v_pages,
                                                  code_pages, dt, B, Hq, Hkv, d, lay,
                                                  max_seq_len, k, t, workspace, ws_bytes,
                                                  idx_out, od, stream);
                           });
}

adamas_status adamas_decode_step_absmax(const void* q, const void* k_cache, const void* v_cache,
                                        const uint8_t* codes, adamas_dtype dt, int B, int Hq,
                                        int Hkv, int d, int64_t Lmax, int64_t L, int k,
                                        float ratio, int shared, void* workspace,
                                        size_t ws_bytes, int32_t* idx_out, float* out,
                                        cudaStream_t stream) {
  return absmax_common(q, k_cache, v_cache, codes, dt, B, Hq, Hkv, d, Lmax, L, k, ratio, shared,
                       workspace, ws_bytes, idx_out, out, stream, false);
}

adamas_status adamas_decode_step_absmax_host(const void* q_host, void* q_dev,
                                             const void* k_cache, const void* v_cache,
                                             const uint8_t* codes, adamas_dtype dt, int B,
                                             int Hq, int Hkv, int d, int64_t Lmax, int64_t L,
                                             int k, float ratio, int shared, void* workspace,
                                             size_t ws_bytes, int32_t* idx_out, float* out_dev,
                                             float* out_host, cudaStream_t stream) {
  if (!q_host || !out_host) return ADAMAS_ERR_INVALID_ARG;
  // every argument of the device call is checked before anything is queued (the
  // aligned dummy pointer stands in for the q / out buffer the mapping decides)
  void* probe = workspace;
  const adamas_status c = absmax_common(probe, k_cache, v_cache, codes, dt, B, Hq, Hkv, d, Lmax, L,
                                        k, ratio, shared, workspace, ws_bytes, idx_out,
                                        static_cast<float*>(probe), stream, true);
  if (c != ADAMAS_OK) return c;
  const size_t qbytes = size_t(B) * Hq * kD * (dt == ADAMAS_F32 ? 4 : 2);
  const size_t obytes = size_t(B) * Hq * kD * sizeof(float);
  return with_host_buffers(q_host, q_dev, out_dev, out_host, qbytes, obytes, stream,
                           [&](const void* qd, float* od) {
                             return absmax_common(qd, k_cache, v_cache, codes, dt, B, Hq, Hkv, d,
                                                  Lmax, L, k, ratio, shared, workspace, ws_bytes,
                                                  idx_out, od, stream, false);
                           });
}

adamas_status adamas_select_topk_paged(const uint8_t* qcodes, const uint8_t* code_pages, int B,
                                       int Hq, int Hkv, int page_size, int64_t num_pages,
                                       const int32_t* block_table, int max_blocks_per_seq,
                                       const int32_t* seq_lens, int64_t max_seq_len, int k,
                                       int shared, void* workspace, size_t ws_bytes,
                                       int32_t* idx_out, cudaStream_t stream) {
  if (!qcodes || (shared != 0 && shared != 1)) return ADAMAS_ERR_INVALID_ARG;
  CacheLayout lay;
  const adamas_status s = check_pages(page_size, num_pages, block_table, max_blocks_per_seq,
                                      seq_lens, max_seq_len, lay);
  if (s != ADAMAS_OK) return s;
  return layout_common(shared != 0, nullptr, qcodes, nullptr, nullptr, code_pages, ADAMAS_BF16, B,
                       Hq, Hkv, kD, lay, max_seq_len, k, 0.0f, workspace, ws_bytes, idx_out,
                       nullptr, stream);
}


size_t adamas_cp_workspace_bytes(int B, int Hq, int Hkv, int d, int64_t L, int k, int shared) {
  if (check_decode_sizes(B, Hq, Hkv, d, L, L, k) != ADAMAS_OK || (shared != 0 && shared != 1))
    return 0;
  return cp_workspace_bytes(B, Hq, Hkv, L, k, shared != 0);
}

size_t adamas_cp_hist_elems(int B, int Hq, int Hkv, int shared) {
  if (B <= 0 || !good_group(Hq, Hkv) || (shared != 0 && shared != 1)) return 0;
  const int G = Hq / Hkv;
  return size_t(B) * (shared ? Hkv : Hq) * selection_bins(G, shared != 0);
}

adamas_status adamas_cp_histograms(const void* q, const uint8_t* codes, adamas_dtype dt, int B,
                                   int Hq, int Hkv, int d, int64_t Lmax, int64_t L, int k,
                                   float t, int shared, void* workspace, size_t ws_bytes,
                                   uint32_t* hist_out, cudaStream_t stream) {
  if (!q || !codes || !workspace || !hist_out || (shared != 0 && shared != 1))
    return ADAMAS_ERR_INVALID_ARG;
  if (!good_dtype(dt) || !good_t(t)) return ADAMAS_ERR_INVALID_ARG;
  const adamas_status s = check_decode_sizes(B, Hq, Hkv, d, Lmax, L, k);
  if (s != ADAMAS_OK) return s;
  if (!aligned(q, 16) || !aligned(codes, 16) || !aligned(workspace, 256) ||
      !aligned(hist_out, 4))
    return ADAMAS_ERR_INVALID_ARG;
  Plan p;
  if (!decode_plan_for_current_device(B, Hq, Hkv, L, k, shared != 0, -1, p))
    return ADAMAS_ERR_UNSUPPORTED;
  if (ws_bytes < cp_workspace_bytes(B, Hq, Hkv, L, k, shared != 0))
    return ADAMAS_ERR_INVALID_ARG;
  CpArgs cpa = {};
  cpa.phase = 1;
  cpa.L_total = L;
  cpa.hist_out = hist_out;
  return from_cuda(launch_decode(q, nullptr, nullptr, nullptr, codes, dt, B, Hq, Hkv,
                                 contiguous(Lmax), L, k, t, workspace, nullptr, nullptr,
                                 shared != 0, p, stream, 0.0f, &cpa));
}

adamas_status adamas_cp_attend(const void* q, const void* k_cache, const void* v_cache,
                               const uint8_t* codes, adamas_dtype dt, int B, int Hq, int Hkv,
                               int d, int64_t Lmax, int64_t L, int64_t L_total,
                               int64_t pos_offset, int k, float t, int shared,
                               const uint32_t* hist_all, int world, int rank, void* workspace,
                               size_t ws_bytes, int32_t* idx_out, float* partial_out,
                               cudaStream_t stream) {
  if (!q || !k_cache || !v_cache || !codes || !hist_all || !workspace || !partial_out ||
      (shared != 0 && shared != 1) || world < 1 || rank < 0 || rank >= world)
    return ADAMAS_ERR_INVALID_ARG;
  if (!good_dtype(dt) || !good_t(t)) return ADAMAS_ERR_INVALID_ARG;
  const adamas_status s = check_decode_sizes(B, Hq, Hkv, d, Lmax, L, k);
  if (s != ADAMAS_OK) return s;
  if (pos_offset < 0 || L_total < pos_offset + L || L_total > INT32_MAX)
    return ADAMAS_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(codes, 16) ||
      !aligned(hist_all, 4) || !aligned(partial_out, 16) || !aligned(workspace, 256) ||
      (idx_out && !aligned(idx_out, 4)))
    return ADAMAS_ERR_INVALID_ARG;
  Plan p;
  if (!decode_plan_for_current_device(B, Hq, Hkv, L, k, shared != 0, -1, p))
    return ADAMAS_ERR_UNSUPPORTED;
  if (ws_bytes < cp_workspace_bytes(B, Hq, Hkv, L, k, shared != 0))
    return ADAMAS_ERR_INVALID_ARG;
  CpArgs cpa = {};
  cpa.phase = 2;
  cpa.L_total = L_total;
  cpa.pos_offset = pos_offset;
  cpa.hist_all = hist_all;
  cpa.world = world;
  cpa.rank = rank;
  cpa.partial_out = partial_out;
  return from_cuda(launch_decode(q, nullptr, k_cache, v_cache, codes, dt, B, Hq, Hkv,
                                 contiguous(Lmax), L, k, t, workspace, idx_out, nullptr,
                                 shared != 0, p, stream, 0.0f, &cpa));
}

adamas_status adamas_cp_combine(const float* partials_all, int world, int B, int Hq, float* out,
                                cudaStream_t stream) {
  if (!partials_all || !out || world < 1 || B <= 0 || Hq <= 0) return ADAMAS_ERR_INVALID_ARG;
  if (!aligned(partials_all, 16) || !aligned(out, 16)) return ADAMAS_ERR_INVALID_ARG;
  return from_cuda(launch_cp_combine(partials_all, world, int64_t(B) * Hq, out, stream));
}

adamas_status adamas_select_topk_shared(const uint8_t* qcodes, const uint8_t* codes, int B,
                                        int Hq, int Hkv, int64_t Lmax, int64_t L, int k,
                                        void* workspace, size_t ws_bytes, int32_t* idx_out,
                                        cudaStream_t stream) {
  return select_common(true, qcodes, codes, B, Hq, Hkv, Lmax, L, k, workspace, ws_bytes,
                       idx_out, stream);
}

size_t adamas_sparse_attention_workspace_bytes(int B, int Hq, int k_eff) {
  if (B <= 0 || Hq <= 0 || k_eff <= 0) return 0;
  return attention_workspace_bytes(B, Hq, k_eff);
}

adamas_status adamas_sparse_attention(const void* q, const void* k_cache, const void* v_cache,
                                      adamas_dtype dt, const int32_t* idx, int B, int Hq,
                                      int Hkv, int d, int64_t Lmax, int k_eff, void* workspace,
                                      size_t ws_bytes, float* out, cudaStream_t stream) {
  if (!q || !k_cache || !v_cache || !idx || !workspace || !out || !good_dtype(dt))
    return ADAMAS_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Lmax <= 0 || k_eff <= 0 || Hq % Hkv)
    return ADAMAS_ERR_INVALID_ARG;
  if (d != kD) return ADAMAS_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
      !aligned(idx, 4) || !aligned(workspace, 256))
    return ADAMAS_ERR_INVALID_ARG;
  if (ws_bytes < attention_workspace_bytes(B, Hq, k_eff)) return ADAMAS_ERR_INVALID_ARG;
  return from_cuda(launch_sparse_attention(q, k_cache, v_cache, dt, idx, B, Hq, Hkv, Lmax, k_eff,
                                           workspace, out, stream));
}

adamas_status adamas_sparse_attention_noalloc(const void* q, const void* k_cache,
                                              const void* v_cache, adamas_dtype dt,
                                              const int32_t* idx, int B, int Hq, int Hkv, int d,
                                              int64_t Lmax, int k_eff, float* out,
                                              cudaStream_t stream) {
  if (!q || !k_cache || !v_cache || !idx || !out || !good_dtype(dt)) return ADAMAS_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Lmax <= 0 || k_eff <= 0 || Hq % Hkv)
    return ADAMAS_ERR_INVALID_ARG;
  if (d != kD) return ADAMAS_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
      !aligned(idx, 4))
    return ADAMAS_ERR_INVALID_ARG;
  if (!noalloc_fits(B, Hq)) return ADAMAS_ERR_UNSUPPORTED;   // B * Hq above the fixed scratch
  return from_cuda(launch_sparse_attention_noalloc(q, k_cache, v_cache, dt, idx, B, Hq, Hkv, Lmax,
                                                   k_eff, out, stream));
}

}  // extern "C"

// Split-k gather attention + combine over explicit positions.
//
// Method: "Adamas: Hadamard Sparse Attention for Efficient Long-Context
// Inference", v2 abstract — the selected positions gather the ORIGINAL KV states
// for sparse attention.  Softmax of (q . K_j) / sqrt(d) over the positions,
// fp32 accumulation.
//
// Grid: (batch x query head) x S splits, 8 warps per CTA, 8 rows in flight per
// warp.  Each CTA writes one softmax partial (m, l, acc[128]); the last CTA of a
// (batch, head) — atomic counter in the workspace — merges the S partials and
// resets its counter, so the workspace stays zero between calls.
#include <algorithm>
#include <mutex>

#include "adamas_internal.cuh"

namespace adamas {

constexpr int kAttnThreads = 256;
constexpr int kAttnWarps = kAttnThreads / 32;

template <typename T>
__global__ void __launch_bounds__(kAttnThreads) sparse_attention_kernel(
    const T* __restrict__ q, const T* __restrict__ kc, const T* __restrict__ vc,
    const int32_t* __restrict__ idx, int Hq, int Hkv, int64_t Lmax, int k_eff, int S,
    float scale_log2, uint32_t* done, float* part, float* __restrict__ out) {
  __shared__ float merge[kAttnWarps][kPartStride];
  __shared__ int last;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.x / S, sp = blockIdx.x % S;
  const int b = bh / Hq, h = bh % Hq, kvh = h / (Hq / Hkv);
  const int per = (k_eff + S - 1) / S;
  const int j0 = min(k_eff, sp * per), j1 = min(k_eff, j0 + per);
  float qv[4];
  load4(q + int64_t(bh) * kD, lane, qv);
  const T* kb = kc + (int64_t(b) * Hkv + kvh) * Lmax * kD;
  const T* vb = vc + (int64_t(b) * Hkv + kvh) * Lmax * kD;
  const int32_t* irow = idx + int64_t(bh) * k_eff + j0;
  // positions outside [0, Lmax) are clamped into range rather than read out of
  // bounds; callers must pass valid positions
  auto pos_of = [&](int j) {
    int64_t p = irow[j];
    return p < 0 ? int64_t(0) : (p >= Lmax ? Lmax - 1 : p);
  };
  SoftmaxState st;
  st.init();
  attend_rows<T>(kb, vb, j1 - j0, warp, kAttnWarps, pos_of, qv, scale_log2, lane, st);
  if (lane == 0) { merge[warp][0] = st.m; merge[warp][1] = st.l; }
#pragma unroll
  for (int r = 0; r < 4; ++r) merge[warp][4 + 4 * lane + r] = st.acc[r];
  __syncthreads();
  float* prow = part + (int64_t(bh) * S + sp) * kPartStride;
  if (tid < kD) {
    float M = -INFINITY, Ls = 0.f, A = 0.f;
    for (int w = 0; w < kAttnWarps; ++w) merge_into(merge[w][0], merge[w][1], merge[w][4 + tid], M, Ls, A);
    if (tid == 0) { prow[0] = M; prow[1] = Ls; }
    prow[4 + tid] = A;
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    last = (atomicAdd(&done[bh], 1u) + 1u == uint32_t(S)) ? 1 : 0;
  }
  __syncthreads();
  if (last) {
    __threadfence();
    if (tid < kD) {
      float M = -INFINITY, Ls = 0.f, A = 0.f;
      for (int s = 0; s < S; ++s) {
        const float* pr = part + (int64_t(bh) * S + s) * kPartStride;
        merge_into(__ldcg(pr), __ldcg(pr + 1), __ldcg(pr + 4 + tid), M, Ls, A);
      }
      out[int64_t(bh) * kD + tid] = A / Ls;
    }
    if (tid == 0) done[bh] = 0u;
  }
}

int attention_splits(int B, int Hq, int k_eff, int sms) {
  const int64_t heads = int64_t(B) * Hq;
  int64_t s = (2 * int64_t(sms) + heads - 1) / heads;            // ~2 CTAs per SM
  s = std::min<int64_t>(s, (k_eff + 15) / 16);                   // >= 16 rows per split
  return int(std::max<int64_t>(1, std::min<int64_t>(s, 64)));
}

size_t attention_workspace_bytes(int B, int Hq, int k_eff) {
  const int sms = current_device_sms(nullptr);
  const int S = attention_splits(B, Hq, k_eff, sms > 0 ? sms : 148);
  const size_t heads = size_t(B) * Hq;
  return align_up(heads * 4, 256) + align_up(heads * S * kPartStride * 4, 256);
}

cudaError_t launch_sparse_attention(const void* q, const void* k, const void* v,
                                    adamas_dtype dt, const int32_t* idx, int B, int Hq,
                                    int Hkv, int64_t Lmax, int k_eff, void* ws, float* out,
                                    cudaStream_t stream) {
  const int sms = current_device_sms(nullptr);
  const int S = attention_splits(B, Hq, k_eff, sms > 0 ? sms : 148);
  const size_t heads = size_t(B) * Hq;
  uint32_t* done = static_cast<uint32_t*>(ws);
  float* part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + align_up(heads * 4, 256));
  const float scale_log2 = float(1.4426950408889634 / 11.313708498984761);
  const unsigned grid = unsigned(heads * S);
  if (dt == ADAMAS_BF16) {
    sparse_attention_kernel<__nv_bfloat16><<<grid, kAttnThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<const __nv_bfloat16*>(v), idx, Hq, Hkv, Lmax, k_eff, S, scale_log2, done,
        part, out);
  } else {
    sparse_attention_kernel<float><<<grid, kAttnThreads, 0, stream>>>(
        static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
        idx, Hq, Hkv, Lmax, k_eff, S, scale_log2, done, part, out);
  }
  return cudaGetLastError();
}

}  // namespace adamas

// ------------------------------------------------------------------------------
// Allocation-free variant of adamas_sparse_attention.
//
// Some callers cannot hand the library a workspace: code that runs where
// cudaMalloc is off limits (inside a custom allocator's own callbacks, in
// real-time paths that must not block on the driver's allocator, or under a
// framework whose memory pool owns every device allocation).  For them the split
// partials and per-head counters live in this fixed, file-scope device array,
// which every GPU that loads the library holds until the process exits.
// ------------------------------------------------------------------------------
namespace adamas {

constexpr int kNoAllocMaxHeads = 4096;      // B * Hq per call
constexpr int kNoAllocMaxPartials = 4096;   // B * Hq * splits per call
constexpr size_t kNoAllocCounterBytes = 256 * ((kNoAllocMaxHeads * 4 + 255) / 256);
constexpr size_t kNoAllocBytes =
    kNoAllocCounterBytes + size_t(kNoAllocMaxPartials) * kPartStride * 4;

// Host code may not use this name as a device address: the symbol's device
// address is looked up once per device below and passed to the kernel.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

constexpr int kNoAllocMaxDevices = 64;
static std::mutex g_noalloc_mutex;
static void* g_noalloc_cleared[kNoAllocMaxDevices] = {};   // address whose counters were cleared

// With the calling device current: the scratch's device address, looked up on every
// call (cheap; a device reset reloads the module and may move the array), and its
// counters cleared the first time that address is seen (each completed call returns
// them to zero by itself).
static cudaError_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return cudaErrorInvalidDevice;
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_cleared[dev] != p) {
    e = cudaMemset(p, 0, kNoAllocCounterBytes);
    if (e != cudaSuccess) return e;
    e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return e;
    g_noalloc_cleared[dev] = p;
  }
  *out = p;
  return cudaSuccess;
}

bool noalloc_fits(int B, int Hq) { return int64_t(B) * Hq <= kNoAllocMaxHeads; }

cudaError_t launch_sparse_attention_noalloc(const void* q, const void* k, const void* v,
                                            adamas_dtype dt, const int32_t* idx, int B,
                                            int Hq, int Hkv, int64_t Lmax, int k_eff,
                                            float* out, cudaStream_t stream) {
  void* scratch = nullptr;
  const cudaError_t e = noalloc_scratch(&scratch);
  if (e != cudaSuccess) return e;
  const int sms = current_device_sms(nullptr);
  const int heads = B * Hq;
  int S = attention_splits(B, Hq, k_eff, sms > 0 ? sms : 148);
  S = std::max(1, std::min(S, kNoAllocMaxPartials / heads));
  uint32_t* done = static_cast<uint32_t*>(scratch);
  float* part = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) + kNoAllocCounterBytes);
  const float scale_log2 = float(1.4426950408889634 / 11.313708498984761);
  const unsigned grid = unsigned(heads) * unsigned(S);
  if (dt == ADAMAS_BF16) {
    sparse_attention_kernel<__nv_bfloat16><<<grid, kAttnThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<const __nv_bfloat16*>(v), idx, Hq, Hkv, Lmax, k_eff, S, scale_log2, done,
        part, out);
  } else {
    sparse_attention_kernel<float><<<grid, kAttnThreads, 0, stream>>>(
        static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
        idx, Hq, Hkv, Lmax, k_eff, S, scale_log2, done, part, out);
  }
  return cudaGetLastError();
}

}  // namespace adamas

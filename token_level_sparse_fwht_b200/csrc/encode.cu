// Key and query encoders: orthonormal FWHT (d = 128), 2-bit buckets at
// {-t, 0, +t}, 4 codes per byte.  One warp per vector, four vectors in flight per
// warp (256 B read + 32 B written per bf16 key).
//
// Method: "Adamas: Hadamard Sparse Attention for Efficient Long-Context
// Inference", v2 abstract (Hadamard transform, bucketization, 2-bit compression)
// and the blog section 2.2 bucket rule (three thresholds, strict "<").
#include "adamas_internal.cuh"

namespace adamas {

// rows [nvec] of 128 elements: vector v lives at src + row_of(v) * 128 and its code
// at dst + row_of(v) * 32, with row_of(v) = grp(v / per) * stride + off + v % per and
// grp(i) = i, or ids[i] when a group list is given (groups whose id is outside
// [0, id_limit) are skipped).  Each warp encodes the contiguous run of `run` vectors
// starting at warp * run: one division finds its first (group, position), after which
// both advance by increment; kVecs vectors are loaded before any is transformed.
constexpr int kVecs = 4;

template <typename T>
__global__ void __launch_bounds__(256) encode_rows_kernel(const T* __restrict__ src,
                                                          uint8_t* __restrict__ dst,
                                                          int64_t nvec, int64_t per,
                                                          int64_t stride, int64_t off,
                                                          int64_t run, float t,
                                                          const int32_t* __restrict__ ids,
                                                          int64_t id_limit, float ratio) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  using R = Raw4<T>;
  int64_t v = warp * run;
  const int64_t vend = min(nvec, v + run);
  if (v >= vend) return;
  int64_t grp = v / per;
  int64_t pos = v - grp * per;
  for (; v < vend; v += kVecs) {
    typename R::type x[kVecs];
    int64_t row[kVecs];
    bool ok[kVecs];
#pragma unroll
    for (int u = 0; u < kVecs; ++u) {
      ok[u] = v + u < vend;
      int64_t g = grp;
      if (ids != nullptr && ok[u]) {
        g = ids[grp];
        ok[u] = g >= 0 && g < id_limit;
      }
      row[u] = g * stride + off + pos;
      if (ok[u]) x[u] = R::load(src + row[u] * kD, lane);
      if (++pos == per) {
        pos = 0;
        ++grp;
      }
    }
#pragma unroll
    for (int u = 0; u < kVecs; ++u) {
      if (ok[u]) {
        float e[4];
        R::decode(x[u], e);
        dst[row[u] * kCodeBytes + lane] = static_cast<uint8_t>(warp_fwht_code(e, t, lane, ratio));
      }
    }
  }
}

cudaError_t launch_encode_rows(const void* src, adamas_dtype dt, uint8_t* dst, int64_t nvec,
                               int64_t per, int64_t stride, int64_t off, float t,
                               cudaStream_t stream, const int32_t* ids, int64_t id_limit,
                               float ratio) {
  if (nvec <= 0) return cudaSuccess;
  const int sms = current_device_sms(nullptr);
  // 8 blocks of 8 warps per SM; each warp a run of at least kVecs vectors
  const int64_t max_warps = int64_t(sms > 0 ? sms : 148) * 64;
  const int64_t want = (nvec + kVecs - 1) / kVecs;
  const int64_t warps = want < max_warps ? want : max_warps;
  const int64_t run = (nvec + warps - 1) / warps;
  const int64_t used = (nvec + run - 1) / run;
  const int grid = static_cast<int>((used + 7) / 8);
  if (dt == ADAMAS_BF16) {
    encode_rows_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(src), dst, nvec, per, stride, off, run, t, ids,
        id_limit, ratio);
  } else {
    encode_rows_kernel<float><<<grid, 256, 0, stream>>>(static_cast<const float*>(src), dst,
                                                         nvec, per, stride, off, run, t, ids,
                                                         id_limit, ratio);
  }
  return cudaGetLastError();
}

}  // namespace adamas

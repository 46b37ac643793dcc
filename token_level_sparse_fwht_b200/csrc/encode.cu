// Key and query encoders: orthonormal FWHT (d = 128), 2-bit buckets at
// {-t, 0, +t}, 4 codes per byte.  One warp per vector, two vectors in flight per
// warp; HBM-bound (256 B read + 32 B written per bf16 key).
//
// Method: "Adamas: Hadamard Sparse Attention for Efficient Long-Context
// Inference", v2 abstract (Hadamard transform, bucketization, 2-bit compression)
// and the blog section 2.2 bucket rule (three thresholds, strict "<").
#include "adamas_internal.cuh"

namespace adamas {

// rows [nvec] of 128 elements: vector v lives at src + row_of(v) * 128 and its code
// at dst + row_of(v) * 32, with row_of(v) = grp(v / per) * stride + off + v % per and
// grp(i) = i, or ids[i] when a group list is given (groups whose id is outside
// [0, id_limit) are skipped).
template <typename T>
__global__ void __launch_bounds__(256) encode_rows_kernel(const T* __restrict__ src,
                                                          uint8_t* __restrict__ dst,
                                                          int64_t nvec, int64_t per,
                                                          int64_t stride, int64_t off,
                                                          float t,
                                                          const int32_t* __restrict__ ids,
                                                          int64_t id_limit, float ratio) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  using R = Raw4<T>;
  const auto row_of = [&](int64_t v, bool& ok) -> int64_t {
    int64_t grp = v / per;
    ok = true;
    if (ids != nullptr) {
      grp = ids[grp];
      ok = grp >= 0 && grp < id_limit;
    }
    return grp * stride + off + v % per;
  };
  for (int64_t v0 = warp; v0 < nvec; v0 += 2 * nwarps) {
    const int64_t v1 = v0 + nwarps;
    bool ok0, ok1 = false;
    const int64_t r0 = row_of(v0, ok0);
    const bool has1 = v1 < nvec;
    const int64_t r1 = has1 ? row_of(v1, ok1) : 0;
    typename R::type x0, x1;
    if (ok0) x0 = R::load(src + r0 * kD, lane);
    if (ok1) x1 = R::load(src + r1 * kD, lane);
    if (ok0) {
      float a[4];
      R::decode(x0, a);
      dst[r0 * kCodeBytes + lane] = static_cast<uint8_t>(warp_fwht_code(a, t, lane, ratio));
    }
    if (ok1) {
      float b[4];
      R::decode(x1, b);
      dst[r1 * kCodeBytes + lane] = static_cast<uint8_t>(warp_fwht_code(b, t, lane, ratio));
    }
  }
}

static int encode_grid(int64_t nvec, int sms) {
  const int64_t warps_needed = (nvec + 1) / 2;
  const int64_t blocks = (warps_needed + 7) / 8;           // 8 warps per block
  const int64_t cap = int64_t(sms) * 8;                    // 8 x 256 threads per SM
  return static_cast<int>(blocks < cap ? (blocks < 1 ? 1 : blocks) : cap);
}

cudaError_t launch_encode_rows(const void* src, adamas_dtype dt, uint8_t* dst, int64_t nvec,
                               int64_t per, int64_t stride, int64_t off, float t,
                               cudaStream_t stream, const int32_t* ids, int64_t id_limit,
                               float ratio) {
  if (nvec <= 0) return cudaSuccess;
  const int sms = current_device_sms(nullptr);
  const int grid = encode_grid(nvec, sms > 0 ? sms : 148);
  if (dt == ADAMAS_BF16) {
    encode_rows_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(src), dst, nvec, per, stride, off, t, ids, id_limit,
        ratio);
  } else {
    encode_rows_kernel<float><<<grid, 256, 0, stream>>>(static_cast<const float*>(src), dst,
                                                         nvec, per, stride, off, t, ids,
                                                         id_limit, ratio);
  }
  return cudaGetLastError();
}

}  // namespace adamas

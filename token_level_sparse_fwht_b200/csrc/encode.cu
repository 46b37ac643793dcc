// Key and query encoders: orthonormal FWHT (d = 128), 2-bit buckets at
// {-t, 0, +t}, 4 codes per byte (256 B read + 32 B written per bf16 key).  bf16
// vectors with a fixed threshold go through the tensor cores, 16 vectors per warp;
// fp32 vectors and per-vector (absmax) thresholds through a warp-shuffle FWHT, one
// warp per vector with four in flight.
//
// Method: "Adamas: Hadamard Sparse Attention for Efficient Long-Context
// Inference", v2 abstract (Hadamard transform, bucketization, 2-bit compression)
// and the blog section 2.2 bucket rule (three thresholds, strict "<").
#include <mutex>

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
  pdl_wait();
  pdl_trigger();
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

// Tensor-core encoder for bf16 vectors with a fixed threshold: a warp transforms 16
// vectors at a time.  In natural (Sylvester) order H_128 = H_8 (x) H_16: for
// i = 16a + b and k = 16c + d, (-1)^popc(i & k) = (-1)^popc(a & c) (-1)^popc(b & d).
// So each 16-dimension block c of the 16 vectors is multiplied by H_16 with
// mma.m16n8k16 (bf16 x +-1 products are exact; fp32 accumulation), and the 8 blocks
// are then butterflied in registers (H_8).  The MMA's k order inside a block is
// permuted so that a lane's A registers hold 4 consecutive dimensions (one 8-byte
// load per row and block): k = 2q, 2q+1 -> dimensions 4q, 4q+1 and k = 2q+8, 2q+9 ->
// 4q+2, 4q+3 (q = lane % 4); B = H_16 takes its rows in the same order, and its
// columns in an order that leaves block coordinates 4q .. 4q+3 in lane q's
// accumulators (one byte of each code word).  Codes are compared against t sqrt(128)
// on the unscaled sums.
constexpr int kMmaVecs = 16;
// staging: a 256-byte row padded to 288 bytes, so that the 8-byte fragment reads of a
// warp (rows gid, columns 32 a + 8 q) touch every bank once per 16 lanes
constexpr int kRowPitch = 288;
constexpr int kStageBytes = kMmaVecs * kRowPitch;
constexpr int kEncStages = 2;                            // tiles in flight per warp
constexpr int kEncSmem = 8 * kEncStages * kStageBytes;   // 8 warps per block
extern __shared__ __align__(16) uint8_t enc_smem[];

// bf16 bits of H_16[d0][n] (low half) and H_16[d1][n] (high half): +-1.0
__device__ __forceinline__ uint32_t h16_pair(int d0, int d1, int n) {
  const uint32_t lo = (__popc(d0 & n) & 1) ? 0xBF80u : 0x3F80u;
  const uint32_t hi = (__popc(d1 & n) & 1) ? 0xBF80u : 0x3F80u;
  return lo | (hi << 16);
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Bucket of an unscaled coordinate y (thresholds at -tt, 0, +tt, tt = t sqrt(128) > 0):
// floor(y / tt + 2) clamped to [0, 3] — one fused multiply-add and one saturating
// float -> unsigned conversion (NaN and negatives give 0) plus a min.  It agrees with
// the three compares except within rounding of a threshold.
__device__ __forceinline__ uint32_t code_fma(float y, float inv_tt) {
  return min(__float2uint_rd(fmaf(y, inv_tt, 2.0f)), 3u);
}
// t = 0: the thresholds collapse to 0 and only the sign decides (codes 0 and 3).
__device__ __forceinline__ uint32_t code_sign(float y) { return y >= 0.0f ? 3u : 0u; }

// Packed pairs of fp32 values (sm_100 f32x2 arithmetic: one instruction per pair,
// each lane IEEE round-to-nearest, the same results as two scalar operations).
__device__ __forceinline__ void add_sub2(float& a0, float& a1, float& b0, float& b1) {
  // (a, b) <- (a + b, a - b), elementwise on the pairs (a0, a1) and (b0, b1)
  asm("{\n\t.reg .b64 pa, pb, ps, pd;\n\t"
      "mov.b64 pa, {%0, %1};\n\t"
      "mov.b64 pb, {%2, %3};\n\t"
      "add.rn.f32x2 ps, pa, pb;\n\t"
      "sub.rn.f32x2 pd, pa, pb;\n\t"
      "mov.b64 {%0, %1}, ps;\n\t"
      "mov.b64 {%2, %3}, pd;\n\t}"
      : "+f"(a0), "+f"(a1), "+f"(b0), "+f"(b1));
}
// (y0 m + 2, y1 m + 2) as one packed fused multiply-add
__device__ __forceinline__ void fma2_plus2(float y0, float y1, float m, float& f0, float& f1) {
  asm("{\n\t.reg .b64 py, pm, pc, pr;\n\t"
      "mov.b64 py, {%2, %3};\n\t"
      "mov.b64 pm, {%4, %4};\n\t"
      "mov.b64 pc, {%5, %5};\n\t"
      "fma.rn.f32x2 pr, py, pm, pc;\n\t"
      "mov.b64 {%0, %1}, pr;\n\t}"
      : "=f"(f0), "=f"(f1)
      : "f"(y0), "f"(y1), "f"(m), "f"(2.0f));
}

// Same vector and row mapping as encode_rows_kernel; run is a multiple of 16.  A
// lane's two rows (vectors v + gid and v + gid + 8 of the tile) advance by 16 per
// tile: their (group, position) pairs are found by one division at the start of the
// run and then carried forward.
// kSign: t = 0 (codes by sign alone).  Tiles are staged in shared memory: each warp
// keeps kEncStages buffers of 16 rows and copies the tile kEncStages - 1 ahead with
// 16-byte asynchronous copies (lane (gid, q): chunks q, q + 4, q + 8, q + 12 of its two
// rows) before it transforms the current one, so HBM reads overlap the arithmetic.
// Rows whose copy is skipped (past the run, or an invalid page id) leave stale bytes in
// their buffer rows; the MMA keeps rows apart and their codes are not stored.
template <bool kSign>
__global__ void __launch_bounds__(256) encode_rows_mma_kernel(
    const __nv_bfloat16* __restrict__ src, uint8_t* __restrict__ dst, int64_t nvec, int64_t per,
    int64_t stride, int64_t off, int64_t run, float t, const int32_t* __restrict__ ids,
    int64_t id_limit) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int gid = lane >> 2, q = lane & 3;
  const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  int64_t v = warp * run;
  const int64_t vend = min(nvec, v + run);
  if (v >= vend) return;
  // H_16 fragments: n-tile nt holds outputs 8 nt .. 8 nt + 7 (column n = 8 nt + gid)
  uint32_t bfr[2][2];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    // output column n = gid of tile nt is block coordinate 4 (n >> 1) + 2 nt + (n & 1),
    // so that lane q ends up holding coordinates 4 q .. 4 q + 3 of every block
    const int col = 4 * (gid >> 1) + 2 * nt + (gid & 1);
    bfr[nt][0] = h16_pair(4 * q, 4 * q + 1, col);
    bfr[nt][1] = h16_pair(4 * q + 2, 4 * q + 3, col);
  }
  const float tt = t * 11.313708498984761f;   // sqrt(128)
  const float inv_tt = 1.0f / tt;             // +inf at t = 0 (the sign path is used)
  // byte-transpose selectors of the quad exchange (partner q ^ 1, then q ^ 2)
  const uint32_t selA = (q & 1) ? 0x3715u : 0x6240u;
  const uint32_t selB = (q & 2) ? 0x3276u : 0x5410u;
  int64_t grp[2], pos[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int64_t vv = v + gid + 8 * h;
    grp[h] = vv / per;
    pos[h] = vv - grp[h] * per;
  }
  // this warp's staging buffers: [kEncStages][16 rows][kRowPitch bytes]
  uint8_t* const stage = enc_smem + (threadIdx.x >> 5) * kEncStages * kStageBytes;
  // rows (and validity) of this lane's two vectors in the tile at vt; advances grp, pos
  const auto tile_rows = [&](int64_t vt, int64_t (&row)[2], bool (&ok)[2]) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      ok[h] = vt + gid + 8 * h < vend;
      int64_t g = grp[h];
      if (ids != nullptr && ok[h]) {
        g = ids[g];
        ok[h] = g >= 0 && g < id_limit;
      }
      row[h] = g * stride + off + pos[h];
      pos[h] += kMmaVecs;
      while (pos[h] >= per) {
        pos[h] -= per;
        ++grp[h];
      }
    }
  };
  // lane (gid, q) copies 16-byte chunks q, q + 4, q + 8, q + 12 of its two rows
  const auto copy_tile = [&](int sb, const int64_t (&row)[2], const bool (&ok)[2]) {
    uint8_t* dstb = stage + sb * kStageBytes;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (ok[h]) {
        const uint8_t* g = reinterpret_cast<const uint8_t*>(src + row[h] * kD);
#pragma unroll
        for (int m = 0; m < 4; ++m)
          cp_async_16(dstb + (gid + 8 * h) * kRowPitch + 16 * (q + 4 * m), g + 16 * (q + 4 * m));
      }
    }
    cp_async_commit();
  };
  // rows of the tiles in flight: ring[i] belongs to the tile i tiles after this one
  int64_t row[kEncStages][2];
  bool ok[kEncStages][2];
#pragma unroll
  for (int i = 0; i < kEncStages - 1; ++i) {
    const int64_t vt = v + i * kMmaVecs;
    if (vt < vend) {
      tile_rows(vt, row[i], ok[i]);
      copy_tile(i, row[i], ok[i]);
    } else {
      cp_async_commit();
    }
  }
  for (int sb = 0; v < vend; v += kMmaVecs, sb = sb + 1 == kEncStages ? 0 : sb + 1) {
    // the copies of the tile kEncStages - 1 ahead go out before this tile is transformed
    {
      const int64_t vt = v + (kEncStages - 1) * kMmaVecs;
      int sn = sb + kEncStages - 1;
      if (sn >= kEncStages) sn -= kEncStages;
      if (vt < vend) {
        tile_rows(vt, row[kEncStages - 1], ok[kEncStages - 1]);
        copy_tile(sn, row[kEncStages - 1], ok[kEncStages - 1]);
      } else {
        cp_async_commit();   // an empty group keeps the wait count uniform
      }
    }
    cp_async_wait_pending(kEncStages - 1);
    __syncwarp();
    uint2 x[2][8];
    const uint8_t* cur = stage + sb * kStageBytes;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int a = 0; a < 8; ++a)
        x[h][a] = *reinterpret_cast<const uint2*>(cur + (gid + 8 * h) * kRowPitch + 32 * a + 8 * q);
    }
    __syncwarp();   // every lane has read this buffer before it is refilled
    // z[c][nt][.]: block c times H_16; rows (gid, gid + 8) x columns 8 nt + 2 q + {0, 1}
    float z[8][2][4];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        z[c][nt][0] = z[c][nt][1] = z[c][nt][2] = z[c][nt][3] = 0.0f;
        mma_bf16_16816(z[c][nt], x[0][c].x, x[1][c].x, x[0][c].y, x[1][c].y, bfr[nt][0],
                       bfr[nt][1]);
      }
    }
    // H_8 over the block index, on packed pairs (e, e + 1)
#pragma unroll
    for (int s = 1; s < 8; s <<= 1) {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        if (c & s) continue;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
          for (int e = 0; e < 4; e += 2)
            add_sub2(z[c][nt][e], z[c][nt][e + 1], z[c | s][nt][e], z[c | s][nt][e + 1]);
        }
      }
    }
    // codes: lane q holds coordinates 16 a + 4 q .. 16 a + 4 q + 3 of each row, i.e.
    // byte q of code word a.  Its bytes of the even and the odd words go into two
    // registers, a 4 x 4 byte transpose across the lane quad (two exchanges) turns
    // them into whole words 2 q and 2 q + 1, and lane q stores those.
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t pw[2] = {0u, 0u};   // bytes of words 0, 2, 4, 6 and of words 1, 3, 5, 7
#pragma unroll
      for (int a = 0; a < 8; ++a) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const float y0 = z[a][nt][2 * h], y1 = z[a][nt][2 * h + 1];
          uint32_t c0, c1;
          if constexpr (kSign) {
            c0 = code_sign(y0);
            c1 = code_sign(y1);
          } else {
            float f0, f1;
            fma2_plus2(y0, y1, inv_tt, f0, f1);
            c0 = min(__float2uint_rd(f0), 3u);
            c1 = min(__float2uint_rd(f1), 3u);
          }
          const int sh = 8 * (a >> 1) + 4 * nt;   // coordinates 4 q + 2 nt, + 1
          pw[a & 1] |= (c0 | (c1 << 2)) << sh;
        }
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        pw[i] = __byte_perm(pw[i], __shfl_xor_sync(0xffffffffu, pw[i], 1), selA);
        pw[i] = __byte_perm(pw[i], __shfl_xor_sync(0xffffffffu, pw[i], 2), selB);
      }
      if (ok[0][h]) {
        uint2* d = reinterpret_cast<uint2*>(dst + row[0][h] * kCodeBytes) + q;
        *d = make_uint2(pw[0], pw[1]);
      }
    }
#pragma unroll
    for (int i = 0; i + 1 < kEncStages; ++i) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        row[i][h] = row[i + 1][h];
        ok[i][h] = ok[i + 1][h];
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
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (dt == ADAMAS_BF16 && ratio == 0.0f && reinterpret_cast<uintptr_t>(dst) % 16 == 0 &&
      reinterpret_cast<uintptr_t>(src) % 16 == 0) {
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
      attr_err = cudaFuncSetAttribute(encode_rows_mma_kernel<false>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, kEncSmem);
      if (attr_err == cudaSuccess)
        attr_err = cudaFuncSetAttribute(encode_rows_mma_kernel<true>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, kEncSmem);
    });
    if (attr_err != cudaSuccess) return attr_err;
    cfg.dynamicSmemBytes = kEncSmem;
    // 2 blocks of 8 warps per SM; each warp a run of whole 16-vector tiles
    const int64_t mw_max = int64_t(sms > 0 ? sms : 148) * 16;
    const int64_t tiles = (nvec + kMmaVecs - 1) / kMmaVecs;
    const int64_t mw = tiles < mw_max ? tiles : mw_max;
    const int64_t mrun = (tiles + mw - 1) / mw * kMmaVecs;
    const int64_t mused = (nvec + mrun - 1) / mrun;
    cfg.gridDim = dim3(static_cast<unsigned>((mused + 7) / 8));
    if (!(t > 0.0f))
      return cudaLaunchKernelEx(&cfg, encode_rows_mma_kernel<true>,
                                static_cast<const __nv_bfloat16*>(src), dst, nvec, per, stride,
                                off, mrun, t, ids, id_limit);
    return cudaLaunchKernelEx(&cfg, encode_rows_mma_kernel<false>,
                              static_cast<const __nv_bfloat16*>(src), dst, nvec, per, stride, off,
                              mrun, t, ids, id_limit);
  }
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  if (dt == ADAMAS_BF16)
    return cudaLaunchKernelEx(&cfg, encode_rows_kernel<__nv_bfloat16>,
                              static_cast<const __nv_bfloat16*>(src), dst, nvec, per, stride, off,
                              run, t, ids, id_limit, ratio);
  return cudaLaunchKernelEx(&cfg, encode_rows_kernel<float>, static_cast<const float*>(src), dst,
                            nvec, per, stride, off, run, t, ids, id_limit, ratio);
}

}  // namespace adamas

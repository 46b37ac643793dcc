// Internal device helpers of the Adamas decode path (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "adamas.h"

namespace adamas {

constexpr int kD = 128;                 // head dimension
constexpr int kCodeBytes = kD / 4;      // 32 B of 2-bit codes per vector
constexpr int kNBins = 3 * kD + 1;      // Manhattan distances 0..384
constexpr int kBinStride = 388;         // padded histogram row
constexpr int kPartStride = 132;        // m, l, 2 pad, acc[128] (floats)

// error word bits (workspace header)
constexpr uint32_t kErrBarrier = 1u;
constexpr uint32_t kErrCopy = 2u;
constexpr uint32_t kErrSelect = 4u;   // top-k bookkeeping found no k-th distance
constexpr uint32_t kErrInput = 8u;    // a device-resident length or page id out of range
constexpr unsigned long long kWaitLimitNs = 1000000000ull;   // 1 s per wait

// ----------------------------------------------------------------- PTX helpers
__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

// 1-D bulk copy global -> shared, completion counted on `bar` (16-B aligned,
// bytes a multiple of 16).
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// 16-byte asynchronous copy global -> shared (both 16-B aligned), completed by the
// issuing thread's commit groups.
__device__ __forceinline__ void cp_async_16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src)
               : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}

// Waits until at most `pending` (0..7) of this thread's commit groups are in flight.
__device__ __forceinline__ void cp_async_wait_pending(int pending) {
  switch (pending) {
    case 0: asm volatile("cp.async.wait_group 0;" ::: "memory"); break;
    case 1: asm volatile("cp.async.wait_group 1;" ::: "memory"); break;
    case 2: asm volatile("cp.async.wait_group 2;" ::: "memory"); break;
    case 3: asm volatile("cp.async.wait_group 3;" ::: "memory"); break;
    case 4: asm volatile("cp.async.wait_group 4;" ::: "memory"); break;
    case 5: asm volatile("cp.async.wait_group 5;" ::: "memory"); break;
    case 6: asm volatile("cp.async.wait_group 6;" ::: "memory"); break;
    default: asm volatile("cp.async.wait_group 7;" ::: "memory"); break;
  }
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Programmatic dependent launch.  pdl_wait: block until the grid launched before this
// one in the stream has completed and its memory is visible (a no-op when there is no
// such dependency); every kernel calls it before its first global-memory access.
// pdl_trigger: let the next grid in the stream begin launching its blocks (they run
// up to their own pdl_wait).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Bounded wait on an mbarrier phase; records kErrCopy and returns false on timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint32_t* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      atomicOr(err, kErrCopy);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_gpu(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void red_add_gpu(uint32_t* p, uint32_t v) {
  asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Grid-wide barrier for a cooperative launch (all CTAs co-resident).  Sense by
// generation counter; the arrival counter returns to zero, so the workspace stays
// reusable.  Bounded: gives up after kWaitLimitNs and records kErrBarrier.
__device__ __forceinline__ void grid_barrier(uint32_t* count, uint32_t* gen, uint32_t nblocks,
                                             uint32_t* err) {
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t g0 = ld_acquire_gpu(gen);
    __threadfence();
    const uint32_t arrived = atomicAdd(count, 1u) + 1u;
    if (arrived == nblocks) {
      atomicExch(count, 0u);
      __threadfence();
      st_release_gpu(gen, g0 + 1u);
    } else {
      const unsigned long long t0 = globaltimer_ns();
      while (ld_acquire_gpu(gen) == g0) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
          atomicOr(err, kErrBarrier);
          break;
        }
        __nanosleep(32);
      }
    }
    __threadfence();
  }
  __syncthreads();
}

// L2 prefetch of one 128-element row (256 B bf16 / 512 B fp32), 128 B per line.
template <typename T>
__device__ __forceinline__ void prefetch_row_l2(const T* row) {
  const char* p = reinterpret_cast<const char*>(row);
#pragma unroll
  for (int o = 0; o < int(kD * sizeof(T)); o += 128)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p + o));
}

// ----------------------------------------------------------- element loading
// Lane l of a warp owns elements 4l .. 4l+3 of a 128-vector.
__device__ __forceinline__ void load4(const float* row, int lane, float v[4]) {
  const float4 x = __ldg(reinterpret_cast<const float4*>(row) + lane);
  v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
}

__device__ __forceinline__ void bf16x2_to_f32(uint32_t w, float& lo, float& hi) {
  lo = __uint_as_float(w << 16);
  hi = __uint_as_float(w & 0xffff0000u);
}

__device__ __forceinline__ void load4(const __nv_bfloat16* row, int lane, float v[4]) {
  const uint2 x = __ldg(reinterpret_cast<const uint2*>(row) + lane);
  bf16x2_to_f32(x.x, v[0], v[1]);
  bf16x2_to_f32(x.y, v[2], v[3]);
}

// Raw 4-element chunks kept undecoded while loads are in flight.
template <typename T> struct Raw4;
template <> struct Raw4<float> {
  using type = float4;
  static __device__ __forceinline__ type load(const float* row, int lane) {
    return __ldg(reinterpret_cast<const float4*>(row) + lane);
  }
  static __device__ __forceinline__ void decode(const type& x, float v[4]) {
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
  }
};
template <> struct Raw4<__nv_bfloat16> {
  using type = uint2;
  static __device__ __forceinline__ type load(const __nv_bfloat16* row, int lane) {
    return __ldg(reinterpret_cast<const uint2*>(row) + lane);
  }
  static __device__ __forceinline__ void decode(const type& x, float v[4]) {
    bf16x2_to_f32(x.x, v[0], v[1]);
    bf16x2_to_f32(x.y, v[2], v[3]);
  }
};

// ------------------------------------------------------------ FWHT + codes
// Orthonormal fast Walsh–Hadamard transform of one 128-vector held by a warp
// (lane l: elements 4l..4l+3), natural (Sylvester) order, fp32.  Index bits 0-1
// are butterflied inside the lane, bits 2-6 across lanes with xor-shuffles.
// Returns the lane's byte of the packed code: 4 coordinates, 2 bits each,
// coordinate 4l+r at bits 2r, code = [y >= -t] + [y >= 0] + [y >= t].  With
// ratio > 0 the threshold is the vector's own: t = ratio * max_i |y_i| (blog
// "ADAMAS：稀疏注意力优化技术解析与应用实践", section 2.2, one 128-dimension group).
__device__ __forceinline__ uint32_t warp_fwht_code(float v[4], float t, int lane,
                                                   float ratio = 0.0f) {
  const float a0 = v[0] + v[1], a1 = v[0] - v[1];
  const float a2 = v[2] + v[3], a3 = v[2] - v[3];
  v[0] = a0 + a2; v[1] = a1 + a3; v[2] = a0 - a2; v[3] = a1 - a3;
#pragma unroll
  for (int s = 1; s < 32; s <<= 1) {
    // lower lane of the pair: v + o; upper: o - v.  One fma with a +-1 factor (the
    // product is exact, so this rounds exactly like the add or subtract)
    const float sg = (lane & s) ? -1.0f : 1.0f;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float o = __shfl_xor_sync(0xffffffffu, v[r], s);
      v[r] = fmaf(v[r], sg, o);
    }
  }
  const float inv_sqrt_d = 0.088388347648318440550f;   // 1 / sqrt(128)
#pragma unroll
  for (int r = 0; r < 4; ++r) v[r] *= inv_sqrt_d;
  if (ratio > 0.0f) {
    float m = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, s));
    t = ratio * m;
  }
  uint32_t byte = 0;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const float y = v[r];
    const uint32_t c = (uint32_t)(y >= -t) + (uint32_t)(y >= 0.0f) + (uint32_t)(y >= t);
    byte |= c << (2 * r);
  }
  return byte;
}

// --------------------------------------------------------- code arithmetic
// Thermometer form of a word of 16 packed codes: for code c = 2h + l the field
// becomes (odd, even) = ([c >= 3], [c >= 1]).  Only c = 2 (binary 10) changes, to
// 01: subtracting d = h & ~l at the even bit does it without borrows, as one
// integer multiply-add w + d * neg1 (neg1 = 0xffffffff, held in a register the
// compiler cannot fold) on the FMA pipe, leaving the logic pipe one op lighter.
__device__ __forceinline__ uint32_t therm13(uint32_t w, uint32_t neg1) {
  const uint32_t d = (w >> 1) & ~w & 0x55555555u;      // h & ~l, at the even bit
  uint32_t r;
  asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(r) : "r"(d), "r"(neg1), "r"(w));
  return r;
}
// [c >= 2] of two words, the first at even bits, the second at odd bits.
__device__ __forceinline__ uint32_t therm2(uint32_t w0, uint32_t w1) {
  return ((w0 >> 1) & 0x55555555u) | (w1 & 0xaaaaaaaau);
}

// Thermometer words of one packed 32-byte code: 8 x therm13 + 4 x therm2.
struct Therm {
  uint32_t a[8];
  uint32_t b[4];
};

// `one` is 1 at run time, opaque to the compiler (see therm_dist_csa).
__device__ __forceinline__ void make_therm(const uint32_t w[8], Therm& t, uint32_t one) {
  const uint32_t neg1 = 0u - one;
#pragma unroll
  for (int i = 0; i < 8; ++i) t.a[i] = therm13(w[i], neg1);
#pragma unroll
  for (int i = 0; i < 4; ++i) t.b[i] = therm2(w[2 * i], w[2 * i + 1]);
}

// Manhattan distance of two code vectors from their thermometer words:
// |a - b| = [a>=1]^[b>=1] + [a>=2]^[b>=2] + [a>=3]^[b>=3] per coordinate.
__device__ __forceinline__ uint32_t therm_dist(const Therm& k, const Therm& q) {
  uint32_t s0 = 0, s1 = 0, s2 = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    s0 += __popc(k.a[2 * i] ^ q.a[2 * i]);
    s1 += __popc(k.a[2 * i + 1] ^ q.a[2 * i + 1]);
    s2 += __popc(k.b[i] ^ q.b[i]);
  }
  return s0 + s1 + s2;
}

// Same distance with two carry-save levels.  The 12 XOR words are added bitwise three
// at a time (sum word = a^b^c, carry word = majority(a,b,c), both single LOP3s) into
// four weight-1 and four weight-2 words; three of each are added again, leaving
// weight-1 words O and o3, weight-2 words T1, T2 and t3, and one weight-4 word F:
// 6 popcounts replace 12.  POPC issues at a quarter of the integer-logic rate on
// sm_100, so this moves work from the popcount pipe to the logic pipe, where the
// thermometer words' multiply-adds (therm13) made room.
__device__ __forceinline__ uint32_t therm_dist_csa(const Therm& k, const Therm& q,
                                                   uint32_t one) {
  uint32_t x[12];
#pragma unroll
  for (int i = 0; i < 8; ++i) x[i] = k.a[i] ^ q.a[i];
#pragma unroll
  for (int i = 0; i < 4; ++i) x[8 + i] = k.b[i] ^ q.b[i];
  // The sums run as integer multiply-adds with a multiplier the compiler cannot
  // fold (one == 1 at run time), which keeps them on the FMA pipe and leaves the
  // integer-logic pipe, the scan's bottleneck, to the XOR / carry-save work.
  uint32_t o[4], tw[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t a = x[3 * j], b = x[3 * j + 1], c = x[3 * j + 2];
    o[j] = a ^ b ^ c;
    tw[j] = (a & b) | (c & (a | b));
  }
  const uint32_t O = o[0] ^ o[1] ^ o[2];
  const uint32_t T1 = (o[0] & o[1]) | (o[2] & (o[0] | o[1]));
  const uint32_t T2 = tw[0] ^ tw[1] ^ tw[2];
  const uint32_t F = (tw[0] & tw[1]) | (tw[2] & (tw[0] | tw[1]));
  // sum = popc(O) + popc(o3) + 2 (popc(T1) + popc(T2) + popc(t3)) + 4 popc(F)
  uint32_t s1 = uint32_t(__popc(O)), s2 = uint32_t(__popc(T1));
  asm("mad.lo.u32 %0, %1, %2, %0;" : "+r"(s1) : "r"(uint32_t(__popc(o[3]))), "r"(one));
  asm("mad.lo.u32 %0, %1, %2, %0;" : "+r"(s2) : "r"(uint32_t(__popc(T2))), "r"(one));
  asm("mad.lo.u32 %0, %1, %2, %0;" : "+r"(s2) : "r"(uint32_t(__popc(tw[3]))), "r"(one));
  uint32_t r;
  asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(r) : "r"(s2), "r"(one + one), "r"(s1));
  asm("mad.lo.u32 %0, %1, %2, %0;" : "+r"(r) : "r"(uint32_t(__popc(F))), "r"(4u * one));
  return r;
}

// ---------------------------------------------------------- warp utilities
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Online-softmax state of one (warp, head): scores are kept in the log2 domain.
struct SoftmaxState {
  float m;       // running max of scaled scores (log2 domain)
  float l;       // running sum of exp2(s - m)
  float acc[4];  // lane's 4 output coordinates, unnormalised
  __device__ __forceinline__ void init() {
    m = -INFINITY; l = 0.f;
    acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
  }
};

// Gathers up to `n` rows (positions from `pos_of(j)` for j = j0, j0+step, ...)
// and folds them into `st`.  K/V row r of this (batch, kv head) starts at
// base + r * kD.  kRows rows (K and V) are in flight per warp per batch.
template <typename T, typename PosFn>
__device__ __forceinline__ void attend_rows(const T* __restrict__ kbase,
                                            const T* __restrict__ vbase, int n, int j0,
                                            int step, PosFn pos_of, const float q[4],
                                            float scale_log2, int lane, SoftmaxState& st) {
  using R = Raw4<T>;
  constexpr int kRows = 8;
  for (int j = j0; j < n; j += kRows * step) {
    typename R::type kr[kRows], vr[kRows];
    bool valid[kRows];
#pragma unroll
    for (int u = 0; u < kRows; ++u) {
      const int jj = j + u * step;
      valid[u] = jj < n;
      if (valid[u]) {
        const int64_t pos = pos_of(jj);
        kr[u] = R::load(kbase + pos * kD, lane);
        vr[u] = R::load(vbase + pos * kD, lane);
      }
    }
    float s[kRows];
#pragma unroll
    for (int u = 0; u < kRows; ++u) {
      float kv[4];
      if (valid[u]) {
        R::decode(kr[u], kv);
        s[u] = q[0] * kv[0] + q[1] * kv[1] + q[2] * kv[2] + q[3] * kv[3];
      } else {
        s[u] = 0.f;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
      for (int u = 0; u < kRows; ++u) s[u] += __shfl_xor_sync(0xffffffffu, s[u], o);
    }
    float mx = st.m;
#pragma unroll
    for (int u = 0; u < kRows; ++u) {
      s[u] = valid[u] ? s[u] * scale_log2 : -INFINITY;
      mx = fmaxf(mx, s[u]);
    }
    const float corr = exp2f(st.m - mx);   // st.m = -inf -> 0
    st.l *= corr;
#pragma unroll
    for (int r = 0; r < 4; ++r) st.acc[r] *= corr;
#pragma unroll
    for (int u = 0; u < kRows; ++u) {
      if (valid[u]) {
        const float p = exp2f(s[u] - mx);
        float vv[4];
        R::decode(vr[u], vv);
        st.l += p;
#pragma unroll
        for (int r = 0; r < 4; ++r) st.acc[r] = fmaf(p, vv[r], st.acc[r]);
      }
    }
    st.m = mx;
  }
}

// attend_rows for a group of GM query heads that share one selection: each K/V row
// is loaded once and scored against all GM queries (q[g][4] is lane's slice of
// query g); st[g] is head g's state.  kRows rows are in flight per warp.
template <typename T, int GM, int kRows, typename PosFn>
__device__ __forceinline__ void attend_rows_group(const T* __restrict__ kbase,
                                                  const T* __restrict__ vbase, int n, int j0,
                                                  int step, PosFn pos_of,
                                                  const float (&q)[GM][4], float scale_log2,
                                                  int lane, SoftmaxState (&st)[GM]) {
  using R = Raw4<T>;
  for (int j = j0; j < n; j += kRows * step) {
    typename R::type kr[kRows], vr[kRows];
    bool valid[kRows];
#pragma unroll
    for (int u = 0; u < kRows; ++u) {
      const int jj = j + u * step;
      valid[u] = jj < n;
      if (valid[u]) {
        const int64_t pos = pos_of(jj);
        kr[u] = R::load(kbase + pos * kD, lane);
        vr[u] = R::load(vbase + pos * kD, lane);
      }
    }
    float s[GM][kRows];
#pragma unroll
    for (int u = 0; u < kRows; ++u) {
      float kv[4] = {0.f, 0.f, 0.f, 0.f};
      if (valid[u]) R::decode(kr[u], kv);
#pragma unroll
      for (int g = 0; g < GM; ++g)
        s[g][u] = q[g][0] * kv[0] + q[g][1] * kv[1] + q[g][2] * kv[2] + q[g][3] * kv[3];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
      for (int g = 0; g < GM; ++g) {
#pragma unroll
        for (int u = 0; u < kRows; ++u) s[g][u] += __shfl_xor_sync(0xffffffffu, s[g][u], o);
      }
    }
    float vv[kRows][4];
#pragma unroll
    for (int u = 0; u < kRows; ++u) {
      vv[u][0] = vv[u][1] = vv[u][2] = vv[u][3] = 0.f;
      if (valid[u]) R::decode(vr[u], vv[u]);
    }
#pragma unroll
    for (int g = 0; g < GM; ++g) {
      float mx = st[g].m;
#pragma unroll
      for (int u = 0; u < kRows; ++u) {
        s[g][u] = valid[u] ? s[g][u] * scale_log2 : -INFINITY;
        mx = fmaxf(mx, s[g][u]);
      }
      const float corr = exp2f(st[g].m - mx);   // st.m = -inf -> 0
      st[g].l *= corr;
#pragma unroll
      for (int r = 0; r < 4; ++r) st[g].acc[r] *= corr;
#pragma unroll
      for (int u = 0; u < kRows; ++u) {
        if (valid[u]) {
          const float p = exp2f(s[g][u] - mx);
          st[g].l += p;
#pragma unroll
          for (int r = 0; r < 4; ++r) st[g].acc[r] = fmaf(p, vv[u][r], st[g].acc[r]);
        }
      }
      st[g].m = mx;
    }
  }
}

// Merge two softmax partials (m, l, acc) into (M, Lsum, A) accumulators.
__device__ __forceinline__ void merge_into(float m, float l, float a, float& M, float& Ls,
                                           float& A) {
  if (l == 0.f) return;
  if (m > M) {
    const float c = exp2f(M - m);
    Ls = Ls * c + l;
    A = A * c + a;
    M = m;
  } else {
    const float c = exp2f(m - M);
    Ls += l * c;
    A += a * c;
  }
}

// ------------------------------------------------------------- host side
int current_device_sms(int* dev_out);
size_t align_up(size_t x, size_t a);

// Launch plan of the fused decode kernel (one thread-block cluster per unit).
struct Plan {
  int grid;              // CTAs = units x cluster
  int cluster;           // CTAs per (batch, kv head) unit
  int waves;             // modelled waves of clusters over the device
  int64_t keys_per_cta;  // R = ceil(L / cluster)
  int list_cap;          // selected-position slots per head per CTA
  int stages;            // bulk-copy ring depth
  size_t smem;           // dynamic shared memory bytes
  int64_t l2_bytes;      // device L2 capacity (0: unknown)
  bool dist_global;      // distances in workspace scratch, not shared memory
};
// page_shift: log2(page size) for paged caches, -1 for contiguous caches.  allow_gd:
// the plan may keep distances in workspace scratch (contiguous per-head kernels).
bool decode_plan_for_current_device(int B, int Hq, int Hkv, int64_t L, int k, bool shared,
                                    int page_shift, Plan& p, bool allow_gd = false);
size_t decode_workspace_bytes(int B, int Hq, int Hkv, int64_t L, int k);
size_t cp_workspace_bytes(int B, int Hq, int Hkv, int64_t L, int k, bool shared);
size_t decode_workspace_error_offset();
// Where a unit's positions live.  Contiguous caches: unit (b, kv head) owns rows
// [unit * Lmax, unit * Lmax + L).  Paged caches (block_table != nullptr): position p
// of sequence b is row p & (page - 1) of kv head h in page block_table[b][p >> shift],
// pages laid out [page][Hkv][page size][...].  seq_lens (nullable) gives each
// sequence its own length <= L.
struct CacheLayout {
  int64_t Lmax = 0;
  const int32_t* seq_lens = nullptr;
  const int32_t* block_table = nullptr;
  int max_blocks = 0;
  int page_shift = 0;
  int64_t num_pages = 0;
};
// One rank's part of a context-parallel step: the rank holds positions
// [pos_offset, pos_offset + L) of a context of L_total positions.
struct CpArgs {
  int phase;               // 1: export distance histograms; 2: select + attend + export partials
  int64_t L_total;
  int64_t pos_offset;
  uint32_t* hist_out;      // phase 1: [B][rows][bins] cumulative counts over the slice
                           //          (rows: Hq, or Hkv for shared selection)
  const uint32_t* hist_all;  // phase 2: [world][B][rows][bins], every rank's hist_out
  int world, rank;
  float* partial_out;      // phase 2: [B][Hq][kPartStride]: m (log2 domain), l, 0, 0, acc[128]
};
cudaError_t launch_decode(const void* q, const uint8_t* qcodes, const void* k, const void* v,
                          const uint8_t* codes, adamas_dtype dt, int B, int Hq, int Hkv,
                          const CacheLayout& lay, int64_t L, int kk, float t, void* ws,
                          int32_t* idx_out, float* out, bool shared, const Plan& p,
                          cudaStream_t stream, float t_ratio = 0.0f,
                          const CpArgs* cpa = nullptr);
// Distance bins of a selection row: 385 per query head, 384 G + 1 for shared selection.
inline int selection_bins(int G, bool shared) { return shared ? 384 * G + 1 : 3 * kD + 1; }
cudaError_t launch_cp_combine(const float* partials, int world, int64_t rows, float* out,
                              cudaStream_t stream);
cudaError_t launch_encode_rows(const void* src, adamas_dtype dt, uint8_t* dst, int64_t nvec,
                               int64_t per, int64_t stride, int64_t off, float t,
                               cudaStream_t stream, const int32_t* ids = nullptr,
                               int64_t id_limit = 0, float ratio = 0.0f);
size_t attention_workspace_bytes(int B, int Hq, int k_eff);
bool noalloc_fits(int B, int Hq);
cudaError_t launch_sparse_attention_noalloc(const void* q, const void* k, const void* v,
                                            adamas_dtype dt, const int32_t* idx, int B,
                                            int Hq, int Hkv, int64_t Lmax, int k_eff,
                                            float* out, cudaStream_t stream);
cudaError_t launch_sparse_attention(const void* q, const void* k, const void* v,
                                    adamas_dtype dt, const int32_t* idx, int B, int Hq,
                                    int Hkv, int64_t Lmax, int k_eff, void* ws, float* out,
                                    cudaStream_t stream);

}  // namespace adamas

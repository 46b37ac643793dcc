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
constexpr uint32_t kErrWait = 1u;     // a bounded wait for peer CTAs gave up
constexpr uint32_t kErrCopy = 2u;     // a bounded wait for a copy into shared memory gave up
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
// bytes a multiple of 16).  The source is read once: it is marked first to go from
// L2 (evict-first), so a long stream of it does not push out data the kernel reads
// again later (distances kept in workspace scratch, K/V rows pulled ahead).
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  uint64_t policy;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(policy));
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
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

// Packed fp32 pairs (sm_100 f32x2 arithmetic): one instruction per pair, each
// element rounded to nearest exactly as the scalar operation would be.
// (d0, d1) += (a0, a1) * (b0, b1)
__device__ __forceinline__ void fma_pair(float& d0, float& d1, float a0, float a1, float b0,
                                         float b1) {
  asm("{\n\t.reg .b64 pd, pa, pb;\n\t"
      "mov.b64 pd, {%0, %1};\n\t"
      "mov.b64 pa, {%2, %3};\n\t"
      "mov.b64 pb, {%4, %5};\n\t"
      "fma.rn.f32x2 pd, pa, pb, pd;\n\t"
      "mov.b64 {%0, %1}, pd;\n\t}"
      : "+f"(d0), "+f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
// (d0, d1) *= (m, m)
__device__ __forceinline__ void mul_pair(float& d0, float& d1, float m) {
  asm("{\n\t.reg .b64 pd, pm;\n\t"
      "mov.b64 pd, {%0, %1};\n\t"
      "mov.b64 pm, {%2, %2};\n\t"
      "mul.rn.f32x2 pd, pd, pm;\n\t"
      "mov.b64 {%0, %1}, pd;\n\t}"
      : "+f"(d0), "+f"(d1)
      : "f"(m));
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
// Packed-pair form of one 32-byte code, for exact Manhattan distances with few
// integer-logic operations.  A code word holds 16 fields c = 2h + l (l at the even
// bit, h at the odd bit).  For 2-bit codes k, q:
//   |k - q| = r0 + 2 r1,  r0 = l_k ^ l_q,
//   r1 = [|k - q| >= 2] = (h_k ^ h_q) & (e_q | (l_k ^ h_q)),  e_q = [q in {0, 3}],
// (all 16 cases check out: q = 0 gives h_k, q = 1 gives h_k l_k, q = 2 gives
// ~h_k ~l_k, q = 3 gives ~h_k).  Words A = w[2j] and B = w[2j+1] are packed into three
// words carrying one bit per coordinate of both, so that each of r0 and r1 costs one
// or two LOP3 per 32 coordinates:
//   p[j] = (A & EVEN) | ((B << 1) & ODD)   low bits: A's at even bits, B's at odd bits
//   h[j] = (A & ODD) | ((B >> 1) & EVEN)   high bits: A's at odd bits, B's at even bits
//   l[j] = ((A << 1) & ODD) | (B & EVEN)   low bits at the positions of h[j]
// A key keeps p, h, l; a query keeps p, h and e = ~(h ^ l).  The two left shifts are
// integer multiplies by an opaque 2 (`two`), so they run on the FMA pipe and leave
// the integer-logic pipe, the scan's bottleneck, to the rest.
struct PairWords {
  uint32_t p[4], h[4], x[4];   // x: l for a key, e for a query
};

__device__ __forceinline__ uint32_t mul_opaque(uint32_t a, uint32_t m) {
  uint32_t r;
  asm("mul.lo.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(m));
  return r;
}

// Key words of one packed code; `two` is 2 at run time, opaque to the compiler.
__device__ __forceinline__ void make_pairs(const uint32_t w[8], PairWords& t, uint32_t two) {
  constexpr uint32_t kEven = 0x55555555u;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t A = w[2 * j], B = w[2 * j + 1];
    const uint32_t A2 = mul_opaque(A, two), B2 = mul_opaque(B, two);
    t.p[j] = (A & kEven) | (B2 & ~kEven);
    t.h[j] = (A & ~kEven) | ((B >> 1) & kEven);
    t.x[j] = (A2 & ~kEven) | (B & kEven);
  }
}

// Query words of one packed code: p, h and e = [q in {0, 3}] at the positions of h.
__device__ __forceinline__ void make_query_pairs(const uint32_t w[8], PairWords& t) {
  make_pairs(w, t, 2u);
#pragma unroll
  for (int j = 0; j < 4; ++j) t.x[j] = ~(t.h[j] ^ t.x[j]);
}

// Manhattan distance of a key code (k) and a query code (q) in packed-pair form.
// The four r0 words (weight 1) and four r1 words (weight 2) are added bitwise by one
// carry-save level on three of each (sum word a^b^c, carry word majority(a,b,c), both
// single LOP3s), which leaves weight-1 words O and u1[3], weight-2 words T1, T2 and
// u2[3], and one weight-4 word F: 6 popcounts.  The popcount sums are integer
// multiply-adds with the opaque multiplier `one` (1 at run time), on the FMA pipe.
__device__ __forceinline__ uint32_t pair_dist(const PairWords& k, const PairWords& q,
                                              uint32_t one) {
  uint32_t u1[4], u2[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    u1[j] = k.p[j] ^ q.p[j];
    u2[j] = (k.h[j] ^ q.h[j]) & (q.x[j] | (k.x[j] ^ q.h[j]));
  }
  const uint32_t O = u1[0] ^ u1[1] ^ u1[2];
  const uint32_t T1 = (u1[0] & u1[1]) | (u1[2] & (u1[0] | u1[1]));
  const uint32_t T2 = u2[0] ^ u2[1] ^ u2[2];
  const uint32_t F = (u2[0] & u2[1]) | (u2[2] & (u2[0] | u2[1]));
  // sum = popc(O) + popc(u1[3]) + 2 (popc(T1) + popc(T2) + popc(u2[3])) + 4 popc(F)
  uint32_t s1 = uint32_t(__popc(O)), s2 = uint32_t(__popc(T1));
  asm("mad.lo.u32 %0, %1, %2, %0;" : "+r"(s1) : "r"(uint32_t(__popc(u1[3]))), "r"(one));
  asm("mad.lo.u32 %0, %1, %2, %0;" : "+r"(s2) : "r"(uint32_t(__popc(T2))), "r"(one));
  asm("mad.lo.u32 %0, %1, %2, %0;" : "+r"(s2) : "r"(uint32_t(__popc(u2[3]))), "r"(one));
  uint32_t r;
  asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(r) : "r"(s2), "r"(one + one), "r"(s1));
  asm("mad.lo.u32 %0, %1, %2, %0;" : "+r"(r) : "r"(uint32_t(__popc(F))), "r"(4u * one));
  return r;
}

// ------------------------------------------------------ decode block shape
constexpr int kThreads = 512;              // threads per decode CTA
constexpr int kWarps = kThreads / 32;
constexpr int kChunk = kThreads;           // keys per bulk copy (16 KiB of codes), one per thread

// Row stride (u16 elements) of a CTA's per-head distance array: a multiple of 8, so
// rows start on 16-byte boundaries.
__host__ __device__ inline int dist_stride(int R) { return (R + 7) & ~7; }

// Bit 15 and bit 31 of w0, then of w1, as bits 0..3 (the sign bits of four packed
// 16-bit lanes): a byte permute gathers the four high bytes, one multiply moves
// their top bits to bits 28..31 without carries.
__device__ __forceinline__ uint32_t lane_sign_bits(uint32_t w0, uint32_t w1) {
  const uint32_t b = __byte_perm(w0, w1, 0x7531) & 0x80808080u;
  return (b * 0x00204081u) >> 28;
}

// Exclusive prefix over the block (thread order) of G counters per thread, and the
// block totals, with one barrier: warp totals go to shared memory, then in every warp
// lanes 0..kWarps-1 take one total each and a shuffle scan over them gives each
// warp its offset and the block total.  `scan` holds two buffers of kWarps x G
// words used alternately (by `parity`), so a call never overwrites totals that a
// slower warp may still be reading from the previous call.
template <int G>
__device__ __forceinline__ void block_exclusive_scan(uint32_t (&v)[G], uint32_t (&total)[G],
                                                     uint32_t* scan, int parity, int lane,
                                                     int warp) {
  static_assert(kWarps <= 32, "one warp total per lane");
  uint32_t* buf = scan + parity * kWarps * G;
  uint32_t inc[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    uint32_t x = v[g];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    inc[g] = x;
    if (lane == 31) buf[warp * G + g] = x;
  }
  __syncthreads();
#pragma unroll
  for (int g = 0; g < G; ++g) {
    uint32_t x = lane < kWarps ? buf[lane * G + g] : 0u;
#pragma unroll
    for (int o = 1; o < kWarps; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    // x: inclusive prefix of the warp totals (lane w: warps 0..w)
    const uint32_t upto = __shfl_sync(0xffffffffu, x, (warp + 31) & 31);
    total[g] = __shfl_sync(0xffffffffu, x, kWarps - 1);
    v[g] = (warp > 0 ? upto : 0u) + inc[g] - v[g];
  }
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

// attend_rows for bf16 rows with 8 lanes per row: lane l is sub-lane sl = l & 7 of
// group gq = l >> 3 and holds dimensions 16 sl .. 16 sl + 15 (two 16-byte loads per
// row of K and of V); the warp's four groups take rows j0 + (4 u + gq) step, so a
// warp step covers 4 kR rows with three xor-shuffle levels per row instead of five.
// Each group keeps its own online softmax; at the end the four groups are merged
// (xor 8, xor 16) and the result is handed over in attend_rows' layout (lane l:
// dimensions 4 l .. 4 l + 3) in `st`.  qrow: the query, 128 floats (shared memory).
// With `ahead`, the K/V rows of the warp step kAhead steps on are pulled into L2 at
// every step (lanes 0-3 of each group: one 128-byte line each), so many more rows
// are on their way from HBM than the registers can hold; callers pass it when the
// rows were not pulled into L2 earlier.
template <typename PosFn>
__device__ __forceinline__ void attend_rows_bf16_g8(const __nv_bfloat16* __restrict__ kbase,
                                                    const __nv_bfloat16* __restrict__ vbase,
                                                    int n, int j0, int step, PosFn pos_of,
                                                    const float* qrow, float scale_log2,
                                                    int lane, SoftmaxState& st,
                                                    bool ahead = false) {
  constexpr int kR = 2;       // rows in flight per group
  constexpr int kAhead = 2;   // warp steps between a row's L2 pull and its loads
  const int gq = lane >> 3, sl = lane & 7;
  const int span = 4 * kR * step;
  const auto pull = [&](int jb) {
    if (sl < 4) {
#pragma unroll
      for (int u = 0; u < kR; ++u) {
        const int jj = jb + (4 * u + gq) * step;
        if (jj < n) {
          const __nv_bfloat16* row = (sl < 2 ? kbase : vbase) + pos_of(jj) * kD;
          asm volatile("prefetch.global.L2 [%0];" ::"l"(row + 64 * (sl & 1)));
        }
      }
    }
  };
  if (ahead) {
    for (int d = 0; d < kAhead; ++d) pull(j0 + d * span);
  }
  float q[16];
#pragma unroll
  for (int i = 0; i < 16; i += 4) {
    const float4 x = *reinterpret_cast<const float4*>(qrow + 16 * sl + i);
    q[i] = x.x; q[i + 1] = x.y; q[i + 2] = x.z; q[i + 3] = x.w;
  }
  float m = -INFINITY, l = 0.f, acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  for (int jb = j0; jb < n; jb += span) {
    if (ahead) pull(jb + kAhead * span);
    uint4 kr[kR][2], vr[kR][2];
    bool valid[kR];
#pragma unroll
    for (int u = 0; u < kR; ++u) {
      const int jj = jb + (4 * u + gq) * step;
      valid[u] = jj < n;
      if (valid[u]) {
        const int64_t pos = pos_of(jj);
        const uint4* kp = reinterpret_cast<const uint4*>(kbase + pos * kD) + 2 * sl;
        const uint4* vp = reinterpret_cast<const uint4*>(vbase + pos * kD) + 2 * sl;
        kr[u][0] = __ldg(kp);
        kr[u][1] = __ldg(kp + 1);
        vr[u][0] = __ldg(vp);
        vr[u][1] = __ldg(vp + 1);
      } else {
        kr[u][0] = kr[u][1] = vr[u][0] = vr[u][1] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    float s[kR];
#pragma unroll
    for (int u = 0; u < kR; ++u) {
      const uint32_t w[8] = {kr[u][0].x, kr[u][0].y, kr[u][0].z, kr[u][0].w,
                             kr[u][1].x, kr[u][1].y, kr[u][1].z, kr[u][1].w};
      float d0 = 0.f, d1 = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float lo, hi;
        bf16x2_to_f32(w[i], lo, hi);
        fma_pair(d0, d1, q[2 * i], q[2 * i + 1], lo, hi);
      }
      s[u] = d0 + d1;
    }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
#pragma unroll
      for (int u = 0; u < kR; ++u) s[u] += __shfl_xor_sync(0xffffffffu, s[u], o);
    }
    float mx = m;
#pragma unroll
    for (int u = 0; u < kR; ++u) {
      s[u] = valid[u] ? s[u] * scale_log2 : -INFINITY;
      mx = fmaxf(mx, s[u]);
    }
    if (mx != -INFINITY) {   // the same in all 8 lanes of a group
      const float corr = exp2f(m - mx);   // m = -inf -> 0
      l *= corr;
#pragma unroll
      for (int i = 0; i < 16; i += 2) mul_pair(acc[i], acc[i + 1], corr);
#pragma unroll
      for (int u = 0; u < kR; ++u) {
        if (valid[u]) {
          const float p = exp2f(s[u] - mx);
          l += p;
          const uint32_t w[8] = {vr[u][0].x, vr[u][0].y, vr[u][0].z, vr[u][0].w,
                                 vr[u][1].x, vr[u][1].y, vr[u][1].z, vr[u][1].w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float lo, hi;
            bf16x2_to_f32(w[i], lo, hi);
            fma_pair(acc[2 * i], acc[2 * i + 1], p, p, lo, hi);
          }
        }
      }
      m = mx;
    }
  }
  // merge the four groups' states (an empty group has m = -inf, l = 0)
#pragma unroll
  for (int o = 8; o < 32; o <<= 1) {
    const float mo = __shfl_xor_sync(0xffffffffu, m, o);
    const float lo = __shfl_xor_sync(0xffffffffu, l, o);
    const float M = fmaxf(m, mo);
    const float c1 = M == -INFINITY ? 0.f : exp2f(m - M);
    const float c2 = M == -INFINITY ? 0.f : exp2f(mo - M);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float ao = __shfl_xor_sync(0xffffffffu, acc[i], o);
      acc[i] = acc[i] * c1 + ao * c2;
    }
    l = l * c1 + lo * c2;
    m = M;
  }
  // hand over: lane L takes dimensions 4 L .. 4 L + 3, held (identically) by every
  // lane of sub-lane L >> 2; the lane of group L & 3 offers entries 4 (L & 3) + r
  float mine[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    float v = acc[r];
#pragma unroll
    for (int g = 1; g < 4; ++g) v = gq == g ? acc[4 * g + r] : v;
    mine[r] = v;
  }
  const int src = (lane >> 2) + 8 * (lane & 3);
  st.m = m;
  st.l = l;
#pragma unroll
  for (int r = 0; r < 4; ++r) st.acc[r] = __shfl_sync(0xffffffffu, mine[r], src);
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
  bool flat;             // grid-wide kernel: `cluster` = 1, exchange through the workspace
  int cand_cap;          // flat: candidate slots per head per CTA
};
// Test hook of the copy-wait error path (adamas_test_set_copy_fault): extra bytes the
// first code chunk's barrier is armed for (the copy never delivers them); 0 restores
// normal operation.
void set_copy_fault(uint32_t extra_tx_bytes);
// Which decode kernel the planner may choose: 0 = the faster by its cost model,
// 1 = thread-block clusters only, 2 = the grid-wide kernel wherever it applies.
void set_decode_policy(int policy);
int decode_policy();
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
// Grid-wide decode step (contiguous caches, per-query-head selection): plan and launch.
bool make_flat_plan(int B, int Hq, int Hkv, int64_t L, int k, int sms, int smem_cap, Plan& p);
size_t flat_workspace_bytes(int B, int Hq, int Hkv, const Plan& p);
cudaError_t launch_decode_flat(const void* q, const uint8_t* qcodes, const void* k,
                               const void* v, const uint8_t* codes, adamas_dtype dt, int B,
                               int Hq, int Hkv, const CacheLayout& lay, int64_t L, int kk,
                               float t, float t_ratio, void* ws, int32_t* idx_out, float* out,
                               const Plan& p, cudaStream_t stream);
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

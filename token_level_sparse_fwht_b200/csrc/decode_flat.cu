// Grid-wide ("flat") Adamas decode step: ONE launch, one CTA per SM, for contiguous
// caches with per-query-head selection when the (batch, kv head) units are too few
// for thread-block clusters to fill the device (the 32K Llama-shaped layer has 8
// units; clusters of at most 10 co-resident CTAs leave 68 of 148 SMs idle).
//
//   query encode -> distance scan -> exact per-head top-k -> gather attention
//   (one split per CTA) -> combine of the splits
//
// Method: "Adamas: Hadamard Sparse Attention for Efficient Long-Context
// Inference" — v2 abstract (compact 2-bit codes, distance-based top-k, gather of
// the original KV states for sparse attention), v1 abstract (Manhattan distance).
//
// Work split.  Unit u = (b, kv head) gets S CTAs; CTA c owns key positions
// [c R, min(L, (c + 1) R)).  All U S CTAs are co-resident (the plan keeps U S at or
// below the device's SM count at one CTA per SM), so CTAs of a unit can wait for
// each other.  Every wait is bounded (1 s by %globaltimer); a wait that gives up
// records kErrWait in the workspace error word and the kernel still returns.
//
// Exact top-k with ties to the lower position.  Each CTA builds per head a 385-bin
// histogram of its distances (kept in shared memory with the distances), makes it
// cumulative and publishes it to the workspace as u16 counts.  After a per-unit
// barrier (arrival counter + generation word in the workspace) each CTA reads a
// 64-bin window of every peer's cumulative counts around its own estimate of the
// k-th distance D* (its local counts scaled up to the unit); one window usually
// brackets D*, otherwise the window moves toward it.  The window gives D*, the
// unit's count below D* and the counts below and at D* in lower-ranked CTAs, so the
// CTA knows how many of its D*-ties it takes and where its positions go.
//
// Latency hiding.  Between arriving at the barrier and waiting on it, every CTA
// collects its "candidates" — keys whose distance is at most a generous local
// bound tau — into a short list in shared memory, and pulls the K/V rows of those
// at or below its D* estimate into L2.  Selection then ranks only the candidates
// (a full pass over the distances is the fallback when D* exceeds tau).
//
// Attention and combine.  Each CTA gathers its selected rows (one split of each
// head's softmax), writes a partial (m, l, acc[128]) per head to the workspace, and
// the last CTA of the unit to finish (arrival counter) merges the S partials and
// writes the output.  Every counter is back at zero when the launch completes, so
// consecutive launches share one zero-initialised workspace.
#include <algorithm>
#include <mutex>
#include <type_traits>

#include "adamas_internal.cuh"

namespace adamas {

constexpr int kWin = 64;            // bins per window of the D* search
constexpr int kHistRow = 392;       // u16 counts per published row: bins 0..384, padded
constexpr int kFlatMaxS = 64;       // CTAs per unit
constexpr int kFlatMinKeys = 512;   // fewest keys worth a CTA
constexpr int kFlatMaxStages = 8;
constexpr int kCandSelectMax = 256; // candidates per head ranked pairwise; more: full pass
constexpr int kNS = kThreads / 32;  // warps

__host__ __device__ inline size_t al_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct FlatArgs {
  const void* q;             // [B][Hq][128] (encode mode) or nullptr
  const uint8_t* qcodes;     // [B][Hq][32] (select mode) or nullptr
  const void* k;             // [B][Hkv][Lmax][128]
  const void* v;
  const uint8_t* codes;      // [B][Hkv][Lmax][32]
  int B, Hq, Hkv;
  int64_t Lmax, L;
  int budget;
  int idx_stride;            // idx_out row length, min(k, L)
  const int32_t* seq_lens;   // [B] or nullptr
  float t, t_ratio, scale_log2;
  int32_t* idx_out;          // [B][Hq][idx_stride] or nullptr
  float* out;                // [B][Hq][128] or nullptr (select mode)
  uint32_t* err;
  int S;                     // CTAs per unit
  int R;                     // keys per CTA, a multiple of 8
  int stages;
  int cand_cap;
  int list_cap;
  int attend;
  int prefetch;
  uint32_t* sync;            // [U][4]: barrier count, barrier generation, done count, pad
  uint16_t* ghist;           // [U][G][S][kHistRow] cumulative counts
  float* gpart;              // [U][G][S][kPartStride] partials
};

struct FlatLayout {
  size_t ring, mbar, hist, dist, fine, cand, list, qf, qc, qth, scan, merge, info, misc, total;
};

__host__ __device__ inline FlatLayout flat_layout(int G, int R, int S, int stages, int cand_cap,
                                                  int list_cap) {
  FlatLayout s;
  size_t o = 0;
  s.ring = o;  o = al_up(o + size_t(stages) * kChunk * kCodeBytes, 128);
  s.mbar = o;  o = al_up(o + 8 * kFlatMaxStages, 128);
  s.hist = o;  o = al_up(o + size_t(G) * kBinStride * 4, 128);
  s.dist = o;  o = al_up(o + size_t(G) * dist_stride(R) * 2, 128);
  s.fine = o;  o = al_up(o + size_t(G) * S * kWin * 2, 128);
  s.cand = o;  o = al_up(o + size_t(G) * cand_cap * 4, 128);
  s.list = o;  o = al_up(o + size_t(G) * list_cap * 2, 128);
  s.qf = o;    o = al_up(o + size_t(G) * kD * 4, 128);
  s.qc = o;    o = al_up(o + size_t(G) * kCodeBytes, 128);
  s.qth = o;   o = al_up(o + size_t(G) * 12 * 4, 128);
  s.scan = o;  o = al_up(o + size_t(2) * kNS * G * 4, 128);
  s.merge = o; o = al_up(o + size_t(kNS) * kPartStride * 4, 128);
  s.info = o;  o = al_up(o + size_t(G) * 16 * 4, 128);
  s.misc = o;  o = al_up(o + 64 * 4, 128);
  s.total = o;
  return s;
}

// Workspace after the 256-byte error header: per-unit sync words, published
// histograms, partials (each region 256-byte aligned).
__host__ __device__ inline size_t flat_sync_bytes(int64_t U) { return al_up(size_t(U) * 16, 256); }
__host__ __device__ inline size_t flat_hist_bytes(int64_t U, int G, int S) {
  return al_up(size_t(U) * G * S * kHistRow * 2, 256);
}
__host__ __device__ inline size_t flat_part_bytes(int64_t U, int G, int S) {
  return al_up(size_t(U) * G * S * kPartStride * 4, 256);
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_u32(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// misc words in shared memory
constexpr int kMiscAbort = 0;      // a bounded wait gave up in this CTA
constexpr int kMiscLast = 1;       // this CTA merges the unit's partials
constexpr int kMiscFull = 2;       // some head needs the full selection pass
constexpr int kMiscCount = 8;      // [G] candidate counts
// info words per head: [0] window start, [1] resolved, [2] D*, [3] base, [4] take,
// [5] selected here, [6] D* estimate, [7] tau (candidate bound), [8] prefetch bound
template <int G, typename T>
__global__ void __launch_bounds__(kThreads, 1) decode_flat_kernel(const FlatArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  pdl_wait();
  const int S = a.S, R = a.R, RS = dist_stride(R);
  const FlatLayout lo = flat_layout(G, R, S, a.stages, a.cand_cap, a.list_cap);
  uint8_t* ring = smem + lo.ring;
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + lo.mbar);
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + lo.hist);   // [G][kBinStride]
  uint16_t* dist = reinterpret_cast<uint16_t*>(smem + lo.dist);   // [G][RS]
  uint16_t* fine = reinterpret_cast<uint16_t*>(smem + lo.fine);   // [G][S][kWin]
  uint32_t* cand = reinterpret_cast<uint32_t*>(smem + lo.cand);   // [G][cand_cap]
  uint16_t* list = reinterpret_cast<uint16_t*>(smem + lo.list);   // [G][list_cap]
  float* qf = reinterpret_cast<float*>(smem + lo.qf);             // [G][128]
  uint8_t* qc = smem + lo.qc;                                      // [G][32]
  uint32_t* qth = reinterpret_cast<uint32_t*>(smem + lo.qth);     // [G][12]
  uint32_t* scan = reinterpret_cast<uint32_t*>(smem + lo.scan);   // [2][kNS][G]
  float* merge = reinterpret_cast<float*>(smem + lo.merge);       // [kNS][kPartStride]
  int* info = reinterpret_cast<int*>(smem + lo.info);             // [G][16]
  int* misc = reinterpret_cast<int*>(smem + lo.misc);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int unit = blockIdx.x / S, c = blockIdx.x % S;
  const int b = unit / a.Hkv, kvh = unit % a.Hkv;
  int64_t L = a.L;
  if (a.seq_lens != nullptr) {
    const int64_t Lb = a.seq_lens[b];
    if ((Lb < 0 || Lb > a.L) && tid == 0 && c == 0) atomicOr(a.err, kErrInput);
    L = min(max(Lb, int64_t(0)), a.L);
  }
  const int keff = int(min(int64_t(a.budget), L));
  const int64_t p0 = int64_t(c) * R;
  const int n = int(max(int64_t(0), min(int64_t(R), L - p0)));   // keys of this CTA
  const int nch = (n + kChunk - 1) / kChunk;
  const int NST = a.stages;
  const uint8_t* codes = a.codes + (int64_t(unit) * a.Lmax + p0) * kCodeBytes;
  uint32_t* sync = a.sync + size_t(unit) * 4;

  const auto issue_chunk = [&](int qi, int slot) {
    const int c0 = qi * kChunk;
    const int keys = min(kChunk, n - c0);
    mbar_expect_tx(&mbar[slot], uint32_t(keys * kCodeBytes));
    bulk_g2s(ring + size_t(slot) * kChunk * kCodeBytes, codes + int64_t(c0) * kCodeBytes,
             uint32_t(keys * kCodeBytes), &mbar[slot]);
  };
  // ---- code copies first (last warp), so HBM traffic starts at once.  `issued`
  // (meaningful in the issuing thread only) counts the chunks in flight or landed.
  int issued = 0;
  if (tid == kThreads - 32) {
    for (int s = 0; s < NST; ++s) mbar_init(&mbar[s], 1);
    fence_mbar_init();
    for (int qi = 0; qi < min(nch, NST); ++qi) issue_chunk(qi, qi);
    issued = min(nch, NST);
  }
  // after a bounded wait gave up, no copy may still be writing this CTA's shared
  // memory when it exits: the issuing thread waits (bounded again) for the last
  // phase of every slot it filled
  const auto drain_copies = [&]() {
    if (misc[kMiscAbort] && tid == kThreads - 32) {
      for (int qi = max(0, issued - NST); qi < issued; ++qi)
        mbar_wait_bounded(&mbar[qi % NST], uint32_t((qi / NST) & 1), a.err);
    }
  };

  // ---- prologue: zero histograms and counters, encode (or fetch) the G query codes
  for (int i = tid; i < G * kBinStride; i += kThreads) hist[i] = 0u;
  if (tid < 64) misc[tid] = 0;
  if (warp < G) {
    const int g = warp, h = kvh * G + g;
    if (a.qcodes != nullptr) {
      qc[g * kCodeBytes + lane] = a.qcodes[(int64_t(b) * a.Hq + h) * kCodeBytes + lane];
    } else {
      float v[4];
      const T* qsrc = static_cast<const T*>(a.q) + (int64_t(b) * a.Hq + h) * kD;
      if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        // 16-byte loads by lanes 0-15 (q may live in mapped host memory), then
        // redistributed to 4 elements per lane
        uint4 x = make_uint4(0u, 0u, 0u, 0u);
        if (lane < 16) x = __ldg(reinterpret_cast<const uint4*>(qsrc) + lane);
        const int from = lane >> 1;
        const uint32_t w0 = __shfl_sync(0xffffffffu, x.x, from);
        const uint32_t w1 = __shfl_sync(0xffffffffu, x.y, from);
        const uint32_t w2 = __shfl_sync(0xffffffffu, x.z, from);
        const uint32_t w3 = __shfl_sync(0xffffffffu, x.w, from);
        bf16x2_to_f32((lane & 1) ? w2 : w0, v[0], v[1]);
        bf16x2_to_f32((lane & 1) ? w3 : w1, v[2], v[3]);
      } else {
        load4(qsrc, lane, v);
      }
      float* qrow = qf + g * kD + 4 * lane;
      qrow[0] = v[0]; qrow[1] = v[1]; qrow[2] = v[2]; qrow[3] = v[3];
      qc[g * kCodeBytes + lane] = static_cast<uint8_t>(warp_fwht_code(v, a.t, lane, a.t_ratio));
    }
  }
  __syncthreads();
  if (tid < G) {
    const uint32_t* wq = reinterpret_cast<const uint32_t*>(qc + tid * kCodeBytes);
    uint32_t wd[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) wd[i] = wq[i];
    PairWords th;
    make_query_pairs(wd, th);
    uint32_t* dst = qth + tid * 12;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      dst[j] = th.p[j];
      dst[4 + j] = th.h[j];
      dst[8 + j] = th.x[j];
    }
  }
  __syncthreads();

  // ---- distance scan: one key per thread per chunk, G heads per key (same word order
  // and arithmetic as the cluster kernel: key pair j against query pair (j + 2 swz) % 4)
  {
    constexpr int GR = G > 4 ? 4 : G;
    const int swz = (tid >> 2) & 1;
    PairWords qreg[GR];
    const auto load_q = [&](int g, PairWords& qt) {
      const uint2* s = reinterpret_cast<const uint2*>(qth + g * 12);
      const uint2 p0v = s[swz], p1v = s[swz ^ 1];
      const uint2 h0 = s[2 + swz], h1 = s[2 + (swz ^ 1)];
      const uint2 x0 = s[4 + swz], x1 = s[4 + (swz ^ 1)];
      qt.p[0] = p0v.x; qt.p[1] = p0v.y; qt.p[2] = p1v.x; qt.p[3] = p1v.y;
      qt.h[0] = h0.x; qt.h[1] = h0.y; qt.h[2] = h1.x; qt.h[3] = h1.y;
      qt.x[0] = x0.x; qt.x[1] = x0.y; qt.x[2] = x1.x; qt.x[3] = x1.y;
    };
    if constexpr (G <= 4) {
#pragma unroll
      for (int g = 0; g < GR; ++g) load_q(g, qreg[g]);
    }
    const uint32_t one = uint32_t(a.R > 0);   // 1, opaque to the compiler
    const uint32_t two = one + one;
    const auto load_key = [&](int sl, PairWords& kt) {
      const uint4* src =
          reinterpret_cast<const uint4*>(ring + (size_t(sl) * kChunk + tid) * kCodeBytes);
      const uint4 xa = src[swz], xb = src[swz ^ 1];
      const uint32_t wd[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
      make_pairs(wd, kt, two);
    };
    const auto score = [&](const PairWords& kt, int r) {
#pragma unroll
      for (int g0 = 0; g0 < G; g0 += GR) {
        if constexpr (G > 4) {
#pragma unroll
          for (int g = 0; g < GR; ++g) load_q(g0 + g, qreg[g]);
        }
#pragma unroll
        for (int g = 0; g < GR; ++g) {
          const uint32_t dd = pair_dist(kt, qreg[g], one);
          dist[size_t(g0 + g) * RS + r] = static_cast<uint16_t>(dd);
          atomicAdd(&hist[(g0 + g) * kBinStride + dd], 1u);
        }
      }
    };
    int slot = 0;
    uint32_t parity = 0;
    int qi = 0;
    if constexpr (G <= 2) {
      // one or two heads per key leave each key's chain short: two chunks per
      // iteration while the ring holds at least four
      if (NST >= 4) {
        for (; qi + 1 < nch; qi += 2) {
          int slot2 = slot + 1;
          uint32_t par2 = parity;
          if (slot2 == NST) { slot2 = 0; par2 ^= 1u; }
          if (!mbar_wait_bounded(&mbar[slot], parity, a.err)) misc[kMiscAbort] = 1;
          if (!mbar_wait_bounded(&mbar[slot2], par2, a.err)) misc[kMiscAbort] = 1;
          PairWords kt0, kt1;
          load_key(slot, kt0);
          load_key(slot2, kt1);
          const int r0 = qi * kChunk + tid, r1 = r0 + kChunk;
          if (r0 < n) score(kt0, r0);
          if (r1 < n) score(kt1, r1);
          if (nch > NST) __syncthreads();
          if (tid == kThreads - 32 && !misc[kMiscAbort]) {
            if (qi + NST < nch) { issue_chunk(qi + NST, slot); ++issued; }
            if (qi + 1 + NST < nch) { issue_chunk(qi + 1 + NST, slot2); ++issued; }
          }
          slot = slot2 + 1;
          parity = par2;
          if (slot == NST) { slot = 0; parity ^= 1u; }
        }
      }
    }
    for (; qi < nch; ++qi) {
      if (!mbar_wait_bounded(&mbar[slot], parity, a.err)) misc[kMiscAbort] = 1;
      const int r = qi * kChunk + tid;
      if (r < n) {
        PairWords kt;
        load_key(slot, kt);
        score(kt, r);
      }
      // a slot is refilled only when the CTA's keys need more chunks than the ring
      // holds; otherwise every chunk has its own slot and warps run ahead freely
      if (nch > NST) __syncthreads();
      if (tid == kThreads - 32 && qi + NST < nch && !misc[kMiscAbort]) {
        issue_chunk(qi + NST, slot);
        ++issued;
      }
      if (++slot == NST) { slot = 0; parity ^= 1u; }
    }
  }
  __syncthreads();   // every key's distances and histogram counts are in

  // ---- cumulative histograms (a warp per head, lane l owning bins 13 l .. 13 l + 12)
  // and the local estimates: D* estimate = the first bin where the local count scaled
  // to the unit (x L / n) reaches k_eff; candidate bound tau = the first bin where it
  // reaches 2 k_eff + 64, lowered until the candidates fit the list
  if (warp < G) {
    constexpr int CB = 13;
    const int g = warp;
    uint32_t* row = hist + g * kBinStride;
    uint32_t loc[CB];
    uint32_t sum = 0;
#pragma unroll
    for (int i = 0; i < CB; ++i) {
      const int bin = CB * lane + i;
      loc[i] = bin < kNBins ? row[bin] : 0u;
      sum += loc[i];
    }
    uint32_t inc = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    uint32_t run = inc - sum;
    const int64_t nn = max(n, 1);
    const int64_t x_est = int64_t(keff) * nn, x_tau = int64_t(2 * keff + 64) * nn;
    int f_est = 1 << 30, f_tau = 1 << 30, f_cap = -1;
#pragma unroll
    for (int i = 0; i < CB; ++i) {
      const int bin = CB * lane + i;
      run += loc[i];
      if (bin < kNBins) {
        row[bin] = run;
        const int64_t scaled = int64_t(run) * L;
        if (scaled >= x_est && f_est > bin) f_est = bin;
        if (scaled >= x_tau && f_tau > bin) f_tau = bin;
        if (run <= uint32_t(a.cand_cap)) f_cap = bin;
      }
    }
    // warp minima / maxima
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      f_est = min(f_est, __shfl_xor_sync(0xffffffffu, f_est, o));
      f_tau = min(f_tau, __shfl_xor_sync(0xffffffffu, f_tau, o));
      f_cap = max(f_cap, __shfl_xor_sync(0xffffffffu, f_cap, o));
    }
    if (lane == 0) {
      const int est = min(f_est, kNBins - 1);
      const int tau = min(min(f_tau, kNBins - 1), f_cap);   // f_cap = -1: no candidates
      int* in = info + g * 16;
      in[0] = min(max(0, (est - 24) & ~7), kHistRow - kWin);
      in[1] = 0;
      in[6] = est;
      in[7] = tau;
      in[8] = a.prefetch ? min(est, tau) : -1;
    }
  }
  __syncthreads();
  // publish the cumulative counts as u16 rows [U][G][S][kHistRow] (bins past 384 hold
  // the total), 16-byte stores
  for (int i = tid; i < G * (kHistRow / 8); i += kThreads) {
    const int g = i / (kHistRow / 8), j = i % (kHistRow / 8);
    const uint32_t* row = hist + g * kBinStride;
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int b0 = min(8 * j + 2 * e, kNBins - 1), b1 = min(8 * j + 2 * e + 1, kNBins - 1);
      w[e] = (row[b0] & 0xffffu) | (row[b1] << 16);
    }
    uint4* dst = reinterpret_cast<uint4*>(
        a.ghist + ((size_t(unit) * G + g) * S + c) * kHistRow + 8 * j);
    *dst = make_uint4(w[0], w[1], w[2], w[3]);
  }
  __syncthreads();

  // ---- arrive at the unit's barrier (the generation is read before arriving, so it
  // cannot have moved on yet); the last to arrive resets the count and releases
  uint32_t gen0 = 0;
  bool passed = false;
  if (tid == 0) {
    gen0 = ld_acquire_u32(sync + 1);
    __threadfence();
    const uint32_t arrived = atomicAdd(sync, 1u) + 1u;
    if (arrived == uint32_t(S)) {
      atomicExch(sync, 0u);
      __threadfence();
      st_release_u32(sync + 1, gen0 + 1u);
      passed = true;
    }
  }

  // ---- while the peers arrive: candidates (distance <= tau) into the per-head
  // lists, K/V rows at or below the D* estimate into L2
  {
    const int per_head = RS / 8;
    for (int i = tid; i < G * per_head; i += kThreads) {
      const int g = i / per_head, r0 = 8 * (i % per_head);
      const int tau = info[g * 16 + 7], pre = info[g * 16 + 8];
      const uint4 v = *reinterpret_cast<const uint4*>(dist + size_t(g) * RS + r0);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int r = r0 + e;
        const int d = int((w[e >> 1] >> (16 * (e & 1))) & 0xffffu);
        if (r < n && d <= tau) {
          const int slot = atomicAdd(&misc[kMiscCount + g], 1);
          if (slot < a.cand_cap) cand[g * a.cand_cap + slot] = (uint32_t(d) << 16) | uint32_t(r);
          if (d <= pre && a.attend) {
            const int64_t row_off = (int64_t(unit) * a.Lmax + p0 + r) * kD;
            prefetch_row_l2(static_cast<const T*>(a.k) + row_off);
            prefetch_row_l2(static_cast<const T*>(a.v) + row_off);
          }
        }
      }
    }
  }

  // ---- wait for the unit's other CTAs
  if (tid == 0 && !passed) {
    const unsigned long long t0 = globaltimer_ns();
    while (ld_acquire_u32(sync + 1) == gen0) {
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        atomicOr(a.err, kErrWait);
        misc[kMiscAbort] = 1;
        break;
      }
    }
    __threadfence();
  }
  __syncthreads();

  // ---- resolve D*, the unit's count below it, the lower-ranked CTAs' counts below
  // and at it (each head: windows of kWin bins of every CTA's published counts)
  for (int iter = 0;; ++iter) {
    for (int i = tid; i < G * S * (kWin / 8); i += kThreads) {
      const int g = i / (S * (kWin / 8));
      if (info[g * 16 + 1]) continue;
      const int cc = (i / (kWin / 8)) % S, j = i % (kWin / 8);
      const uint4 v = __ldcg(reinterpret_cast<const uint4*>(
          a.ghist + ((size_t(unit) * G + g) * S + cc) * kHistRow + info[g * 16] + 8 * j));
      *reinterpret_cast<uint4*>(fine + (size_t(g) * S + cc) * kWin + 8 * j) = v;
    }
    __syncthreads();
    if (warp < G && !info[warp * 16 + 1]) {
      const int g = warp;
      int* in = info + g * 16;
      const int wlo = in[0];
      uint32_t C0 = 0, C1 = 0, B0 = 0, B1 = 0;   // unit / lower-ranked counts at 2 bins
#pragma unroll 8
      for (int cc = 0; cc < S; ++cc) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(fine + (size_t(g) * S + cc) * kWin +
                                                             2 * lane);
        const uint32_t x0 = w & 0xffffu, x1 = w >> 16;
        C0 += x0; C1 += x1;
        if (cc < c) { B0 += x0; B1 += x1; }
      }
      const uint32_t ke = uint32_t(keff);
      const uint32_t first = __shfl_sync(0xffffffffu, C0, 0);
      const uint32_t last = __shfl_sync(0xffffffffu, C1, 31);
      const bool below = wlo > 0 && first >= ke;
      const bool above = last < ke;
      if (below || above) {
        if (lane == 0) {
          in[0] = below ? max(0, wlo - (kWin - 8)) : min(kHistRow - kWin, wlo + (kWin - 8));
        }
      } else {
        const uint32_t h0 = __ballot_sync(0xffffffffu, C0 >= ke);
        const uint32_t h1 = __ballot_sync(0xffffffffu, C1 >= ke);
        // first bin reaching k_eff: bin 2 l (h0) comes before bin 2 l + 1 (h1)
        const int l0 = h0 ? __ffs(h0) - 1 : 64, l1 = h1 ? __ffs(h1) - 1 : 64;
        const int off = (l0 <= l1) ? 2 * l0 : 2 * l1 + 1;   // offset of D* in the window
        const int dstar = wlo + off;
        // counts one bin below D* (offset off - 1), if inside the window
        const int pl = (off - 1) >> 1;
        const uint32_t pC0 = __shfl_sync(0xffffffffu, C0, max(pl, 0));
        const uint32_t pC1 = __shfl_sync(0xffffffffu, C1, max(pl, 0));
        const uint32_t pB0 = __shfl_sync(0xffffffffu, B0, max(pl, 0));
        const uint32_t pB1 = __shfl_sync(0xffffffffu, B1, max(pl, 0));
        const int ql = off >> 1;
        const uint32_t qB0 = __shfl_sync(0xffffffffu, B0, ql);
        const uint32_t qB1 = __shfl_sync(0xffffffffu, B1, ql);
        uint32_t less = 0, lt_before = 0;
        if (off > 0) {
          less = ((off - 1) & 1) ? pC1 : pC0;
          lt_before = ((off - 1) & 1) ? pB1 : pB0;
        }
        const uint32_t eq_before = ((off & 1) ? qB1 : qB0) - lt_before;
        const uint32_t* own = hist + g * kBinStride;
        const int dcl = min(dstar, kNBins - 1);
        const uint32_t lt_own = dcl > 0 ? own[dcl - 1] : 0u;
        const uint32_t eq_own = own[dcl] - lt_own;
        const uint32_t need = ke - less;
        const uint32_t base = lt_before + min(eq_before, need);
        const uint32_t take = need > eq_before ? min(need - eq_before, eq_own) : 0u;
        if (lane == 0) {
          in[2] = dcl;
          in[3] = int(base);
          in[4] = int(take);
          in[5] = int(lt_own + take);
          in[1] = 1;
        }
      }
    }
    __syncthreads();
    bool done = true;
#pragma unroll
    for (int g = 0; g < G; ++g) done = done && info[g * 16 + 1];
    if (done) break;
    if (iter >= 16 || misc[kMiscAbort]) {
      // inconsistent counts (a peer gave up waiting): select nothing rather than guess
      if (tid == 0) atomicOr(a.err, kErrSelect);
      if (tid < G && !info[tid * 16 + 1]) {
        info[tid * 16 + 2] = kNBins - 1;
        info[tid * 16 + 3] = 0;
        info[tid * 16 + 4] = 0;
        info[tid * 16 + 5] = 0;
        info[tid * 16 + 1] = 1;
      }
      __syncthreads();
      break;
    }
  }

  // ---- select, in position order.  Usually from the candidate lists: a candidate
  // below D* is taken, one at D* if fewer than `take` D*-candidates sit before it;
  // its slot is the number of taken candidates before it.  Full pass over the
  // distances when some head's D* lies above its candidate bound (or it has too
  // many candidates to rank pairwise).
  if (tid < G) {
    const int m = misc[kMiscCount + tid];
    if (info[tid * 16 + 2] > info[tid * 16 + 7] || m > kCandSelectMax || m > a.cand_cap)
      atomicOr(&misc[kMiscFull], 1);
  }
  __syncthreads();
  const auto orow_of = [&](int g) -> int32_t* {
    return a.idx_out != nullptr
               ? a.idx_out + (int64_t(b) * a.Hq + kvh * G + g) * a.idx_stride + info[g * 16 + 3]
               : nullptr;
  };
  if (!misc[kMiscFull]) {
    constexpr int TPH = kThreads / G;   // threads per head
    const int g = tid / TPH, sub = tid % TPH;
    const int m = misc[kMiscCount + g];
    const int dstar = info[g * 16 + 2], take = info[g * 16 + 4], nsel = info[g * 16 + 5];
    const uint32_t* cl = cand + g * a.cand_cap;
    int32_t* orow = orow_of(g);
    const int base = info[g * 16 + 3];
    uint16_t* lrow = list + size_t(g) * a.list_cap;
    for (int i = sub; i < m; i += TPH) {
      const uint32_t ci = cl[i];
      const int di = int(ci >> 16), ri = int(ci & 0xffffu);
      if (di > dstar) continue;
      int lt_b = 0, eq_b = 0;   // candidates before ri below D* / at D*
      for (int j = 0; j < m; ++j) {
        const uint32_t cj = cl[j];
        const int dj = int(cj >> 16), rj = int(cj & 0xffffu);
        lt_b += (rj < ri && dj < dstar);
        eq_b += (rj < ri && dj == dstar);
      }
      if (di == dstar && eq_b >= take) continue;
      const int rk = lt_b + min(eq_b, take);
      if (rk < nsel && rk < a.list_cap && base + rk < keff) {
        lrow[rk] = static_cast<uint16_t>(ri);
        if (orow) orow[rk] = int32_t(p0 + ri);
      }
    }
  } else {
    // full pass: each thread owns up to 32 consecutive positions per round; "< D*" and
    // "== D*" masks by packed 16-bit compares, one block scan ranks them
    int dstar[G], take[G], nsel[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      dstar[g] = info[g * 16 + 2];
      take[g] = info[g * 16 + 4];
      nsel[g] = info[g * 16 + 5];
    }
    uint32_t carry_lt[G], carry_eq[G];
#pragma unroll
    for (int g = 0; g < G; ++g) carry_lt[g] = carry_eq[g] = 0;
    constexpr int kRoundKeys = kThreads * 32;
    for (int rb = 0, par = 0; rb < n; rb += kRoundKeys, par ^= 1) {
      const int nr = min(kRoundKeys, n - rb);
      const int per = (((nr + kThreads - 1) / kThreads) + 7) & ~7;
      const int s0 = rb + tid * per;
      const int cntv = max(0, min(per, rb + nr - s0));
      uint32_t ltm[G], eqm[G], cnt[G], tot[G], cle[G], clt[G];
      const uint32_t valid = cntv >= 32 ? 0xffffffffu : ((1u << cntv) - 1u);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        cle[g] = (0x8000u + uint32_t(dstar[g])) * 0x10001u;
        clt[g] = cle[g] - 0x10001u;
        ltm[g] = eqm[g] = 0;
      }
      for (int i8 = 0; i8 < cntv; i8 += 8) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const uint4 v = *reinterpret_cast<const uint4*>(dist + size_t(g) * RS + s0 + i8);
          const uint32_t l0 = lane_sign_bits(clt[g] - v.x, clt[g] - v.y);
          const uint32_t l1 = lane_sign_bits(clt[g] - v.z, clt[g] - v.w);
          const uint32_t e0 = lane_sign_bits(cle[g] - v.x, cle[g] - v.y) & ~l0;
          const uint32_t e1 = lane_sign_bits(cle[g] - v.z, cle[g] - v.w) & ~l1;
          ltm[g] |= (l0 | (l1 << 4)) << i8;
          eqm[g] |= (e0 | (e1 << 4)) << i8;
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        ltm[g] &= valid;
        eqm[g] &= valid;
        cnt[g] = (uint32_t(__popc(ltm[g])) << 16) | uint32_t(__popc(eqm[g]));
      }
      block_exclusive_scan<G>(cnt, tot, scan, par, lane, warp);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const int lt_b = int(carry_lt[g] + (cnt[g] >> 16));
        const int eq_b = int(carry_eq[g] + (cnt[g] & 0xffffu));
        uint32_t sel_eq = 0;
        const int te = take[g] - eq_b;
        if (te > 0) {
          uint32_t rest = eqm[g];
          for (int cc = 0; cc < te && rest; ++cc) rest &= rest - 1u;
          sel_eq = eqm[g] ^ rest;
        }
        uint32_t sel = ltm[g] | sel_eq;
        int rk = lt_b + min(eq_b, take[g]);
        int32_t* orow = orow_of(g);
        const int base = info[g * 16 + 3];
        uint16_t* lrow = list + size_t(g) * a.list_cap;
        while (sel) {
          const int i = __ffs(sel) - 1;
          sel &= sel - 1u;
          const int r = s0 + i;
          if (rk < nsel[g] && rk < a.list_cap && base + rk < keff) {
            lrow[rk] = static_cast<uint16_t>(r);
            if (orow) orow[rk] = int32_t(p0 + r);
          }
          ++rk;
        }
        carry_lt[g] += tot[g] >> 16;
        carry_eq[g] += tot[g] & 0xffffu;
      }
    }
  }
  // a sequence shorter than the budget fills only keff slots of its rows: CTA 0 marks
  // the rest -1
  if (a.seq_lens != nullptr && a.idx_out != nullptr && c == 0 && keff < a.idx_stride) {
    const int pad = a.idx_stride - keff;
    for (int i = tid; i < G * pad; i += kThreads) {
      const int g = i / pad;
      a.idx_out[(int64_t(b) * a.Hq + kvh * G + g) * a.idx_stride + keff + i % pad] = -1;
    }
  }
  __syncthreads();

  if (!a.attend) {
    drain_copies();
    return;
  }

  // ---- attention over the selected rows: 16 / G warps per head
  {
    constexpr int WPG = kNS / G;
    const int g = warp % G, sub = warp / G;
    const int nsel = min(info[g * 16 + 5], a.list_cap);
    const uint16_t* lrow = list + size_t(g) * a.list_cap;
    const int64_t base_row = int64_t(unit) * a.Lmax + p0;
    const T* kb = static_cast<const T*>(a.k) + base_row * kD;
    const T* vb = static_cast<const T*>(a.v) + base_row * kD;
    float qv[4];
    {
      const float* qrow = qf + g * kD + 4 * lane;
      qv[0] = qrow[0]; qv[1] = qrow[1]; qv[2] = qrow[2]; qv[3] = qrow[3];
    }
    SoftmaxState st;
    st.init();
    const auto pos_of = [&](int j) { return int64_t(lrow[j]); };
    // more than 8 rows per warp: bf16 rows go 8 lanes per row
    bool done = false;
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
      if (nsel > 8 * WPG) {
        attend_rows_bf16_g8(kb, vb, nsel, sub, WPG, pos_of, qf + g * kD, a.scale_log2, lane, st);
        done = true;
      }
    }
    if (!done) attend_rows<T>(kb, vb, nsel, sub, WPG, pos_of, qv, a.scale_log2, lane, st);
    float* mw = merge + (sub * G + g) * kPartStride;
    if (lane == 0) { mw[0] = st.m; mw[1] = st.l; }
#pragma unroll
    for (int r = 0; r < 4; ++r) mw[4 + 4 * lane + r] = st.acc[r];
  }
  __syncthreads();
  // this CTA's partial per head -> workspace
  for (int i = tid; i < G * kD; i += kThreads) {
    constexpr int WPG = kNS / G;
    const int gg = i / kD, dim = i % kD;
    float M = -INFINITY, Ls = 0.f, A = 0.f;
    for (int sw = 0; sw < WPG; ++sw) {
      const float* mm = merge + (sw * G + gg) * kPartStride;
      merge_into(mm[0], mm[1], mm[4 + dim], M, Ls, A);
    }
    float* prow = a.gpart + ((size_t(unit) * G + gg) * S + c) * kPartStride;
    if (dim == 0) { prow[0] = M; prow[1] = Ls; }
    prow[4 + dim] = A;
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    misc[kMiscLast] = (atomicAdd(sync + 2, 1u) + 1u == uint32_t(S)) ? 1 : 0;
  }
  __syncthreads();
  if (misc[kMiscLast]) {
    __threadfence();
    // the unit's S partials per head: four coordinates per thread, 16-byte stores (out
    // may live in mapped host memory).  Every partial's loads are issued before any is
    // used, eight at a time, so their L2 latencies overlap.
    for (int i = tid; i < G * (kD / 4); i += kThreads) {
      const int gg = i / (kD / 4), d4 = 4 * (i % (kD / 4));
      const float* pr0 = a.gpart + (size_t(unit) * G + gg) * S * kPartStride;
      float M = -INFINITY, Ls = 0.f;
      float4 A = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int c0 = 0; c0 < S; c0 += 8) {
        float m8[8], l8[8];
        float4 x8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (c0 + u < S) {
            const float* pr = pr0 + (c0 + u) * kPartStride;
            const float2 ml = __ldcg(reinterpret_cast<const float2*>(pr));
            m8[u] = ml.x;
            l8[u] = ml.y;
            x8[u] = __ldcg(reinterpret_cast<const float4*>(pr + 4 + d4));
          } else {
            m8[u] = -INFINITY;
            l8[u] = 0.f;
            x8[u] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
        // fold the eight into the running state (an empty split has l = 0, m = -inf)
        float Mn = M;
#pragma unroll
        for (int u = 0; u < 8; ++u) Mn = fmaxf(Mn, l8[u] > 0.f ? m8[u] : -INFINITY);
        if (Mn != -INFINITY) {
          const float cs = M == -INFINITY ? 0.f : exp2f(M - Mn);
          Ls *= cs;
          A.x *= cs; A.y *= cs; A.z *= cs; A.w *= cs;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            if (l8[u] > 0.f) {
              const float e = exp2f(m8[u] - Mn);
              Ls = fmaf(l8[u], e, Ls);
              A.x = fmaf(x8[u].x, e, A.x);
              A.y = fmaf(x8[u].y, e, A.y);
              A.z = fmaf(x8[u].z, e, A.z);
              A.w = fmaf(x8[u].w, e, A.w);
            }
          }
          M = Mn;
        }
      }
      const float inv = Ls > 0.f ? 1.f / Ls : 0.f;   // an empty sequence outputs zeros
      *reinterpret_cast<float4*>(a.out + (int64_t(b) * a.Hq + kvh * G + gg) * kD + d4) =
          make_float4(A.x * inv, A.y * inv, A.z * inv, A.w * inv);
    }
    if (tid == 0) atomicExch(sync + 2, 0u);
  }
  drain_copies();
}

// ------------------------------------------------------------------- host side
namespace {
int max_smem_optin_flat(int dev) {
  int v = 0;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) {
    cudaGetLastError();
    return 232448;
  }
  return v;
}

size_t flat_smem(int G, int R, int S, int stages, int cand_cap, int list_cap) {
  return flat_layout(G, R, S, stages, cand_cap, list_cap).total;
}
}  // namespace

bool make_flat_plan(int B, int Hq, int Hkv, int64_t L, int k, int sms, int smem_cap, Plan& p) {
  const int G = Hq / Hkv;
  const int64_t U = int64_t(B) * Hkv;
  if (U <= 0 || sms <= 0 || U > sms / 2) return false;
  const int64_t k_eff = std::min<int64_t>(k, L);
  int S = int(std::min<int64_t>({int64_t(kFlatMaxS), int64_t(sms) / U,
                                 (L + kFlatMinKeys - 1) / kFlatMinKeys}));
  if (S < 2) return false;
  int64_t R = (L + S - 1) / S;
  R = (R + 7) & ~int64_t(7);
  S = int((L + R - 1) / R);                     // no CTA without keys
  if (S < 2 || R > 65535) return false;
  const int cand_cap = int(std::min<int64_t>(R, 4 * ((k_eff + S - 1) / S) + 128));
  const int list_cap = int(std::max<int64_t>(1, std::min<int64_t>(R, k_eff)));
  const int64_t nchunks = (R + kChunk - 1) / kChunk;
  int stages = int(std::min<int64_t>(kFlatMaxStages, nchunks));
  while (stages > 1 && flat_smem(G, int(R), S, stages, cand_cap, list_cap) > size_t(smem_cap))
    --stages;
  const size_t smem = flat_smem(G, int(R), S, stages, cand_cap, list_cap);
  if (smem > size_t(smem_cap)) return false;
  p.grid = int(U * S);
  p.cluster = 1;
  p.waves = 1;
  p.keys_per_cta = R;
  p.list_cap = list_cap;
  p.stages = stages;
  p.smem = smem;
  p.l2_bytes = 0;
  p.dist_global = false;
  p.flat = true;
  p.cand_cap = cand_cap;
  return true;
}

size_t flat_workspace_bytes(int B, int Hq, int Hkv, const Plan& p) {
  const int G = Hq / Hkv;
  const int64_t U = int64_t(B) * Hkv;
  const int S = int(p.grid / U);
  return 256 + flat_sync_bytes(U) + flat_hist_bytes(U, G, S) + flat_part_bytes(U, G, S);
}

template <int G, typename T>
static cudaError_t prepare_flat() {
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    int dev = 0;
    cudaGetDevice(&dev);
    err = cudaFuncSetAttribute(decode_flat_kernel<G, T>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               max_smem_optin_flat(dev));
  });
  return err;
}

template <int G, typename T>
static cudaError_t launch_flat_g(const FlatArgs& a, const Plan& p, cudaStream_t stream) {
  const cudaError_t e = prepare_flat<G, T>();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_flat_kernel<G, T>, a);
}

template <typename T>
static cudaError_t launch_flat_t(int G, const FlatArgs& a, const Plan& p, cudaStream_t s) {
  switch (G) {
    case 1: return launch_flat_g<1, T>(a, p, s);
    case 2: return launch_flat_g<2, T>(a, p, s);
    case 4: return launch_flat_g<4, T>(a, p, s);
    case 8: return launch_flat_g<8, T>(a, p, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_decode_flat(const void* q, const uint8_t* qcodes, const void* k,
                               const void* v, const uint8_t* codes, adamas_dtype dt, int B,
                               int Hq, int Hkv, const CacheLayout& lay, int64_t L, int kk,
                               float t, float t_ratio, void* ws, int32_t* idx_out, float* out,
                               const Plan& p, cudaStream_t stream) {
  const int G = Hq / Hkv;
  const int64_t U = int64_t(B) * Hkv;
  FlatArgs a;
  a.q = q; a.qcodes = qcodes; a.k = k; a.v = v; a.codes = codes;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Lmax = lay.Lmax; a.L = L;
  a.budget = kk;
  a.idx_stride = int(std::min<int64_t>(kk, L));
  a.seq_lens = lay.seq_lens;
  a.t = t;
  a.t_ratio = t_ratio;
  a.scale_log2 = float(1.4426950408889634 / 11.313708498984761);  // log2(e) / sqrt(128)
  a.idx_out = idx_out;
  a.out = out;
  uint8_t* w = static_cast<uint8_t*>(ws);
  a.err = reinterpret_cast<uint32_t*>(w + decode_workspace_error_offset());
  a.S = int(p.grid / U);
  a.R = int(p.keys_per_cta);
  a.stages = p.stages;
  a.cand_cap = p.cand_cap;
  a.list_cap = p.list_cap;
  a.attend = out != nullptr ? 1 : 0;
  {
    const int64_t sel_bytes = int64_t(B) * Hq * a.idx_stride * 2 * kD * (dt == ADAMAS_F32 ? 4 : 2);
    a.prefetch = (p.l2_bytes <= 0 || 4 * sel_bytes <= 3 * p.l2_bytes) ? 1 : 0;
  }
  a.sync = reinterpret_cast<uint32_t*>(w + 256);
  a.ghist = reinterpret_cast<uint16_t*>(w + 256 + flat_sync_bytes(U));
  a.gpart = reinterpret_cast<float*>(w + 256 + flat_sync_bytes(U) + flat_hist_bytes(U, G, a.S));
  if (dt == ADAMAS_F32) return launch_flat_t<float>(G, a, p, stream);
  return launch_flat_t<__nv_bfloat16>(G, a, p, stream);
}

}  // namespace adamas

// Fused Adamas decode step: ONE launch of a thread-block-cluster kernel runs
//   query encode -> distance scan -> exact per-head top-k -> gather attention
//   (one split per CTA) -> combine of the splits,
// with every cross-CTA exchange in distributed shared memory.
//
// Method: "Adamas: Hadamard Sparse Attention for Efficient Long-Context
// Inference" — v2 abstract (compact 2-bit codes, distance-based top-k, gather of
// the original KV states for sparse attention), v1 abstract (Manhattan distance).
//
// Work split.  A (batch, kv head) pair is a "unit".  Each unit gets one cluster
// of CS CTAs (CS <= 16, one CTA per SM); CTA r of the cluster owns key positions
// [r*R, min(L, (r+1)*R)), R = ceil(L / CS).  Clusters are independent, so more
// units than fit at once simply run in waves.
//
// Exact top-k with ties to the lower position.  Distances are integers 0..384.
// Each CTA keeps its distances in shared memory (plans for long CTA ranges keep them
// in workspace scratch, read back from L2) and builds, per query head, a 385-bin
// histogram that it turns into a cumulative one.  Before a cluster barrier every CTA
// pushes its cumulative counts at the ends of 30 coarse chunks (13 bins each) into
// the shared memory of every peer; after it, each CTA finds locally the chunk where
// the unit's count reaches k, then pulls from each peer a 20-bin window of the
// cumulative histogram around that chunk through distributed shared memory.  That
// gives the k-th distance D*, how many tokens of lower-ranked CTAs are selected, and
// how many of its own D*-ties it takes.  One block scan in position order then emits
// its selected positions.  The key codes cross HBM exactly once, and no global-memory
// atomic or barrier is involved.
//
// Attention.  Each CTA gathers the original K/V rows it selected (one split of
// the unit's softmax) and stores its partial (m, l, acc[128]) per head into the
// shared memory of cluster rank 0; after a second cluster barrier rank 0 merges
// the CS partials and writes the output.
#include <algorithm>
#include <atomic>
#include <map>
#include <mutex>
#include <tuple>
#include <type_traits>

#include <cooperative_groups.h>

#include "adamas_internal.cuh"

namespace cg = cooperative_groups;

namespace adamas {

constexpr int kMaxStages = 8;    // bulk-copy ring depth (runtime: 1..8, as shared memory allows)
constexpr int kMaxCluster = 16;  // non-portable cluster size limit
// kernel flavours: contiguous caches, paged caches, one rank of a context-parallel step,
// contiguous caches with each CTA's distances in workspace scratch instead of shared
// memory (per-head selection over long CTA ranges: fewer, longer CTAs in one wave)
constexpr int kModeContiguous = 0, kModePaged = 1, kModeCP = 2, kModeContigGD = 3;
constexpr int kNCoarse = 30;     // coarse chunks of the D* search (30 x chunk >= bins)
constexpr int kCoarseRow = 32;   // coarse counts per (CTA, head), padded to 128 B
constexpr int kRound = kThreads * 32;   // tokens per select round (32 per thread)

struct DecodeArgs {
  const void* q;             // [B][Hq][128] (encode mode) or nullptr
  const uint8_t* qcodes;     // [B][Hq][32] (select mode) or nullptr
  const void* k;             // [B][Hkv][Lmax][128], or pages [P][Hkv][page][128]
  const void* v;
  const uint8_t* codes;      // [B][Hkv][Lmax][32], or pages [P][Hkv][page][32]
  int B, Hq, Hkv;
  int64_t Lmax, L;           // cache rows per unit (contiguous layout); longest context
  int budget;                // k; a unit selects min(k, its length) positions
  int idx_stride;            // idx_out row length, min(k, L)
  const int32_t* seq_lens;   // [B] context lengths, or nullptr (every sequence has L)
  const int32_t* block_table;  // [B][max_blocks] page ids, or nullptr (contiguous)
  int max_blocks;
  int page_shift;            // log2(page size)
  int64_t num_pages;
  float t;
  float t_ratio;             // > 0: each query's threshold is t_ratio * its rotated absmax
  float scale_log2;
  int32_t* idx_out;          // [B][rows][idx_stride] or nullptr (-1 past a unit's count)
  float* out;                // [B][Hq][128] or nullptr (select mode)
  uint32_t* err;             // device error word
  int cluster;               // CTAs per unit
  int keys_per_cta;          // R
  int list_cap;
  int stages;                // bulk-copy ring depth
  int attend;
  int prefetch;              // pull rows below D* into L2 during the select
  uint16_t* dist_scratch;    // kModeContigGD: per CTA [GS][RS] distances (workspace)
  // context-parallel slice (kModeCP): see CpArgs
  int cp_phase;
  int64_t L_total, pos_offset;
  uint32_t* cp_hist_out;
  uint8_t* cp_scratch;       // per CTA: distances [GS][RS] u16, then cumulative hist [GS][BS]
  const uint32_t* cp_hist_all;
  int cp_world, cp_rank;
  float* cp_partial;
  // extra bytes the first chunk's barrier expects (test hook of the copy-wait timeout)
  uint32_t inject_tx;
};

// Selection geometry of one kernel flavour.  Per-head selection (SH = false):
// G selection heads, distances 0..384.  Shared selection (SH = true): one selection
// per kv head over the sum of the G heads' distances, 0..384 G.
template <int G, bool SH>
struct Sel {
  static constexpr int GS = SH ? 1 : G;                // selection heads
  static constexpr int NB = SH ? 384 * G + 1 : kNBins;  // distance bins
  static constexpr int BS = (NB + 3) / 4 * 4;           // histogram row stride (16 B multiple)
  static constexpr int C = (NB + kNCoarse - 1) / kNCoarse;   // bins per coarse chunk
  static constexpr int FW = (C + 4 + 3) / 4 * 4;        // fine-window bins (covers C + 1)
  static constexpr int GM = SH ? (G < 4 ? G : 4) : 1;  // query heads (softmax states) per warp
};

// per-head selection: 385 bins, 30 coarse chunks of 13, a 20-bin (5 x 16 B) fine window
static_assert(Sel<1, false>::NB == kNBins && Sel<1, false>::BS == kBinStride &&
                  Sel<1, false>::C == 13 && Sel<1, false>::FW == 20,
              "per-head selection geometry");
static_assert(Sel<8, true>::NB <= 0x7fff, "summed distances must fit a signed 16-bit lane");

struct SmemLayout {
  size_t ring, mbar, hist, coarse, fine, dist, list, qf, qc, qth, scan, merge, info, ptab, misc,
      total;
};

__host__ __device__ inline size_t al(size_t x, size_t a) { return (x + a - 1) / a * a; }

// GS, BS, FW, GM as in Sel<G, SH>; G = query heads of the unit.  With GM > 1 the
// per-warp merge buffer (kWarps x GM partials) is placed in the ring region right
// after the partials: the ring is idle once the scan is over, and rank 0 receives
// the peers' partials only after the first cluster barrier.
__host__ __device__ inline SmemLayout make_layout(int G, int GS, int BS, int FW, int GM, int R,
                                                 int list_cap, int CS, int stages, int ptab,
                                                 bool dist_smem) {
  SmemLayout s;
  size_t o = 0;
  const size_t ring = size_t(stages) * kChunk * kCodeBytes;
  const size_t merge = size_t(kWarps) * GM * kPartStride * 4;
  const size_t part = size_t(CS) * G * kPartStride * 4 + (GM > 1 ? merge : 0);
  s.ring = o;  o = al(o + (ring > part ? ring : part), 128);
  s.mbar = o;  o = al(o + 8 * kMaxStages, 128);
  s.hist = o;  o = al(o + size_t(GS) * BS * 4, 128);
  s.coarse = o; o = al(o + size_t(CS) * GS * kCoarseRow * 4, 128);   // pushed by the peers
  s.fine = o;  o = al(o + size_t(CS) * GS * FW * 4, 128);            // pulled from the peers
  s.dist = o;  o = al(o + (dist_smem ? size_t(GS) * dist_stride(R) * 2 : 0), 128);
  s.list = o;  o = al(o + size_t(GS) * list_cap * 2, 128);
  s.qf = o;    o = al(o + size_t(G) * kD * 4, 128);
  s.qc = o;    o = al(o + size_t(G) * kCodeBytes, 128);
  s.qth = o;   o = al(o + size_t(G) * 12 * 4, 128);
  s.scan = o;  o = al(o + size_t(2) * kWarps * GS * 4, 128);
  if (GM > 1) {
    s.merge = s.ring + size_t(CS) * G * kPartStride * 4;
  } else {
    s.merge = o; o = al(o + merge, 128);
  }
  s.info = o;  o = al(o + size_t(GS) * 9 * 4, 128);
  s.ptab = o;  o = al(o + size_t(ptab) * 4, 128);   // page ids of the CTA's range (paged)
  s.misc = o;  o = al(o + 128, 128);
  s.total = o;
  return s;
}

template <int G, bool SH>
__host__ __device__ inline SmemLayout layout_of(int R, int list_cap, int CS, int stages,
                                                int ptab, bool dist_smem = true) {
  using X = Sel<G, SH>;
  return make_layout(G, X::GS, X::BS, X::FW, X::GM, R, list_cap, CS, stages, ptab, dist_smem);
}

// Bytes a CTA keeps between the two context-parallel phases: its distances and its
// cumulative histograms (16-byte multiples).
__host__ __device__ inline size_t cp_scratch_per_cta(int GS, int BS, int R) {
  return size_t(GS) * dist_stride(R) * 2 + size_t(GS) * BS * 4;
}

// Page-table entries a CTA stages: the pages its R positions can span.
__host__ __device__ inline int ptab_entries(int R, int page_shift, bool paged) {
  return paged ? ((R + (1 << page_shift) - 1) >> page_shift) + 1 : 0;
}

template <int G, bool SH, int MD, typename T>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const DecodeArgs a) {
  using X = Sel<G, SH>;
  constexpr int GS = X::GS, BS = X::BS, NB = X::NB, CB = X::C, FW = X::FW, GM = X::GM;
  constexpr bool paged = MD == kModePaged;
  constexpr bool cp = MD == kModeCP;   // one rank's slice of a context-parallel step
  extern __shared__ __align__(128) uint8_t smem[];
  pdl_wait();
  cg::cluster_group cluster = cg::this_cluster();
  const int CS = a.cluster;
  const int rank = int(cluster.block_rank());
  const int S = a.stages;
  const SmemLayout lo = layout_of<G, SH>(a.keys_per_cta, a.list_cap, CS, S,
                                         ptab_entries(a.keys_per_cta, a.page_shift, MD == kModePaged),
                                         MD != kModeContigGD);
  uint8_t* ring = smem + lo.ring;
  float* part = reinterpret_cast<float*>(smem + lo.ring);           // [CS][G][kPartStride]
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + lo.mbar);
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + lo.hist);    // [GS][BS]
  uint32_t* coarse = reinterpret_cast<uint32_t*>(smem + lo.coarse);  // [CS][GS][kCoarseRow]
  uint32_t* fine = reinterpret_cast<uint32_t*>(smem + lo.fine);      // [CS][GS][FW]
  uint16_t* dist;                                                   // [GS][RS]
  if constexpr (MD == kModeContigGD) {
    dist = a.dist_scratch + size_t(blockIdx.x) * X::GS * dist_stride(a.keys_per_cta);
  } else {
    dist = reinterpret_cast<uint16_t*>(smem + lo.dist);
  }
  uint16_t* list = reinterpret_cast<uint16_t*>(smem + lo.list);    // [GS][list_cap]
  float* qf = reinterpret_cast<float*>(smem + lo.qf);              // [G][128]
  uint8_t* qc = smem + lo.qc;                                       // [G][32]
  uint32_t* qth = reinterpret_cast<uint32_t*>(smem + lo.qth);      // [G][12]
  uint32_t* scan = reinterpret_cast<uint32_t*>(smem + lo.scan);    // [2][kWarps][GS]
  float* merge = reinterpret_cast<float*>(smem + lo.merge);        // [kWarps][GM][kPartStride]
  int* info = reinterpret_cast<int*>(smem + lo.info);              // [GS][8], then [GS]
  int32_t* ptab = reinterpret_cast<int32_t*>(smem + lo.ptab);      // paged: row bases

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int unit = blockIdx.x / CS;
  const int b = unit / a.Hkv, kvh = unit % a.Hkv;
  // this unit's context length (a length outside [0, L] is an input error: flagged,
  // clamped) and the number of positions it selects
  int64_t L = a.L;
  if (a.seq_lens != nullptr) {
    const int64_t Lb = a.seq_lens[b];
    if (Lb < 0 || Lb > a.L) {
      if (tid == 0) atomicOr(a.err, kErrInput);
    }
    L = min(max(Lb, int64_t(0)), a.L);
  }
  const int keff = int(min(int64_t(a.budget), cp ? a.L_total : L));
  const int R = a.keys_per_cta;
  const int RS = dist_stride(R);
  const int64_t p0 = int64_t(rank) * R;
  const int n = int(max(int64_t(0), min(int64_t(R), L - p0)));   // keys of this CTA
  const int nch = (n + kChunk - 1) / kChunk;
  const uint8_t* codes = a.codes + (int64_t(unit) * a.Lmax + p0) * kCodeBytes;
  // paged caches: position p of this unit lives in page block_table[b][p >> shift]
  // (rows [page][kv head][p & mask]).  The last warp stages, for every page of this
  // CTA's range, the row of its first position for this kv head in shared memory
  // (pool rows number below 2^31: a row is at least 256 bytes); a page id outside
  // [0, num_pages) is an input error: flagged, and page 0 is used instead so that no
  // access leaves the pool.
  const int psh = a.page_shift;
  const int pmask = (1 << psh) - 1;
  const int64_t pfirst = p0 >> psh;
  // row of position p in the K/V (and code) storage
  const auto row_of = [&](int64_t p) -> int64_t {
    if constexpr (!paged) {
      return int64_t(unit) * a.Lmax + p;
    } else {
      return int64_t(ptab[(p >> psh) - pfirst] + (int(p) & pmask));
    }
  };
  // chunk qi of this CTA's codes into ring slot `slot`.  Contiguous caches: one
  // bulk copy on the slot's mbarrier, issued by one thread.  Paged caches: each warp
  // copies the 32 keys its threads scan (1 KB) with 16-byte asynchronous copies, one
  // commit group per chunk: lanes 2m, 2m + 1 take the two halves of key m (then of
  // key m + 16), so each instruction reads 512 contiguous bytes of a page, and a
  // page of any size costs no extra copy instruction.
  const auto issue_chunk = [&](int qi, int slot) {
    if constexpr (!paged) {
      const int c0 = qi * kChunk;
      const int keys = min(kChunk, n - c0);
      mbar_expect_tx(&mbar[slot], uint32_t(keys * kCodeBytes) + (qi == 0 ? a.inject_tx : 0u));
      bulk_g2s(ring + size_t(slot) * kChunk * kCodeBytes, codes + int64_t(c0) * kCodeBytes,
               uint32_t(keys * kCodeBytes), &mbar[slot]);
    } else {
      // positions and rows fit 32 bits (a CTA range starts below 2^20; pool rows
      // number below 2^31)
      const int kk = warp * 32 + (lane >> 1);       // key of this lane's first half
      const int half = (lane & 1) * 16;
      uint8_t* dst = ring + (slot * kChunk + kk) * kCodeBytes + half;
      const int r = qi * kChunk + kk;
      const int pos = int(p0) + r;
#pragma unroll
      for (int i = 0; i < 2; ++i) {               // keys kk and kk + 16
        if (qi < nch && r + 16 * i < n) {
          const int pi = pos + 16 * i;
          const int row = ptab[(pi >> psh) - int(pfirst)] + (pi & pmask);
          cp_async_16(dst + 16 * i * kCodeBytes, a.codes + int64_t(row) * kCodeBytes + half);
        }
      }
      cp_async_commit();
    }
  };

  // ---- issue the code copies first: HBM traffic starts before anything else.  The
  // last warp issues them, so the warps that encode the queries are not delayed.
  // (context-parallel phase 2 reads its distances back from phase 1: no copies)
  const bool scan_codes = !(cp && a.cp_phase == 2);
  // chunks the issuing thread has put in flight (meaningful in that thread only)
  int issued = 0;
  if constexpr (!paged) {
    if (tid == kThreads - 32 && scan_codes) {
      for (int s = 0; s < S; ++s) mbar_init(&mbar[s], 1);
      fence_mbar_init();
      for (int qi = 0; qi < min(nch, S); ++qi) issue_chunk(qi, qi);
      issued = min(nch, S);
    }
  } else {
    // paged: the whole block stages the page table, four independent loads in
    // flight per thread (the copies start after the prologue's barrier)
    const int32_t* bt = a.block_table + int64_t(b) * a.max_blocks + pfirst;
    const int npages = n > 0 ? int(((p0 + n - 1) >> psh) - pfirst + 1) : 0;
    for (int i0 = tid; i0 < npages; i0 += 4 * kThreads) {
      int32_t pg[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * kThreads;
        pg[u] = i < npages ? bt[i] : 0;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * kThreads;
        if (i < npages) {
          if (pg[u] < 0 || int64_t(pg[u]) >= a.num_pages) {
            atomicOr(a.err, kErrInput);
            pg[u] = 0;
          }
          ptab[i] = int32_t((int64_t(pg[u]) * a.Hkv + kvh) << psh);
        }
      }
    }
  }

  // A copy wait that gives up sets this thread's copy_abort.  The issuing thread also
  // scans keys, so it waits on every chunk it issued: once its own wait gave up it
  // issues no more copies, and before the CTA exits it waits (bounded again) for the
  // last phase of every slot it filled, so no bulk copy is still writing this CTA's
  // shared memory when it exits.
  bool copy_abort = false;
  const auto drain_copies = [&]() {
    if constexpr (!paged) {
      if (tid == kThreads - 32 && copy_abort) {
        for (int qi = max(0, issued - S); qi < issued; ++qi)
          mbar_wait_bounded(&mbar[qi % S], uint32_t((qi / S) & 1), a.err);
      }
    }
  };

  // ---- prologue: zero histograms, encode (or fetch) the G query codes
  for (int i = tid; i < GS * BS; i += kThreads) hist[i] = 0u;
  if (warp < G) {
    const int g = warp, h = kvh * G + g;
    if (a.qcodes != nullptr) {
      qc[g * kCodeBytes + lane] = a.qcodes[(int64_t(b) * a.Hq + h) * kCodeBytes + lane];
    } else {
      float v[4];
      const T* qsrc = static_cast<const T*>(a.q) + (int64_t(b) * a.Hq + h) * kD;
      if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        // 16-byte loads by lanes 0-15 (q may live in mapped host memory, where
        // fewer, wider requests matter), redistributed to 4 elements per lane
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
      qc[g * kCodeBytes + lane] =
          static_cast<uint8_t>(warp_fwht_code(v, a.t, lane, a.t_ratio));
    }
  }
  __syncthreads();
  if constexpr (paged) {
    // page table staged: every thread starts its copies of the first S chunks (one
    // commit group each, empty past the CTA's last chunk)
    for (int qi = 0; qi < S; ++qi) issue_chunk(qi, qi);
  }
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

  // ---- distance scan: one key per thread per chunk, G heads per key
  {
    constexpr int GR = G > 4 ? 4 : G;
    // A thread reads its key's 32-byte code as two 16-byte halves, the second half
    // first where swz = 1 (neighbouring lane quads then hit different banks), and
    // scores the words in that order.  The distance is a sum over coordinates, so the
    // query's packed-pair words are taken in the same order instead: key pair j (code
    // words 2j, 2j+1 in load order) pairs with query pair (j + 2 swz) mod 4.
    const int swz = (tid >> 2) & 1;
    PairWords qreg[GR];
    // query words of head g in this thread's pair order
    const auto load_q = [&](int g, PairWords& qt) {
      const uint2* s = reinterpret_cast<const uint2*>(qth + g * 12);
      const uint2 p0 = s[swz], p1 = s[swz ^ 1];
      const uint2 h0 = s[2 + swz], h1 = s[2 + (swz ^ 1)];
      const uint2 x0 = s[4 + swz], x1 = s[4 + (swz ^ 1)];
      qt.p[0] = p0.x; qt.p[1] = p0.y; qt.p[2] = p1.x; qt.p[3] = p1.y;
      qt.h[0] = h0.x; qt.h[1] = h0.y; qt.h[2] = h1.x; qt.h[3] = h1.y;
      qt.x[0] = x0.x; qt.x[1] = x0.y; qt.x[2] = x1.x; qt.x[3] = x1.y;
    };
    if constexpr (G <= 4) {
#pragma unroll
      for (int g = 0; g < GR; ++g) load_q(g, qreg[g]);
    }
    const uint32_t one = uint32_t(a.keys_per_cta > 0);   // 1, opaque to the compiler
    const uint32_t two = one + one;
    // the packed-pair words of this thread's key in ring slot `sl`
    const auto load_key = [&](int sl, PairWords& kt) {
      const uint4* src = reinterpret_cast<const uint4*>(ring + (size_t(sl) * kChunk + tid) *
                                                        kCodeBytes);
      const uint4 xa = src[swz], xb = src[swz ^ 1];
      const uint32_t wd[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
      make_pairs(wd, kt, two);
    };
    // distances of NK keys (positions r[]; side effects only where valid[]), with the
    // keys' work in one block so that their dependency chains interleave (the pair
    // loop below; the one-chunk loop keeps its own branch-guarded body)
    const auto score_keys = [&](auto nk_tag, const PairWords* kt, const int* r, const bool* valid) {
      constexpr int NK = decltype(nk_tag)::value;
      uint32_t dsum[NK];
#pragma unroll
      for (int u = 0; u < NK; ++u) dsum[u] = 0;   // shared selection: sum over the heads
#pragma unroll
      for (int g0 = 0; g0 < G; g0 += GR) {
        if constexpr (G > 4) {
#pragma unroll
          for (int g = 0; g < GR; ++g) load_q(g0 + g, qreg[g]);
        }
#pragma unroll
        for (int g = 0; g < GR; ++g) {
#pragma unroll
          for (int u = 0; u < NK; ++u) {
            const uint32_t dd = pair_dist(kt[u], qreg[g], one);
            if constexpr (SH) {
              dsum[u] += dd;
            } else if (valid[u]) {
              dist[size_t(g0 + g) * RS + r[u]] = static_cast<uint16_t>(dd);
              atomicAdd(&hist[(g0 + g) * BS + dd], 1u);
            }
          }
        }
      }
      if constexpr (SH) {
#pragma unroll
        for (int u = 0; u < NK; ++u) {
          if (valid[u]) {
            dist[r[u]] = static_cast<uint16_t>(dsum[u]);
            atomicAdd(&hist[dsum[u]], 1u);
          }
        }
      }
    };
    using Two = std::integral_constant<int, 2>;
    int slot = 0;
    uint32_t parity = 0;
    int qi = 0;
    if constexpr (!paged && G <= 2) {
      // one or two heads per key leave each key's chain short and latency-bound: two
      // chunks per iteration while the ring holds at least four, their keys scored
      // together (the next copies are issued once both are consumed).  With four or
      // more heads the heads already interleave and the popcount pipe is the limit.
      if (S >= 4) {
        for (; qi + 1 < (scan_codes ? nch : 0); qi += 2) {
          int slot2 = slot + 1;
          uint32_t par2 = parity;
          if (slot2 == S) { slot2 = 0; par2 ^= 1u; }
          if (!mbar_wait_bounded(&mbar[slot], parity, a.err)) copy_abort = true;
          if (!mbar_wait_bounded(&mbar[slot2], par2, a.err)) copy_abort = true;
          PairWords kt[2];
          load_key(slot, kt[0]);
          load_key(slot2, kt[1]);
          const int r[2] = {qi * kChunk + tid, (qi + 1) * kChunk + tid};
          const bool valid[2] = {r[0] < n, r[1] < n};
          score_keys(Two{}, kt, r, valid);
          if (nch > S) __syncthreads();
          if (tid == kThreads - 32 && !copy_abort) {
            if (qi + S < nch) { issue_chunk(qi + S, slot); ++issued; }
            if (qi + 1 + S < nch) { issue_chunk(qi + 1 + S, slot2); ++issued; }
          }
          slot = slot2 + 1;
          parity = par2;
          if (slot == S) { slot = 0; parity ^= 1u; }
        }
      }
    }
    for (; qi < (scan_codes ? nch : 0); ++qi) {
      if constexpr (paged) {
        cp_async_wait_pending(S - 1);   // this thread's copies of chunk qi have landed
        __syncwarp();                   // ... and its warp-mates' (the key it scans)
      } else {
        if (!mbar_wait_bounded(&mbar[slot], parity, a.err)) copy_abort = true;
      }
      const int r = qi * kChunk + tid;
      if (r < n) {
        PairWords kt;
        load_key(slot, kt);
        uint32_t dsum = 0;   // shared selection: sum of the G heads' distances
#pragma unroll
        for (int g0 = 0; g0 < G; g0 += GR) {
          if constexpr (G > 4) {
#pragma unroll
            for (int g = 0; g < GR; ++g) load_q(g0 + g, qreg[g]);
          }
#pragma unroll
          for (int g = 0; g < GR; ++g) {
            const uint32_t dd = pair_dist(kt, qreg[g], one);
            if constexpr (SH) {
              dsum += dd;
            } else {
              dist[size_t(g0 + g) * RS + r] = static_cast<uint16_t>(dd);
              atomicAdd(&hist[(g0 + g) * BS + dd], 1u);
            }
          }
        }
        if constexpr (SH) {
          dist[r] = static_cast<uint16_t>(dsum);
          atomicAdd(&hist[dsum], 1u);
        }
      }
      if constexpr (paged) {
        // the slot's entries for this warp's keys: every lane has read its own key
        __syncwarp();
        issue_chunk(qi + S, slot);
      } else {
        // a slot is refilled only when the CTA's keys need more chunks than the ring
        // holds; otherwise every chunk has its own slot and warps run ahead freely
        if (nch > S) __syncthreads();
        if (tid == kThreads - 32 && qi + S < nch && !copy_abort) {
          issue_chunk(qi + S, slot);
          ++issued;
        }
      }
      if (++slot == S) { slot = 0; parity ^= 1u; }
    }
  }
  __syncthreads();   // every key's distances and histogram counts are in

  // ---- histograms -> inclusive cumulative histograms, in place.  Then every CTA
  // pushes its cumulative counts at the 30 coarse-chunk ends (+2 pad) into every
  // peer, so the coarse level of the D* search reads local memory after the
  // barrier: lane j of the pushing warp holds the count at the end of chunk j
  // (lanes 30, 31: the total); four lanes are gathered per 16-byte remote store.
  const auto push_coarse = [&](int g, uint32_t run) {
    const uint32_t c0 = __shfl_sync(0xffffffffu, run, (lane & 7) * 4 + 0);
    const uint32_t c1 = __shfl_sync(0xffffffffu, run, (lane & 7) * 4 + 1);
    const uint32_t c2 = __shfl_sync(0xffffffffu, run, (lane & 7) * 4 + 2);
    const uint32_t c3 = __shfl_sync(0xffffffffu, run, (lane & 7) * 4 + 3);
    if (lane < kCoarseRow / 4) {
      for (int cc = 0; cc < CS; ++cc) {
        uint4* dst = reinterpret_cast<uint4*>(cluster.map_shared_rank(coarse, cc) +
                                              (size_t(rank) * GS + g) * kCoarseRow) + lane;
        *dst = make_uint4(c0, c1, c2, c3);
      }
    }
  };
  uint8_t* scratch = nullptr;
  if constexpr (cp) {
    scratch = a.cp_scratch + size_t(blockIdx.x) * cp_scratch_per_cta(GS, BS, R);
  }
  if (cp && a.cp_phase == 2) {
    // phase 2: this CTA's distances and cumulative histograms, kept by phase 1
    const uint4* src = reinterpret_cast<const uint4*>(scratch);
    uint4* dd = reinterpret_cast<uint4*>(dist);
    const int nd = GS * RS * 2 / 16;
    for (int i = tid; i < nd; i += kThreads) dd[i] = src[i];
    uint4* hh = reinterpret_cast<uint4*>(hist);
    for (int i = tid; i < GS * BS / 4; i += kThreads) hh[i] = src[nd + i];
    __syncthreads();
    if (warp < GS) push_coarse(warp, hist[warp * BS + min(CB * lane + CB - 1, NB - 1)]);
  } else if constexpr (CB <= 16) {
    // 385 bins (per head, or one shared head of G = 1): a warp per selection head,
    // lane l owning bins CB*l .. CB*l + CB-1 in registers
    if (warp < GS) {
      uint32_t* row = hist + warp * BS;
      uint32_t loc[CB];
      uint32_t sum = 0;
#pragma unroll
      for (int i = 0; i < CB; ++i) {
        const int bin = CB * lane + i;
        loc[i] = bin < NB ? row[bin] : 0u;
        sum += loc[i];
      }
      uint32_t inc = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      uint32_t run = inc - sum;
#pragma unroll
      for (int i = 0; i < CB; ++i) {
        const int bin = CB * lane + i;
        run += loc[i];
        if (bin < NB) row[bin] = run;
      }
      push_coarse(warp, run);
    }
  } else {
    // wide shared-selection histogram (384 G + 1 bins, one row): the whole block,
    // each thread owning PB consecutive bins read and written as 16-byte words
    // (bins NB .. BS-1 are zero padding), one block scan
    constexpr int PB = (NB + 4 * kThreads - 1) / (4 * kThreads) * 4;
    uint32_t loc[PB];
    uint32_t sum = 0;
#pragma unroll
    for (int i4 = 0; i4 < PB; i4 += 4) {
      const int bin = tid * PB + i4;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (bin < BS) v = *reinterpret_cast<const uint4*>(hist + bin);
      loc[i4] = v.x; loc[i4 + 1] = v.y; loc[i4 + 2] = v.z; loc[i4 + 3] = v.w;
      sum += v.x + v.y + v.z + v.w;
    }
    uint32_t ex[1] = {sum}, tot[1];
    block_exclusive_scan<1>(ex, tot, scan, 0, lane, warp);
    uint32_t run = ex[0];
#pragma unroll
    for (int i4 = 0; i4 < PB; i4 += 4) {
      const int bin = tid * PB + i4;
      uint4 v;
      v.x = run += loc[i4];
      v.y = run += loc[i4 + 1];
      v.z = run += loc[i4 + 2];
      v.w = run += loc[i4 + 3];
      if (bin < BS) *reinterpret_cast<uint4*>(hist + bin) = v;
    }
    __syncthreads();
    if (warp == 0) push_coarse(0, hist[min(CB * lane + CB - 1, NB - 1)]);
  }

  cluster.sync();   // cumulative histograms complete; coarse counts delivered
  pdl_trigger();    // the next grid's blocks may take the SMs this one leaves idle

  if constexpr (cp) {
    if (a.cp_phase == 1) {
      // context-parallel phase 1: every CTA keeps its distances and cumulative
      // histograms for phase 2; the unit's cumulative histogram over this rank's
      // slice (the sum of its CTAs', gathered by rank 0 through distributed shared
      // memory; the second barrier keeps the peers alive until it has read them)
      // is exported for the other ranks
      {
        uint4* dst = reinterpret_cast<uint4*>(scratch);
        const uint4* dd = reinterpret_cast<const uint4*>(dist);
        const int nd = GS * RS * 2 / 16;
        for (int i = tid; i < nd; i += kThreads) dst[i] = dd[i];
        const uint4* hh = reinterpret_cast<const uint4*>(hist);
        for (int i = tid; i < GS * BS / 4; i += kThreads) dst[nd + i] = hh[i];
      }
      if (rank == 0) {
        for (int i = tid; i < GS * NB; i += kThreads) {
          const int g = i / NB, bin = i % NB;
          uint32_t c = 0;
          for (int cc = 0; cc < CS; ++cc) c += cluster.map_shared_rank(hist, cc)[g * BS + bin];
          a.cp_hist_out[(int64_t(unit) * GS + g) * NB + bin] = c;
        }
      }
      cluster.sync();
      drain_copies();
      return;
    }
  }

  // ---- resolve D*, the count selected in lower-ranked CTAs, and the ties taken.
  // Level 1 (local): the coarse chunk j* where the unit's cumulative count reaches
  // k_eff.  Level 2: each peer's FW-bin window around chunk j* is pulled with
  // 16-byte loads, then bins CB j* - 1 .. CB j* + CB - 1 give D* exactly.
  int* jst = info + GS * 8;   // [GS] coarse chunk per selection head
  if (warp < GS) {
    const int g = warp;
    uint32_t S1 = 0;
    if (lane < kNCoarse) {
      for (int cc = 0; cc < CS; ++cc) S1 += coarse[(cc * GS + g) * kCoarseRow + lane];
      if constexpr (cp) {   // the other ranks' cumulative counts at the chunk end
        const int64_t rows = int64_t(a.B) * a.Hkv * GS;
        const int64_t e = (int64_t(unit) * GS + g) * NB + min(CB * lane + CB - 1, NB - 1);
#pragma unroll 4
        for (int w = 0; w < a.cp_world; ++w) {
          if (w != a.cp_rank) S1 += a.cp_hist_all[int64_t(w) * rows * NB + e];
        }
      }
    }
    const uint32_t hit1 = __ballot_sync(0xffffffffu, lane < kNCoarse && S1 >= uint32_t(keff));
    if (lane == 0) jst[g] = __ffs(hit1) - 1;   // exists: chunk 29 ends at the last bin, count L
  }
  __syncthreads();
  for (int i = tid; i < CS * GS * (FW / 4); i += kThreads) {
    const int cc = i / (GS * (FW / 4));
    const int g = (i / (FW / 4)) % GS;
    const int q4 = i % (FW / 4);
    const int lo_bin = min(max(0, CB * jst[g] - 1) & ~3, BS - FW);
    const uint4 v = *(reinterpret_cast<const uint4*>(cluster.map_shared_rank(hist, cc) +
                                                      g * BS + lo_bin) + q4);
    *(reinterpret_cast<uint4*>(fine + (cc * GS + g) * FW) + q4) = v;
  }
  __syncthreads();
  if (warp < GS) {
    const int g = warp;
    const uint32_t ke = uint32_t(keff);
    const int jstar = jst[g];
    const int lo_bin = min(max(0, CB * jstar - 1) & ~3, BS - FW);
    // level 2, 32 bins per pass: lane l of pass p -> bin CB j* - 1 + 32 p + l.  The
    // first bin reaching k_eff is D*; the counts one bin lower are the "less than"
    // counts (carried across passes in lane 31's values).
    int dstar = -1;
    uint32_t less = 0, lt_before = 0, eq_before = 0, carry2 = 0, carryb = 0;
    for (int base = 0; base < CB + 1 && dstar < 0; base += 32) {
      const int l = base + lane;
      const int d = CB * jstar - 1 + l;
      uint32_t S2 = 0, Sb = 0;
      if (l < CB + 1 && d >= 0) {
        const int off = min(d, NB - 1) - lo_bin;
        for (int cc = 0; cc < CS; ++cc) {
          const uint32_t x = fine[(cc * GS + g) * FW + off];
          S2 += x;
          if (cc < rank) Sb += x;
        }
        if constexpr (cp) {   // other ranks count in the total, lower ranks also come first
          const int64_t rows = int64_t(a.B) * a.Hkv * GS;
          const int64_t e = (int64_t(unit) * GS + g) * NB + min(d, NB - 1);
#pragma unroll 4
          for (int w = 0; w < a.cp_world; ++w) {
            if (w == a.cp_rank) continue;
            const uint32_t x = a.cp_hist_all[int64_t(w) * rows * NB + e];
            S2 += x;
            if (w < a.cp_rank) Sb += x;
          }
        }
      }
      const uint32_t hit2 = __ballot_sync(0xffffffffu, l >= 1 && l < CB + 1 && S2 >= ke);
      uint32_t p2 = __shfl_up_sync(0xffffffffu, S2, 1);
      uint32_t pb = __shfl_up_sync(0xffffffffu, Sb, 1);
      if (lane == 0) { p2 = carry2; pb = carryb; }
      if (hit2) {
        const int ls = __ffs(hit2) - 1;
        dstar = CB * jstar - 1 + l - lane + ls;
        less = __shfl_sync(0xffffffffu, p2, ls);        // unit count d < D*
        lt_before = __shfl_sync(0xffffffffu, pb, ls);
        eq_before = __shfl_sync(0xffffffffu, Sb, ls) - lt_before;
      }
      carry2 = __shfl_sync(0xffffffffu, S2, 31);
      carryb = __shfl_sync(0xffffffffu, Sb, 31);
    }
    if (dstar < 0) {   // impossible when the counts are consistent; never index with it
      if (lane == 0) atomicOr(a.err, kErrSelect);
      dstar = NB - 1;
      less = lt_before = eq_before = 0;
    }
    const uint32_t* own = hist + g * BS;
    const uint32_t lt_own = dstar > 0 ? own[dstar - 1] : 0u;
    const uint32_t eq_own = own[dstar] - lt_own;
    const uint32_t need = ke - less;                 // ties at D* the unit takes
    const uint32_t base = lt_before + min(eq_before, need);
    const uint32_t take = need > eq_before ? min(need - eq_before, eq_own) : 0u;
    if (lane == 0) {
      int* in = info + g * 8;
      in[0] = dstar;
      in[1] = int(base);
      in[2] = int(take);
      in[3] = int(lt_own + take);   // selected in this CTA
    }
  }
  __syncthreads();

  // ---- select, in position order: per round each thread owns up to 32 consecutive
  // tokens; one pass over the distances builds "< D*" and "== D*" bit masks, one
  // block scan ranks them, and only the selected bits are then visited
  {
    int dstar[GS], take[GS], base[GS], nsel[GS];
#pragma unroll
    for (int g = 0; g < GS; ++g) {
      const int* in = info + g * 8;
      dstar[g] = in[0];
      base[g] = in[1];
      take[g] = in[2];
      nsel[g] = in[3];
    }
    uint32_t carry_lt[GS], carry_eq[GS];
#pragma unroll
    for (int g = 0; g < GS; ++g) carry_lt[g] = carry_eq[g] = 0;
    for (int rb = 0, parity = 0; rb < n; rb += kRound, parity ^= 1) {
      const int nr = min(kRound, n - rb);
      const int per = (((nr + kThreads - 1) / kThreads) + 7) & ~7;   // multiple of 8, <= 32
      const int s0 = rb + tid * per;
      const int cntv = max(0, min(per, rb + nr - s0));
      uint32_t ltm[GS], eqm[GS], cnt[GS], tot[GS];
      const uint32_t valid = cntv >= 32 ? 0xffffffffu : ((1u << cntv) - 1u);
      // packed compares, two distances per word: in each 16-bit lane
      // (0x8000 + D*) - d keeps bit 15 iff d <= D*, (0x7fff + D*) - d iff d < D*
      // (distances <= 384 G <= 3072, so no lane borrows from its neighbour).  All
      // selection heads' loads of a group of 8 positions are issued before any compare.
      uint32_t cle[GS], clt[GS];
#pragma unroll
      for (int g = 0; g < GS; ++g) {
        cle[g] = (0x8000u + uint32_t(dstar[g])) * 0x10001u;
        clt[g] = cle[g] - 0x10001u;
        ltm[g] = eqm[g] = 0;
      }
      for (int i8 = 0; i8 < cntv; i8 += 8) {
        uint4 v[GS];
#pragma unroll
        for (int g = 0; g < GS; ++g)
          v[g] = *reinterpret_cast<const uint4*>(dist + size_t(g) * RS + s0 + i8);
#pragma unroll
        for (int g = 0; g < GS; ++g) {
          const uint32_t l0 = lane_sign_bits(clt[g] - v[g].x, clt[g] - v[g].y);
          const uint32_t l1 = lane_sign_bits(clt[g] - v[g].z, clt[g] - v[g].w);
          const uint32_t e0 = lane_sign_bits(cle[g] - v[g].x, cle[g] - v[g].y) & ~l0;
          const uint32_t e1 = lane_sign_bits(cle[g] - v[g].z, cle[g] - v[g].w) & ~l1;
          ltm[g] |= (l0 | (l1 << 4)) << i8;
          eqm[g] |= (e0 | (e1 << 4)) << i8;
        }
      }
#pragma unroll
      for (int g = 0; g < GS; ++g) {
        ltm[g] &= valid;
        eqm[g] &= valid;
        cnt[g] = (uint32_t(__popc(ltm[g])) << 16) | uint32_t(__popc(eqm[g]));
        // tokens below D* are selected whatever the tie rule decides: start pulling
        // their K/V rows into L2 now, so the gather finds them there (when the step's
        // selected rows fit in 3/4 of the L2; beyond that the prefetches evict each
        // other and only add work)
        if (a.attend && a.prefetch) {
          uint32_t m = ltm[g];
          while (m) {
            const int i = __ffs(m) - 1;
            m &= m - 1u;
            const int64_t row_off = row_of(p0 + s0 + i) * kD;
            prefetch_row_l2(static_cast<const T*>(a.k) + row_off);
            prefetch_row_l2(static_cast<const T*>(a.v) + row_off);
          }
        }
      }
      block_exclusive_scan<GS>(cnt, tot, scan, parity, lane, warp);
#pragma unroll
      for (int g = 0; g < GS; ++g) {
        const int lt_b = int(carry_lt[g] + (cnt[g] >> 16));
        const int eq_b = int(carry_eq[g] + (cnt[g] & 0xffffu));
        // this thread's ties that still fit: the lowest (take - eq_b) bits of eqm
        uint32_t sel_eq = 0;
        const int te = take[g] - eq_b;
        if (te > 0) {
          uint32_t rest = eqm[g];
          for (int c = 0; c < te && rest; ++c) rest &= rest - 1u;
          sel_eq = eqm[g] ^ rest;
        }
        uint32_t sel = ltm[g] | sel_eq;
        int rk = lt_b + min(eq_b, take[g]);
        // idx_out rows: [B][Hq] for per-head selection, [B][Hkv] for shared selection
        const int64_t orow_id = SH ? int64_t(b) * a.Hkv + kvh : int64_t(b) * a.Hq + kvh * G + g;
        int32_t* orow =
            a.idx_out != nullptr ? a.idx_out + orow_id * a.idx_stride + base[g] : nullptr;
        uint16_t* lrow = list + size_t(g) * a.list_cap;
        while (sel) {
          const int i = __ffs(sel) - 1;
          sel &= sel - 1u;
          const int r = s0 + i;
          // rk < nsel and base + rk < k_eff hold by construction; the guard keeps a
          // broken invariant from writing outside the list or the output row
          if (rk < nsel[g] && base[g] + rk < keff) {
            lrow[rk] = static_cast<uint16_t>(r);
            if (orow) orow[rk] = int32_t(a.pos_offset + p0 + r);
          }
          ++rk;
        }
        carry_lt[g] += tot[g] >> 16;
        carry_eq[g] += tot[g] & 0xffffu;
      }
    }
  }
  // a sequence shorter than the budget fills only keff slots of its rows: rank 0
  // marks the rest -1
  if (a.seq_lens != nullptr && a.idx_out != nullptr && rank == 0 && keff < a.idx_stride) {
    const int pad = a.idx_stride - keff;
    for (int i = tid; i < GS * pad; i += kThreads) {
      const int g = i / pad;
      const int64_t orow_id = SH ? int64_t(b) * a.Hkv + kvh : int64_t(b) * a.Hq + kvh * G + g;
      a.idx_out[orow_id * a.idx_stride + keff + i % pad] = -1;
    }
  }
  __syncthreads();

  // ---- attention over the selected rows: this CTA's split of the unit's softmax.
  // The warps form G / GM groups; group gi serves query heads gi GM .. gi GM + GM-1,
  // its warps taking rows sub, sub + WPG, ... of the heads' list.  Per-head
  // selection: GM = 1, one group per head.  Shared selection: one list, GM <= 4
  // heads scored per loaded K/V row (for G = 8 the second group's reads of a row
  // hit L2).
  if (a.attend) {
    constexpr int NGR = G / GM;          // warp groups
    constexpr int WPG = kWarps / NGR;    // warps per group
    const int gi = warp % NGR, sub = warp / NGR;
    const int sel_head = SH ? 0 : gi;
    const int nsel = info[sel_head * 8 + 3];
    const uint16_t* lrow = list + size_t(sel_head) * a.list_cap;
    // contiguous caches: rows relative to the unit's base; paged: absolute pool rows
    const int64_t base_row = paged ? 0 : int64_t(unit) * a.Lmax;
    const T* kb = static_cast<const T*>(a.k) + base_row * kD;
    const T* vb = static_cast<const T*>(a.v) + base_row * kD;
    float qv[GM][4];
#pragma unroll
    for (int h = 0; h < GM; ++h) {
      const float* qrow = qf + (gi * GM + h) * kD + 4 * lane;
      qv[h][0] = qrow[0]; qv[h][1] = qrow[1]; qv[h][2] = qrow[2]; qv[h][3] = qrow[3];
    }
    SoftmaxState st[GM];
#pragma unroll
    for (int h = 0; h < GM; ++h) st[h].init();
    const auto pos_of = [&](int j) {
      if constexpr (paged) {
        return row_of(p0 + int64_t(lrow[j]));
      } else {
        return p0 + int64_t(lrow[j]);
      }
    };
    if constexpr (GM == 1) {
      // more than 8 rows per warp: bf16 rows go 8 lanes per row (fewer shuffles and
      // softmax updates per row); otherwise one row per warp instruction, which has
      // no group merge to pay for
      bool done = false;
      if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        if (nsel > 8 * WPG) {
          // rows not pulled into L2 by the select pass are pulled a few steps ahead here
          attend_rows_bf16_g8(kb, vb, nsel, sub, WPG, pos_of, qf + gi * kD, a.scale_log2, lane,
                              st[0], a.prefetch == 0);
          done = true;
        }
      }
      if (!done) attend_rows<T>(kb, vb, nsel, sub, WPG, pos_of, qv[0], a.scale_log2, lane, st[0]);
    } else {
      constexpr int kRowsG = GM <= 2 ? 8 : 4;
      attend_rows_group<T, GM, kRowsG>(kb, vb, nsel, sub, WPG, pos_of, qv, a.scale_log2, lane,
                                       st);
    }
    // merge row (sub * G + head) holds warp `sub` of the head's group's partial
#pragma unroll
    for (int h = 0; h < GM; ++h) {
      float* mw = merge + (sub * G + gi * GM + h) * kPartStride;
      if (lane == 0) { mw[0] = st[h].m; mw[1] = st[h].l; }
#pragma unroll
      for (int r = 0; r < 4; ++r) mw[4 + 4 * lane + r] = st[h].acc[r];
    }
    __syncthreads();
    float* dstp = cluster.map_shared_rank(part, 0) + size_t(rank) * G * kPartStride;
    for (int i = tid; i < G * kD; i += kThreads) {
      const int gg = i / kD, dim = i % kD;
      float M = -INFINITY, Ls = 0.f, A = 0.f;
      for (int sw = 0; sw < WPG; ++sw) {
        const float* mm = merge + (sw * G + gg) * kPartStride;
        merge_into(mm[0], mm[1], mm[4 + dim], M, Ls, A);
      }
      float* prow = dstp + gg * kPartStride;
      if (dim == 0) { prow[0] = M; prow[1] = Ls; }
      prow[4 + dim] = A;
    }
  }

  cluster.sync();   // partials are in rank 0; no CTA reads a peer's memory after this

  if (cp && a.attend && rank == 0) {
    // context-parallel phase 2: this rank's partial of every head (log2 domain; a
    // rank that selected nothing for a head exports m = -inf, l = 0)
    for (int i = tid; i < G * kD; i += kThreads) {
      const int gg = i / kD, dim = i % kD;
      float M = -INFINITY;
      for (int cc = 0; cc < CS; ++cc) M = fmaxf(M, part[(cc * G + gg) * kPartStride]);
      float Ls = 0.f, A = 0.f;
      if (M != -INFINITY) {
        for (int cc = 0; cc < CS; ++cc) {
          const float* prow = part + (cc * G + gg) * kPartStride;
          const float e = exp2f(prow[0] - M);
          Ls = fmaf(prow[1], e, Ls);
          A = fmaf(prow[4 + dim], e, A);
        }
      }
      float* pr = a.cp_partial + (int64_t(b) * a.Hq + kvh * G + gg) * kPartStride;
      if (dim == 0) { pr[0] = M; pr[1] = Ls; pr[2] = 0.f; pr[3] = 0.f; }
      pr[4 + dim] = A;
    }
  } else if (a.attend && rank == 0) {
    // four coordinates per thread: 16-byte partial reads and one 16-byte output store
    // (out may live in mapped host memory, where fewer, wider requests matter)
    for (int i = tid; i < G * (kD / 4); i += kThreads) {
      const int gg = i / (kD / 4), d4 = 4 * (i % (kD / 4));
      float M = -INFINITY;
      for (int cc = 0; cc < CS; ++cc) M = fmaxf(M, part[(cc * G + gg) * kPartStride]);
      if (M == -INFINITY) M = 0.f;   // every split empty (length 0): all terms below are 0
      float Ls = 0.f;
      float4 A = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int cc = 0; cc < CS; ++cc) {
        const float* prow = part + (cc * G + gg) * kPartStride;
        const float e = exp2f(prow[0] - M);     // empty split: m = -inf -> 0
        const float4 x = *reinterpret_cast<const float4*>(prow + 4 + d4);
        Ls = fmaf(prow[1], e, Ls);
        A.x = fmaf(x.x, e, A.x);
        A.y = fmaf(x.y, e, A.y);
        A.z = fmaf(x.z, e, A.z);
        A.w = fmaf(x.w, e, A.w);
      }
      // an empty sequence (length 0) selects nothing: its output is zero
      const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
      *reinterpret_cast<float4*>(a.out + (int64_t(b) * a.Hq + kvh * G + gg) * kD + d4) =
          make_float4(A.x * inv, A.y * inv, A.z * inv, A.w * inv);
    }
  }
  drain_copies();
}

// ------------------------------------------------------------------- host side
static int max_smem_optin(int dev) {
  int v = 0;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) {
    cudaGetLastError();
    return 232448;
  }
  return v;
}

template <int G, bool SH, int MD, typename T>
static cudaError_t prepare_kernel() {
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    int dev = 0;
    cudaGetDevice(&dev);
    err = cudaFuncSetAttribute(decode_kernel<G, SH, MD, T>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem_optin(dev));
    if (err == cudaSuccess)
      err = cudaFuncSetAttribute(decode_kernel<G, SH, MD, T>,
                                 cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  });
  return err;
}

template <int G, bool SH, typename T>
static int active_clusters_g(int cs, size_t smem) {
  if (prepare_kernel<G, SH, kModeContiguous, T>() != cudaSuccess) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int nclusters = 0;
  if (cudaOccupancyMaxActiveClusters(&nclusters, decode_kernel<G, SH, kModeContiguous, T>, &cfg) !=
      cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return nclusters;
}

template <bool SH>
static int active_clusters_s(int G, int cs, size_t smem) {
  switch (G) {
    case 1: return active_clusters_g<1, SH, __nv_bfloat16>(cs, smem);
    case 2: return active_clusters_g<2, SH, __nv_bfloat16>(cs, smem);
    case 4: return active_clusters_g<4, SH, __nv_bfloat16>(cs, smem);
    case 8: return active_clusters_g<8, SH, __nv_bfloat16>(cs, smem);
  }
  return 0;
}

static int active_clusters(int G, bool shared, int cs, size_t smem) {
  return shared ? active_clusters_s<true>(G, cs, smem) : active_clusters_s<false>(G, cs, smem);
}

static size_t layout_total(int G, bool shared, int R, int list_cap, int cs, int stages,
                           int ptab, bool dist_smem = true) {
#define ADAMAS_LAYOUT_CASE(GG)                                                        \
  case GG:                                                                            \
    return shared ? layout_of<GG, true>(R, list_cap, cs, stages, ptab, dist_smem).total \
                  : layout_of<GG, false>(R, list_cap, cs, stages, ptab, dist_smem).total;
  switch (G) {
    ADAMAS_LAYOUT_CASE(1)
    ADAMAS_LAYOUT_CASE(2)
    ADAMAS_LAYOUT_CASE(4)
    ADAMAS_LAYOUT_CASE(8)
  }
#undef ADAMAS_LAYOUT_CASE
  return ~size_t(0);
}

// Chooses the cluster size: among sizes whose shared memory fits (and, on a device,
// whose clusters can be scheduled), the one with the least modelled time
// waves x (per-key scan cost x keys per CTA + fixed per-wave latency).
bool make_decode_plan(int B, int Hq, int Hkv, int64_t L, int k, bool shared, int page_shift,
                      bool allow_gd, int sms, int smem_cap, bool query_device, Plan& p) {
  const int G = Hq / Hkv;
  const int64_t U = int64_t(B) * Hkv;
  const int64_t k_eff = std::min<int64_t>(k, L);
  double best = 0;
  bool found = false;
  for (int cs = 1; cs <= kMaxCluster; ++cs) {
    const int64_t R = (L + cs - 1) / cs;
    if (R > 65535) continue;                       // positions in a CTA are 16-bit
    if (cs > 1 && (L + R - 1) / R < cs) continue;  // an all-empty tail CTA: use fewer
    const int list_cap = int(std::max<int64_t>(1, std::min<int64_t>(R, k_eff)));
    const int64_t nchunks = (R + kChunk - 1) / kChunk;
    const int ptab = ptab_entries(int(R), page_shift, page_shift >= 0);
    // distances in shared memory; or, where allowed, in workspace scratch (their global
    // stores and reloads cost about 15 % of the scan, modelled below)
    for (int gd = 0; gd <= (allow_gd ? 1 : 0); ++gd) {
      int stages = int(std::min<int64_t>(kMaxStages, std::max<int64_t>(1, nchunks)));
      while (stages > 1 && layout_total(G, shared, int(R), list_cap, cs, stages, ptab, !gd) >
                               size_t(smem_cap))
        --stages;
      const size_t smem = layout_total(G, shared, int(R), list_cap, cs, stages, ptab, !gd);
      if (smem > size_t(smem_cap)) continue;
      int conc_clusters = sms / cs;
      if (query_device) {
        conc_clusters = active_clusters(G, shared, cs, smem);
      } else if (sms == 148) {
        // no device to ask: the co-resident clusters of one CTA per SM that
        // cudaOccupancyMaxActiveClusters reports on a 148-SM B200 (its SMs sit in
        // GPCs of unequal size, so large clusters fit fewer times than 148 / cs)
        static const int kB200Clusters[17] = {0, 148, 74, 45, 33, 26, 22, 15, 15, 15, 11,
                                              7, 7, 7, 7, 7, 7};
        conc_clusters = kB200Clusters[cs];
      }
      if (conc_clusters < 1) continue;
      const int64_t total = U * cs;
      const int64_t conc = int64_t(conc_clusters) * cs;
      const int64_t waves = (total + conc - 1) / conc;
      const double per_key_ns = (0.45 * G + 0.35) * (gd ? 1.15 : 1.0);
      const double cost = double(waves) * (per_key_ns * double(R) + 6000.0);
      if (!found || cost < best) {
        best = cost;
        found = true;
        p.grid = int(total);
        p.cluster = cs;
        p.keys_per_cta = R;
        p.list_cap = list_cap;
        p.stages = stages;
        p.smem = smem;
        p.waves = int(waves);
        p.l2_bytes = 0;
        p.dist_global = gd != 0;
        p.flat = false;
        p.cand_cap = 0;
      }
    }
  }
  return found && p.grid > 0 && int64_t(p.grid) == U * p.cluster && U * p.cluster < (1ll << 31);
}

namespace {
// Plans are memoised per device, problem and policy: making one queries the cluster
// occupancy of every candidate cluster size, far more host time than a launch.
struct PlanKey {
  int dev, B, Hq, Hkv, k, page_shift, policy;
  int64_t L;
  bool shared, allow_gd;
  bool operator<(const PlanKey& o) const {
    return std::tie(dev, B, Hq, Hkv, k, page_shift, policy, L, shared, allow_gd) <
           std::tie(o.dev, o.B, o.Hq, o.Hkv, o.k, o.page_shift, o.policy, o.L, o.shared,
                    o.allow_gd);
  }
};
std::atomic<int> g_policy{0};
std::atomic<uint32_t> g_inject_tx{0};

// Modelled step time of a plan (ns), fitted to B200 measurements of both kernels:
// waves x (per-key scan cost x keys per CTA + fixed latency of the stage chain).  The
// cluster kernel's chain (exchanges in distributed shared memory) costs about 8 us.
// The grid-wide kernel's exchanges are round trips through L2 and its last CTA merges
// every split, so its chain costs about 14.4 us plus 0.11 us per CTA of a unit: it
// wins only where clusters would leave most SMs idle over very long contexts (one kv
// head at 256K: 26.3 against 31.5 us; the 32K Llama layer: 18.7 against 13.0 us).
double plan_cost(int G, const Plan& p, int64_t units) {
  const double per_key_ns = (0.477 + 0.243 * G) * (p.dist_global ? 1.15 : 1.0);
  const double per_unit = units > 0 ? double(p.grid) / double(units) : 1.0;
  const double fixed = p.flat ? 14400.0 + 110.0 * per_unit : 8000.0;
  return double(p.waves) * (per_key_ns * double(p.keys_per_cta) + fixed);
}

// Where it applies (contiguous caches, per-head selection, not a context-parallel
// slice: callers say so with allow_gd), the grid-wide plan replaces the cluster plan
// when the policy asks for it or its modelled time is lower.
void consider_flat(int B, int Hq, int Hkv, int64_t L, int k, bool shared, int page_shift,
                   bool allow_gd, int sms, int smem_cap, bool have_cluster, Plan& p) {
  const int policy = g_policy.load();
  if (policy == 1 || shared || page_shift >= 0 || !allow_gd) return;
  Plan f;
  if (!make_flat_plan(B, Hq, Hkv, L, k, sms, smem_cap, f)) return;
  const int G = Hq / Hkv;
  const int64_t U = int64_t(B) * Hkv;
  // by default only where it puts clearly more SMs to work and is modelled faster
  const bool wider = have_cluster && 4 * int64_t(f.grid) >= 5 * int64_t(p.grid) &&
                     plan_cost(G, f, U) < plan_cost(G, p, U);
  if (!have_cluster || policy == 2 || wider) p = f;
}
std::mutex g_plan_mutex;
std::map<PlanKey, std::pair<bool, Plan>> g_plans;
constexpr size_t kMaxPlans = 4096;
}  // namespace

bool decode_plan_for_current_device(int B, int Hq, int Hkv, int64_t L, int k, bool shared,
                                    int page_shift, Plan& p, bool allow_gd) {
  int dev = 0;
  const int sms = current_device_sms(&dev);
  if (sms <= 0) {
    // no device visible: plan for a 148-SM part with the sm_100 shared-memory cap
    const bool ok = make_decode_plan(B, Hq, Hkv, L, k, shared, page_shift, allow_gd, 148, 232448,
                                     false, p);
    consider_flat(B, Hq, Hkv, L, k, shared, page_shift, allow_gd, 148, 232448, ok, p);
    return ok || p.flat;
  }
  const PlanKey key{dev, B, Hq, Hkv, k, page_shift, g_policy.load(), L, shared, allow_gd};
  std::lock_guard<std::mutex> lock(g_plan_mutex);
  const auto it = g_plans.find(key);
  if (it != g_plans.end()) {
    p = it->second.second;
    return it->second.first;
  }
  p.flat = false;
  bool ok = make_decode_plan(B, Hq, Hkv, L, k, shared, page_shift, allow_gd, sms,
                             max_smem_optin(dev), true, p);
  consider_flat(B, Hq, Hkv, L, k, shared, page_shift, allow_gd, sms, max_smem_optin(dev), ok, p);
  ok = ok || p.flat;
  int l2 = 0;
  if (cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess) {
    cudaGetLastError();
    l2 = 0;
  }
  p.l2_bytes = l2;
  if (g_plans.size() >= kMaxPlans) g_plans.clear();
  g_plans.emplace(key, std::make_pair(ok, p));
  return ok;
}

// Context-parallel workspace: the error word, then every CTA's scratch.
size_t cp_workspace_bytes(int B, int Hq, int Hkv, int64_t L, int k, bool shared) {
  Plan p;
  if (!decode_plan_for_current_device(B, Hq, Hkv, L, k, shared, -1, p)) return 0;
  const int G = Hq / Hkv;
  const int NB = selection_bins(G, shared);
  const int BS = (NB + 3) / 4 * 4;
  return 256 + size_t(p.grid) * cp_scratch_per_cta(shared ? 1 : G, BS, int(p.keys_per_cta));
}

// The decode workspace carries the device error word (bounded copy waits) and, when
// the plan keeps distances outside shared memory (per-head selection over long CTA
// ranges), every CTA's distances.
size_t decode_workspace_bytes(int B, int Hq, int Hkv, int64_t L, int k) {
  Plan p;
  if (Hkv <= 0 || Hq % Hkv ||
      !decode_plan_for_current_device(B, Hq, Hkv, L, k, false, -1, p, true))
    return 256;
  if (p.flat) return flat_workspace_bytes(B, Hq, Hkv, p);
  if (!p.dist_global) return 256;
  return 256 + size_t(p.grid) * (Hq / Hkv) * dist_stride(int(p.keys_per_cta)) * 2;
}

void set_decode_policy(int policy) { g_policy.store(policy); }
void set_copy_fault(uint32_t extra_tx_bytes) { g_inject_tx.store(extra_tx_bytes); }
int decode_policy() { return g_policy.load(); }
size_t decode_workspace_error_offset() { return 8; }

template <int G, bool SH, int MD, typename T>
static cudaError_t launch_g(const DecodeArgs& a, const Plan& p, cudaStream_t stream) {
  const cudaError_t e = prepare_kernel<G, SH, MD, T>();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, decode_kernel<G, SH, MD, T>, a);
}

template <bool SH, int MD, typename T>
static cudaError_t launch_t(int G, const DecodeArgs& a, const Plan& p, cudaStream_t s) {
  switch (G) {
    case 1: return launch_g<1, SH, MD, T>(a, p, s);
    case 2: return launch_g<2, SH, MD, T>(a, p, s);
    case 4: return launch_g<4, SH, MD, T>(a, p, s);
    case 8: return launch_g<8, SH, MD, T>(a, p, s);
    default: return cudaErrorInvalidValue;
  }
}

template <bool SH, int MD>
static cudaError_t launch_dt(adamas_dtype dt, int G, const DecodeArgs& a, const Plan& p,
                             cudaStream_t s) {
  if (dt == ADAMAS_F32) return launch_t<SH, MD, float>(G, a, p, s);
  return launch_t<SH, MD, __nv_bfloat16>(G, a, p, s);
}

cudaError_t launch_decode(const void* q, const uint8_t* qcodes, const void* k, const void* v,
                          const uint8_t* codes, adamas_dtype dt, int B, int Hq, int Hkv,
                          const CacheLayout& lay, int64_t L, int kk, float t, void* ws,
                          int32_t* idx_out, float* out, bool shared, const Plan& p,
                          cudaStream_t stream, float t_ratio, const CpArgs* cpa) {
  if (p.flat) {
    if (shared || cpa != nullptr || lay.block_table != nullptr) return cudaErrorInvalidValue;
    return launch_decode_flat(q, qcodes, k, v, codes, dt, B, Hq, Hkv, lay, L, kk, t, t_ratio, ws,
                              idx_out, out, p, stream);
  }
  const int G = Hq / Hkv;
  DecodeArgs a;
  a.q = q; a.qcodes = qcodes; a.k = k; a.v = v; a.codes = codes;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Lmax = lay.Lmax; a.L = L;
  a.budget = kk;
  a.idx_stride = int(std::min<int64_t>(kk, L));
  a.seq_lens = lay.seq_lens;
  a.block_table = lay.block_table;
  a.max_blocks = lay.max_blocks;
  a.page_shift = lay.page_shift;
  a.num_pages = lay.num_pages;
  a.t = t;
  a.t_ratio = t_ratio;
  a.scale_log2 = float(1.4426950408889634 / 11.313708498984761);  // log2(e) / sqrt(128)
  a.idx_out = idx_out; a.out = out;
  a.err = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + decode_workspace_error_offset());
  a.cluster = p.cluster;
  a.keys_per_cta = int(p.keys_per_cta);
  a.list_cap = p.list_cap;
  a.stages = p.stages;
  a.attend = (out != nullptr || (cpa != nullptr && cpa->phase == 2)) ? 1 : 0;
  {
    // selected K and V bytes of the whole step (rows gathered once per selection row)
    const int64_t rows = int64_t(B) * (shared ? Hkv : Hq) * a.idx_stride;
    const int64_t sel_bytes = rows * 2 * kD * (dt == ADAMAS_F32 ? 4 : 2);
    a.prefetch = (p.l2_bytes <= 0 || 4 * sel_bytes <= 3 * p.l2_bytes) ? 1 : 0;
  }
  a.inject_tx = lay.block_table == nullptr ? g_inject_tx.load() : 0u;
  a.cp_phase = cpa ? cpa->phase : 0;
  a.L_total = cpa ? cpa->L_total : L;
  a.pos_offset = cpa ? cpa->pos_offset : 0;
  a.cp_hist_out = cpa ? cpa->hist_out : nullptr;
  a.cp_scratch = cpa ? static_cast<uint8_t*>(ws) + 256 : nullptr;
  a.cp_hist_all = cpa ? cpa->hist_all : nullptr;
  a.cp_world = cpa ? cpa->world : 1;
  a.cp_rank = cpa ? cpa->rank : 0;
  a.cp_partial = cpa ? cpa->partial_out : nullptr;
  if (cpa) a.idx_stride = int(std::min<int64_t>(kk, cpa->L_total));
  const int mode = cpa != nullptr ? kModeCP
                   : lay.block_table != nullptr ? kModePaged
                   : p.dist_global ? kModeContigGD : kModeContiguous;
  if (mode == kModeContigGD) {   // planned for per-head selection only
    if (shared) return cudaErrorInvalidValue;
    a.dist_scratch = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(ws) + 256);
    return launch_dt<false, kModeContigGD>(dt, G, a, p, stream);
  }
  a.dist_scratch = nullptr;
  if (shared) {
    return mode == kModeCP      ? launch_dt<true, kModeCP>(dt, G, a, p, stream)
           : mode == kModePaged ? launch_dt<true, kModePaged>(dt, G, a, p, stream)
                                : launch_dt<true, kModeContiguous>(dt, G, a, p, stream);
  }
  return mode == kModeCP      ? launch_dt<false, kModeCP>(dt, G, a, p, stream)
         : mode == kModePaged ? launch_dt<false, kModePaged>(dt, G, a, p, stream)
                              : launch_dt<false, kModeContiguous>(dt, G, a, p, stream);
}

}  // namespace adamas

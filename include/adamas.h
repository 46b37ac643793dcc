/*
 * adamas.h — C ABI of the Adamas decode hot path on B200 (sm_100a).
 *
 * The method ("Adamas: Hadamard Sparse Attention for Efficient Long-Context
 * Inference", arXiv 2510.18413, v2 abstract): every key and every decode query is
 * passed through a Hadamard transform, bucketized and compressed to 2-bit codes; a
 * distance between the query code and every key code (a Manhattan distance, per
 * the v1 abstract) picks the top-k candidate positions; the ORIGINAL K/V rows at
 * those positions are gathered for exact sparse attention.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers, owned by the caller.  The library
 *    never allocates, frees or synchronizes in these calls (except
 *    adamas_check_workspace, which says so), and keeps no per-call host state.
 *  - Every call is asynchronous on `stream`; argument checks run on the host
 *    before any launch, and a rejected call launches nothing.
 *  - Stream order is kept.  The decode and key-encode kernels are launched with
 *    programmatic dependent launch: their blocks may become resident while the
 *    previous kernel in the stream is still running, but wait for its completion
 *    (and for its memory) before they touch any buffer.
 *  - Layouts are contiguous, row-major:
 *        q        [B][Hq][d]           elements of `dt`
 *        k_cache  [B][Hkv][Lmax][d]    elements of `dt`   (original keys)
 *        v_cache  [B][Hkv][Lmax][d]    elements of `dt`
 *        codes    [B][Hkv][Lmax][d/4]  bytes: 2-bit codes, 4 per byte, coordinate
 *                                      i in byte i>>2 at bits 2*(i&3)
 *        qcodes   [B][Hq][d/4]         bytes, same packing
 *        idx      [B][Hq][k_eff]       int32 positions, ascending
 *        out      [B][Hq][d]           float32
 *    with d = 128, G = Hq / Hkv query heads per kv head (query head h reads kv
 *    head h / G), and k_eff = min(k, L).
 *  - Pointers must be 16-byte aligned (idx: 4-byte, workspace: 256-byte).
 *  - Codes: y = H x / sqrt(d) with H the natural-order Sylvester Hadamard matrix,
 *    then code = [y >= -t] + [y >= 0] + [y >= t] in {0,1,2,3} (the blog section 2.2
 *    rule of three thresholds compared with strict "<", here at {-t, 0, +t} with a
 *    fixed per-run t >= 0 shared by keys and queries).
 *  - Selection: query head h keeps the k_eff positions with the smallest
 *    Manhattan distance between its code and the key codes of kv head h / G, ties
 *    going to the lower position.
 *  - Attention: softmax over the selected positions of (q . K_j) / sqrt(d), fp32
 *    accumulation, fp32 output.
 *
 * Errors: ADAMAS_ERR_INVALID_ARG for null or misaligned pointers, non-positive
 * sizes, L > Lmax, Hq % Hkv != 0, t < 0 or not finite, a too-small workspace;
 * ADAMAS_ERR_UNSUPPORTED for d != 128, G not in {1, 2, 4, 8}, or a context too long
 * for the on-chip plan; ADAMAS_ERR_CUDA when a launch fails (no C++ exception ever
 * crosses this boundary).
 */
#ifndef ADAMAS_H
#define ADAMAS_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ADAMAS_OK = 0,
  ADAMAS_ERR_INVALID_ARG = 1,
  ADAMAS_ERR_UNSUPPORTED = 2,
  ADAMAS_ERR_CUDA = 3,
  ADAMAS_ERR_TIMEOUT = 4,
  ADAMAS_ERR_INTERNAL = 5
} adamas_status;

typedef enum { ADAMAS_F32 = 0, ADAMAS_BF16 = 1 } adamas_dtype;

/* Human-readable name of a status code (static string, never NULL). */
const char* adamas_status_string(adamas_status s);

/* ABI version, bumped when a signature or layout changes. */
int adamas_abi_version(void);

/*
 * Which kernel the decode and select entry points may plan with (process-wide, for
 * tuning and testing; results are the same either way): 0 = whichever the launch
 * planner models as faster (the default), 1 = thread-block clusters only (one
 * cluster per (batch, kv head) unit, exchange in distributed shared memory), 2 =
 * the grid-wide kernel wherever it applies (contiguous caches with per-query-head
 * selection and few enough units that every unit gets at least two CTAs, all CTAs
 * co-resident at one per SM; exchange through the workspace).  Changing it changes
 * adamas_decode_workspace_bytes for some sizes.  ADAMAS_ERR_INVALID_ARG outside 0..2.
 */
adamas_status adamas_set_decode_policy(int policy);

/*
 * Test hook of the bounded-wait error path (process-wide; not for production use).
 * While extra_tx_bytes (a multiple of 16, at most 2^20) is nonzero, decode launches
 * on contiguous caches through thread-block clusters arm the barrier of each CTA's
 * first code chunk for that many bytes more than the bulk copy delivers, so every
 * wait on it runs into its 1 s limit.  The kernel then records the timeout in the
 * workspace error word, stops issuing copies, waits (bounded again) for the copies
 * it has in flight and returns: adamas_check_workspace reports ADAMAS_ERR_TIMEOUT, the
 * results of that launch are unspecified, and the device stays usable.  0 restores
 * normal operation.  ADAMAS_ERR_INVALID_ARG for a negative, unaligned or larger count.
 */
adamas_status adamas_test_set_copy_fault(int extra_tx_bytes);

/*
 * Key encoder, run when keys are appended to the cache (v2 abstract: Hadamard
 * transform, bucketization, 2-bit compression of the keys).  Encodes positions
 * [pos0, pos0 + n_new) of every (batch, kv head) from k_cache into codes.
 * Reads n_new * B * Hkv * d elements, writes n_new * B * Hkv * d/4 bytes.
 * The transform runs in fp32 (bf16 keys with a fixed t: on the tensor cores, as
 * H_8 x H_16), so a coordinate within rounding distance of a threshold may land
 * in either neighbouring bucket; the fused decode step encodes its queries with a
 * differently ordered fp32 FWHT.
 */
adamas_status adamas_encode_keys(const void* k_cache, adamas_dtype dt, int B, int Hkv, int d,
                                 int64_t Lmax, int64_t pos0, int64_t n_new, float t,
                                 uint8_t* codes, cudaStream_t stream);

/* Query encoder: the same transform on q [B][Hq][d] into qcodes [B][Hq][d/4]. */
adamas_status adamas_encode_queries(const void* q, adamas_dtype dt, int B, int Hq, int d,
                                    float t, uint8_t* qcodes, cudaStream_t stream);

/*
 * Workspace of adamas_decode_step and adamas_select_topk, in bytes; 0 if the
 * arguments are invalid or unsupported.  It serves the selection stage (v2 abstract of
 * "Adamas: Hadamard Sparse Attention for Efficient Long-Context Inference": the
 * top-k candidates are the positions whose codes lie closest to the query's code),
 * which needs, beyond the kernel's own shared memory, only this buffer.  The first 256 bytes hold the device error
 * word that a bounded wait sets when it gives up (see adamas_check_workspace).
 * Where the launch plan keeps every CTA's distances on chip (the 32K layer, for
 * one) that is all of it.  Plans for long contexts over many (batch, kv head) units
 * keep the distances in workspace scratch instead: one u16 per key and query head,
 * written and read back by the same launch (it stays in L2).  Zero-fill the
 * workspace once before first use (adamas_workspace_init); the scratch needs no
 * initialisation.  Calls that run one after another on one stream may share a
 * workspace; concurrent calls whose plans use scratch need one workspace each.
 */
size_t adamas_decode_workspace_bytes(int B, int Hq, int Hkv, int d, int64_t L, int k);

/* Zero-fills a workspace (cudaMemsetAsync on `stream`). */
adamas_status adamas_workspace_init(void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * SYNCHRONIZES `stream`, then reads the device error word of a decode workspace.
 * Returns ADAMAS_ERR_TIMEOUT if a kernel gave up a bounded wait (completion of a
 * bulk copy into shared memory) since the workspace was initialised,
 * ADAMAS_ERR_INVALID_ARG if a kernel met a device-resident length or page id out of
 * range (adamas_decode_step_varlen / _paged), ADAMAS_ERR_INTERNAL if the top-k
 * bookkeeping of a kernel found no k-th distance
 * (inconsistent counts: a bug, never expected), else ADAMAS_OK (or ADAMAS_ERR_CUDA
 * if the stream reported an error).
 */
adamas_status adamas_check_workspace(const void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * One decode step of the Adamas method (v2 abstract of "Adamas: Hadamard Sparse
 * Attention for Efficient Long-Context Inference": Hadamard transform, bucketing and
 * 2-bit compression of the query, a code distance to every cached key (Manhattan, v1
 * abstract), top-k candidates, and sparse attention over the ORIGINAL K/V rows of
 * those candidates; the blog "ADAMAS：稀疏注意力优化技术解析与应用实践", section 4,
 * puts the cost of a 32K decode step in memory traffic), all five stages in ONE
 * kernel launch (thread-block clusters,
 * one cluster per (batch, kv head) pair, cross-CTA exchange in distributed shared
 * memory): query encode, distance scan over the key codes, exact per-head top-k,
 * gather of the original K/V rows with split softmax attention, and the combine of
 * the splits.
 * Uses the first L positions of every cache row; codes must hold the keys' codes
 * for those positions (adamas_encode_keys).  idx_out may be NULL; when given it
 * receives the selected positions [B][Hq][k_eff], ascending.
 */
adamas_status adamas_decode_step(const void* q, const void* k_cache, const void* v_cache,
                                 const uint8_t* codes, adamas_dtype dt, int B, int Hq,
                                 int Hkv, int d, int64_t Lmax, int64_t L, int k, float t,
                                 void* workspace, size_t ws_bytes, int32_t* idx_out,
                                 float* out, cudaStream_t stream);

/*
 * adamas_decode_step for a caller whose queries and outputs live in (preferably
 * pinned) host memory: queues the copy q_host -> q_dev ([B][Hq][d] elements of
 * `dt`), the decode step, and the copy out_dev -> out_host ([B][Hq][d] float32),
 * all asynchronous on `stream` (synchronize before reading out_host).  q_dev and
 * out_dev are caller-owned device staging buffers; the caches, codes, workspace
 * and idx_out are as in adamas_decode_step.  When both host buffers are
 * page-locked and mapped into the device's address space (cudaHostAlloc /
 * cudaMallocHost memory on a unified-addressing system), the kernel reads q and
 * writes the output through that mapping and the staging buffers are not used.
 */
adamas_status adamas_decode_step_host(const void* q_host, void* q_dev, const void* k_cache,
                                      const void* v_cache, const uint8_t* codes, adamas_dtype dt,
                                      int B, int Hq, int Hkv, int d, int64_t Lmax, int64_t L,
                                      int k, float t, void* workspace, size_t ws_bytes,
                                      int32_t* idx_out, float* out_dev, float* out_host,
                                      cudaStream_t stream);

/*
 * Stage entry point: distance scan + top-k from given query codes (no attention).
 * Same kernel as adamas_decode_step with the attention stages switched off.  The
 * stage is the candidate search of the v2 abstract of "Adamas: Hadamard Sparse
 * Attention for Efficient Long-Context Inference" (smallest code distances to the
 * query), with the distance the v1 abstract names (Manhattan, summed over the 128
 * 2-bit codes: 0 .. 384).  qcodes [B][Hq][32] as adamas_encode_queries writes them;
 * idx_out [B][Hq][k_eff] receives the positions ascending.
 */
adamas_status adamas_select_topk(const uint8_t* qcodes, const uint8_t* codes, int B, int Hq,
                                 int Hkv, int64_t Lmax, int64_t L, int k, void* workspace,
                                 size_t ws_bytes, int32_t* idx_out, cudaStream_t stream);

/*
 * Shared GQA selection (a variant the Adamas pages leave open: the v2 abstract of
 * "Adamas: Hadamard Sparse Attention for Efficient Long-Context Inference" picks
 * top-k positions per query but does not treat grouped-query attention).  For
 * each (batch, kv head) the score of key j is the SUM over the G = Hq / Hkv query
 * heads of the group of their Manhattan code distances to key j (0 .. 384 G); the
 * first min(k, L) positions under (score ascending, position ascending) are
 * selected ONCE, and every query head of the group attends over that one set, so
 * each selected K/V row is read once per group instead of once per query head.
 * Arguments, layouts, ownership and errors are those of adamas_decode_step, except
 * idx_out, which receives [B][Hkv][k_eff] positions, ascending.
 */
adamas_status adamas_decode_step_shared(const void* q, const void* k_cache, const void* v_cache,
                                        const uint8_t* codes, adamas_dtype dt, int B, int Hq,
                                        int Hkv, int d, int64_t Lmax, int64_t L, int k, float t,
                                        void* workspace, size_t ws_bytes, int32_t* idx_out,
                                        float* out, cudaStream_t stream);

/* adamas_decode_step_host for the shared selection (idx_out [B][Hkv][k_eff]). */
adamas_status adamas_decode_step_shared_host(const void* q_host, void* q_dev,
                                             const void* k_cache, const void* v_cache,
                                             const uint8_t* codes, adamas_dtype dt, int B,
                                             int Hq, int Hkv, int d, int64_t Lmax, int64_t L,
                                             int k, float t, void* workspace, size_t ws_bytes,
                                             int32_t* idx_out, float* out_dev, float* out_host,
                                             cudaStream_t stream);

/* adamas_select_topk for the shared selection: idx_out [B][Hkv][k_eff]. */
adamas_status adamas_select_topk_shared(const uint8_t* qcodes, const uint8_t* codes, int B,
                                        int Hq, int Hkv, int64_t Lmax, int64_t L, int k,
                                        void* workspace, size_t ws_bytes, int32_t* idx_out,
                                        cudaStream_t stream);

/*
 * Per-sequence context lengths (serving form of the same step; the Adamas pages run
 * each sequence over its own context and the method is unchanged).  Contiguous
 * caches as in adamas_decode_step, [B][Hkv][Lmax][d]; sequence b uses its first
 * seq_lens[b] positions (device array [B] of int32, each in [0, Lmax]).  shared = 0
 * selects per query head (idx_out [B][Hq][min(k, Lmax)]), shared = 1 per kv head
 * as adamas_decode_step_shared (idx_out [B][Hkv][min(k, Lmax)]).  A row holds the
 * min(k, seq_lens[b]) selected positions, ascending, then -1.  A sequence of length
 * 0 selects nothing and its output is all zeros.  The launch plan is made for Lmax.
 * A length outside [0, Lmax] is read on the device: it is clamped and recorded in
 * the workspace error word (adamas_check_workspace returns ADAMAS_ERR_INVALID_ARG).
 */
adamas_status adamas_decode_step_varlen(const void* q, const void* k_cache, const void* v_cache,
                                        const uint8_t* codes, adamas_dtype dt, int B, int Hq,
                                        int Hkv, int d, int64_t Lmax, const int32_t* seq_lens,
                                        int k, float t, int shared, void* workspace,
                                        size_t ws_bytes, int32_t* idx_out, float* out,
                                        cudaStream_t stream);

/*
 * Paged caches (block tables, the layout of paged-attention serving engines).  A
 * pool of num_pages pages, each holding page_size consecutive positions of every
 * kv head: k_pages, v_pages [num_pages][Hkv][page_size][d] elements of `dt`,
 * code_pages [num_pages][Hkv][page_size][d/4] bytes (adamas_encode_pages).
 * Position p of sequence b lives in page block_table[b * max_blocks_per_seq +
 * p / page_size], row p % page_size.  page_size is a power of two in [1, 2^20];
 * max_blocks_per_seq * page_size >= max_seq_len; seq_lens [B] int32 in
 * [0, max_seq_len] (device).  Entries of a block-table row past the sequence's
 * last page are never read.  The kernel copies each page's codes straight into
 * shared memory and gathers the selected K/V rows through the table.  idx_out,
 * out, shared and the error behaviour are those of adamas_decode_step_varlen with
 * Lmax = max_seq_len; a page id outside [0, num_pages) is read on the device: page
 * 0 is used instead and the error word records it (ADAMAS_ERR_INVALID_ARG).
 */
adamas_status adamas_decode_step_paged(const void* q, const void* k_pages, const void* v_pages,
                                       const uint8_t* code_pages, adamas_dtype dt, int B, int Hq,
                                       int Hkv, int d, int page_size, int64_t num_pages,
                                       const int32_t* block_table, int max_blocks_per_seq,
                                       const int32_t* seq_lens, int64_t max_seq_len, int k,
                                       float t, int shared, void* workspace, size_t ws_bytes,
                                       int32_t* idx_out, float* out, cudaStream_t stream);

/*
 * adamas_decode_step_paged for a caller whose queries and outputs live in host memory
 * (the serving loop of a paged engine): q_host [B][Hq][d] elements of `dt` in,
 * out_host [B][Hq][d] float32 back, both asynchronous on `stream` (synchronize
 * before reading out_host).  Page-locked host buffers mapped into the device's
 * address space are read and written by the kernel in place (no copies); otherwise
 * q goes through the caller's device staging buffer q_dev and the output through
 * out_dev.  Every argument is checked before anything is queued; the rest is as in
 * adamas_decode_step_paged.
 */
adamas_status adamas_decode_step_paged_host(const void* q_host, void* q_dev, const void* k_pages,
                                            const void* v_pages, const uint8_t* code_pages,
                                            adamas_dtype dt, int B, int Hq, int Hkv, int d,
                                            int page_size, int64_t num_pages,
                                            const int32_t* block_table, int max_blocks_per_seq,
                                            const int32_t* seq_lens, int64_t max_seq_len, int k,
                                            float t, int shared, void* workspace,
                                            size_t ws_bytes, int32_t* idx_out, float* out_dev,
                                            float* out_host, cudaStream_t stream);

/* Stage entry point: distance scan + top-k over paged codes from query codes. */
adamas_status adamas_select_topk_paged(const uint8_t* qcodes, const uint8_t* code_pages, int B,
                                       int Hq, int Hkv, int page_size, int64_t num_pages,
                                       const int32_t* block_table, int max_blocks_per_seq,
                                       const int32_t* seq_lens, int64_t max_seq_len, int k,
                                       int shared, void* workspace, size_t ws_bytes,
                                       int32_t* idx_out, cudaStream_t stream);

/*
 * Key encoder for paged caches: encodes every row (all kv heads, all page_size
 * positions) of the pages page_ids[0 .. n_ids) of k_pages into code_pages (layouts
 * as in adamas_decode_step_paged); page_ids == NULL encodes all num_pages pages.
 * Appending a token re-encodes its page.  Page ids outside [0, num_pages) are
 * skipped.
 */
adamas_status adamas_encode_pages(const void* k_pages, adamas_dtype dt, int Hkv, int d,
                                  int page_size, int64_t num_pages, const int32_t* page_ids,
                                  int64_t n_ids, float t, uint8_t* code_pages,
                                  cudaStream_t stream);

/*
 * Dynamic (per-vector) bucket thresholds: blog "ADAMAS：稀疏注意力优化技术解析与应用实践",
 * section 2.2, sets the thresholds at -0.5 absmax, 0, +0.5 absmax of the values being
 * bucketed, with groups of 128 dimensions.  Here every key and query vector (one
 * 128-dimension group) gets t_v = ratio * max_i |y_i| of its own rotated values y;
 * 0 < ratio <= 1 (the blog's 0.5); other values return ADAMAS_ERR_INVALID_ARG.
 * Layouts and errors are those of the fixed-threshold encoders.
 */
adamas_status adamas_encode_keys_absmax(const void* k_cache, adamas_dtype dt, int B, int Hkv,
                                        int d, int64_t Lmax, int64_t pos0, int64_t n_new,
                                        float ratio, uint8_t* codes, cudaStream_t stream);
adamas_status adamas_encode_queries_absmax(const void* q, adamas_dtype dt, int B, int Hq, int d,
                                           float ratio, uint8_t* qcodes, cudaStream_t stream);
adamas_status adamas_encode_pages_absmax(const void* k_pages, adamas_dtype dt, int Hkv, int d,
                                         int page_size, int64_t num_pages,
                                         const int32_t* page_ids, int64_t n_ids, float ratio,
                                         uint8_t* code_pages, cudaStream_t stream);

/*
 * adamas_decode_step (shared = 0) or adamas_decode_step_shared (shared = 1) with the
 * fused query encode using per-vector absmax thresholds; `codes` must hold keys
 * encoded by adamas_encode_keys_absmax with the same ratio.
 */
adamas_status adamas_decode_step_absmax(const void* q, const void* k_cache, const void* v_cache,
                                        const uint8_t* codes, adamas_dtype dt, int B, int Hq,
                                        int Hkv, int d, int64_t Lmax, int64_t L, int k,
                                        float ratio, int shared, void* workspace,
                                        size_t ws_bytes, int32_t* idx_out, float* out,
                                        cudaStream_t stream);

/* adamas_decode_step_absmax with host-memory queries and outputs: the same buffer
 * rules as adamas_decode_step_paged_host (mapped page-locked buffers in place, else
 * copies through q_dev / out_dev; every argument checked before anything is queued). */
adamas_status adamas_decode_step_absmax_host(const void* q_host, void* q_dev,
                                             const void* k_cache, const void* v_cache,
                                             const uint8_t* codes, adamas_dtype dt, int B,
                                             int Hq, int Hkv, int d, int64_t Lmax, int64_t L,
                                             int k, float ratio, int shared, void* workspace,
                                             size_t ws_bytes, int32_t* idx_out, float* out_dev,
                                             float* out_host, cudaStream_t stream);

/*
 * Context-parallel decode (one GPU per contiguous slice of a long context).  The
 * pages run one device; this split is the implementation's.  Rank r of `world`
 * holds positions [pos_offset, pos_offset + L) of a context of L_total positions
 * (lower ranks hold lower positions) in contiguous caches [B][Hkv][Lmax][d] and
 * codes [B][Hkv][Lmax][d/4].  One step:
 *   1. adamas_cp_histograms: per selection row (query head, or kv head if shared),
 *      the cumulative histogram of Manhattan distances over the slice -> hist
 *      [B][rows][bins] uint32 (count of distances <= bin), bins = 385 (per head) or
 *      384 G + 1 (shared); adamas_cp_hist_elems gives B * rows * bins.
 *   2. the caller all-gathers the histograms of all ranks, rank order:
 *      hist_all [world][B][rows][bins].
 *   3. adamas_cp_attend: the global top-k (the first min(k, L_total) positions by
 *      (distance, global position)) restricted to this slice, attention over it,
 *      and one softmax partial per query head -> partial [B][Hq][132] float
 *      (m in the log2 domain, l, 0, 0, acc[128]; l = 0: nothing selected here).
 *      idx_out (nullable, [B][rows][min(k, L_total)]) receives this rank's global
 *      positions at their global slots; other slots are left untouched, so
 *      -1-filled arrays of all ranks merge by elementwise max.
 *   4. the caller all-gathers the partials: partials_all [world][B][Hq][132].
 *   5. adamas_cp_combine: out [B][Hq][d] float, equal to adamas_decode_step (or
 *      _shared) over the whole context.
 * Steps 1 and 3 are launches of the fused decode kernel (q encoded inside, as in
 * adamas_decode_step); step 3 reads back the distances step 1 computed (the codes
 * are scanned once).  Errors as adamas_decode_step, plus ADAMAS_ERR_INVALID_ARG for
 * pos_offset < 0, pos_offset + L > L_total, L_total > 2^31 - 1 or rank outside
 * [0, world).
 */
size_t adamas_cp_hist_elems(int B, int Hq, int Hkv, int shared);
/* Workspace of adamas_cp_histograms / adamas_cp_attend for this rank's L positions:
 * the error word plus the distances and histograms each CTA keeps from step 1 to
 * step 3 (zero-fill once with adamas_workspace_init; both steps must get the same
 * workspace and sizes); 0 if the arguments are invalid. */
size_t adamas_cp_workspace_bytes(int B, int Hq, int Hkv, int d, int64_t L, int k, int shared);
adamas_status adamas_cp_histograms(const void* q, const uint8_t* codes, adamas_dtype dt, int B,
                                   int Hq, int Hkv, int d, int64_t Lmax, int64_t L, int k,
                                   float t, int shared, void* workspace, size_t ws_bytes,
                                   uint32_t* hist_out, cudaStream_t stream);
adamas_status adamas_cp_attend(const void* q, const void* k_cache, const void* v_cache,
                               const uint8_t* codes, adamas_dtype dt, int B, int Hq, int Hkv,
                               int d, int64_t Lmax, int64_t L, int64_t L_total,
                               int64_t pos_offset, int k, float t, int shared,
                               const uint32_t* hist_all, int world, int rank, void* workspace,
                               size_t ws_bytes, int32_t* idx_out, float* partial_out,
                               cudaStream_t stream);
adamas_status adamas_cp_combine(const float* partials_all, int world, int B, int Hq, float* out,
                                cudaStream_t stream);

/* Workspace of adamas_sparse_attention, in bytes (zero-filled once, self-cleaning). */
size_t adamas_sparse_attention_workspace_bytes(int B, int Hq, int k_eff);

/*
 * Stage entry point: split-k gather attention + combine over explicit positions
 * idx [B][Hq][k_eff] (any order, each in [0, Lmax)); writes out [B][Hq][d] fp32.
 * This is the last stage of the v2 abstract of "Adamas: Hadamard Sparse Attention
 * for Efficient Long-Context Inference": the ORIGINAL K/V states at the selected
 * positions are gathered and attention runs over them alone, softmax of
 * (q . K_j) / sqrt(d) with fp32 accumulation.  Positions may repeat; each copy
 * counts as its own term.  Query head h reads kv head h / G.
 */
adamas_status adamas_sparse_attention(const void* q, const void* k_cache, const void* v_cache,
                                      adamas_dtype dt, const int32_t* idx, int B, int Hq,
                                      int Hkv, int d, int64_t Lmax, int k_eff, void* workspace,
                                      size_t ws_bytes, float* out, cudaStream_t stream);

/*
 * adamas_sparse_attention without a workspace, for callers that cannot allocate
 * device memory: code running inside a memory allocator's own hooks, latency
 * paths that must not call into the driver's allocator, or hosts whose memory
 * pool owns every device allocation.  The paper has no counterpart to this entry
 * point; it is an interface convenience.
 *
 * Same arguments, layouts and result as adamas_sparse_attention, minus the
 * workspace.  Scratch (per-head counters and split partials, about 2.2 MB) is a
 * fixed array inside the library that every GPU loading the library keeps until
 * the process exits.  Limit: B * Hq <= 4096 (larger calls return
 * ADAMAS_ERR_UNSUPPORTED); the split count is reduced so that B * Hq * splits
 * <= 4096 (on a 148-SM B200 the default split count never exceeds that).  Every
 * call looks up the array's device address; the FIRST call on each device (and the
 * first after a device reset moved the array) clears its counters, synchronizing the
 * device: make that first call outside any stream capture.  All calls share the one array (each completed call leaves
 * its counters at zero again), so calls that run concurrently on the GPU — from
 * several streams or host threads — race and must be serialized by the caller.
 */
adamas_status adamas_sparse_attention_noalloc(const void* q, const void* k_cache,
                                              const void* v_cache, adamas_dtype dt,
                                              const int32_t* idx, int B, int Hq, int Hkv, int d,
                                              int64_t Lmax, int k_eff, float* out,
                                              cudaStream_t stream);

/*
 * Launch plan of adamas_decode_step for these sizes on the current device (host
 * only, no launch): total CTAs, CTAs per thread-block cluster (one cluster per
 * (batch, kv head) pair), key positions per CTA, dynamic shared memory bytes per
 * CTA.  Any output pointer may be NULL.
 */
adamas_status adamas_decode_plan(int B, int Hq, int Hkv, int d, int64_t L, int k, int* ctas,
                                 int* cluster, int64_t* tokens_per_cta, int* smem_bytes);

/* adamas_decode_plan of adamas_decode_step_shared / adamas_select_topk_shared. */
adamas_status adamas_decode_plan_shared(int B, int Hq, int Hkv, int d, int64_t L, int k,
                                        int* ctas, int* cluster, int64_t* tokens_per_cta,
                                        int* smem_bytes);

#ifdef __cplusplus
}
#endif

#endif /* ADAMAS_H */

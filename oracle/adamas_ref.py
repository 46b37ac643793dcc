"""Float64 CPU oracle of the Adamas decode hot path.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference legs of ``bench.py`` may import it.  It shares no
code, table or constant with the CUDA path in ``token_level_sparse_fwht_b200`` and
imports nothing from it.

What the method computes (sources are the pages on "Adamas: Hadamard Sparse
Attention for Efficient Long-Context Inference", arXiv 2510.18413):

* v2 abstract: a Hadamard transform, bucketization and 2-bit compression give a
  compact code per key and query; a distance-based estimate picks the top-k
  candidate positions; the ORIGINAL K/V rows at those positions are gathered for
  sparse attention.
* v1 abstract: the distance estimate is a Manhattan distance.
* third-party blog "ADAMAS：稀疏注意力优化技术解析与应用实践", section 2.1: QK^T is
  rewritten as (HQ)(HK)^T with a recursively built Hadamard matrix; section 2.2:
  three thresholds and strict "<" comparisons map a value to a bucket 0..3;
  section 3.1: the 2-bit codes are packed several to a machine word.

Readings where the pages are silent or garbled:

* H is the Sylvester matrix in natural order, H[i, j] = (-1)^popcount(i & j),
  scaled by 1/sqrt(d) so that it is orthonormal (the (HQ)(HK)^T identity of blog
  section 2.1 needs that); no random sign flips.
* Thresholds are {-t, 0, +t} with t a per-run constant, shared by keys and queries
  (the blog's per-batch 0.5*absmax rule is replaced by a fixed t).
* A value exactly on a threshold goes to the upper bucket (strict "<" chain).
* Codes are packed 4 per byte: coordinate i sits in byte i >> 2 at bits
  2*(i & 3) .. 2*(i & 3) + 1, so a key code is 32 bytes for d = 128.
* Smaller Manhattan distance means more relevant.  Top-k keeps the first
  k_eff = min(k, L) positions in the order (distance ascending, position
  ascending) and reports them ascending by position.
* GQA: query head h is scored against kv head h // G, G = Hq / Hkv, and selects
  its own top-k.
* Attention uses the original (untransformed) q and K, scale 1/sqrt(d), softmax
  over the selected positions only.

Parity pins (tests/test_oracle_pins.py) tie every function below to something
other than itself: scipy's textbook Hadamard routine, closed forms, hand-written
golden cases under tests/golden/, brute force on tiny inputs, the t = 0 reduction
to 3 x Hamming distance of sign bits, and torch's dense attention.
"""
from __future__ import annotations

import numpy as np

D = 128                 # head dimension the method is run at
CODE_BYTES = D // 4     # 2-bit codes, 4 per byte
MAX_DIST = 3 * D        # largest Manhattan distance between two code vectors


# --------------------------------------------------------------------------- H
def sylvester_hadamard(n: int = D) -> np.ndarray:
    """Unnormalised Sylvester Hadamard matrix, entries +1/-1, natural order.

    Blog section 2.1 builds H recursively; the recursion H_{2m} = [[H, H], [H, -H]]
    gives H[i, j] = (-1)^popcount(i & j).
    """
    if n < 1 or n & (n - 1):
        raise ValueError("n must be a power of two")
    idx = np.arange(n)
    anded = np.bitwise_and.outer(idx, idx)
    parity = np.zeros_like(anded)
    for bit in range(int(n).bit_length()):
        parity ^= (anded >> bit) & 1
    return np.where(parity == 1, -1, 1).astype(np.int64)


def hadamard_rotate(x: np.ndarray) -> np.ndarray:
    """y = H x / sqrt(d) over the last axis, in float64 (v2 abstract; blog 2.1)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    H = sylvester_hadamard(d).astype(np.float64)
    return (x @ H.T) / np.sqrt(d)


# --------------------------------------------------------------------- codes
def bucketize(y: np.ndarray, t: float) -> np.ndarray:
    """2-bit bucket of every coordinate (blog section 2.2, thresholds -t, 0, +t).

    y < -t -> 0;  -t <= y < 0 -> 1;  0 <= y < t -> 2;  y >= t -> 3.
    The threshold t is taken as the float32 value the kernels receive.
    """
    y = np.asarray(y, dtype=np.float64)
    t = float(np.float32(t))
    codes = np.full(y.shape, 3, dtype=np.uint8)
    codes[y < t] = 2
    codes[y < 0.0] = 1
    codes[y < -t] = 0
    return codes


def threshold_margin(y: np.ndarray, t: float) -> np.ndarray:
    """Distance of every coordinate to the nearest bucket threshold."""
    y = np.asarray(y, dtype=np.float64)
    t = float(np.float32(t))
    return np.minimum(np.minimum(np.abs(y + t), np.abs(y)), np.abs(y - t))


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """Pack 2-bit codes 4 per byte: coordinate i -> byte i>>2, bits 2*(i&3)."""
    codes = np.asarray(codes, dtype=np.uint8)
    if codes.shape[-1] % 4:
        raise ValueError("last axis must be a multiple of 4")
    c = codes.reshape(codes.shape[:-1] + (codes.shape[-1] // 4, 4)).astype(np.uint16)
    packed = c[..., 0] | (c[..., 1] << 2) | (c[..., 2] << 4) | (c[..., 3] << 6)
    return packed.astype(np.uint8)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    """Inverse of pack_codes."""
    p = np.asarray(packed, dtype=np.uint8)
    parts = [(p >> (2 * r)) & 3 for r in range(4)]
    return np.stack(parts, axis=-1).reshape(p.shape[:-1] + (p.shape[-1] * 4,))


def encode(x: np.ndarray, t: float) -> np.ndarray:
    """Packed code of each vector: Hadamard, then bucketize, then pack."""
    return pack_codes(bucketize(hadamard_rotate(x), t))


# ------------------------------------------------------------------ selection
def manhattan(cq: np.ndarray, ck: np.ndarray) -> np.ndarray:
    """Manhattan distance between code vectors (v1 abstract), integer.

    cq: [..., d] codes of one query; ck: [..., L, d] codes of the keys.
    """
    a = np.asarray(cq, dtype=np.int64)
    b = np.asarray(ck, dtype=np.int64)
    return np.abs(b - a[..., None, :]).sum(axis=-1)


def select_topk(dist: np.ndarray, k: int) -> np.ndarray:
    """First min(k, L) positions under (distance asc, position asc), ascending."""
    dist = np.asarray(dist)
    L = dist.shape[-1]
    k_eff = min(int(k), L)
    pos = np.arange(L)
    order = np.lexsort((pos, dist))          # full stable sort, last key primary
    return np.sort(order[:k_eff]).astype(np.int64)


# ------------------------------------------------------------------ attention
def sparse_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray,
                     idx: np.ndarray) -> np.ndarray:
    """Softmax attention of one query over the gathered ORIGINAL rows K[idx], V[idx].

    v2 abstract: the selected positions gather the original KV states; scale
    1/sqrt(d), float64.
    """
    q = np.asarray(q, dtype=np.float64)
    Ks = np.asarray(K, dtype=np.float64)[idx]
    Vs = np.asarray(V, dtype=np.float64)[idx]
    s = Ks @ q / np.sqrt(q.shape[-1])
    p = np.exp(s - s.max())
    p /= p.sum()
    return p @ Vs


# --------------------------------------------------------------- whole step
def decode_step(q: np.ndarray, K: np.ndarray, V: np.ndarray, k: int, t: float,
                key_codes: np.ndarray | None = None,
                query_codes: np.ndarray | None = None):
    """One Adamas decode step for every (batch, query head).

    q: [B, Hq, d]; K, V: [B, Hkv, L, d] (only the first L positions are used);
    key_codes: optional packed [B, Hkv, L, d/4] (else encoded here);
    query_codes: optional packed [B, Hq, d/4] (else encoded here).
    Returns (idx [B, Hq, k_eff] int64 ascending, out [B, Hq, d] float64).
    """
    q = np.asarray(q)
    B, Hq, d = q.shape
    _, Hkv, L, _ = K.shape
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    if key_codes is None:
        key_codes = encode(K, t)
    if query_codes is None:
        query_codes = encode(q, t)
    ck = unpack_codes(np.asarray(key_codes)[:, :, :L])
    cq = unpack_codes(np.asarray(query_codes))
    k_eff = min(int(k), L)
    idx = np.zeros((B, Hq, k_eff), dtype=np.int64)
    out = np.zeros((B, Hq, d), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            kvh = h // G
            dist = manhattan(cq[b, h], ck[b, kvh])
            sel = select_topk(dist, k)
            idx[b, h] = sel
            out[b, h] = sparse_attention(q[b, h], K[b, kvh, :L], V[b, kvh, :L], sel)
    return idx, out


def decode_head(q_vec, K_rows, V_rows, k, t, key_codes_rows=None, query_code=None):
    """decode_step for one (batch, query head) pair; used to sample big configs.

    q_vec [d]; K_rows, V_rows [L, d]; key_codes_rows [L, d/4] packed (optional).
    """
    if key_codes_rows is None:
        key_codes_rows = encode(K_rows, t)
    if query_code is None:
        query_code = encode(q_vec, t)
    dist = manhattan(unpack_codes(query_code), unpack_codes(key_codes_rows))
    sel = select_topk(dist, k)
    return sel, sparse_attention(q_vec, K_rows, V_rows, sel), dist


# ------------------------------------------------ shared GQA selection variant
def decode_step_shared(q: np.ndarray, K: np.ndarray, V: np.ndarray, k: int, t: float,
                       key_codes: np.ndarray | None = None,
                       query_codes: np.ndarray | None = None):
    """Decode step with one selection per kv head, shared by its G query heads.

    A variant the pages leave open (the v2 abstract selects top-k positions but
    says nothing about grouped-query attention): the score of key j for kv head
    h_kv is the SUM over the group's query heads of their Manhattan distances to
    key j's code; the first min(k, L) positions under (sum asc, position asc) are
    gathered once and every query head of the group attends over them.
    Returns (idx [B, Hkv, k_eff] ascending, out [B, Hq, d] float64).
    """
    q = np.asarray(q)
    B, Hq, d = q.shape
    _, Hkv, L, _ = K.shape
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    if key_codes is None:
        key_codes = encode(K, t)
    if query_codes is None:
        query_codes = encode(q, t)
    ck = unpack_codes(np.asarray(key_codes)[:, :, :L])
    cq = unpack_codes(np.asarray(query_codes))
    k_eff = min(int(k), L)
    idx = np.zeros((B, Hkv, k_eff), dtype=np.int64)
    out = np.zeros((B, Hq, d), dtype=np.float64)
    for b in range(B):
        for kvh in range(Hkv):
            score = np.zeros(L, dtype=np.int64)
            for g in range(G):
                score += manhattan(cq[b, kvh * G + g], ck[b, kvh])
            sel = select_topk(score, k)
            idx[b, kvh] = sel
            for g in range(G):
                h = kvh * G + g
                out[b, h] = sparse_attention(q[b, h], K[b, kvh, :L], V[b, kvh, :L], sel)
    return idx, out


# ------------------------------------- per-sequence context lengths (serving form)
def decode_step_varlen(q: np.ndarray, K: np.ndarray, V: np.ndarray, seq_lens, k: int,
                       t: float, key_codes: np.ndarray | None = None,
                       query_codes: np.ndarray | None = None, shared: bool = False):
    """Decode step where sequence b has its own context length seq_lens[b].

    The pages run every sequence over its own context; nothing in the method
    changes: sequence b is decode_step (or decode_step_shared) over its first
    seq_lens[b] positions.  The result is laid out for a batch:
    idx [B, rows, min(k, Lmax)] with entries past min(k, seq_lens[b]) set to -1
    (rows = Hq, or Hkv when shared), out [B, Hq, d]; a sequence of length 0 selects
    nothing and its output is all zeros (a reading: softmax over an empty set is
    undefined).  K, V: [B, Hkv, Lmax, d] logical caches; paging is only a storage
    layout and is not modelled here.
    """
    q = np.asarray(q)
    B, Hq, d = q.shape
    _, Hkv, Lmax, _ = K.shape
    seq_lens = [int(x) for x in seq_lens]
    if len(seq_lens) != B or min(seq_lens) < 0 or max(seq_lens) > Lmax:
        raise ValueError("seq_lens must hold B lengths in [0, Lmax]")
    k_row = min(int(k), Lmax)
    rows = Hkv if shared else Hq
    idx = np.full((B, rows, k_row), -1, dtype=np.int64)
    out = np.zeros((B, Hq, d), dtype=np.float64)
    step = decode_step_shared if shared else decode_step
    for b, Lb in enumerate(seq_lens):
        if Lb == 0:
            continue
        kc = None if key_codes is None else np.asarray(key_codes)[b:b + 1, :, :Lb]
        qc = None if query_codes is None else np.asarray(query_codes)[b:b + 1]
        ib, ob = step(q[b:b + 1], K[b:b + 1, :, :Lb], V[b:b + 1, :, :Lb], k, t,
                      key_codes=kc, query_codes=qc)
        idx[b, :, :ib.shape[-1]] = ib[0]
        out[b] = ob[0]
    return idx, out


# ------------------------------------------ dynamic (absmax) bucket thresholds
def absmax_thresholds(x: np.ndarray, ratio: float = 0.5) -> np.ndarray:
    """Per-vector threshold t_v = ratio * max_i |y_i| of the rotated vector y = H x / sqrt(d).

    Blog "ADAMAS：稀疏注意力优化技术解析与应用实践", section 2.2: the bucket
    thresholds are -0.5 absmax, 0, +0.5 absmax of the values being bucketed, and
    groups of 128 dimensions beat one global absmax.  Reading: one group per head
    vector (d = 128), the absmax taken after the Hadamard rotation (the values that
    are bucketed), ratio 0.5 by default; float64, not rounded.
    """
    y = hadamard_rotate(x)
    return float(ratio) * np.abs(y).max(axis=-1)


def bucketize_per_vector(y: np.ndarray, t: np.ndarray) -> np.ndarray:
    """bucketize with one threshold per vector (t has y's shape minus the last axis)."""
    y = np.asarray(y, dtype=np.float64)
    tt = np.asarray(t, dtype=np.float64)[..., None]
    codes = np.full(y.shape, 3, dtype=np.uint8)
    codes[y < tt] = 2
    codes[y < 0.0] = 1
    codes[y < -tt] = 0
    return codes


def encode_absmax(x: np.ndarray, ratio: float = 0.5) -> np.ndarray:
    """Packed codes with per-vector absmax thresholds (see absmax_thresholds)."""
    return pack_codes(bucketize_per_vector(hadamard_rotate(x), absmax_thresholds(x, ratio)))


def decode_step_absmax(q: np.ndarray, K: np.ndarray, V: np.ndarray, k: int,
                       ratio: float = 0.5, shared: bool = False):
    """decode_step (or decode_step_shared) with every key and query encoded under its
    own absmax threshold instead of one fixed t."""
    step = decode_step_shared if shared else decode_step
    return step(q, K, V, k, 0.0, key_codes=encode_absmax(K, ratio),
                query_codes=encode_absmax(q, ratio))

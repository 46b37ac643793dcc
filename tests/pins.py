"""Checks that pin the float64 oracle to facts outside itself.

Each check_* function raises AssertionError on failure.  test_oracle_pins.py runs
them as tests; test_oracle_mutations.py plants plausible mistakes in the oracle
(on the CPU) and confirms that at least one check catches each mistake.

What pins what:
* Hadamard: scipy.linalg.hadamard (textbook Sylvester routine), H H^T = d I in
  integers, involution of H/sqrt(d), q.k preserved (blog section 2.1), Walsh
  closed forms.
* Codes: hand-written golden cases (tests/golden/bucket_cases.txt) for the strict
  "<" chain of blog section 2.2.
* Threshold margin (which GPU encoder mismatches are forgiven): hand-worked rows
  (tests/golden/margin_cases.txt, float32 rounding of t included) and the property
  that moving y by less than its margin never changes its bucket, by slightly more
  always can.
* Packing: hand-worked bytes (tests/golden/pack_cases.txt).
* Distance: the |a-b| table (tests/golden/manhattan_table.txt), a pure-Python brute
  force, and the t = 0 reduction to 3 x Hamming distance of sign bits (SimHash).
* Top-k: pure-Python full sort by (distance, position); all-equal and k >= L cases.
* Attention: budget = L equals torch's dense scaled-dot-product attention; budget 1
  returns the V row.
* GQA mapping and recall of planted keys on the seeded single-head workload.
* decode_head (one query head, used to sample the big workloads and to enumerate the
  admissible query codes): equal to decode_step's row for that head, with natural
  and with explicitly given (different) key and query codes, and to a pure-Python
  brute force of distance, selection and dense attention.
* Shared selection: G = 1 reduction, pure-Python brute force, identical heads.
* Per-sequence lengths: pure-Python brute force (empty, short and long sequences,
  -1 padding), invariance to cache slots past a length, full-length reduction.
* Absmax thresholds: hand-worked cases (tests/golden/absmax_cases.txt), reduction to
  the fixed-threshold bucketize, the extreme coordinate's end bucket, per-vector
  scale invariance, and a brute-force decode over the absmax codes.
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch

import oracle.adamas_ref as ref

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows


# ---------------------------------------------------------------- Hadamard
def check_hadamard_matches_scipy():
    import scipy.linalg
    for n in (1, 2, 4, 8, 16, 32, 64, 128):
        H = ref.sylvester_hadamard(n)
        assert np.array_equal(H, scipy.linalg.hadamard(n).astype(np.int64)), n


def check_hadamard_orthogonal():
    H = ref.sylvester_hadamard(128)
    assert np.array_equal(H @ H.T, 128 * np.eye(128, dtype=np.int64))


def check_rotate_involution_and_dot():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((16, 128))
    y = ref.hadamard_rotate(x)
    assert np.allclose(ref.hadamard_rotate(y), x, rtol=0, atol=1e-12)
    q, k = rng.standard_normal((2, 64, 128))
    lhs = (ref.hadamard_rotate(q) * ref.hadamard_rotate(k)).sum(-1)
    rhs = (q * k).sum(-1)
    assert np.allclose(lhs, rhs, rtol=1e-12, atol=1e-12)
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-12)


def check_rotate_closed_forms():
    s = 1.0 / math.sqrt(128)
    ones = np.ones(128)
    e0 = np.zeros(128)
    e0[0] = 1
    assert np.allclose(ref.hadamard_rotate(ones), math.sqrt(128) * e0, atol=1e-12)
    assert np.allclose(ref.hadamard_rotate(e0), s * ones, atol=1e-15)
    # Walsh functions in natural order: e_1 -> + - + - ..., e_2 -> + + - - ...,
    # e_64 -> 64 x (+) then 64 x (-)
    e1 = np.zeros(128)
    e1[1] = 1
    assert np.allclose(ref.hadamard_rotate(e1), s * np.tile([1.0, -1.0], 64), atol=1e-15)
    e2 = np.zeros(128)
    e2[2] = 1
    assert np.allclose(ref.hadamard_rotate(e2), s * np.tile([1.0, 1.0, -1.0, -1.0], 32),
                       atol=1e-15)
    e64 = np.zeros(128)
    e64[64] = 1
    assert np.allclose(ref.hadamard_rotate(e64),
                       s * np.concatenate([np.ones(64), -np.ones(64)]), atol=1e-15)


# ------------------------------------------------------------------- codes
def check_bucket_golden():
    for t, v, c in _golden("bucket_cases.txt"):
        got = ref.bucketize(np.array([float(v)]), float(t))[0]
        assert int(got) == int(c), (t, v, c, int(got))


def check_pack_golden():
    for row in _golden("pack_cases.txt"):
        codes = np.array([int(x) for x in row[:4]], dtype=np.uint8)
        byte = int(row[4])
        assert int(ref.pack_codes(codes)[0]) == byte, (row, int(ref.pack_codes(codes)[0]))
        assert np.array_equal(ref.unpack_codes(np.array([byte], np.uint8)), codes)
    rng = np.random.default_rng(3)
    c = rng.integers(0, 4, size=(5, 7, 128), dtype=np.uint8)
    p = ref.pack_codes(c)
    assert p.shape == (5, 7, 32)
    assert np.array_equal(ref.unpack_codes(p), c)
    # coordinate order across bytes: codes i % 4 -> every byte 0b11100100
    assert np.all(ref.pack_codes(np.arange(128, dtype=np.uint8) % 4) == 228)


# --------------------------------------------------------------- distances
def check_margin_golden():
    """threshold_margin on hand-worked rows, float32(t) rounding included."""
    for t, y, m in _golden("margin_cases.txt"):
        got = float(ref.threshold_margin(np.array([float(y)]), float(t))[0])
        assert abs(got - float(m)) <= 1e-15 + 1e-12 * float(m), (t, y, m, got)


def check_margin_is_bucket_distance():
    """Moving y by less than its margin keeps its bucket; by slightly more, one way
    or the other changes it (bucketize is pinned by its own golden cases)."""
    rng = np.random.default_rng(83)
    for t in (0.0, 0.5, 1.01165):
        y = rng.uniform(-3.5, 3.5, 4000)
        m = ref.threshold_margin(y, t)
        y, m = y[m > 1e-6], m[m > 1e-6]
        c = ref.bucketize(y, t)
        assert np.array_equal(ref.bucketize(y - 0.999 * m, t), c)
        assert np.array_equal(ref.bucketize(y + 0.999 * m, t), c)
        moved = (ref.bucketize(y - 1.001 * m, t) != c) | (ref.bucketize(y + 1.001 * m, t) != c)
        assert moved.all()


def check_manhattan_table():
    table = np.array([[int(x) for x in r] for r in _golden("manhattan_table.txt")])
    for a in range(4):
        for b in range(4):
            d = ref.manhattan(np.array([a]), np.array([[b]]))
            assert int(d[0]) == table[a, b]


def check_manhattan_bruteforce():
    rng = np.random.default_rng(11)
    for _ in range(5):
        cq = rng.integers(0, 4, size=128)
        ck = rng.integers(0, 4, size=(9, 128))
        got = ref.manhattan(cq, ck)
        for j in range(9):
            s = 0
            for i in range(128):
                s += abs(int(cq[i]) - int(ck[j, i]))
            assert got[j] == s
    assert ref.manhattan(np.zeros(128, int), np.full((1, 128), 3))[0] == 384


def check_simhash_reduction():
    """t = 0: codes are 0/3 by sign, so distance = 3 x Hamming(sign bits)."""
    rng = np.random.default_rng(5)
    q = rng.standard_normal(128)
    K = rng.standard_normal((50, 128))
    cq = ref.unpack_codes(ref.encode(q, 0.0))
    ck = ref.unpack_codes(ref.encode(K, 0.0))
    dist = ref.manhattan(cq, ck)
    sq = ref.hadamard_rotate(q) >= 0
    sk = ref.hadamard_rotate(K) >= 0
    ham = (sq[None, :] != sk).sum(-1)
    assert np.array_equal(dist, 3 * ham)


# ------------------------------------------------------------------- top-k
def check_topk_bruteforce():
    rng = np.random.default_rng(13)
    for L, k in ((1, 1), (5, 3), (37, 10), (100, 100), (100, 250), (300, 64)):
        dist = rng.integers(0, 6, size=L)          # many ties
        want = sorted(sorted(range(L), key=lambda j: (int(dist[j]), j))[:min(k, L)])
        got = ref.select_topk(dist, k)
        assert list(got) == want, (L, k)


def check_topk_special():
    assert list(ref.select_topk(np.full(50, 7), 8)) == list(range(8))
    assert list(ref.select_topk(np.arange(10)[::-1].copy(), 20)) == list(range(10))
    assert list(ref.select_topk(np.array([5, 1, 5, 0, 1]), 2)) == [1, 3]


# --------------------------------------------------------------- attention
def check_attention_dense():
    rng = np.random.default_rng(17)
    L = 200
    q = rng.standard_normal(128)
    K = rng.standard_normal((L, 128)) * 2
    V = rng.standard_normal((L, 128))
    got = ref.sparse_attention(q, K, V, np.arange(L))
    want = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None, None, :], torch.from_numpy(K)[None, None],
        torch.from_numpy(V)[None, None])[0, 0, 0].numpy()
    assert np.allclose(got, want, rtol=0, atol=1e-12)
    # a subset equals dense attention over just those rows
    sub = np.array([3, 17, 50, 199])
    want_sub = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None, None, :], torch.from_numpy(K[sub])[None, None],
        torch.from_numpy(V[sub])[None, None])[0, 0, 0].numpy()
    assert np.allclose(ref.sparse_attention(q, K, V, sub), want_sub, atol=1e-12)


def check_attention_budget1():
    rng = np.random.default_rng(19)
    q = rng.standard_normal(128)
    K = rng.standard_normal((10, 128))
    V = rng.standard_normal((10, 128))
    assert np.array_equal(ref.sparse_attention(q, K, V, np.array([4])), V[4])


# -------------------------------------------------------------- whole step
def check_decode_dense_limit():
    """Budget = L: the sparse step is dense attention (v2 abstract's premise)."""
    rng = np.random.default_rng(23)
    B, Hq, Hkv, L = 2, 4, 2, 40
    q = rng.standard_normal((B, Hq, 128))
    K = rng.standard_normal((B, Hkv, L, 128))
    V = rng.standard_normal((B, Hkv, L, 128))
    idx, out = ref.decode_step(q, K, V, k=L, t=0.5)
    assert np.array_equal(idx, np.broadcast_to(np.arange(L), (B, Hq, L)))
    Kr = np.repeat(K, Hq // Hkv, axis=1)
    Vr = np.repeat(V, Hq // Hkv, axis=1)
    want = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[:, :, None, :], torch.from_numpy(Kr),
        torch.from_numpy(Vr))[:, :, 0].numpy()
    assert np.allclose(out, want, atol=1e-12)


def check_gqa_and_planted():
    """Query head h reads kv head h // G: a copy of q_h planted only in that kv
    head is its nearest key; the other kv heads never see it."""
    rng = np.random.default_rng(29)
    B, Hq, Hkv, L = 1, 8, 2, 256
    G = Hq // Hkv
    q = rng.standard_normal((B, Hq, 128))
    K = rng.standard_normal((B, Hkv, L, 128))
    V = rng.standard_normal((B, Hkv, L, 128))
    pos = {}
    for h in range(Hq):
        p = 10 + 30 * h
        K[0, h // G, p] = q[0, h]
        pos[h] = p
    idx, _ = ref.decode_step(q, K, V, k=1, t=0.5)
    for h in range(Hq):
        assert idx[0, h, 0] == pos[h], (h, idx[0, h, 0], pos[h])


def check_planted_recall_single_head():
    """Seeded single-head workload: its 4 planted keys (q + 0.1 noise) are in the
    budget-64 selection."""
    from workloads import WORKLOADS, generate
    w = WORKLOADS[1]
    inp = generate(w, "cpu")
    q = inp.q.double().numpy()
    K = inp.k_cache.double().numpy()
    V = inp.v_cache.double().numpy()
    idx, _ = ref.decode_step(q, K, V, k=64, t=inp.t)
    planted = set(inp.planted[0, 0].tolist())
    assert planted <= set(idx[0, 0].tolist())


# ---------------------------------------------------- shared GQA selection
def check_decode_head_matches_step():
    """decode_head(one head) = decode_step's row for that head, both with the codes it
    encodes itself and with given key / query codes that differ from those; and equal
    to a pure-Python brute force of the distances, the selection and the attention."""
    rng = np.random.default_rng(89)
    t, k = 0.5, 9
    q = rng.standard_normal((1, 4, 128))
    K = rng.standard_normal((1, 2, 60, 128))
    V = rng.standard_normal((1, 2, 60, 128))
    kc_alt = ref.encode(rng.standard_normal((1, 2, 60, 128)), t)
    qc_alt = ref.encode(rng.standard_normal((1, 4, 128)), t)
    i0, o0 = ref.decode_step(q, K, V, k, t)
    i1, o1 = ref.decode_step(q, K, V, k, t, key_codes=kc_alt, query_codes=qc_alt)
    differs = 0
    for h in range(4):
        kv = h // 2
        sel, out, dist = ref.decode_head(q[0, h], K[0, kv], V[0, kv], k, t)
        assert np.array_equal(sel, i0[0, h]) and np.allclose(out, o0[0, h], atol=1e-12)
        sel1, out1, dist1 = ref.decode_head(q[0, h], K[0, kv], V[0, kv], k, t,
                                            key_codes_rows=kc_alt[0, kv],
                                            query_code=qc_alt[0, h])
        assert np.array_equal(sel1, i1[0, h]) and np.allclose(out1, o1[0, h], atol=1e-12)
        cq = ref.unpack_codes(qc_alt[0, h])
        ck = ref.unpack_codes(kc_alt[0, kv])
        brute = [sum(abs(int(cq[i]) - int(ck[j, i])) for i in range(128)) for j in range(60)]
        assert [int(x) for x in dist1] == brute
        want = _brute_select(brute, k)
        assert list(sel1) == want
        assert np.allclose(out1, _dense(q[0, h], K[0, kv, want], V[0, kv, want]), atol=1e-12)
        differs += not np.array_equal(sel, sel1)
    assert differs, "the substituted codes must change some selection"


def check_shared_g1_is_per_head():
    """With one query head per kv head, shared selection IS per-head selection."""
    rng = np.random.default_rng(31)
    q = rng.standard_normal((2, 3, 128))
    K = rng.standard_normal((2, 3, 90, 128))
    V = rng.standard_normal((2, 3, 90, 128))
    i1, o1 = ref.decode_step(q, K, V, k=17, t=0.4)
    i2, o2 = ref.decode_step_shared(q, K, V, k=17, t=0.4)
    assert np.array_equal(i1, i2) and np.allclose(o1, o2, atol=1e-12)


def check_shared_bruteforce():
    """Pure-Python sum of per-head Manhattan distances, full sort by (sum, position),
    and torch dense attention over the selected rows for every head of the group."""
    rng = np.random.default_rng(37)
    B, Hq, Hkv, L, k, t = 1, 4, 2, 40, 9, 0.3
    G = Hq // Hkv
    q = rng.standard_normal((B, Hq, 128))
    K = rng.standard_normal((B, Hkv, L, 128))
    V = rng.standard_normal((B, Hkv, L, 128))
    idx, out = ref.decode_step_shared(q, K, V, k=k, t=t)
    cq = ref.unpack_codes(ref.encode(q, t))
    ck = ref.unpack_codes(ref.encode(K, t))
    for kvh in range(Hkv):
        score = []
        for j in range(L):
            s = 0
            for g in range(G):
                for i in range(128):
                    s += abs(int(cq[0, kvh * G + g, i]) - int(ck[0, kvh, j, i]))
            score.append(s)
        want = sorted(sorted(range(L), key=lambda j: (score[j], j))[:k])
        assert list(idx[0, kvh]) == want, (kvh, list(idx[0, kvh]), want)
        for g in range(G):
            h = kvh * G + g
            dense = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(q[0, h])[None, None, None, :],
                torch.from_numpy(K[0, kvh, want])[None, None],
                torch.from_numpy(V[0, kvh, want])[None, None])[0, 0, 0].numpy()
            assert np.allclose(out[0, h], dense, atol=1e-12)


def check_shared_identical_heads():
    """If every query head of a group is the same vector, the summed score is G times
    each head's distance, so the shared selection equals each head's own."""
    rng = np.random.default_rng(41)
    q0 = rng.standard_normal((1, 2, 128))
    q = np.repeat(q0, 4, axis=1)                  # Hq = 8, Hkv = 2, G = 4
    K = rng.standard_normal((1, 2, 120, 128))
    V = rng.standard_normal((1, 2, 120, 128))
    i_head, o_head = ref.decode_step(q, K, V, k=20, t=0.5)
    i_sh, o_sh = ref.decode_step_shared(q, K, V, k=20, t=0.5)
    for kvh in range(2):
        for g in range(4):
            assert np.array_equal(i_sh[0, kvh], i_head[0, kvh * 4 + g])
    assert np.allclose(o_sh, o_head, atol=1e-12)


# ------------------------------------------- per-sequence context lengths
def _brute_select(dist, k):
    return sorted(sorted(range(len(dist)), key=lambda j: (dist[j], j))[:k])


def _dense(qv, Ks, Vs):
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(qv)[None, None, None, :], torch.from_numpy(Ks)[None, None],
        torch.from_numpy(Vs)[None, None])[0, 0, 0].numpy()


def check_varlen_bruteforce():
    """Lengths 0, 5, 37 in a 40-slot cache: per head, a pure-Python Manhattan
    distance over the sequence's own positions, full sort by (distance, position),
    dense attention over the selection; -1 padding past min(k, L_b); an empty
    sequence selects nothing and outputs zeros.  Same for the shared selection with
    the group's distances summed."""
    rng = np.random.default_rng(43)
    B, Hq, Hkv, Lmax, k, t = 3, 4, 2, 40, 8, 0.35
    G = Hq // Hkv
    lens = [0, 5, 37]
    q = rng.standard_normal((B, Hq, 128))
    K = rng.standard_normal((B, Hkv, Lmax, 128))
    V = rng.standard_normal((B, Hkv, Lmax, 128))
    cq = ref.unpack_codes(ref.encode(q, t))
    ck = ref.unpack_codes(ref.encode(K, t))

    def dist(b, h, kvh, Lb):
        return [sum(abs(int(cq[b, h, i]) - int(ck[b, kvh, j, i])) for i in range(128))
                for j in range(Lb)]

    idx, out = ref.decode_step_varlen(q, K, V, lens, k, t)
    sidx, sout = ref.decode_step_varlen(q, K, V, lens, k, t, shared=True)
    assert idx.shape == (B, Hq, k) and sidx.shape == (B, Hkv, k)
    for b, Lb in enumerate(lens):
        ke = min(k, Lb)
        for kvh in range(Hkv):
            per = [dist(b, kvh * G + g, kvh, Lb) for g in range(G)]
            swant = _brute_select([sum(c) for c in zip(*per)], k) if Lb else []
            assert list(sidx[b, kvh, :ke]) == swant and (sidx[b, kvh, ke:] == -1).all()
            for g in range(G):
                h = kvh * G + g
                want = _brute_select(per[g], k) if Lb else []
                assert list(idx[b, h, :ke]) == want, (b, h)
                assert (idx[b, h, ke:] == -1).all()
                if Lb == 0:
                    assert (out[b, h] == 0).all() and (sout[b, h] == 0).all()
                    continue
                assert np.allclose(out[b, h], _dense(q[b, h], K[b, kvh, want], V[b, kvh, want]),
                                   atol=1e-12)
                assert np.allclose(sout[b, h],
                                   _dense(q[b, h], K[b, kvh, swant], V[b, kvh, swant]),
                                   atol=1e-12)


def check_varlen_ignores_tail():
    """Cache slots at or past a sequence's length take no part: overwriting them
    changes neither the selection nor the output."""
    rng = np.random.default_rng(47)
    B, Hq, Hkv, Lmax = 2, 2, 1, 64
    lens = [30, 64]
    q = rng.standard_normal((B, Hq, 128))
    K = rng.standard_normal((B, Hkv, Lmax, 128))
    V = rng.standard_normal((B, Hkv, Lmax, 128))
    i1, o1 = ref.decode_step_varlen(q, K, V, lens, 12, 0.5)
    K2, V2 = K.copy(), V.copy()
    K2[0, :, 30:] = np.repeat(q[0, :1, None, :], 34, axis=1) * 3.0   # would win if scanned
    V2[0, :, 30:] = 1e6
    i2, o2 = ref.decode_step_varlen(q, K2, V2, lens, 12, 0.5)
    assert np.array_equal(i1, i2) and np.array_equal(o1, o2)


def check_varlen_uniform_is_decode_step():
    """Every sequence at full length: the batch step of decode_step."""
    rng = np.random.default_rng(53)
    q = rng.standard_normal((2, 4, 128))
    K = rng.standard_normal((2, 2, 50, 128))
    V = rng.standard_normal((2, 2, 50, 128))
    i1, o1 = ref.decode_step(q, K, V, 16, 0.5)
    i2, o2 = ref.decode_step_varlen(q, K, V, [50, 50], 16, 0.5)
    assert np.array_equal(i1, i2) and np.array_equal(o1, o2)


# ------------------------------------------- dynamic (absmax) thresholds
def check_absmax_golden():
    """Hand-worked per-vector thresholds (tests/golden/absmax_cases.txt)."""
    cases = {}
    for case, ratio, idx, y, want in _golden("absmax_cases.txt"):
        cases.setdefault(int(case), (float(ratio), {}))[1][int(idx)] = (float(y), int(want))
    for case, (ratio, entries) in cases.items():
        y = np.zeros(128)
        for i, (v, _) in entries.items():
            y[i] = v
        x = ref.hadamard_rotate(y)               # H / sqrt(d) is its own inverse
        t = ref.absmax_thresholds(x, ratio)
        assert abs(t - ratio * np.abs(y).max()) <= 1e-12 * np.abs(y).max(), (case, t)
        codes = ref.unpack_codes(ref.encode_absmax(x, ratio))
        for i, (_, want) in entries.items():
            assert codes[i] == want, (case, i, codes[i], want)


def check_bucket_per_vector_golden():
    """The per-vector bucketize on the hand-worked threshold cases
    (tests/golden/bucket_cases.txt, values on and beside each threshold), each case a
    one-coordinate vector with its own t."""
    rows = _golden("bucket_cases.txt")
    t = np.array([float(r[0]) for r in rows])
    y = np.array([[float(r[1])] for r in rows])
    want = np.array([int(r[2]) for r in rows])
    assert np.array_equal(ref.bucketize_per_vector(y, t)[:, 0], want)


def check_absmax_reduces_to_fixed():
    """With each vector's threshold handed to the fixed-threshold bucketize, the
    per-vector rule gives the same codes."""
    rng = np.random.default_rng(59)
    x = rng.standard_normal((6, 128)) * rng.uniform(0.1, 10, (6, 1))
    y = ref.hadamard_rotate(x)
    t = np.float32(ref.absmax_thresholds(x, 0.5)).astype(np.float64)
    per_vec = ref.bucketize_per_vector(y, t)
    for v in range(6):
        assert np.array_equal(per_vec[v], ref.bucketize(y[v], t[v]))


def check_absmax_extreme_coordinate():
    """ratio <= 1: the coordinate of largest magnitude always lands in an end bucket."""
    rng = np.random.default_rng(61)
    x = rng.standard_normal((50, 128))
    y = ref.hadamard_rotate(x)
    codes = ref.unpack_codes(ref.encode_absmax(x, 0.7))
    j = np.abs(y).argmax(-1)
    for v in range(50):
        assert codes[v, j[v]] == (3 if y[v, j[v]] > 0 else 0)


def check_absmax_per_vector_scale_invariance():
    """Scaling one vector by a power of two leaves its codes and every other vector's
    codes unchanged (the threshold is per vector, not global)."""
    rng = np.random.default_rng(67)
    x = rng.standard_normal((8, 128))
    scales = 2.0 ** np.arange(-4, 4)[:, None]
    a = ref.encode_absmax(x, 0.5)
    b = ref.encode_absmax(x * scales, 0.5)
    assert np.array_equal(a, b)


def check_decode_absmax_uses_both_codes():
    """decode_step_absmax = decode_step over the absmax codes of keys and queries."""
    rng = np.random.default_rng(71)
    q = rng.standard_normal((1, 4, 128))
    K = rng.standard_normal((1, 2, 80, 128)) * rng.uniform(0.2, 5, (1, 2, 80, 1))
    V = rng.standard_normal((1, 2, 80, 128))
    i1, o1 = ref.decode_step_absmax(q, K, V, 11, 0.5)
    cq = ref.unpack_codes(ref.encode_absmax(q, 0.5))
    ck = ref.unpack_codes(ref.encode_absmax(K, 0.5))
    for h in range(4):
        d = [int(np.abs(cq[0, h].astype(int) - ck[0, h // 2, j].astype(int)).sum())
             for j in range(80)]
        want = _brute_select(d, 11)
        assert list(i1[0, h]) == want
        assert np.allclose(o1[0, h], _dense(q[0, h], K[0, h // 2, want], V[0, h // 2, want]),
                           atol=1e-12)


ALL_CHECKS = [
    check_hadamard_matches_scipy, check_hadamard_orthogonal,
    check_rotate_involution_and_dot, check_rotate_closed_forms, check_bucket_golden,
    check_pack_golden, check_manhattan_table, check_manhattan_bruteforce,
    check_simhash_reduction, check_topk_bruteforce, check_topk_special,
    check_attention_dense, check_attention_budget1, check_decode_dense_limit,
    check_gqa_and_planted, check_planted_recall_single_head,
    check_margin_golden, check_margin_is_bucket_distance, check_decode_head_matches_step,
    check_shared_g1_is_per_head, check_shared_bruteforce, check_shared_identical_heads,
    check_varlen_bruteforce, check_varlen_ignores_tail, check_varlen_uniform_is_decode_step,
    check_absmax_golden, check_bucket_per_vector_golden, check_absmax_reduces_to_fixed, check_absmax_extreme_coordinate,
    check_absmax_per_vector_scale_invariance, check_decode_absmax_uses_both_codes,
]

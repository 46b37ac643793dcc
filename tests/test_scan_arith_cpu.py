"""The decode scan's integer plan, emulated on the CPU against the oracle's distance.

A 32-byte code is 8 words of 16 packed 2-bit fields c = 2h + l.  For codes k, q the
scan uses |k - q| = r0 + 2 r1 with r0 = l_k ^ l_q and r1 = (h_k ^ h_q) & (e_q | (l_k ^
h_q)), e_q = [q in {0, 3}].  Code words A = w[2j], B = w[2j+1] are packed into three
words with one bit per coordinate of both (low bits p, high bits h, low bits aligned
with h), so r0 and r1 of 32 coordinates take one and two logic operations.  One
carry-save level on three of the four r0 words and three of the four r1 words leaves
two weight-1, three weight-2 and one weight-4 word for six popcounts.  A thread scores
its key's words in load order (the second 16-byte half first on alternate lane quads)
against the query's pairs rotated the same way.  This restates those steps on integers
and compares them with oracle.manhattan."""
import numpy as np

import oracle

M = 0xFFFFFFFF
EVEN = 0x55555555
ODD = 0xAAAAAAAA


def _pairs(w):
    p, h, l = [], [], []
    for j in range(4):
        a, b = w[2 * j], w[2 * j + 1]
        p.append((a & EVEN) | ((b << 1) & ODD))
        h.append((a & ODD) | ((b >> 1) & EVEN))
        l.append(((a << 1) & ODD) | (b & EVEN))
    return p, h, l


def _query_pairs(w):
    p, h, l = _pairs(w)
    return p, h, [~(hh ^ ll) & M for hh, ll in zip(h, l)]


def _pop(x):
    return bin(x).count("1")


def _dist(k, q):
    kp, kh, kl = k
    qp, qh, qe = q
    u1 = [a ^ b for a, b in zip(kp, qp)]
    u2 = [(kh[j] ^ qh[j]) & (qe[j] | (kl[j] ^ qh[j])) for j in range(4)]
    O = u1[0] ^ u1[1] ^ u1[2]
    T1 = (u1[0] & u1[1]) | (u1[2] & (u1[0] | u1[1]))
    T2 = u2[0] ^ u2[1] ^ u2[2]
    F = (u2[0] & u2[1]) | (u2[2] & (u2[0] | u2[1]))
    return _pop(O) + _pop(u1[3]) + 2 * (_pop(T1) + _pop(T2) + _pop(u2[3])) + 4 * _pop(F)


def _words(code_bytes):
    return [int(v) for v in np.frombuffer(bytes(code_bytes), dtype="<u4")]


def test_per_coordinate_rule_all_code_pairs():
    # r0 + 2 r1 equals |k - q| for all 16 pairs of 2-bit codes
    for k in range(4):
        for q in range(4):
            lk, hk, lq, hq = k & 1, k >> 1, q & 1, q >> 1
            e = 1 if q in (0, 3) else 0
            r0 = lk ^ lq
            r1 = (hk ^ hq) & (e | (lk ^ hq))
            assert r0 + 2 * r1 == abs(k - q)


def test_scan_plan_matches_manhattan():
    rng = np.random.default_rng(5)
    keys = rng.integers(0, 256, size=(300, 32), dtype=np.uint8)
    keys[0] = 0x00                       # all codes 0
    keys[1] = 0xFF                       # all codes 3
    keys[2] = 0xAA                       # all codes 2
    keys[3] = 0x55                       # all codes 1
    queries = rng.integers(0, 256, size=(6, 32), dtype=np.uint8)
    queries[0] = 0xFF
    queries[1] = 0x55
    queries[2] = 0x00
    for qb in queries:
        want = oracle.manhattan(oracle.unpack_codes(qb), oracle.unpack_codes(keys))
        qp, qh, qe = _query_pairs(_words(qb))
        for swz in (0, 1):
            # the query's pairs in this thread's order: pair (j + 2 swz) mod 4
            rot = [(j + 2 * swz) % 4 for j in range(4)]
            qt = ([qp[i] for i in rot], [qh[i] for i in rot], [qe[i] for i in rot])
            for kb, w in zip(keys, want):
                kw = _words(kb)
                kt = _pairs(kw[4:] + kw[:4] if swz else kw)
                assert _dist(kt, qt) == w

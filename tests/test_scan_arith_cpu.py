"""The decode scan's integer plan, emulated on the CPU against the oracle's distance.

A 32-byte code is 8 words of 16 packed 2-bit codes.  The scan turns each word into
thermometer form: [c>=1] and [c>=3] at the even and odd bit of every field
(w - (h & ~l) at the even bit), and [c>=2] of two words packed into one.  With
|a - b| = sum over t of [a>=t] xor [b>=t], the 12 XOR words of a (key, query) pair are
added by two carry-save levels: triples of words give sum and majority words, then
three of each again.  Two popcounts of weight 1, three of weight 2 and one of weight
4 give the distance.  A thread scores its key's words in load order (the second
16-byte half first on alternate lane quads) against the query's words permuted the
same way.  This restates those steps on integers and compares them with
oracle.manhattan."""
import numpy as np

import oracle

M = 0xFFFFFFFF


def _therm(w):
    a = [(x - ((x >> 1) & ~x & 0x55555555)) & M for x in w]
    b = [((w[2 * j] >> 1) & 0x55555555) | (w[2 * j + 1] & 0xAAAAAAAA) for j in range(4)]
    return a, b


def _pop(x):
    return bin(x).count("1")


def _dist_csa(k, q):
    x = [ka ^ qa for ka, qa in zip(k[0], q[0])] + [kb ^ qb for kb, qb in zip(k[1], q[1])]
    o, tw = [], []
    for j in range(4):
        a, b, c = x[3 * j:3 * j + 3]
        o.append(a ^ b ^ c)
        tw.append((a & b) | (c & (a | b)))
    O = o[0] ^ o[1] ^ o[2]
    T1 = (o[0] & o[1]) | (o[2] & (o[0] | o[1]))
    T2 = tw[0] ^ tw[1] ^ tw[2]
    F = (tw[0] & tw[1]) | (tw[2] & (tw[0] | tw[1]))
    return _pop(O) + _pop(o[3]) + 2 * (_pop(T1) + _pop(T2) + _pop(tw[3])) + 4 * _pop(F)


def _words(code_bytes):
    return [int(v) for v in np.frombuffer(bytes(code_bytes), dtype="<u4")]


def test_scan_plan_matches_manhattan():
    rng = np.random.default_rng(5)
    keys = rng.integers(0, 256, size=(300, 32), dtype=np.uint8)
    keys[0] = 0x00                       # all codes 0
    keys[1] = 0xFF                       # all codes 3
    keys[2] = 0xAA                       # all codes 2
    queries = rng.integers(0, 256, size=(6, 32), dtype=np.uint8)
    queries[0] = 0xFF
    queries[1] = 0x55                    # all codes 1
    for qb in queries:
        want = oracle.manhattan(oracle.unpack_codes(qb), oracle.unpack_codes(keys))
        qa, qbw = _therm(_words(qb))
        for swz in (0, 1):
            # the query's words in this thread's order: a[(i + 4 swz) mod 8], b[(j + 2 swz) mod 4]
            qt = ([qa[(i + 4 * swz) % 8] for i in range(8)], [qbw[(j + 2 * swz) % 4] for j in range(4)])
            for kb, w in zip(keys, want):
                kw = _words(kb)
                kt = _therm(kw[4:] + kw[:4] if swz else kw)
                assert _dist_csa(kt, qt) == w

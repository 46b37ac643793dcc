"""The tensor-core key encoder's index plan, checked on the CPU against the oracle.

The kernel factors the Sylvester H_128 as H_8 (x) H_16 (index i = 16 a + b), multiplies
each 16-dimension block by H_16 with m16n8k16 MMAs whose k order is permuted (k = 2q,
2q+1 -> dimensions 4q, 4q+1; k = 2q+8, 2q+9 -> 4q+2, 4q+3) and whose output columns are
permuted too (column n of n-tile nt -> block coordinate 4 (n >> 1) + 2 nt + (n & 1)), so
that lane q's accumulators hold block coordinates 4q .. 4q+3.  It butterflies the 8
blocks, buckets each unscaled coordinate y as min(floor(y / tt + 2), 3) (one float32
fused multiply-add, a saturating conversion; tt = t sqrt(128); only the sign when
t = 0), and builds byte q of every code word in lane q: the bytes of the even words in
one register, of the odd words in another.  A 4 x 4 byte transpose across the lane quad
(byte permutes after an xor-1 and an xor-2 exchange) turns them into whole words 2q and
2q + 1, which lane q stores.  This emulates those formulas lane by lane and compares the
bytes with oracle.encode; a code may differ only within float32 rounding of a
threshold."""
import numpy as np

import oracle


def _h16(d, n):
    return -1.0 if bin(d & n).count("1") & 1 else 1.0


def _byte_perm(x, y, s):
    b = [(x >> (8 * i)) & 255 for i in range(4)] + [(y >> (8 * i)) & 255 for i in range(4)]
    return sum(b[(s >> (4 * i)) & 7] << (8 * i) for i in range(4))


def _emulate(X, t):
    perm = np.zeros(16, int)
    for q in range(4):
        perm[2 * q], perm[2 * q + 1], perm[2 * q + 8], perm[2 * q + 9] = (4 * q, 4 * q + 1,
                                                                          4 * q + 2, 4 * q + 3)

    def col(nt, n):
        return 4 * (n >> 1) + 2 * nt + (n & 1)

    # z[block][nt][row][n]: block c times the permuted H_16 columns of n-tile nt
    z = np.zeros((8, 2, 16, 8))
    for nt in range(2):
        B = np.array([[_h16(perm[k], col(nt, n)) for n in range(8)] for k in range(16)])
        for c in range(8):
            z[c, nt] = X[:, 16 * c + perm] @ B
    for s in (1, 2, 4):
        for c in range(8):
            if not c & s:
                z[c], z[c | s] = z[c] + z[c | s], z[c] - z[c | s]
    tt = np.float32(t) * np.float32(np.sqrt(128.0))
    inv = np.float32(1.0) / tt if tt > 0 else np.float32(np.inf)

    def code(y):
        if not tt > 0:
            return 3 if y >= 0 else 0
        f = np.float32(float(np.float32(y)) * float(inv) + 2.0)   # one rounding, like an fma
        return int(min(max(np.floor(f), 0.0), 3.0))

    out = np.zeros((16, 32), np.uint8)
    for h in range(2):
        regs = {}
        for ln in range(32):
            q, row = ln & 3, (ln >> 2) + 8 * h
            pw = [0, 0]
            for a in range(8):
                for nt in range(2):
                    c0 = code(z[a, nt, row, 2 * q])
                    c1 = code(z[a, nt, row, 2 * q + 1])
                    pw[a & 1] |= (c0 | (c1 << 2)) << (8 * (a >> 1) + 4 * nt)
            regs[ln] = pw
        stage = {ln: [_byte_perm(regs[ln][i], regs[ln ^ 1][i], 0x3715 if ln & 1 else 0x6240)
                      for i in range(2)] for ln in range(32)}
        final = {ln: [_byte_perm(stage[ln][i], stage[ln ^ 2][i], 0x3276 if ln & 2 else 0x5410)
                      for i in range(2)] for ln in range(32)}
        for ln in range(32):
            q, row = ln & 3, (ln >> 2) + 8 * h
            words = np.array(final[ln], np.uint32)
            out[row, 8 * q:8 * q + 8] = np.frombuffer(words.tobytes(), np.uint8)
    return out


def test_mma_encoder_plan_matches_oracle():
    rng = np.random.default_rng(11)
    for t in (0.0, 0.5, 1.01165):
        X = rng.standard_normal((16, 128)).astype(np.float32)
        X[:, [3, 77]] *= 10.0
        X = (X.view(np.uint32) & 0xFFFF0000).view(np.float32).astype(np.float64)   # bf16 values
        got, want = _emulate(X, t), oracle.encode(X, t)
        y = oracle.hadamard_rotate(X)
        margin = np.minimum(np.minimum(abs(y + t), abs(y)), abs(y - t))
        diff = oracle.unpack_codes(got) != oracle.unpack_codes(want)
        assert not (diff & (margin >= 1e-5)).any()


def test_byte_transpose_is_a_transpose():
    # byte j of lane q's register ends up as byte q of lane j's register
    M = {q: sum(((16 * q + j) & 255) << (8 * j) for j in range(4)) for q in range(4)}
    A = {q: _byte_perm(M[q], M[q ^ 1], 0x3715 if q & 1 else 0x6240) for q in range(4)}
    T = {q: _byte_perm(A[q], A[q ^ 2], 0x3276 if q & 2 else 0x5410) for q in range(4)}
    for q in range(4):
        for j in range(4):
            assert (T[q] >> (8 * j)) & 255 == (M[j] >> (8 * q)) & 255

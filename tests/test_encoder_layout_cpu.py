"""The tensor-core key encoder's index plan, checked on the CPU against the oracle.

The kernel factors the Sylvester H_128 as H_8 (x) H_16 (index i = 16 a + b), multiplies
each 16-dimension block by H_16 with m16n8k16 MMAs whose k order is permuted (k = 2q,
2q+1 -> dimensions 4q, 4q+1; k = 2q+8, 2q+9 -> 4q+2, 4q+3), butterflies the 8 blocks,
buckets each unscaled coordinate y as min(floor(y / tt + 2), 3) (one float32 fused
multiply-add, a saturating conversion; tt = t sqrt(128); only the sign when t = 0),
and packs codes from the accumulator layout (row = lane/4 (+8), column = 8 nt + 2
(lane % 4) + e): lane q puts its nibbles at bits 16 nt + 4 q + 2 e of each block's
word, the quad ORs the words together (xor-1 and xor-2 exchanges) and lane q stores
words 2q and 2q + 1.  This emulates those formulas lane by lane and compares the
bytes with oracle.encode; a code may differ only within float32 rounding of a
threshold."""
import numpy as np

import oracle


def _h16(d, n):
    return -1.0 if bin(d & n).count("1") & 1 else 1.0


def _emulate(X, t):
    perm = np.zeros(16, int)
    for q in range(4):
        perm[2 * q], perm[2 * q + 1], perm[2 * q + 8], perm[2 * q + 9] = (4 * q, 4 * q + 1,
                                                                          4 * q + 2, 4 * q + 3)
    B = np.array([[_h16(perm[k], n) for n in range(16)] for k in range(16)])
    z = np.stack([X[:, 16 * c + perm] @ B for c in range(8)])     # [block][row][col]
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
        part = {}
        for ln in range(32):
            q = ln & 3
            row = (ln >> 2) + 8 * h
            for a in range(8):
                w = 0
                for nt in range(2):
                    c0 = code(z[a][row][8 * nt + 2 * q])
                    c1 = code(z[a][row][8 * nt + 2 * q + 1])
                    w |= (c0 | (c1 << 2)) << (16 * nt + 4 * q)
                part[(ln, a)] = w
        for ln in range(32):
            q = ln & 3
            row = (ln >> 2) + 8 * h
            full = [part[(ln, a)] | part[(ln ^ 1, a)] | part[(ln ^ 2, a)] | part[(ln ^ 3, a)]
                    for a in range(8)]
            words = np.array([full[2 * q], full[2 * q + 1]], np.uint32)
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

"""The tensor-core key encoder's index plan, checked on the CPU against the oracle.

The kernel factors the Sylvester H_128 as H_8 (x) H_16 (index i = 16 a + b), multiplies
each 16-dimension block by H_16 with m16n8k16 MMAs whose k order is permuted (k = 2q,
2q+1 -> dimensions 4q, 4q+1; k = 2q+8, 2q+9 -> 4q+2, 4q+3), butterflies the 8 blocks,
and packs codes from the accumulator layout (row = lane/4 (+8), column = 8 nt + 2
(lane % 4) + e) through xor-1 and xor-2 lane exchanges.  This emulates those formulas
lane by lane and compares the bytes with oracle.encode."""
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
    tt = t * np.sqrt(128.0)
    code = lambda y: int(y >= -tt) + int(y >= 0) + int(y >= tt)
    out = np.zeros((16, 32), np.uint8)
    for h in range(2):
        nib = {(ln, a, nt): code(z[a][(ln >> 2) + 8 * h][8 * nt + 2 * (ln & 3)])
               | (code(z[a][(ln >> 2) + 8 * h][8 * nt + 2 * (ln & 3) + 1]) << 2)
               for ln in range(32) for a in range(8) for nt in range(2)}
        byte = {}
        for (ln, a, nt), mine in nib.items():
            other = nib[(ln ^ 1, a, nt)]
            byte[(ln, a, nt)] = (other | (mine << 4)) if ln & 1 else (mine | (other << 4))
        for ln in range(0, 32, 4):           # lane q = 0 of each quad stores its row
            words = []
            for a in range(8):
                half = [byte[(ln, a, nt)] | (byte[(ln ^ 2, a, nt)] << 8) for nt in range(2)]
                words.append(half[0] | (half[1] << 16))
            out[(ln >> 2) + 8 * h] = np.frombuffer(np.array(words, np.uint32).tobytes(), np.uint8)
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
        assert not (diff & (margin >= 1e-9)).any()

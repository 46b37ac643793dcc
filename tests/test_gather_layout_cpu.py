"""The 8-lane gather's lane plan, emulated on the CPU.

attend_rows_bf16_g8 gives each bf16 row 8 lanes: lane l is sub-lane sl = l % 8 of group
gq = l / 8 and holds dimensions 16 sl .. 16 sl + 15 of q, K and V.  The warp's rows are
j0, j0 + step, ...; a warp step takes kR = 2 rows per group, group gq taking rows
jb + (4 u + gq) step.  A row's score is the lane's partial dot product summed over the
group's 8 lanes (xor 1, 2, 4), scaled into the log2 domain; each group keeps its own
online softmax (running max m, sum l, 16 accumulators).  At the end the four groups
are merged (xor 8, then xor 16: max of the two maxima, each side rescaled by exp2 of
its distance to it), and lane L takes over dimensions 4 L .. 4 L + 3 from lane
(L / 4) + 8 (L % 4), whose group index picks which quarter of its 16 dimensions it
offers.  This emulates those steps lane by lane and compares the result with a direct
softmax over the same rows."""
import numpy as np


def _emulate(q, K, V, rows, scale_log2):
    n = len(rows)
    kR = 2
    lanes = range(32)
    m = {l: -np.inf for l in lanes}
    s_l = {l: 0.0 for l in lanes}
    acc = {l: np.zeros(16) for l in lanes}
    for jb in range(0, n, 4 * kR):
        # scores: partial dot products, summed over the group's 8 lanes
        s = {}
        for l in lanes:
            gq, sl = l >> 3, l & 7
            for u in range(kR):
                jj = jb + 4 * u + gq
                part = float(q[16 * sl:16 * sl + 16] @ K[rows[jj], 16 * sl:16 * sl + 16]) \
                    if jj < n else 0.0
                s[(l, u)] = part
        for l in lanes:
            gq = l >> 3
            for u in range(kR):
                tot = sum(s[((gq << 3) | t, u)] for t in range(8))
                jj = jb + 4 * u + gq
                s[(l, u, 'full')] = tot * scale_log2 if jj < n else -np.inf
        for l in lanes:
            gq, sl = l >> 3, l & 7
            mx = max([m[l]] + [s[(l, u, 'full')] for u in range(kR)])
            if mx == -np.inf:
                continue
            corr = 2.0 ** (m[l] - mx)
            s_l[l] *= corr
            acc[l] *= corr
            for u in range(kR):
                jj = jb + 4 * u + gq
                if jj < n:
                    p = 2.0 ** (s[(l, u, 'full')] - mx)
                    s_l[l] += p
                    acc[l] += p * V[rows[jj], 16 * sl:16 * sl + 16]
            m[l] = mx
    for o in (8, 16):
        new = {}
        for l in lanes:
            mo, lo, ao = m[l ^ o], s_l[l ^ o], acc[l ^ o]
            M = max(m[l], mo)
            c1 = 0.0 if M == -np.inf else 2.0 ** (m[l] - M)
            c2 = 0.0 if M == -np.inf else 2.0 ** (mo - M)
            new[l] = (M, s_l[l] * c1 + lo * c2, acc[l] * c1 + ao * c2)
        for l in lanes:
            m[l], s_l[l], acc[l] = new[l]
    out = np.zeros(128)
    for L in lanes:
        src = (L >> 2) + 8 * (L & 3)
        gq_src = src >> 3
        out[4 * L:4 * L + 4] = acc[src][4 * gq_src:4 * gq_src + 4] / s_l[src]
    return out


def test_g8_lane_plan_matches_direct_softmax():
    rng = np.random.default_rng(4)
    q = rng.standard_normal(128)
    K = rng.standard_normal((200, 128))
    V = rng.standard_normal((200, 128))
    scale_log2 = 1.0 / np.sqrt(128.0) / np.log(2.0)
    for n in (1, 7, 8, 9, 37, 64):
        rows = rng.choice(200, n, replace=False)
        got = _emulate(q, K, V, rows, scale_log2)
        s = (K[rows] @ q) * scale_log2
        p = 2.0 ** (s - s.max())
        want = (p / p.sum()) @ V[rows]
        assert np.abs(got - want).max() < 1e-12

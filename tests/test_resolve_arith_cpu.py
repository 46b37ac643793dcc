"""The cluster decode kernel's k-th-distance search, emulated on the CPU.

Each CTA of a unit holds the cumulative histogram of its keys' distances (bins 0 .. NB-1,
rows padded to BS bins).  Level 1: every CTA has its peers' cumulative counts at the ends
of 30 coarse chunks of C bins; the first chunk j* whose unit total reaches k_eff holds D*.
Level 2: each CTA pulls a window of FW bins of every peer's cumulative histogram starting
at min(max(0, C j* - 1) rounded down to 4, BS - FW), and scans bins C j* - 1 .. C j* + C - 1
in passes of 32 (carrying the last bin's counts across passes): the first bin whose unit
count reaches k_eff is D*; the bin before it gives the unit's count below D* and the
lower-ranked CTAs' counts below and at D*.  Each CTA then takes all its keys below D* and
the ties at D* that the unit still needs after the lower-ranked CTAs' ties.  This restates
those steps and checks them against a direct sort, for per-head selection (385 bins) and
shared selection (384 G + 1 bins), with ties spread across CTAs."""
import numpy as np

NCOARSE = 30


def _geometry(nb):
    bs = (nb + 3) // 4 * 4
    c = (nb + NCOARSE - 1) // NCOARSE
    fw = (c + 4 + 3) // 4 * 4
    return bs, c, fw


def _resolve(cum, k, nb):
    """cum: [CS][BS] inclusive cumulative histograms; returns per-CTA (dstar, base, take,
    nsel) as the kernel computes them."""
    cs = len(cum)
    bs, c, fw = _geometry(nb)
    coarse = [[cum[cc][min(c * j + c - 1, nb - 1)] for j in range(NCOARSE)] for cc in range(cs)]
    s1 = [sum(coarse[cc][j] for cc in range(cs)) for j in range(NCOARSE)]
    jstar = next(j for j in range(NCOARSE) if s1[j] >= k)
    lo_bin = min(max(0, c * jstar - 1) & ~3, bs - fw)
    fine = [cum[cc][lo_bin:lo_bin + fw] for cc in range(cs)]
    out = []
    for rank in range(cs):
        dstar, less, lt_before, eq_before = -1, 0, 0, 0
        carry2 = carryb = 0
        base = 0
        while base < c + 1 and dstar < 0:
            S2, Sb = [], []
            for lane in range(32):
                l = base + lane
                d = c * jstar - 1 + l
                s2 = sb = 0
                if l < c + 1 and d >= 0:
                    off = min(d, nb - 1) - lo_bin
                    assert 0 <= off < fw
                    for cc in range(cs):
                        s2 += fine[cc][off]
                        if cc < rank:
                            sb += fine[cc][off]
                S2.append(s2)
                Sb.append(sb)
            hits = [lane for lane in range(32)
                    if base + lane >= 1 and base + lane < c + 1 and S2[lane] >= k]
            p2 = [carry2] + S2[:31]
            pb = [carryb] + Sb[:31]
            if hits:
                ls = hits[0]
                dstar = c * jstar - 1 + base + ls
                less, lt_before = p2[ls], pb[ls]
                eq_before = Sb[ls] - lt_before
            carry2, carryb = S2[31], Sb[31]
            base += 32
        assert dstar >= 0
        own = cum[rank]
        lt_own = own[dstar - 1] if dstar > 0 else 0
        eq_own = own[dstar] - lt_own
        need = k - less
        b = lt_before + min(eq_before, need)
        take = min(need - eq_before, eq_own) if need > eq_before else 0
        out.append((dstar, b, take, lt_own + take))
    return out


def _check(dists_per_cta, k, nb):
    bs, _, _ = _geometry(nb)
    cum = []
    for d in dists_per_cta:
        h = np.bincount(np.asarray(d, int), minlength=bs)[:bs]
        cum.append(np.cumsum(h).tolist())
    allv = np.concatenate([np.asarray(d, int) for d in dists_per_cta])
    keff = min(k, len(allv))
    res = _resolve(cum, keff, nb)
    # direct: the first keff keys by (distance, position); positions are CTA-major
    order = np.lexsort((np.arange(len(allv)), allv))[:keff]
    want_dstar = int(allv[order[-1]])
    sizes = [len(d) for d in dists_per_cta]
    starts = np.concatenate([[0], np.cumsum(sizes)[:-1]])
    taken = np.zeros(len(allv), bool)
    taken[order] = True
    prefix = 0
    for r, (dstar, base, take, nsel) in enumerate(res):
        assert dstar == want_dstar
        n_r = int(taken[starts[r]:starts[r] + sizes[r]].sum())
        assert nsel == n_r and base == prefix
        prefix += n_r
    assert prefix == keff


def test_resolve_per_head_geometry():
    rng = np.random.default_rng(0)
    for _ in range(60):
        cs = int(rng.integers(1, 11))
        mean = rng.integers(0, 385)
        d = [np.clip(rng.normal(mean, rng.integers(1, 40), int(rng.integers(1, 400))), 0, 384)
             .astype(int) for _ in range(cs)]
        total = sum(len(x) for x in d)
        for k in {1, 2, int(rng.integers(1, total + 1)), total, total + 5}:
            _check(d, k, 385)


def test_resolve_ties_across_ctas_and_chunk_edges():
    for value in (0, 12, 13, 25, 26, 376, 377, 384):
        d = [[value] * 50, [value] * 7, [max(0, value - 1)] * 3 + [value] * 20]
        for k in (1, 3, 4, 30, 60, 80):
            _check(d, k, 385)


def test_resolve_shared_geometry():
    rng = np.random.default_rng(1)
    for g in (2, 4, 8):
        nb = 384 * g + 1
        for _ in range(20):
            cs = int(rng.integers(1, 9))
            d = [rng.integers(0, nb, int(rng.integers(1, 300))) for _ in range(cs)]
            total = sum(len(x) for x in d)
            for k in {1, int(rng.integers(1, total + 1)), total}:
                _check(d, k, nb)

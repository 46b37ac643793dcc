"""The grid-wide decode kernel's k-th-distance search, emulated on the CPU.

Each of a unit's S CTAs publishes its cumulative distance counts as 16-bit values over
392 bins (bins past 384 hold its total).  A CTA guesses D* from its own counts scaled to
the unit (the first bin where count x L / n reaches k_eff) and reads a 64-bin window of
every CTA's row starting at a multiple of 8 no higher than 24 bins below the guess.  If
the unit's count at the window's first bin already reaches k_eff (and the window does not
start at 0), or its count at the last bin does not, the window moves down or up by 56
bins; otherwise the first bin reaching k_eff is D*, the bin before it gives the unit's
count below D*, and the lower-ranked CTAs' counts below and at D* give this CTA's base and
tie share.  This restates those steps and checks them against a direct sort, including
skewed CTAs whose own guess lies far from D*."""
import numpy as np

NBINS, ROW, WIN = 385, 392, 64


def _rows(dists):
    rows = []
    for d in dists:
        h = np.bincount(np.asarray(d, int), minlength=NBINS)[:NBINS]
        cum = np.cumsum(h)
        rows.append(np.concatenate([cum, np.full(ROW - NBINS, cum[-1])]).astype(np.int64))
    return rows


def _resolve(rows, rank, keff, L):
    own = rows[rank]
    n = max(int(own[NBINS - 1]), 1)
    scaled = own[:NBINS] * L
    hits = np.nonzero(scaled >= keff * n)[0]
    est = min(int(hits[0]) if len(hits) else 1 << 30, NBINS - 1)
    wlo = min(max(0, (est - 24) & ~7), ROW - WIN)
    for _ in range(17):
        C = sum(r[wlo:wlo + WIN] for r in rows)
        B = sum((r[wlo:wlo + WIN] for r in rows[:rank]), np.zeros(WIN, np.int64))
        assert ROW - WIN >= wlo >= 0 and wlo % 8 == 0
        if wlo > 0 and C[0] >= keff:
            wlo = max(0, wlo - (WIN - 8))
            continue
        if C[WIN - 1] < keff:
            wlo = min(ROW - WIN, wlo + (WIN - 8))
            continue
        off = int(np.nonzero(C >= keff)[0][0])
        dstar = wlo + off
        less = int(C[off - 1]) if off > 0 else 0
        lt_before = int(B[off - 1]) if off > 0 else 0
        eq_before = int(B[off]) - lt_before
        dcl = min(dstar, NBINS - 1)
        lt_own = int(own[dcl - 1]) if dcl > 0 else 0
        eq_own = int(own[dcl]) - lt_own
        need = keff - less
        base = lt_before + min(eq_before, need)
        take = min(need - eq_before, eq_own) if need > eq_before else 0
        return dcl, base, lt_own + take
    raise AssertionError("window search did not settle")


def _check(dists, k):
    rows = _rows(dists)
    allv = np.concatenate([np.asarray(d, int) for d in dists])
    L = len(allv)
    keff = min(k, L)
    order = np.lexsort((np.arange(L), allv))[:keff]
    taken = np.zeros(L, bool)
    taken[order] = True
    want = int(allv[order[-1]])
    start = 0
    prefix = 0
    for rank, d in enumerate(dists):
        dstar, base, nsel = _resolve(rows, rank, keff, L)
        assert dstar == want
        n_r = int(taken[start:start + len(d)].sum())
        assert nsel == n_r and base == prefix
        prefix += n_r
        start += len(d)
    assert prefix == keff


def test_flat_resolve_random_units():
    rng = np.random.default_rng(3)
    for _ in range(80):
        s = int(rng.integers(1, 20))
        mean = int(rng.integers(0, 385))
        dists = [np.clip(rng.normal(mean, rng.integers(1, 60), int(rng.integers(1, 600))), 0, 384)
                 .astype(int) for _ in range(s)]
        total = sum(len(d) for d in dists)
        for k in {1, int(rng.integers(1, total + 1)), total, total + 3}:
            _check(dists, k)


def test_flat_resolve_skewed_ctas_move_their_windows():
    # CTA 0 holds only far distances, CTA 1 only near ones: CTA 0's own guess is far above
    # D*, and a CTA holding only low distances guesses far below it at large budgets
    rng = np.random.default_rng(5)
    dists = [rng.integers(300, 385, 500), rng.integers(0, 20, 500), rng.integers(150, 200, 500)]
    for k in (1, 10, 499, 500, 501, 900, 1200, 1500):
        _check(dists, k)
    ties = [np.full(300, 200), np.full(5, 200), np.concatenate([np.full(10, 199), np.full(40, 200)])]
    for k in (1, 9, 10, 11, 100, 355):
        _check(ties, k)

"""The cluster kernel's select pass, emulated on the CPU: which positions a CTA emits
and where each lands in its list.

Per round of 512 x 32 positions, thread t owns `per` consecutive positions (per = the
round's positions per thread rounded up to a multiple of 8).  It builds "< D*" and "= D*"
bit masks, a block-wide exclusive scan of its two counts (plus the carries of earlier
rounds) gives the selections before it, it keeps the lowest (take - ties before it) of its
tie bits, and emits its selected positions in bit order starting at rank
(less-than before it) + min(ties before it, take).  This restates those steps and checks
that a CTA's list is exactly its positions below D* plus its first `take` ties at D*, in
ascending position order."""
import numpy as np

THREADS = 512
ROUND = THREADS * 32


def _select(d, dstar, take):
    n = len(d)
    out = {}
    carry_lt = carry_eq = 0
    for rb in range(0, n, ROUND):
        nr = min(ROUND, n - rb)
        per = ((nr + THREADS - 1) // THREADS + 7) & ~7
        ltm, eqm, cnt_lt, cnt_eq = [], [], [], []
        for t in range(THREADS):
            s0 = rb + t * per
            cntv = max(0, min(per, rb + nr - s0))
            lt = sum(1 << i for i in range(cntv) if d[s0 + i] < dstar)
            eq = sum(1 << i for i in range(cntv) if d[s0 + i] == dstar)
            ltm.append(lt)
            eqm.append(eq)
            cnt_lt.append(bin(lt).count("1"))
            cnt_eq.append(bin(eq).count("1"))
        ex_lt = np.concatenate([[0], np.cumsum(cnt_lt)[:-1]])
        ex_eq = np.concatenate([[0], np.cumsum(cnt_eq)[:-1]])
        for t in range(THREADS):
            lt_b = carry_lt + int(ex_lt[t])
            eq_b = carry_eq + int(ex_eq[t])
            rest = eqm[t]
            te = take - eq_b
            c = 0
            while c < te and rest:
                rest &= rest - 1
                c += 1
            sel = ltm[t] | (eqm[t] ^ rest if te > 0 else 0)
            rk = lt_b + min(eq_b, take)
            i = 0
            while sel:
                if sel & 1:
                    assert rk not in out
                    out[rk] = rb + t * per + i
                    rk += 1
                sel >>= 1
                i += 1
        carry_lt += sum(cnt_lt)
        carry_eq += sum(cnt_eq)
    return [out[r] for r in range(len(out))]


def test_select_emits_ascending_positions_with_first_ties():
    rng = np.random.default_rng(9)
    for n in (1, 7, 513, 3277, 16384, 16385, 40000):
        d = rng.integers(0, 40, n)
        for dstar in (0, 5, 20, 39):
            eq_total = int((d == dstar).sum())
            for take in sorted({0, 1, eq_total // 2, eq_total}):
                got = _select(d, dstar, take)
                ties = np.nonzero(d == dstar)[0][:take]
                want = np.sort(np.concatenate([np.nonzero(d < dstar)[0], ties]))
                assert got == want.tolist()

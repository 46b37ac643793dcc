"""Distance scan + top-k on the GPU fed the ORACLE's codes: indices bit-exact.

Cases span several CTAs, ragged tails, units straddling CTA ranges, several waves,
every supported GQA group size, ties, k >= L, L = 1 and the full 32K / 128K
workloads at every budget; most run on both decode kernels (thread-block clusters
and the grid-wide kernel)."""
import numpy as np
import pytest
import torch

import oracle
import token_level_sparse_fwht_b200 as ad
from gpu_helpers import f64, oracle_codes, upload
from workloads import WORKLOADS, generate

pytestmark = pytest.mark.gpu


def _oracle_select(qc, kc, k, G):
    """qc [B,Hq,32], kc [B,Hkv,L,32] packed -> idx [B,Hq,k_eff]."""
    B, Hq, _ = qc.shape
    uq = oracle.unpack_codes(qc)
    uk = oracle.unpack_codes(kc)
    out = []
    for b in range(B):
        rows = []
        for h in range(Hq):
            d = oracle.manhattan(uq[b, h], uk[b, h // G])
            rows.append(oracle.select_topk(d, k))
        out.append(rows)
    return np.array(out)


def _run(qc, kc, L, k, Lmax=None):
    B, Hq, _ = qc.shape
    _, Hkv, Lc, _ = kc.shape
    codes = upload(kc)
    ws = ad.decode_workspace(B, Hq, Hkv, L, k)
    idx = ad.select_topk(upload(qc), codes, L, k, ws)
    torch.cuda.synchronize()
    ad.check_workspace(ws)
    return idx.cpu().numpy(), ws


def _random_codes(rng, *shape):
    return rng.integers(0, 256, size=shape, dtype=np.uint8)


@pytest.mark.parametrize("B,Hq,Hkv,L,k", [
    (1, 1, 1, 1024, 64),        # single head, 4 CTAs
    (1, 32, 8, 3001, 128),      # ragged, units straddle CTAs
    (2, 8, 2, 5000, 256),
    (1, 4, 4, 1, 1),            # L = 1
    (3, 4, 4, 100, 7),          # L < a CTA's minimum range
    (1, 8, 1, 2048, 100),       # G = 8
    (2, 4, 2, 999, 999),        # k = L
    (2, 4, 2, 333, 5000),       # k > L
    (75, 4, 4, 64, 8),          # 300 units: three waves
    (1, 2, 1, 70000, 50),       # one unit over all CTAs
])
def test_select_random_codes(B, Hq, Hkv, L, k, decode_policy):
    rng = np.random.default_rng(B * 1000 + L)
    qc = _random_codes(rng, B, Hq, 32)
    kc = _random_codes(rng, B, Hkv, L, 32)
    got, _ = _run(qc, kc, L, k)
    want = _oracle_select(qc, kc, k, Hq // Hkv)
    assert got.shape == want.shape
    assert np.array_equal(got, want)


def test_select_all_ties_take_lowest_positions(decode_policy):
    B, Hq, Hkv, L, k = 2, 8, 2, 4000, 300
    qc = np.zeros((B, Hq, 32), np.uint8)
    kc = np.full((B, Hkv, L, 32), 0x55, np.uint8)
    got, _ = _run(qc, kc, L, k)
    assert np.array_equal(got, np.broadcast_to(np.arange(k), (B, Hq, k)))


def test_select_few_distinct_distances(decode_policy):
    """Codes drawn from 2 values: huge tie groups at the k-th distance across CTAs."""
    rng = np.random.default_rng(5)
    B, Hq, Hkv, L, k = 1, 4, 4, 20000, 777
    qc = np.zeros((B, Hq, 32), np.uint8)
    kc = np.where(rng.random((B, Hkv, L, 1)) < 0.3, 0x01, 0x00).astype(np.uint8)
    kc = np.broadcast_to(kc, (B, Hkv, L, 32)).copy()
    got, _ = _run(qc, kc, L, k)
    assert np.array_equal(got, _oracle_select(qc, kc, k, 1))


def test_select_lmax_padding_and_workspace_reuse(decode_policy):
    """Lmax > L: only the first L positions count; a second call on the same
    workspace returns the same indices."""
    rng = np.random.default_rng(9)
    B, Hq, Hkv, L, Lmax, k = 2, 8, 2, 3000, 4096, 64
    qc = _random_codes(rng, B, Hq, 32)
    kc = _random_codes(rng, B, Hkv, Lmax, 32)
    codes = upload(kc)
    ws = ad.decode_workspace(B, Hq, Hkv, L, k)
    a = ad.select_topk(upload(qc), codes, L, k, ws).cpu().numpy()
    b = ad.select_topk(upload(qc), codes, L, k, ws).cpu().numpy()
    assert np.array_equal(a, b)
    assert np.array_equal(a, _oracle_select(qc, kc[:, :, :L], k, Hq // Hkv))
    # the error word is clear (clusters keep everything else on chip; the grid-wide
    # kernel's exchange words are back at zero after each launch)
    assert int(ws.view(torch.int32)[2]) == 0
    if ws.numel() > 256:
        sync = ws[256:256 + 16 * B * Hkv].view(torch.int32).view(B * Hkv, 4)
        assert int(sync[:, 0].abs().sum()) == 0 and int(sync[:, 2].abs().sum()) == 0


@pytest.mark.parametrize("cfg", [1, 2])
def test_select_workload_oracle_codes(cfg, decode_policy):
    """Seeded workloads (single head 1K; Llama-3.1-8B layer 32K) at every budget, the
    oracle's own codes of the generated q and K."""
    w = WORKLOADS[cfg]
    inp = generate(w, "cuda" if cfg > 1 else "cpu")
    qc = oracle_codes(inp.q, inp.t)
    kc = oracle_codes(inp.k_cache, inp.t)
    for k in w.budgets:
        got, _ = _run(qc, kc, w.L, k)
        assert np.array_equal(got, _oracle_select(qc, kc, k, w.G)), k


@pytest.mark.slow
def test_select_128k_mha_sampled_heads():
    """MHA 32 x 128K with 16 needles per head: all heads scanned on the GPU, 4 heads
    checked against the oracle at both budgets; the needles are recalled."""
    w = WORKLOADS[4]
    inp = generate(w, "cuda")
    qc = oracle_codes(inp.q, inp.t)
    heads = [0, 9, 22, 31]
    kc_full = np.zeros((1, w.Hkv, w.L, 32), np.uint8)
    for h in range(w.Hkv):
        kc_full[0, h] = oracle_codes(inp.k_cache[0, h].cpu(), inp.t)
    for k in w.budgets:
        got, _ = _run(qc, kc_full, w.L, k)
        for h in heads:
            d = oracle.manhattan(oracle.unpack_codes(qc[0, h]), oracle.unpack_codes(kc_full[0, h]))
            assert np.array_equal(got[0, h], oracle.select_topk(d, k)), (k, h)
        planted = inp.planted[0].cpu().numpy()
        recall = np.mean([np.isin(planted[h], got[0, h]).mean() for h in range(w.Hq)])
        assert recall > 0.9, recall

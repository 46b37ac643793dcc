"""Split-k gather attention on the GPU vs the oracle's float64 softmax attention
over the same positions (max-abs error <= 2e-3)."""
import numpy as np
import pytest
import torch

import oracle
import token_level_sparse_fwht_b200 as ad
from gpu_helpers import ATOL_OUT, f64, upload
from workloads import WORKLOADS, generate

pytestmark = pytest.mark.gpu


def _oracle_attn(q, K, V, idx, G):
    B, Hq, _ = q.shape
    out = np.zeros((B, Hq, 128))
    for b in range(B):
        for h in range(Hq):
            out[b, h] = oracle.sparse_attention(q[b, h], K[b, h // G], V[b, h // G], idx[b, h])
    return out


@pytest.mark.parametrize("cfg,L,k", [(1, 1024, 64), (2, 4000, 128), (2, 4000, 1024),
                                     (3, 600, 256), (4, 900, 17)])
def test_attention_random_positions(cfg, L, k):
    w = WORKLOADS[cfg].scaled(L=L, B=min(WORKLOADS[cfg].B, 2))
    inp = generate(w, "cpu")
    rng = np.random.default_rng(L + k)
    k_eff = min(k, L)
    idx = np.stack([np.stack([np.sort(rng.choice(L, k_eff, replace=False))
                              for _ in range(w.Hq)]) for _ in range(w.B)]).astype(np.int32)
    got = ad.sparse_attention(inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(),
                              upload(idx)).cpu().numpy()
    want = _oracle_attn(f64(inp.q), f64(inp.k_cache), f64(inp.v_cache), idx, w.G)
    assert np.abs(got - want).max() <= ATOL_OUT


def test_attention_budget_L_is_dense():
    """All L positions: the result is textbook dense attention (torch, float64)."""
    w = WORKLOADS[2].scaled(L=2500, Hq=8, Hkv=2)
    inp = generate(w, "cpu")
    idx = np.broadcast_to(np.arange(w.L, dtype=np.int32), (1, w.Hq, w.L)).copy()
    got = ad.sparse_attention(inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(),
                              upload(idx)).cpu().numpy()
    q = inp.q.double()[:, :, None, :]
    K = inp.k_cache.double().repeat_interleave(w.G, dim=1)
    V = inp.v_cache.double().repeat_interleave(w.G, dim=1)
    dense = torch.nn.functional.scaled_dot_product_attention(q, K, V)[:, :, 0].numpy()
    assert np.abs(got - dense).max() <= ATOL_OUT


def test_attention_budget_one_is_the_v_row():
    w = WORKLOADS[2].scaled(L=300, Hq=4, Hkv=4)
    inp = generate(w, "cpu")
    idx = np.array([[[7], [299], [0], [150]]], dtype=np.int32)
    got = ad.sparse_attention(inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(),
                              upload(idx)).cpu().numpy()
    want = np.stack([f64(inp.v_cache[0, h, idx[0, h, 0]]) for h in range(4)])[None]
    assert np.array_equal(got, want.astype(np.float32))


def test_attention_workspace_reuse():
    w = WORKLOADS[2].scaled(L=1000, Hq=8, Hkv=2)
    inp = generate(w, "cpu")
    rng = np.random.default_rng(1)
    idx = upload(np.sort(rng.choice(1000, (1, 8, 200)), -1).astype(np.int32))
    ws = ad.sparse_attention_workspace(1, 8, 200)
    a = ad.sparse_attention(inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(), idx, ws)
    b = ad.sparse_attention(inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(), idx, ws)
    assert torch.equal(a, b)
    assert int(ws.view(torch.int32)[:8].abs().sum()) == 0


def test_attention_repeated_unsorted_positions():
    """Positions in any order and repeated: each copy is its own softmax term, as in
    the oracle's K[idx] gather."""
    w = WORKLOADS[2].scaled(L=700, Hq=8, Hkv=2)
    inp = generate(w, "cpu")
    rng = np.random.default_rng(11)
    idx = rng.integers(0, 40, size=(1, 8, 300)).astype(np.int32)   # many repeats
    idx[0, 3] = 5                                                  # one row, 300 copies
    got = ad.sparse_attention(inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(),
                              upload(idx)).cpu().numpy()
    want = _oracle_attn(f64(inp.q), f64(inp.k_cache), f64(inp.v_cache), idx, w.G)
    assert np.abs(got - want).max() <= ATOL_OUT

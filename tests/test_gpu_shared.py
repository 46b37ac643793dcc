"""Shared GQA selection on the GPU vs the oracle's decode_step_shared.

One selection per (batch, kv head) over the sum of the group's Manhattan
distances (0 .. 384 G), shared by the G query heads.  Fed the oracle's codes the
indices are bit-exact; in the fused step the kernel encodes the queries itself, so
a query coordinate within 1e-4 of a threshold may take either bucket: the
selection must equal the oracle's for one admissible combination of the group's
query codes, and the output must be within 2e-3 of the oracle's attention."""
import itertools

import numpy as np
import pytest
import torch

import oracle
import token_level_sparse_fwht_b200 as ad
from gpu_helpers import (ATOL_OUT, check_decode_unit_shared as _check_unit, f64,
                         oracle_codes, query_alternatives, upload)
from workloads import WORKLOADS, generate

pytestmark = pytest.mark.gpu


def _oracle_select_shared(qc, kc, k):
    """Selection of oracle.decode_step_shared from packed codes (the attention part
    runs on zero-filled q/K/V and is ignored)."""
    B, Hq, _ = qc.shape
    _, Hkv, L, _ = kc.shape
    zq = np.zeros((B, Hq, 128))
    zkv = np.broadcast_to(np.zeros(1), (B, Hkv, L, 128))
    idx, _ = oracle.decode_step_shared(zq, zkv, zkv, k, 1.0, key_codes=kc, query_codes=qc)
    return idx


def _select(qc, kc, L, k):
    B, Hq, _ = qc.shape
    _, Hkv, _, _ = kc.shape
    ws = ad.decode_workspace(B, Hq, Hkv, L, k)
    idx = ad.select_topk_shared(upload(qc), upload(kc), L, k, ws)
    torch.cuda.synchronize()
    ad.check_workspace(ws)
    return idx.cpu().numpy()


@pytest.mark.parametrize("B,Hq,Hkv,L,k", [
    (1, 1, 1, 1024, 64),        # G = 1: the per-head selection
    (1, 32, 8, 3001, 128),      # G = 4, ragged, units straddle CTAs
    (2, 8, 4, 5000, 256),       # G = 2
    (1, 8, 1, 2048, 100),       # G = 8: 3073 bins
    (1, 16, 2, 70000, 50),      # G = 8, one unit over all CTAs
    (2, 4, 2, 333, 5000),       # k > L
    (2, 8, 2, 999, 999),        # k = L
    (3, 8, 2, 1, 1),            # L = 1
    (70, 8, 2, 64, 8),          # 140 units: waves
])
def test_select_shared_random_codes(B, Hq, Hkv, L, k):
    rng = np.random.default_rng(7 * B + L)
    qc = rng.integers(0, 256, size=(B, Hq, 32), dtype=np.uint8)
    kc = rng.integers(0, 256, size=(B, Hkv, L, 32), dtype=np.uint8)
    got = _select(qc, kc, L, k)
    want = _oracle_select_shared(qc, kc, k)
    assert got.shape == want.shape == (B, Hkv, min(k, L))
    assert np.array_equal(got, want)


def test_select_shared_ties_across_ctas():
    """Two key codes only: every summed score is one of two values, so the k-th
    score is a huge tie group spread over all CTAs; ties go to lower positions."""
    rng = np.random.default_rng(11)
    B, Hq, Hkv, L, k = 1, 16, 2, 20000, 777
    qc = rng.integers(0, 256, size=(B, Hq, 32), dtype=np.uint8)
    pick = rng.random((B, Hkv, L, 1)) < 0.3
    kc = np.where(pick, np.uint8(0x1b), np.uint8(0xe4)).astype(np.uint8)
    kc = np.broadcast_to(kc, (B, Hkv, L, 32)).copy()
    got = _select(qc, kc, L, k)
    assert np.array_equal(got, _oracle_select_shared(qc, kc, k))


def test_select_shared_extreme_scores():
    """Scores at both ends of 0 .. 384 G: keys equal to or opposite every query."""
    B, Hq, Hkv, L, k = 1, 8, 1, 3000, 1500
    qc = np.zeros((B, Hq, 32), np.uint8)                  # every coordinate bucket 0
    kc = np.full((B, Hkv, L, 32), 0xff, np.uint8)        # bucket 3: distance 384 per head
    kc[0, 0, ::7] = 0                                     # distance 0
    got = _select(qc, kc, L, k)
    assert np.array_equal(got, _oracle_select_shared(qc, kc, k))


def test_select_shared_g1_equals_per_head():
    rng = np.random.default_rng(3)
    B, Hq, Hkv, L, k = 2, 4, 4, 4000, 200
    qc = rng.integers(0, 256, size=(B, Hq, 32), dtype=np.uint8)
    kc = rng.integers(0, 256, size=(B, Hkv, L, 32), dtype=np.uint8)
    ws = ad.decode_workspace(B, Hq, Hkv, L, k)
    per_head = ad.select_topk(upload(qc), upload(kc), L, k, ws).cpu().numpy()
    assert np.array_equal(_select(qc, kc, L, k), per_head)


def _decode_shared(inp, kc, L, k):
    B, Hq, _ = inp.q.shape
    _, Hkv, _, _ = inp.k_cache.shape
    ws = ad.decode_workspace(B, Hq, Hkv, L, k)
    idx = torch.full((B, Hkv, min(k, L)), -1, dtype=torch.int32, device="cuda")
    out = ad.decode_step_shared(inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(), upload(kc),
                                L, k, inp.t, ws, idx_out=idx)
    torch.cuda.synchronize()
    ad.check_workspace(ws)
    return idx.cpu().numpy(), out.cpu().numpy()


@pytest.mark.parametrize("cfg,over,k", [
    (1, {}, 64),                                   # single head, fp32
    (2, dict(L=3001), 128),                        # G = 4
    (2, dict(L=3001), 1024),
    (3, dict(B=3, L=2500), 256),                   # B = 3
    (2, dict(L=5000, Hq=16, Hkv=2), 64),           # G = 8
    (2, dict(L=4000, Hq=8, Hkv=4), 300),           # G = 2
    (2, dict(L=777, Hq=4, Hkv=2), 2000),           # k > L: dense
    (2, dict(B=70, Hq=4, Hkv=2, L=64), 5),         # 140 units: waves
])
def test_decode_shared_matches_oracle(cfg, over, k):
    w = WORKLOADS[cfg].scaled(**over)
    inp = generate(w, "cpu")
    kc = oracle_codes(inp.k_cache, inp.t)
    idx, out = _decode_shared(inp, kc, w.L, k)
    q, K, V = f64(inp.q), f64(inp.k_cache), f64(inp.v_cache)
    G = w.G
    worst = 0.0
    for b in range(w.B):
        for kvh in range(w.Hkv):
            hs = slice(kvh * G, (kvh + 1) * G)
            worst = max(worst, _check_unit(idx[b, kvh], out[b, hs], q[b, hs], K[b, kvh, :w.L],
                                           V[b, kvh, :w.L], kc[b, kvh, :w.L], k, inp.t))
    assert worst <= ATOL_OUT


def test_decode_shared_full_32k_sampled_units():
    """The Llama-3.1-8B layer at 32K, budget 128, in the launch configuration the
    benchmark times: every unit computed on the GPU, three checked in full."""
    w = WORKLOADS[2]
    inp = generate(w, "cpu")
    kc = oracle_codes(inp.k_cache, inp.t)
    idx, out = _decode_shared(inp, kc, w.L, 128)
    q = f64(inp.q)
    G = w.G
    for kvh in (0, 3, 7):
        hs = slice(kvh * G, (kvh + 1) * G)
        err = _check_unit(idx[0, kvh], out[0, hs], q[0, hs], f64(inp.k_cache[0, kvh]),
                          f64(inp.v_cache[0, kvh]), kc[0, kvh], 128, inp.t)
        assert err <= ATOL_OUT


def test_decode_shared_host_buffers_match_device_call():
    w = WORKLOADS[2].scaled(L=4096)
    inp = generate(w, "cpu")
    kc = upload(oracle_codes(inp.k_cache, inp.t))
    kcache, vcache = inp.k_cache.cuda(), inp.v_cache.cuda()
    ws = ad.decode_workspace(w.B, w.Hq, w.Hkv, w.L, 128)
    want = ad.decode_step_shared(inp.q.cuda(), kcache, vcache, kc, w.L, 128, inp.t, ws)
    q_host = inp.q.clone().pin_memory()
    out_host = torch.empty((w.B, w.Hq, 128), dtype=torch.float32).pin_memory()
    q_dev = torch.empty_like(inp.q, device="cuda")
    out_dev = torch.empty((w.B, w.Hq, 128), dtype=torch.float32, device="cuda")
    step = ad.PreparedDecodeHost(q_host, q_dev, kcache, vcache, kc, w.L, 128, inp.t, ws, out_dev,
                                 out_host, shared=True)
    step()
    torch.cuda.synchronize()
    ad.check_workspace(ws)
    assert torch.equal(out_host, want.cpu())
    out_host2 = torch.empty((w.B, w.Hq, 128), dtype=torch.float32)   # pageable: staged copies
    ad.decode_step_shared_host(inp.q.clone(), q_dev, kcache, vcache, kc, w.L, 128, inp.t, ws,
                               out_dev, out_host2)
    torch.cuda.synchronize()
    assert torch.equal(out_host2, want.cpu())

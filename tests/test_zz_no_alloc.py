"""The allocation-free attention entry point (adamas_sparse_attention_noalloc).

It serves callers that cannot allocate device memory themselves, so its scratch
is a fixed array inside the library.  Checked through the C ABI against
adamas_sparse_attention (which takes a caller workspace): two calls in a row must
each match it within the attention tolerance, and oversized calls are refused.  It is
also checked against the float64 oracle's sparse attention for bf16 and fp32 caches,
and at the largest head count it accepts (B * Hq = 4096; on a 148-SM B200 the split
count there is 1, so the scratch's split cap of B * Hq * splits <= 4096 holds without
reducing anything: it only binds on devices with far more SMs).
This file is collected last, so a stop-at-first-failure run has already run
every other test; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

import oracle
import token_level_sparse_fwht_b200 as ad
from gpu_helpers import ATOL_OUT, f64
from workloads import WORKLOADS, generate

pytestmark = pytest.mark.gpu


def _inputs(B, Hq, Hkv, L, k_eff, seed, cfg=2):
    w = WORKLOADS[cfg].scaled(B=B, Hq=Hq, Hkv=Hkv, L=L)
    inp = generate(w, "cpu")
    rng = np.random.default_rng(seed)
    idx = np.stack([np.stack([np.sort(rng.choice(L, k_eff, replace=False)) for _ in range(Hq)])
                    for _ in range(B)]).astype(np.int32)
    return (inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(),
            torch.from_numpy(idx).cuda())


def _call(q, kc, vc, idx, out):
    B, Hq, d = q.shape
    _, Hkv, Lmax, _ = kc.shape
    dt = ad.BF16 if kc.dtype == torch.bfloat16 else ad.F32
    return ad.lib().adamas_sparse_attention_noalloc(
        q.data_ptr(), kc.data_ptr(), vc.data_ptr(), dt, idx.data_ptr(), B, Hq, Hkv, d, Lmax,
        idx.shape[-1], out.data_ptr(), torch.cuda.current_stream().cuda_stream)


def _oracle_heads(q, kc, vc, idx, heads):
    """The float64 oracle's sparse attention for (batch, head) pairs."""
    G = q.shape[1] // kc.shape[1]
    out = {}
    for b, h in heads:
        sel = idx[b, h].cpu().numpy().astype(np.int64)
        out[(b, h)] = oracle.sparse_attention(f64(q[b, h]), f64(kc[b, h // G]),
                                              f64(vc[b, h // G]), sel)
    return out


def test_noalloc_matches_workspace_entry_point_twice():
    q, kc, vc, idx = _inputs(2, 32, 8, 3000, 128, seed=1)
    want = ad.sparse_attention(q, kc, vc, idx)
    for _ in range(2):
        out = torch.full_like(want, float("nan"))
        assert _call(q, kc, vc, idx, out) == ad.OK
        torch.cuda.synchronize()
        assert torch.isfinite(out).all()
        assert float((out - want).abs().max()) <= ATOL_OUT


def test_noalloc_second_shape_and_limit():
    q, kc, vc, idx = _inputs(1, 8, 2, 1000, 1000, seed=2)   # dense: every position
    want = ad.sparse_attention(q, kc, vc, idx)
    got = ad.sparse_attention_noalloc(q, kc, vc, idx)
    torch.cuda.synchronize()
    assert float((got - want).abs().max()) <= ATOL_OUT
    # B * Hq above the fixed scratch is refused before any launch
    big_q = torch.zeros((129, 32, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((129, 32, 128), dtype=torch.float32, device="cuda")
    small_idx = torch.zeros((129, 32, 1), dtype=torch.int32, device="cuda")
    assert ad.lib().adamas_sparse_attention_noalloc(
        big_q.data_ptr(), kc.data_ptr(), vc.data_ptr(), ad.BF16, small_idx.data_ptr(), 129, 32,
        8, 128, kc.shape[2], 1, out.data_ptr(), None) == ad.ERR_UNSUPPORTED


@pytest.mark.parametrize("cfg", [1, 2])
def test_noalloc_matches_oracle_bf16_and_fp32(cfg):
    """Config 1 holds fp32 caches (one head), config 2 bf16 (GQA 32 / 8)."""
    if cfg == 1:
        q, kc, vc, idx = _inputs(1, 1, 1, 1024, 64, seed=3, cfg=1)
    else:
        q, kc, vc, idx = _inputs(1, 32, 8, 2000, 128, seed=4)
    out = torch.full((q.shape[0], q.shape[1], 128), float("nan"), device="cuda")
    assert _call(q, kc, vc, idx, out) == ad.OK
    torch.cuda.synchronize()
    heads = [(0, h) for h in range(q.shape[1])]
    want = _oracle_heads(q, kc, vc, idx, heads)
    got = out.cpu().numpy()
    for b, h in heads:
        assert np.abs(got[b, h] - want[(b, h)]).max() <= ATOL_OUT, (b, h)


def test_noalloc_largest_head_count_matches_oracle():
    """B * Hq = 4096 heads (the limit), 1024 positions each: sampled heads against the
    oracle, and the whole output against the workspace entry point."""
    q, kc, vc, idx = _inputs(128, 32, 8, 1024, 1024, seed=5)
    out = torch.full((128, 32, 128), float("nan"), device="cuda")
    assert _call(q, kc, vc, idx, out) == ad.OK
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    want_ws = ad.sparse_attention(q, kc, vc, idx)
    torch.cuda.synchronize()
    assert float((out - want_ws).abs().max()) <= ATOL_OUT
    heads = [(0, 0), (17, 5), (64, 31), (127, 12)]
    want = _oracle_heads(q, kc, vc, idx, heads)
    got = out.cpu().numpy()
    for b, h in heads:
        assert np.abs(got[b, h] - want[(b, h)]).max() <= ATOL_OUT, (b, h)

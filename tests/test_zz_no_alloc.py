"""The allocation-free attention entry point (adamas_sparse_attention_noalloc).

It serves callers that cannot allocate device memory themselves, so its scratch
is a fixed array inside the library.  Checked through the C ABI against
adamas_sparse_attention (which takes a caller workspace): two calls in a row must
each match it within the attention tolerance, and oversized calls are refused.
This file is collected last, so a stop-at-first-failure run has already run
every other test; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

import token_level_sparse_fwht_b200 as ad
from gpu_helpers import ATOL_OUT
from workloads import WORKLOADS, generate

pytestmark = pytest.mark.gpu


def _inputs(B, Hq, Hkv, L, k_eff, seed):
    w = WORKLOADS[2].scaled(B=B, Hq=Hq, Hkv=Hkv, L=L)
    inp = generate(w, "cpu")
    rng = np.random.default_rng(seed)
    idx = np.stack([np.stack([np.sort(rng.choice(L, k_eff, replace=False)) for _ in range(Hq)])
                    for _ in range(B)]).astype(np.int32)
    return (inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(),
            torch.from_numpy(idx).cuda())


def _call(q, kc, vc, idx, out):
    B, Hq, d = q.shape
    _, Hkv, Lmax, _ = kc.shape
    return ad.lib().adamas_sparse_attention_noalloc(
        q.data_ptr(), kc.data_ptr(), vc.data_ptr(), ad.BF16, idx.data_ptr(), B, Hq, Hkv, d, Lmax,
        idx.shape[-1], out.data_ptr(), torch.cuda.current_stream().cuda_stream)


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

"""Key / query encoder (FWHT + 2-bit buckets + packing) on the GPU vs the oracle.

Codes must match except at coordinates within 1e-4 of a threshold, and the
fraction of coordinates whose code differs must stay below 1e-4."""
import numpy as np
import pytest
import torch

import oracle
import token_level_sparse_fwht_b200 as ad
from gpu_helpers import encoder_mismatch, MAX_MISMATCH_FRACTION, f64
from workloads import WORKLOADS, generate

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg,L", [(1, 1024), (2, 3001), (4, 777)])
def test_encode_keys_matches_oracle(cfg, L):
    w = WORKLOADS[cfg].scaled(L=L)
    inp = generate(w, "cpu")
    k = inp.k_cache.cuda()
    codes = torch.zeros(k.shape[:-1] + (32,), dtype=torch.uint8, device="cuda")
    ad.encode_keys(k, codes, 0, L, inp.t)
    torch.cuda.synchronize()
    bad, frac, near = encoder_mismatch(codes.cpu().numpy(), inp.k_cache, inp.t)
    assert bad == 0
    assert frac < MAX_MISMATCH_FRACTION, (frac, near)


def test_encode_append_touches_only_its_rows():
    w = WORKLOADS[3].scaled(B=2, L=700)
    inp = generate(w, "cpu")
    k = inp.k_cache.cuda()
    codes = torch.full(k.shape[:-1] + (32,), 0xAB, dtype=torch.uint8, device="cuda")
    ad.encode_keys(k, codes, 188, 512, inp.t)
    c = codes.cpu().numpy()
    assert np.all(c[:, :, :188] == 0xAB)
    bad, frac, _ = encoder_mismatch(c[:, :, 188:700], inp.k_cache[:, :, 188:700], inp.t)
    assert bad == 0 and frac < MAX_MISMATCH_FRACTION


def test_encode_closed_forms_exact():
    """Vectors whose transform is known in closed form and far from every
    threshold: all-ones -> (sqrt(128), 0, ..., 0); e_i -> +-1/sqrt(128)."""
    t = 0.05
    x = torch.zeros((1, 1, 130, 128), dtype=torch.float32)
    x[0, 0, 0] = 1.0                           # y = (11.31, 0, ...): codes 3, 2, 2, ...
    for i in range(128):
        x[0, 0, 1 + i, i] = 1.0                # e_i -> +-0.0884: codes 3 or 0
    x[0, 0, 129] = -1.0
    k = x.cuda()
    codes = torch.zeros((1, 1, 130, 32), dtype=torch.uint8, device="cuda")
    ad.encode_keys(k, codes, 0, 130, t)
    got = codes.cpu().numpy()[0, 0]
    want = oracle.encode(x[0, 0].double().numpy(), t)
    assert np.array_equal(got, want)
    assert got[0, 0] == (3 | 2 << 2 | 2 << 4 | 2 << 6)


@pytest.mark.parametrize("t", [0.05, 0.0])
def test_encode_closed_forms_exact_bf16_tensor_core_path(t):
    """The same closed forms in bf16 (exact), which go through the tensor-core encoder;
    t = 0 takes its sign-only bucketing (y = 0 -> code 3)."""
    x = torch.zeros((1, 1, 130, 128), dtype=torch.bfloat16)
    x[0, 0, 0] = 1.0
    for i in range(128):
        x[0, 0, 1 + i, i] = 1.0
    x[0, 0, 129] = -1.0
    codes = torch.zeros((1, 1, 130, 32), dtype=torch.uint8, device="cuda")
    ad.encode_keys(x.cuda(), codes, 0, 130, t)
    got = codes.cpu().numpy()[0, 0]
    want = oracle.encode(x[0, 0].double().numpy(), t)
    assert np.array_equal(got, want)


def test_encode_queries_matches_oracle():
    w = WORKLOADS[2].scaled(B=3)
    inp = generate(w, "cpu")
    qc = ad.encode_queries(inp.q.cuda(), inp.t)
    bad, frac, _ = encoder_mismatch(qc.cpu().numpy(), inp.q, inp.t)
    assert bad == 0 and frac < 1e-3       # 3 x 32 vectors: one coordinate at most


@pytest.mark.slow
def test_encode_full_append_workload():
    """The 512-token append of the batch-8, 32K-context workload (8 x 8 x 512 keys)."""
    w = WORKLOADS[3]
    inp = generate(w, "cuda")
    codes = torch.zeros(inp.k_cache.shape[:-1] + (32,), dtype=torch.uint8, device="cuda")
    pos0 = w.L - w.append
    ad.encode_keys(inp.k_cache, codes, pos0, w.append, inp.t)
    sub = inp.k_cache[:, :, pos0:].cpu()
    bad, frac, near = encoder_mismatch(codes[:, :, pos0:].cpu().numpy(), sub, inp.t)
    print(f"append encode: mismatch fraction {frac:.3g}, near-threshold fraction {near:.3g}")
    assert bad == 0 and frac < MAX_MISMATCH_FRACTION


@pytest.mark.parametrize("n_new,pos0", [(1, 699), (3, 250), (17, 0)])
def test_encode_short_appends(n_new, pos0):
    """Appends shorter than a 16-key tile (one token per sequence per decode step is
    the usual case): a tile then spans several (batch, kv head) rows."""
    w = WORKLOADS[3].scaled(B=3, L=700)
    inp = generate(w, "cpu")
    k = inp.k_cache.cuda()
    codes = torch.full(k.shape[:-1] + (32,), 0xAB, dtype=torch.uint8, device="cuda")
    ad.encode_keys(k, codes, pos0, n_new, inp.t)
    c = codes.cpu().numpy()
    assert np.all(c[:, :, :pos0] == 0xAB) and np.all(c[:, :, pos0 + n_new:] == 0xAB)
    bad, frac, _ = encoder_mismatch(c[:, :, pos0:pos0 + n_new],
                                    inp.k_cache[:, :, pos0:pos0 + n_new], inp.t)
    assert bad == 0 and frac < 1e-2      # few coordinates: one flip is 1/(B Hkv n 128)

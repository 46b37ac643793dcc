"""Seeded generators: determinism, shapes, outlier channels and planted keys."""
import math

import torch

from workloads import WORKLOADS, generate, sigma_of, replicas_for_l2


def test_deterministic_and_shaped():
    w = WORKLOADS[2].scaled(L=300, Hq=8, Hkv=2)
    a = generate(w, "cpu")
    b = generate(w, "cpu")
    assert a.q.shape == (1, 8, 128) and a.k_cache.shape == (1, 2, 300, 128)
    assert a.k_cache.dtype == torch.bfloat16
    assert torch.equal(a.k_cache, b.k_cache) and torch.equal(a.q, b.q)
    c = generate(w, "cpu", layer=1)
    assert not torch.equal(a.k_cache, c.k_cache)


def test_outlier_channels_scaled():
    w = WORKLOADS[2].scaled(L=4096, Hq=4, Hkv=4)
    inp = generate(w, "cpu")
    std = inp.k_cache.float().reshape(-1, 128).std(0)
    ch = inp.outlier_channels
    assert len(set(ch.tolist())) == 4
    others = torch.ones(128, dtype=torch.bool)
    others[ch] = False
    assert torch.all(std[ch] > 8) and torch.all(std[others] < 1.2)
    assert math.isclose(w.t, 0.5 * math.sqrt(524 / 128))
    assert sigma_of(False) == 1.0


def test_planted_rows():
    w = WORKLOADS[1]
    inp = generate(w, "cpu")
    p = inp.planted[0, 0]
    assert p.numel() == 4 and len(set(p.tolist())) == 4
    diff = inp.k_cache[0, 0, p] - inp.q[0, 0][None]
    assert diff.abs().max() < 1.0 and diff.std() < 0.2
    assert inp.k_cache.dtype == torch.float32 and inp.t == 0.5


def test_bytes_model_matches_formula():
    w = WORKLOADS[2]
    # codes 8 MiB + 32 heads x 128 rows x 512 B + q + fp32 out
    assert w.algorithmic_bytes(128) == 10_510_336
    assert WORKLOADS[5].algorithmic_bytes(1024) == 201_424_896
    assert replicas_for_l2(10_510_336, 126 * 2**20) >= 26

"""The fused decode step (one kernel launch: thread-block clusters, or the grid-wide
kernel for few units; both are run) vs the float64 oracle.

The key codes are the oracle's (uploaded); the kernel encodes the queries itself in
fp32, so a query coordinate within 1e-4 of a threshold may take either bucket: the
selection must equal the oracle's for one admissible query code, and the output
must be within 2e-3 of the oracle's attention over that selection."""
import numpy as np
import pytest
import torch

import oracle
import token_level_sparse_fwht_b200 as ad
from gpu_helpers import check_decode_head, f64, oracle_codes, upload
from workloads import WORKLOADS, generate

pytestmark = pytest.mark.gpu


def _decode(inp, kc, L, k):
    B, Hq, _ = inp.q.shape
    _, Hkv, Lmax, _ = inp.k_cache.shape
    q = inp.q.cuda()
    kcache = inp.k_cache.cuda()
    vcache = inp.v_cache.cuda()
    codes = upload(kc)
    ws = ad.decode_workspace(B, Hq, Hkv, L, k)
    idx = torch.full((B, Hq, min(k, L)), -1, dtype=torch.int32, device="cuda")
    out = ad.decode_step(q, kcache, vcache, codes, L, k, inp.t, ws, idx_out=idx)
    torch.cuda.synchronize()
    ad.check_workspace(ws)
    return idx.cpu().numpy(), out.cpu().numpy(), ws


def _check_all(inp, kc, L, k, heads=None):
    B, Hq, _ = inp.q.shape
    G = Hq // inp.k_cache.shape[1]
    idx, out, ws = _decode(inp, kc, L, k)
    q = f64(inp.q)
    worst = 0.0
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hq)]
    for b, h in pairs:
        K = f64(inp.k_cache[b, h // G, :L])
        V = f64(inp.v_cache[b, h // G, :L])
        worst = max(worst, check_decode_head(idx[b, h], out[b, h], q[b, h], K, V,
                                             kc[b, h // G, :L], k, inp.t))
    return worst, idx, out, ws


@pytest.mark.parametrize("cfg,over,k", [
    (1, {}, 64),                                   # single head, fp32, 4 planted keys
    (2, dict(L=3001), 128),
    (2, dict(L=3001), 1024),
    (3, dict(B=3, L=2500), 256),
    (4, dict(L=5000, Hq=8, Hkv=8), 128),           # MHA, 16 needles per head
    (2, dict(L=5000, Hq=16, Hkv=2), 64),           # G = 8
    (2, dict(L=777, Hq=4, Hkv=2), 2000),           # k > L: dense
    (2, dict(B=70, Hq=4, Hkv=4, L=64), 5),         # 280 units: two waves
])
def test_decode_step_matches_oracle(cfg, over, k, decode_policy):
    w = WORKLOADS[cfg].scaled(**over)
    inp = generate(w, "cpu")
    kc = oracle_codes(inp.k_cache, inp.t)
    worst, idx, out, _ = _check_all(inp, kc, w.L, k)
    assert worst <= 2e-3
    if w.planted and k >= 64:
        for b in range(w.B):
            for h in range(w.Hq):
                assert set(inp.planted[b, h].tolist()) <= set(idx[b, h].tolist())


def test_decode_lmax_padding_and_repeat(decode_policy):
    w = WORKLOADS[2].scaled(L=2000, Hq=8, Hkv=2)
    inp = generate(w, "cpu", Lmax=2600)
    kc = oracle_codes(inp.k_cache, inp.t)
    worst, idx, out, ws = _check_all(inp, kc, w.L, 100)
    assert worst <= 2e-3
    idx2, out2, _ = _decode(inp, kc, w.L, 100)
    assert np.array_equal(idx, idx2) and np.array_equal(out, out2)


def test_decode_without_idx_output(decode_policy):
    w = WORKLOADS[2].scaled(L=1500, Hq=8, Hkv=2)
    inp = generate(w, "cpu")
    kc = oracle_codes(inp.k_cache, inp.t)
    ws = ad.decode_workspace(1, 8, 2, w.L, 64)
    out = ad.decode_step(inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(), upload(kc), w.L,
                         64, inp.t, ws).cpu().numpy()
    q = f64(inp.q)
    for h in range(8):
        check_decode_head(None, out[0, h], q[0, h], f64(inp.k_cache[0, h // 4]),
                          f64(inp.v_cache[0, h // 4]), kc[0, h // 4], 64, inp.t)


def test_decode_full_32k_layer_every_budget(decode_policy):
    """Llama-3.1-8B-shaped layer, 32K context: all 32 heads at budgets 64..1024, in
    the launch configuration the benchmark times."""
    w = WORKLOADS[2]
    inp = generate(w, "cuda")
    kc = oracle_codes(inp.k_cache, inp.t)
    cpu = type(inp)(q=inp.q.cpu(), k_cache=inp.k_cache.cpu(), v_cache=inp.v_cache.cpu(),
                    t=inp.t, outlier_channels=None)
    for k in w.budgets:
        worst, _, _, _ = _check_all(cpu, kc, w.L, k)
        assert worst <= 2e-3, (k, worst)


@pytest.mark.slow
def test_decode_batch8_with_append():
    """Batch 8 x 32K: the last 512 positions are encoded on the GPU by
    adamas_encode_keys (checked against the oracle) and the decode step then runs on
    the oracle's codes; 16 (batch, head) pairs are checked at both budgets."""
    w = WORKLOADS[3]
    inp = generate(w, "cuda")
    pos0 = w.L - w.append
    codes = torch.zeros(inp.k_cache.shape[:-1] + (32,), dtype=torch.uint8, device="cuda")
    ad.encode_keys(inp.k_cache, codes, pos0, w.append, inp.t)
    from gpu_helpers import encoder_mismatch, MAX_MISMATCH_FRACTION
    bad, frac, _ = encoder_mismatch(codes[:, :, pos0:].cpu().numpy(),
                                    inp.k_cache[:, :, pos0:].cpu(), inp.t)
    assert bad == 0 and frac < MAX_MISMATCH_FRACTION
    kcache = inp.k_cache.cpu()
    kc = np.stack([oracle_codes(kcache[b], inp.t) for b in range(w.B)])
    cpu = type(inp)(q=inp.q.cpu(), k_cache=kcache, v_cache=inp.v_cache.cpu(), t=inp.t,
                    outlier_channels=None)
    heads = [(b, h) for b in range(w.B) for h in (b, 31 - b)]
    for k in w.budgets:
        worst, _, _, _ = _check_all(cpu, kc, w.L, k, heads=heads)
        assert worst <= 2e-3


@pytest.mark.slow
def test_decode_llama8b_128k_layers_sampled():
    """Layers of the 32-layer Llama-3.1-8B shape at batch 4 x 128K (two waves of
    units per launch): three seeded layers run on the GPU, and two (batch, head)
    pairs per layer are checked against the oracle on the oracle's codes."""
    w = WORKLOADS[5]
    k = w.budgets[0]
    rng = np.random.default_rng(0)
    layers = sorted(rng.choice(w.layers, 3, replace=False).tolist())
    for layer in layers:
        inp = generate(w, "cuda", layer=layer)
        codes = torch.empty(inp.k_cache.shape[:-1] + (32,), dtype=torch.uint8, device="cuda")
        ad.encode_keys(inp.k_cache, codes, 0, w.L, inp.t)
        picks = [(int(rng.integers(w.B)), int(rng.integers(w.Hq))) for _ in range(2)]
        ocodes = {}
        for b, h in picks:
            kv = h // w.G
            ocodes[(b, kv)] = oracle_codes(inp.k_cache[b, kv].cpu(), inp.t)
            codes[b, kv] = upload(ocodes[(b, kv)])
        ws = ad.decode_workspace(w.B, w.Hq, w.Hkv, w.L, k)
        idx = torch.empty((w.B, w.Hq, k), dtype=torch.int32, device="cuda")
        out = ad.decode_step(inp.q, inp.k_cache, inp.v_cache, codes, w.L, k, inp.t, ws,
                             idx_out=idx)
        ad.check_workspace(ws)
        for b, h in picks:
            kv = h // w.G
            check_decode_head(idx[b, h].cpu().numpy(), out[b, h].cpu().numpy(),
                              f64(inp.q[b, h]), f64(inp.k_cache[b, kv]), f64(inp.v_cache[b, kv]),
                              ocodes[(b, kv)], k, inp.t)
        del inp, codes, ws
        torch.cuda.empty_cache()


def test_decode_step_host_buffers(decode_policy):
    """adamas_decode_step_host (pinned q in, fp32 out back, one C call) returns what
    adamas_decode_step returns for the same inputs, bit for bit."""
    w = WORKLOADS[2].scaled(L=2500, Hq=16, Hkv=4)
    inp = generate(w, "cpu")
    kc = oracle_codes(inp.k_cache, inp.t)
    kcache, vcache, codes = inp.k_cache.cuda(), inp.v_cache.cuda(), upload(kc)
    ws = ad.decode_workspace(1, 16, 4, w.L, 128)
    want = ad.decode_step(inp.q.cuda(), kcache, vcache, codes, w.L, 128, inp.t, ws)
    q_host = inp.q.clone().pin_memory()
    out_host = torch.zeros((1, 16, 128), dtype=torch.float32).pin_memory()
    q_dev = torch.empty_like(inp.q, device="cuda")
    out_dev = torch.empty((1, 16, 128), dtype=torch.float32, device="cuda")
    ad.decode_step_host(q_host, q_dev, kcache, vcache, codes, w.L, 128, inp.t, ws, out_dev,
                        out_host)
    torch.cuda.synchronize()
    assert torch.equal(out_host, want.cpu())


def test_prepared_decode_host_call(decode_policy):
    """The prepared (buffer-bound) host call gives the same output as decode_step."""
    w = WORKLOADS[2].scaled(L=1800, Hq=8, Hkv=2)
    inp = generate(w, "cpu")
    kcache, vcache = inp.k_cache.cuda(), inp.v_cache.cuda()
    codes = upload(oracle_codes(inp.k_cache, inp.t))
    ws = ad.decode_workspace(1, 8, 2, w.L, 64)
    want = ad.decode_step(inp.q.cuda(), kcache, vcache, codes, w.L, 64, inp.t, ws).cpu()
    q_host = inp.q.clone().pin_memory()
    out_host = torch.zeros((1, 8, 128), dtype=torch.float32).pin_memory()
    call = ad.PreparedDecodeHost(q_host, torch.empty_like(inp.q, device="cuda"), kcache, vcache,
                                 codes, w.L, 64, inp.t, ws,
                                 torch.empty((1, 8, 128), device="cuda"), out_host,
                                 stream=torch.cuda.current_stream())
    for _ in range(2):
        out_host.zero_()
        call()
        torch.cuda.synchronize()
        assert torch.equal(out_host, want)


def test_long_context_plan_with_scratch_distances_select_exact():
    """Batch 4 x 8 kv heads at 128K: the plan keeps each CTA's distances in workspace
    scratch (fewer, longer CTAs in one wave).  Random codes: sampled rows bit-exact."""
    B, Hq, Hkv, L, k = 4, 32, 8, 131072, 1024
    assert ad.decode_workspace_bytes(B, Hq, Hkv, L, k) > 256      # the scratch plan
    rng = np.random.default_rng(77)
    qc = rng.integers(0, 256, size=(B, Hq, 32), dtype=np.uint8)
    kc = rng.integers(0, 256, size=(B, Hkv, L, 32), dtype=np.uint8)
    ws = ad.decode_workspace(B, Hq, Hkv, L, k)
    idx = ad.select_topk(upload(qc), upload(kc), L, k, ws)
    torch.cuda.synchronize()
    ad.check_workspace(ws)
    idx = idx.cpu().numpy()
    uq, G = oracle.unpack_codes(qc), Hq // Hkv
    for b, h in [(0, 0), (1, 13), (2, 22), (3, 31)]:
        d = oracle.manhattan(uq[b, h], oracle.unpack_codes(kc[b, h // G]))
        assert np.array_equal(idx[b, h], oracle.select_topk(d, k)), (b, h)


def test_long_context_plan_with_scratch_distances_decode():
    """The same plan through the fused step: the oracle's key codes for two sampled kv
    heads (the GPU encoder's elsewhere), their query heads checked against the oracle."""
    w = WORKLOADS[5].scaled(layers=1)
    inp = generate(w, "cuda")
    assert ad.decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.L, 1024) > 256
    codes = torch.empty(inp.k_cache.shape[:-1] + (32,), dtype=torch.uint8, device="cuda")
    ad.encode_keys(inp.k_cache, codes, 0, w.L, inp.t)
    sampled = [(0, 1), (3, 6)]
    kcs = {}
    for b, kvh in sampled:
        kcs[(b, kvh)] = oracle_codes(inp.k_cache[b, kvh].cpu(), inp.t)
        codes[b, kvh] = upload(kcs[(b, kvh)])
    ws = ad.decode_workspace(w.B, w.Hq, w.Hkv, w.L, 1024)
    idx = torch.empty((w.B, w.Hq, 1024), dtype=torch.int32, device="cuda")
    out = ad.decode_step(inp.q, inp.k_cache, inp.v_cache, codes, w.L, 1024, inp.t, ws,
                         idx_out=idx)
    torch.cuda.synchronize()
    ad.check_workspace(ws)
    idx, out, q = idx.cpu().numpy(), out.cpu().numpy(), f64(inp.q)
    G = w.G
    for b, kvh in sampled:
        K, V = f64(inp.k_cache[b, kvh]), f64(inp.v_cache[b, kvh])
        for h in range(kvh * G, (kvh + 1) * G):
            check_decode_head(idx[b, h], out[b, h], q[b, h], K, V, kcs[(b, kvh)], 1024, inp.t)


def test_decode_long_single_kv_head_grid_wide_plan():
    """One kv head over 256K keys (4 query heads): the planner's default is the
    grid-wide kernel (64 CTAs exchanging counts through the workspace).  Selection on
    the oracle's codes must be bit-exact and the outputs within 2e-3 for every head."""
    w = WORKLOADS[2].scaled(Hq=4, Hkv=1, L=262144)
    plan = ad.decode_plan(1, 4, 1, w.L, 128)
    assert plan["cluster"] == 1 and plan["ctas"] > 16
    inp = generate(w, "cuda")
    kc = oracle_codes(inp.k_cache[0, 0].cpu(), inp.t)[None, None]
    worst, idx, out, ws = _check_all(type(inp)(q=inp.q.cpu(), k_cache=inp.k_cache.cpu(),
                                               v_cache=inp.v_cache.cpu(), t=inp.t,
                                               outlier_channels=None), kc, w.L, 128)
    assert worst <= 2e-3
    assert ws.numel() > 256


@pytest.mark.slow
def test_decode_128k_mha_both_budgets_sampled_heads():
    """The 128K MHA workload (32 heads, 16 planted needles each) through the fused step
    at budgets 128 and 1024, in the launch configuration the benchmark times: four
    sampled heads carry the oracle's key codes (the GPU encoder's elsewhere) and are
    checked against the oracle in full; the needles are recalled."""
    w = WORKLOADS[4]
    inp = generate(w, "cuda")
    codes = torch.empty(inp.k_cache.shape[:-1] + (32,), dtype=torch.uint8, device="cuda")
    ad.encode_keys(inp.k_cache, codes, 0, w.L, inp.t)
    heads = [0, 11, 20, 31]
    ocodes = {}
    for h in heads:
        ocodes[h] = oracle_codes(inp.k_cache[0, h].cpu(), inp.t)
        codes[0, h] = upload(ocodes[h])
    q = f64(inp.q)
    for k in w.budgets:
        ws = ad.decode_workspace(w.B, w.Hq, w.Hkv, w.L, k)
        idx = torch.empty((1, w.Hq, k), dtype=torch.int32, device="cuda")
        out = ad.decode_step(inp.q, inp.k_cache, inp.v_cache, codes, w.L, k, inp.t, ws,
                             idx_out=idx)
        torch.cuda.synchronize()
        ad.check_workspace(ws)
        gi, go = idx.cpu().numpy(), out.cpu().numpy()
        for h in heads:
            err = check_decode_head(gi[0, h], go[0, h], q[0, h], f64(inp.k_cache[0, h]),
                                    f64(inp.v_cache[0, h]), ocodes[h], k, inp.t)
            assert err <= 2e-3, (k, h, err)
        planted = inp.planted[0].cpu().numpy()
        assert np.mean([np.isin(planted[h], gi[0, h]).mean() for h in range(w.Hq)]) > 0.9

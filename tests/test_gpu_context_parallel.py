"""Context-parallel kernel steps on one GPU: ranks emulated as independent launches.

Every "rank" runs its steps on its own slice of the caches; stacking tensors stands
in for the all-gathers (no launch waits on another).  The merged selection and
output must match the oracle over the whole context (query codes within 1e-4 of a
threshold may take either bucket) and equal the single-GPU step."""
import numpy as np
import pytest
import torch

import token_level_sparse_fwht_b200 as ad
from gpu_helpers import check_decode_head, check_decode_unit_shared, f64, oracle_codes, upload
from workloads import WORKLOADS, generate

pytestmark = pytest.mark.gpu


def _run_ranks(inp, codes, cuts, k, shared):
    """All steps for every rank; returns (out [B,Hq,128], idx merged by max)."""
    B, Hq, _ = inp.q.shape
    Hkv = inp.k_cache.shape[1]
    L_total = cuts[-1]
    world = len(cuts) - 1
    q = inp.q.cuda()
    slices = []
    for r in range(world):
        lo, hi = cuts[r], cuts[r + 1]
        slices.append((inp.k_cache[:, :, lo:hi].contiguous().cuda(),
                       inp.v_cache[:, :, lo:hi].contiguous().cuda(),
                       codes[:, :, lo:hi].contiguous(), hi - lo, lo))
    wss = [ad.cp_workspace(B, Hq, Hkv, sl[3], k, shared) for sl in slices]
    hists = [ad.cp_histograms(q, sl[2], sl[3], k, inp.t, ws, shared=shared)
             for sl, ws in zip(slices, wss)]
    hist_all = torch.stack(hists)                                  # stands in for all-gather
    rows = Hkv if shared else Hq
    parts, idxs = [], []
    for r, (sl, ws) in enumerate(zip(slices, wss)):
        idx = torch.full((B, rows, min(k, L_total)), -1, dtype=torch.int32, device="cuda")
        parts.append(ad.cp_attend(q, sl[0], sl[1], sl[2], sl[3], L_total, sl[4], k, inp.t,
                                  hist_all, r, ws, shared=shared, idx_out=idx))
        idxs.append(idx)
    out = ad.cp_combine(torch.stack(parts))                         # stands in for all-gather
    torch.cuda.synchronize()
    for ws in wss:
        ad.check_workspace(ws)
    return out.cpu().numpy(), torch.stack(idxs).amax(0).cpu().numpy()


@pytest.mark.parametrize("cfg,over,cuts,k,shared", [
    (2, dict(L=3000), [0, 1500, 3000], 128, False),
    (2, dict(L=3001), [0, 700, 2000, 3001], 256, False),        # three uneven slices
    (2, dict(L=4000, Hq=16, Hkv=2), [0, 1000, 2000, 3000, 4000], 64, False),   # G = 8, 4 ranks
    (2, dict(L=3000, B=2), [0, 1200, 3000], 200, True),          # shared selection
    (1, {}, [0, 512, 1024], 64, False),                          # fp32, single head
    (2, dict(L=1000, Hq=4, Hkv=2), [0, 990, 1000], 600, False),  # a tiny slice, big budget
    (2, dict(L=2500, Hq=16, Hkv=2), [0, 500, 1000, 1500, 2000, 2500], 128, True),  # 5 ranks
    (2, dict(L=1201, Hq=8, Hkv=2), [0, 1, 1200, 1201], 64, False),   # one-position ranks
])
def test_context_parallel_matches_oracle_and_single_gpu(cfg, over, cuts, k, shared):
    w = WORKLOADS[cfg].scaled(**over)
    inp = generate(w, "cpu")
    kc = oracle_codes(inp.k_cache, inp.t)
    codes = upload(kc)
    out, idx = _run_ranks(inp, codes, cuts, k, shared)
    # single-GPU step over the whole context, same kernels' query encode
    ws = ad.decode_workspace(w.B, w.Hq, w.Hkv, w.L, k)
    rows = w.Hkv if shared else w.Hq
    sidx = torch.empty((w.B, rows, min(k, w.L)), dtype=torch.int32, device="cuda")
    f = ad.decode_step_shared if shared else ad.decode_step
    sout = f(inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(), codes, w.L, k, inp.t, ws,
             idx_out=sidx)
    torch.cuda.synchronize()
    assert np.array_equal(idx, sidx.cpu().numpy())
    # same positions, same float32 arithmetic per row, but the rows' softmax terms are
    # summed in a different order (ranks first, or the CTAs of one cluster, and within
    # a warp either one row per instruction or 8-lane row groups merged at the end):
    # the two agree to float32 rounding of a weighted sum over up to 1024 rows, which
    # 1e-4 bounds with room (the oracle comparison below keeps 2e-3)
    assert np.abs(out - sout.cpu().numpy()).max() <= 1e-4
    if not shared:
        q = f64(inp.q)
        G = w.G
        for b in range(w.B):
            for h in range(w.Hq):
                check_decode_head(idx[b, h], out[b, h], q[b, h], f64(inp.k_cache[b, h // G]),
                                  f64(inp.v_cache[b, h // G]), kc[b, h // G], k, inp.t)
    else:
        # every (batch, kv head) row against the oracle, for one admissible combination
        # of the group's query codes
        q = f64(inp.q)
        G = w.G
        for b in range(w.B):
            for kvh in range(w.Hkv):
                hs = slice(kvh * G, (kvh + 1) * G)
                check_decode_unit_shared(idx[b, kvh], out[b, hs], q[b, hs],
                                         f64(inp.k_cache[b, kvh]), f64(inp.v_cache[b, kvh]),
                                         kc[b, kvh], k, inp.t)


@pytest.mark.slow
def test_context_parallel_128k_mha_two_ranks_sampled():
    """The 128K MHA workload split over two emulated ranks (the oracle's key codes):
    equal to the single-GPU step, four heads checked against the oracle, needles
    recalled."""
    w = WORKLOADS[4]
    inp = generate(w, "cuda")
    kc = np.zeros((1, w.Hkv, w.L, 32), np.uint8)
    for h in range(w.Hkv):
        kc[0, h] = oracle_codes(inp.k_cache[0, h].cpu(), inp.t)
    codes = upload(kc)
    half = w.L // 2
    out, idx = _run_ranks(inp, codes, [0, half, w.L], 128, False)
    ws = ad.decode_workspace(w.B, w.Hq, w.Hkv, w.L, 128)
    sidx = torch.empty((1, w.Hq, 128), dtype=torch.int32, device="cuda")
    sout = ad.decode_step(inp.q, inp.k_cache, inp.v_cache, codes, w.L, 128, inp.t, ws,
                          idx_out=sidx)
    torch.cuda.synchronize()
    assert np.array_equal(idx, sidx.cpu().numpy())
    # same positions, same float32 arithmetic per row, but the rows' softmax terms are
    # summed in a different order (ranks first, or the CTAs of one cluster, and within
    # a warp either one row per instruction or 8-lane row groups merged at the end):
    # the two agree to float32 rounding of a weighted sum over up to 1024 rows, which
    # 1e-4 bounds with room (the oracle comparison below keeps 2e-3)
    assert np.abs(out - sout.cpu().numpy()).max() <= 1e-4
    q = f64(inp.q)
    for h in (0, 7, 19, 31):
        check_decode_head(idx[0, h], out[0, h], q[0, h], f64(inp.k_cache[0, h]),
                          f64(inp.v_cache[0, h]), kc[0, h], 128, inp.t)
    planted = inp.planted[0].cpu().numpy()
    assert np.mean([np.isin(planted[h], idx[0, h]).mean() for h in range(w.Hq)]) > 0.9

"""Per-sequence context lengths and paged caches on the GPU vs oracle.decode_step_varlen.

Paging is a storage layout: the seeded logical caches are scattered into a shuffled
page pool (workloads.paging) with spare pages holding a large constant, so a kernel
that reads a page it was not given produces visibly wrong results.  Fed the
oracle's codes, selections are bit-exact (including the -1 padding of short
sequences); in the fused step a query coordinate within 1e-4 of a threshold may
take either bucket, and outputs must be within 2e-3 of the oracle's."""
import itertools

import numpy as np
import pytest
import torch

import oracle
import token_level_sparse_fwht_b200 as ad
from gpu_helpers import (ATOL_OUT, MAX_MISMATCH_FRACTION, encoder_mismatch, f64, oracle_codes,
                         query_alternatives, upload)
from workloads import WORKLOADS, generate
from workloads.paging import make_block_table, scatter_to_pages

pytestmark = pytest.mark.gpu


def _oracle_idx(qc, kc, lens, k, shared):
    B, Hq, _ = qc.shape
    _, Hkv, Lmax, _ = kc.shape
    zq = np.zeros((B, Hq, 128))
    zkv = np.broadcast_to(np.zeros(1), (B, Hkv, Lmax, 128))
    idx, _ = oracle.decode_step_varlen(zq, zkv, zkv, lens, k, 1.0, key_codes=kc,
                                       query_codes=qc, shared=shared)
    return idx


@pytest.mark.parametrize("shared", [False, True])
@pytest.mark.parametrize("B,Hq,Hkv,Lmax,lens,page,k", [
    (3, 8, 2, 5000, [5000, 1, 2777], 16, 128),       # full, single-key, ragged
    (4, 4, 4, 3000, [0, 3000, 999, 64], 64, 100),    # an empty sequence
    (2, 8, 1, 4096, [4096, 4000], 1, 50),            # page size 1: a copy per key
    (2, 32, 8, 2048, [2048, 1500], 4096, 64),        # one page holds a whole sequence
    (2, 16, 2, 9000, [8191, 9000], 512, 700),        # G = 8, chunk-sized pages
    (5, 4, 2, 700, [700, 13, 300, 699, 2], 32, 1000),  # budget above every length
    (3, 16, 2, 3000, [1, 2999, 3000], 1, 77),        # G = 8, one-token pages, length 1
])
def test_select_paged_random_codes(B, Hq, Hkv, Lmax, lens, page, k, shared):
    rng = np.random.default_rng(B * 97 + Lmax + page)
    qc = rng.integers(0, 256, size=(B, Hq, 32), dtype=np.uint8)
    kc = rng.integers(0, 256, size=(B, Hkv, Lmax, 32), dtype=np.uint8)
    pc = make_block_table(lens, Lmax, page, seed=Lmax + page)
    pool = scatter_to_pages(torch.from_numpy(kc), pc, fill=0)   # spare pages: distance-0 bait
    ws = ad.decode_workspace(B, Hq, Hkv, Lmax, k)
    got = ad.select_topk_paged(upload(qc), upload(pool), upload(pc.block_table),
                               upload(pc.seq_lens), Lmax, k, ws, shared=shared)
    torch.cuda.synchronize()
    ad.check_workspace(ws)
    want = _oracle_idx(qc, kc, lens, k, shared)
    assert np.array_equal(got.cpu().numpy(), want)


@pytest.mark.parametrize("shared", [False, True])
def test_select_varlen_contiguous(shared):
    rng = np.random.default_rng(61)
    B, Hq, Hkv, Lmax, k = 4, 8, 2, 3000, 200
    lens = [3000, 0, 150, 2001]
    qc = rng.integers(0, 256, size=(B, Hq, 32), dtype=np.uint8)
    kc = rng.integers(0, 256, size=(B, Hkv, Lmax, 32), dtype=np.uint8)
    # varlen over contiguous caches has no select-only entry point: the paged one with
    # one page per sequence is the same layout ([B][Hkv][Lmax] = pages of Lmax rows)
    table = torch.arange(B, dtype=torch.int32)[:, None]
    page = 4096
    pool = np.zeros((B, Hkv, page, 32), np.uint8)
    pool[:, :, :Lmax] = kc
    ws = ad.decode_workspace(B, Hq, Hkv, Lmax, k)
    got = ad.select_topk_paged(upload(qc), upload(pool), upload(table),
                               upload(torch.tensor(lens, dtype=torch.int32)), Lmax, k, ws,
                               shared=shared)
    torch.cuda.synchronize()
    assert np.array_equal(got.cpu().numpy(), _oracle_idx(qc, kc, lens, k, shared))


def _alternatives(qg, t, cap=64):
    per_head = [query_alternatives(qg[g], t) for g in range(qg.shape[0])]
    for combo in itertools.islice(itertools.product(*per_head), cap):
        yield np.stack(combo)


def _check_group(gpu_idx, gpu_out, qg, Kg, Vg, kcg, Lb, k, t, shared):
    """One (sequence, kv head): qg [G,128], Kg/Vg [Lmax,128], kcg [Lmax,32]; gpu_idx is
    [G, k_row] (per head) or [k_row] (shared); gpu_out [G,128].  Returns max error."""
    G = qg.shape[0]
    errs = []
    for qcg in _alternatives(qg, t):
        idx, out = oracle.decode_step_varlen(qg[None], Kg[None, None], Vg[None, None], [Lb], k,
                                             t, key_codes=kcg[None, None], query_codes=qcg[None],
                                             shared=shared)
        want_idx = idx[0, 0] if shared else idx[0]
        if not np.array_equal(np.asarray(gpu_idx, np.int64), want_idx):
            continue
        err = float(np.abs(np.asarray(gpu_out, np.float64) - out[0]).max())
        errs.append(err)
        if err <= ATOL_OUT:
            return err
    raise AssertionError(f"no admissible oracle result matches (G={G}, L={Lb}): {errs}")


def _run_decode(inp, kc, lens, k, page, shared, paged=True):
    B, Hq, _ = inp.q.shape
    _, Hkv, Lmax, _ = inp.k_cache.shape
    rows = Hkv if shared else Hq
    ws = ad.decode_workspace(B, Hq, Hkv, Lmax, k)
    idx = torch.full((B, rows, min(k, Lmax)), -7, dtype=torch.int32, device="cuda")
    if paged:
        pc = make_block_table(lens, Lmax, page, seed=Lmax * 3 + page)
        big = 1e4                      # spare pages: values that would wreck the output
        kp = upload(scatter_to_pages(inp.k_cache, pc, fill=big))
        vp = upload(scatter_to_pages(inp.v_cache, pc, fill=big))
        cp = upload(scatter_to_pages(torch.from_numpy(kc), pc, fill=0))
        out = ad.decode_step_paged(inp.q.cuda(), kp, vp, cp, upload(pc.block_table),
                                   upload(pc.seq_lens), Lmax, k, inp.t, ws, shared=shared,
                                   idx_out=idx)
    else:
        out = ad.decode_step_varlen(inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(),
                                    upload(kc), upload(torch.tensor(lens, dtype=torch.int32)),
                                    k, inp.t, ws, shared=shared, idx_out=idx)
    torch.cuda.synchronize()
    ad.check_workspace(ws)
    return idx.cpu().numpy(), out.cpu().numpy()


@pytest.mark.parametrize("paged", [True, False])
@pytest.mark.parametrize("shared", [False, True])
@pytest.mark.parametrize("cfg,over,lens,page,k", [
    (2, dict(B=3, L=3001), [3001, 0, 1234], 16, 128),
    (2, dict(B=2, L=2000, Hq=16, Hkv=2), [1999, 77], 64, 256),   # G = 8
    (1, dict(B=2, L=1024), [1024, 500], 32, 64),                 # fp32, single head
    (2, dict(B=4, L=600, Hq=8, Hkv=4), [600, 5, 599, 300], 8, 1000),  # budget > lengths
])
def test_decode_varlen_matches_oracle(cfg, over, lens, page, k, shared, paged, decode_policy):
    w = WORKLOADS[cfg].scaled(**over)
    inp = generate(w, "cpu")
    kc = oracle_codes(inp.k_cache, inp.t)
    idx, out = _run_decode(inp, kc, lens, k, page, shared, paged)
    q, K, V = f64(inp.q), f64(inp.k_cache), f64(inp.v_cache)
    G = w.G
    worst = 0.0
    for b, Lb in enumerate(lens):
        for kvh in range(w.Hkv):
            hs = slice(kvh * G, (kvh + 1) * G)
            gidx = idx[b, kvh] if shared else idx[b, hs]
            if Lb == 0:
                assert (gidx == -1).all() and (out[b, hs] == 0).all()
            worst = max(worst, _check_group(gidx, out[b, hs], q[b, hs], K[b, kvh], V[b, kvh],
                                            kc[b, kvh], Lb, k, inp.t, shared))
    assert worst <= ATOL_OUT


def test_paged_full_32k_layer_sampled():
    """The Llama-3.1-8B layer at 32K, budget 128, held in 16-token pages: every unit
    on the GPU, two query heads checked in full; equals the contiguous step."""
    w = WORKLOADS[2]
    inp = generate(w, "cpu")
    kc = oracle_codes(inp.k_cache, inp.t)
    idx, out = _run_decode(inp, kc, [w.L], 128, 16, shared=False)
    q = f64(inp.q)
    for h in (0, 29):
        kvh = h // w.G
        _check_group(idx[0, h:h + 1], out[0, h:h + 1], q[0, h:h + 1], f64(inp.k_cache[0, kvh]),
                     f64(inp.v_cache[0, kvh]), kc[0, kvh], w.L, 128, inp.t, False)
    ws = ad.decode_workspace(w.B, w.Hq, w.Hkv, w.L, 128)
    cidx = torch.empty((1, w.Hq, 128), dtype=torch.int32, device="cuda")
    cout = ad.decode_step(inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(), upload(kc), w.L,
                          128, inp.t, ws, idx_out=cidx)
    torch.cuda.synchronize()
    assert np.array_equal(cidx.cpu().numpy(), idx)
    assert np.abs(cout.cpu().numpy() - out).max() <= 1e-5


def test_encode_pages_matches_oracle_and_respects_page_list():
    w = WORKLOADS[2].scaled(B=2, L=1000)
    inp = generate(w, "cpu")
    pc = make_block_table([1000, 700], w.L, 16, seed=5)
    kp = scatter_to_pages(inp.k_cache, pc, fill=0).cuda()
    cp = torch.full((pc.num_pages, w.Hkv, 16, 32), 0xAA, dtype=torch.uint8, device="cuda")
    ad.encode_pages(kp, cp, inp.t)
    torch.cuda.synchronize()
    far, frac, _ = encoder_mismatch(cp.cpu().numpy(), kp.cpu(), inp.t)
    assert far == 0 and frac < MAX_MISMATCH_FRACTION
    # a page list rewrites exactly the listed pages; ids outside the pool are skipped
    before = cp.clone()
    kp2 = kp.clone()
    kp2[3] = -kp2[3]
    kp2[7] = -kp2[7]
    ids = torch.tensor([7, pc.num_pages + 4, -1, 3], dtype=torch.int32, device="cuda")
    ad.encode_pages(kp2, cp, inp.t, page_ids=ids)
    torch.cuda.synchronize()
    changed = (cp != before).flatten(1).any(1).cpu().numpy()
    assert set(np.nonzero(changed)[0].tolist()) == {3, 7}
    far, frac, _ = encoder_mismatch(cp[[3, 7]].cpu().numpy(), kp2[[3, 7]].cpu(), inp.t)
    assert far == 0 and frac < MAX_MISMATCH_FRACTION


def test_paged_bad_page_id_and_length_are_reported():
    """Out-of-range device-side inputs are clamped by the kernel (page 0, length in
    [0, max]) and reported through the workspace error word, never dereferenced."""
    rng = np.random.default_rng(71)
    B, Hq, Hkv, Lmax, k = 2, 4, 2, 512, 32
    qc = upload(rng.integers(0, 256, size=(B, Hq, 32), dtype=np.uint8))
    pc = make_block_table([512, 300], Lmax, 64, seed=1)
    pool = upload(scatter_to_pages(torch.from_numpy(
        rng.integers(0, 256, size=(B, Hkv, Lmax, 32), dtype=np.uint8)), pc))
    table = pc.block_table.clone()
    table[1, 2] = pc.num_pages + 100
    ws = ad.decode_workspace(B, Hq, Hkv, Lmax, k)
    ad.select_topk_paged(qc, pool, upload(table), upload(pc.seq_lens), Lmax, k, ws)
    with pytest.raises(ad.AdamasError) as e:
        ad.check_workspace(ws)
    assert e.value.status == ad.ERR_INVALID_ARG
    ws2 = ad.decode_workspace(B, Hq, Hkv, Lmax, k)
    lens = torch.tensor([Lmax + 50, -3], dtype=torch.int32)
    idx = ad.select_topk_paged(qc, pool, upload(pc.block_table), upload(lens), Lmax, k, ws2)
    with pytest.raises(ad.AdamasError) as e:
        ad.check_workspace(ws2)
    assert e.value.status == ad.ERR_INVALID_ARG
    assert (idx[1].cpu().numpy() == -1).all()          # length -3 clamped to 0


@pytest.mark.parametrize("pinned", [True, False])
def test_paged_host_buffers_match_device_call(pinned):
    """adamas_decode_step_paged_host (host q in, host fp32 out, one C call) returns
    what adamas_decode_step_paged returns, bit for bit: with page-locked buffers the
    kernel reads and writes them in place; with pageable ones the call copies through
    the staging buffers."""
    w = WORKLOADS[2].scaled(B=2, L=1500, Hq=8, Hkv=2)
    inp = generate(w, "cpu")
    kc = oracle_codes(inp.k_cache, inp.t)
    pc = make_block_table([1500, 900], w.L, 16, seed=3)
    kp = upload(scatter_to_pages(inp.k_cache, pc))
    vp = upload(scatter_to_pages(inp.v_cache, pc))
    cp = upload(scatter_to_pages(torch.from_numpy(kc), pc))
    bt, lens = upload(pc.block_table), upload(pc.seq_lens)
    ws = ad.decode_workspace(w.B, w.Hq, w.Hkv, w.L, 64)
    want = ad.decode_step_paged(inp.q.cuda(), kp, vp, cp, bt, lens, w.L, 64, inp.t, ws).cpu()
    q_host = inp.q.clone()
    out_host = torch.zeros((w.B, w.Hq, 128), dtype=torch.float32)
    if pinned:
        q_host, out_host = q_host.pin_memory(), out_host.pin_memory()
    call = ad.PreparedPagedDecodeHost(q_host, torch.empty_like(inp.q, device="cuda"), kp, vp, cp,
                                      bt, lens, w.L, 64, inp.t, ws,
                                      torch.empty((w.B, w.Hq, 128), device="cuda"), out_host,
                                      stream=torch.cuda.current_stream())
    for _ in range(2):
        out_host.zero_()
        call()
        torch.cuda.synchronize()
        assert torch.equal(out_host, want)
    ad.check_workspace(ws)

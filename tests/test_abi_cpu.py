"""The C ABI on a machine without a GPU: the library loads, exports every entry point
declared in include/adamas.h, and rejects bad arguments on the host before any
launch (none of these calls reaches a kernel)."""
import math

import pytest

import token_level_sparse_fwht_b200 as ad
from token_level_sparse_fwht_b200 import (OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, F32, BF16)

A = 1 << 20          # a fake, 256-byte aligned "device" address; never dereferenced
MIS = A + 1          # misaligned


def test_library_exports_every_header_symbol():
    lib = ad.lib()
    syms = ad.header_symbols()
    assert "adamas_decode_step" in syms and "adamas_encode_keys" in syms
    for s in syms:
        assert hasattr(lib, s), s
    assert lib.adamas_abi_version() == 2


def test_status_strings():
    assert ad.status_string(OK) == "ok"
    assert "invalid" in ad.status_string(ERR_INVALID_ARG)
    assert ad.status_string(99) == "unknown status"


def _decode(**kw):
    a = dict(q=A, kc=A, v=A, codes=A, dt=BF16, B=1, Hq=32, Hkv=8, d=128, Lmax=4096, L=4096, k=128,
             t=1.0, ws=A, ws_bytes=0, idx=None, out=A, stream=None)
    a.update(kw)
    return ad.lib().adamas_decode_step(a["q"], a["kc"], a["v"], a["codes"], a["dt"], a["B"],
                                       a["Hq"], a["Hkv"], a["d"], a["Lmax"], a["L"], a["k"],
                                       a["t"], a["ws"], a["ws_bytes"], a["idx"], a["out"],
                                       a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), ERR_INVALID_ARG),
    (dict(out=None), ERR_INVALID_ARG),
    (dict(ws=None), ERR_INVALID_ARG),
    (dict(d=64), ERR_UNSUPPORTED),
    (dict(Hq=24, Hkv=8), ERR_UNSUPPORTED),       # G = 3
    (dict(Hq=30, Hkv=8), ERR_INVALID_ARG),       # Hq % Hkv != 0
    (dict(L=5000), ERR_INVALID_ARG),             # L > Lmax
    (dict(L=0), ERR_INVALID_ARG),
    (dict(k=0), ERR_INVALID_ARG),
    (dict(B=0), ERR_INVALID_ARG),
    (dict(t=-0.5), ERR_INVALID_ARG),
    (dict(t=math.nan), ERR_INVALID_ARG),
    (dict(t=math.inf), ERR_INVALID_ARG),
    (dict(dt=7), ERR_INVALID_ARG),
    (dict(q=MIS), ERR_INVALID_ARG),
    (dict(codes=A + 8), ERR_INVALID_ARG),
    (dict(ws=A + 16), ERR_INVALID_ARG),          # workspace needs 256-byte alignment
    (dict(idx=A + 2), ERR_INVALID_ARG),
    (dict(ws_bytes=128), ERR_INVALID_ARG),       # too small (needs 256)
])
def test_decode_rejects_before_launch(kw, status):
    assert _decode(**kw) == status


def test_encode_keys_rejects():
    f = ad.lib().adamas_encode_keys
    assert f(None, BF16, 1, 8, 128, 100, 0, 10, 1.0, A, None) == ERR_INVALID_ARG
    assert f(A, BF16, 1, 8, 128, 100, 95, 10, 1.0, A, None) == ERR_INVALID_ARG   # past Lmax
    assert f(A, BF16, 1, 8, 128, 100, -1, 10, 1.0, A, None) == ERR_INVALID_ARG
    assert f(A, BF16, 1, 8, 128, 100, 0, 0, 1.0, A, None) == ERR_INVALID_ARG
    assert f(A, BF16, 1, 8, 96, 100, 0, 10, 1.0, A, None) == ERR_UNSUPPORTED
    assert f(A, F32, 1, 8, 128, 100, 0, 10, -1.0, A, None) == ERR_INVALID_ARG
    assert f(MIS, F32, 1, 8, 128, 100, 0, 10, 1.0, A, None) == ERR_INVALID_ARG
    g = ad.lib().adamas_encode_queries
    assert g(A, BF16, 1, 32, 128, 1.0, None, None) == ERR_INVALID_ARG
    assert g(A, BF16, 0, 32, 128, 1.0, A, None) == ERR_INVALID_ARG


def test_select_and_attention_reject():
    s = ad.lib().adamas_select_topk
    assert s(None, A, 1, 32, 8, 100, 100, 10, A, 1 << 30, A, None) == ERR_INVALID_ARG
    assert s(A, A, 1, 32, 8, 100, 100, 10, A, 1 << 30, None, None) == ERR_INVALID_ARG
    assert s(A, A, 1, 32, 8, 100, 101, 10, A, 1 << 30, A, None) == ERR_INVALID_ARG
    assert s(A, A, 1, 48, 8, 100, 100, 10, A, 1 << 30, A, None) == ERR_UNSUPPORTED
    assert s(A, A, 1, 32, 8, 100, 100, 10, A, 16, A, None) == ERR_INVALID_ARG
    at = ad.lib().adamas_sparse_attention
    assert at(A, A, A, BF16, None, 1, 32, 8, 128, 100, 10, A, 1 << 30, A, None) == ERR_INVALID_ARG
    assert at(A, A, A, BF16, A, 1, 32, 8, 64, 100, 10, A, 1 << 30, A, None) == ERR_UNSUPPORTED
    assert at(A, A, A, BF16, A, 1, 32, 8, 128, 100, 10, A, 8, A, None) == ERR_INVALID_ARG
    assert at(A, A, A, BF16, A + 1, 1, 32, 8, 128, 100, 10, A, 1 << 30, A, None) == ERR_INVALID_ARG


def test_workspace_sizes_and_plan():
    n = ad.decode_workspace_bytes(1, 32, 8, 32768, 128)
    assert n > 0 and n % 256 == 0
    assert ad.lib().adamas_decode_workspace_bytes(1, 32, 8, 64, 32768, 128) == 0
    assert ad.lib().adamas_decode_workspace_bytes(1, 32, 8, 128, 0, 128) == 0
    assert ad.lib().adamas_sparse_attention_workspace_bytes(1, 32, 128) > 0
    assert ad.lib().adamas_sparse_attention_workspace_bytes(1, 32, 0) == 0
    # without a device the plan assumes a 148-SM B200 (its shared-memory cap and the
    # cluster occupancy it reports).  The 32K layer's 8 units: clusters of 10 (at most
    # 11 fit at once); the grid-wide kernel (18 CTAs of 1824 keys per unit) only on
    # request.  One kv head over 256K: the grid-wide kernel by default.
    p = ad.decode_plan(1, 32, 8, 32768, 128)
    assert p == {"ctas": 80, "cluster": 10, "tokens_per_cta": 3277,
                 "smem_bytes": p["smem_bytes"]} and p["smem_bytes"] <= 232448
    assert ad.decode_workspace_bytes(1, 32, 8, 32768, 128) == 256
    ad.set_decode_policy(ad.POLICY_FLAT)
    try:
        pf = ad.decode_plan(1, 32, 8, 32768, 128)
        assert pf == {"ctas": 144, "cluster": 1, "tokens_per_cta": 1824,
                      "smem_bytes": pf["smem_bytes"]}
        assert ad.decode_workspace_bytes(1, 32, 8, 32768, 128) > 256   # exchange scratch
    finally:
        ad.set_decode_policy(ad.POLICY_AUTO)
    long1 = ad.decode_plan(1, 4, 1, 262144, 128)
    assert long1["cluster"] == 1 and long1["ctas"] == 64 and long1["tokens_per_cta"] == 4096
    ad.set_decode_policy(ad.POLICY_CLUSTER)
    try:
        assert ad.decode_plan(1, 4, 1, 262144, 128)["cluster"] == 16
    finally:
        ad.set_decode_policy(ad.POLICY_AUTO)
    with pytest.raises(ad.AdamasError):
        ad.set_decode_policy(3)
    big = ad.decode_plan(8, 32, 8, 32768, 1024)         # 64 units: clusters of 2
    assert big["cluster"] == 2 and big["tokens_per_cta"] == 16384
    for args in [(4, 32, 8, 131072, 1024), (1, 32, 32, 131072, 1024), (1, 2, 1, 70000, 50),
                 (75, 4, 4, 64, 8), (1, 1, 1, 1024, 64)]:
        q = ad.decode_plan(*args)
        B, Hq, Hkv, L, k = args
        per_unit = q["ctas"] // (B * Hkv)
        assert q["ctas"] == B * Hkv * per_unit and q["cluster"] in (1, per_unit)
        assert 1 <= per_unit <= 148 and (q["cluster"] == 1 or q["cluster"] <= 16)
        assert q["tokens_per_cta"] * per_unit >= L and q["tokens_per_cta"] <= 65535
        assert q["smem_bytes"] <= 232448
    tiny = ad.decode_plan(3, 4, 4, 1, 1)                # L = 1: one key per unit
    assert tiny["cluster"] == 1 and tiny["tokens_per_cta"] == 1 and tiny["ctas"] == 12


def test_shared_entry_points_reject_and_plan():
    f = ad.lib().adamas_decode_step_shared
    args = [A, A, A, A, BF16, 1, 32, 8, 128, 4096, 4096, 128, 1.0, A, 1 << 30, None, A, None]
    bad = list(args); bad[0] = None
    assert f(*bad) == ERR_INVALID_ARG
    bad = list(args); bad[6] = 24                         # G = 3
    assert f(*bad) == ERR_UNSUPPORTED
    bad = list(args); bad[10] = 5000                      # L > Lmax
    assert f(*bad) == ERR_INVALID_ARG
    bad = list(args); bad[14] = 16                        # workspace too small
    assert f(*bad) == ERR_INVALID_ARG
    s = ad.lib().adamas_select_topk_shared
    assert s(None, A, 1, 32, 8, 100, 100, 10, A, 1 << 30, A, None) == ERR_INVALID_ARG
    assert s(A, A, 1, 48, 8, 100, 100, 10, A, 1 << 30, A, None) == ERR_UNSUPPORTED
    h = ad.lib().adamas_decode_step_shared_host
    assert h(None, A, A, A, A, BF16, 1, 32, 8, 128, 4096, 4096, 128, 1.0, A, 1 << 30, None, A,
             A, None) == ERR_INVALID_ARG
    # shared selection needs wider histograms (384 G + 1 bins) and, for G > 1, a
    # per-warp merge buffer for several heads: plans still fit the B200 cap
    for args in [(1, 32, 8, 32768, 128), (4, 32, 8, 131072, 1024), (1, 64, 8, 65536, 256),
                 (2, 16, 8, 10000, 100), (1, 8, 8, 4096, 64), (1, 2, 1, 70000, 50)]:
        q = ad.decode_plan_shared(*args)
        B, Hq, Hkv, L, k = args
        assert q["ctas"] == B * Hkv * q["cluster"] and 1 <= q["cluster"] <= 16
        assert q["tokens_per_cta"] * q["cluster"] >= L and q["tokens_per_cta"] <= 65535
        assert q["smem_bytes"] <= 232448
    assert ad.decode_plan_shared(1, 32, 8, 32768, 128)["cluster"] == 10   # at most 11 fit


def test_varlen_and_paged_entry_points_reject():
    v = ad.lib().adamas_decode_step_varlen
    ok = [A, A, A, A, BF16, 2, 32, 8, 128, 4096, A, 128, 1.0, 0, A, 1 << 30, None, A, None]
    for i, bad in [(10, None), (10, A + 2), (13, 2), (0, None), (8, 64), (9, 0)]:
        args = list(ok); args[i] = bad
        want = ERR_UNSUPPORTED if i == 8 else ERR_INVALID_ARG
        assert v(*args) == want, (i, bad)
    p = ad.lib().adamas_decode_step_paged
    ok = [A, A, A, A, BF16, 2, 32, 8, 128, 16, 100, A, 64, A, 1024, 128, 1.0, 0, A, 1 << 30, None,
          A, None]
    cases = [
        (9, 24),        # page size not a power of two
        (9, 0),
        (9, 1 << 21),   # page size above 2^20
        (10, 0),        # no pages
        (11, None),     # no block table
        (13, None),     # no lengths
        (12, 63),       # 63 blocks x 16 < 1024 positions
        (14, 0),
        (17, 5),        # shared flag not 0/1
        (11, A + 2),    # misaligned table
    ]
    for i, bad in cases:
        args = list(ok); args[i] = bad
        assert p(*args) == ERR_INVALID_ARG, (i, bad)
    args = list(ok); args[8] = 96
    assert p(*args) == ERR_UNSUPPORTED
    s = ad.lib().adamas_select_topk_paged
    assert s(None, A, 2, 32, 8, 16, 100, A, 64, A, 1024, 128, 0, A, 1 << 30, A, None) == ERR_INVALID_ARG
    assert s(A, A, 2, 32, 8, 16, 100, A, 64, A, 1024, 128, 0, A, 1 << 30, None, None) == ERR_INVALID_ARG
    e = ad.lib().adamas_encode_pages
    assert e(None, BF16, 8, 128, 16, 100, None, 0, 1.0, A, None) == ERR_INVALID_ARG
    assert e(A, BF16, 8, 64, 16, 100, None, 0, 1.0, A, None) == ERR_UNSUPPORTED
    assert e(A, BF16, 8, 128, 16, 0, None, 0, 1.0, A, None) == ERR_INVALID_ARG
    assert e(A, BF16, 8, 128, 16, 100, A, -1, 1.0, A, None) == ERR_INVALID_ARG


def test_paging_helper_layout():
    """workloads.paging puts position p of sequence b at page table[b, p // page], row
    p % page, with distinct pages per block and spare pages left at the fill value."""
    import torch
    from workloads.paging import make_block_table, scatter_to_pages
    lens = [37, 0, 16]
    pc = make_block_table(lens, 40, 16, seed=3, spare=2)
    assert pc.num_pages == 3 + 0 + 1 + 2
    used = pc.block_table[pc.block_table >= 0].tolist()
    assert len(used) == len(set(used)) == 4
    x = torch.arange(3 * 2 * 40, dtype=torch.float32).reshape(3, 2, 40, 1)
    pool = scatter_to_pages(x, pc, fill=-1)
    for b, L in enumerate(lens):
        for p in range(L):
            page = int(pc.block_table[b, p // 16])
            assert torch.equal(pool[page, :, p % 16], x[b, :, p])
    spare = set(range(pc.num_pages)) - set(used)
    assert all((pool[s] == -1).all() for s in spare)


def test_absmax_entry_points_reject():
    ek = ad.lib().adamas_encode_keys_absmax
    for ratio in (0.0, -0.5, 1.5, math.nan, math.inf):
        assert ek(A, BF16, 1, 8, 128, 100, 0, 10, ratio, A, None) == ERR_INVALID_ARG, ratio
    assert ek(A, BF16, 1, 8, 96, 100, 0, 10, 0.5, A, None) == ERR_UNSUPPORTED
    eq = ad.lib().adamas_encode_queries_absmax
    assert eq(A, BF16, 1, 32, 128, 0.0, A, None) == ERR_INVALID_ARG
    assert eq(A, BF16, 1, 32, 128, 0.5, None, None) == ERR_INVALID_ARG
    ep = ad.lib().adamas_encode_pages_absmax
    assert ep(A, BF16, 8, 128, 16, 100, None, 0, 2.0, A, None) == ERR_INVALID_ARG
    d = ad.lib().adamas_decode_step_absmax
    ok = [A, A, A, A, BF16, 1, 32, 8, 128, 4096, 4096, 128, 0.5, 0, A, 1 << 30, None, A, None]
    for i, bad in [(12, 0.0), (12, 1.01), (13, 3), (0, None), (14, A + 16), (15, 16)]:
        args = list(ok); args[i] = bad
        assert d(*args) == ERR_INVALID_ARG, (i, bad)
    args = list(ok); args[6] = 24
    assert d(*args) == ERR_UNSUPPORTED


def test_context_parallel_entry_points_reject():
    assert ad.lib().adamas_cp_hist_elems(2, 32, 8, 0) == 2 * 32 * 385
    assert ad.lib().adamas_cp_hist_elems(2, 32, 8, 1) == 2 * 8 * (384 * 4 + 1)
    assert ad.lib().adamas_cp_hist_elems(2, 24, 8, 0) == 0
    h = ad.lib().adamas_cp_histograms
    assert h(None, A, BF16, 1, 32, 8, 128, 100, 100, 10, 1.0, 0, A, 1 << 30, A, None) == ERR_INVALID_ARG
    assert h(A, A, BF16, 1, 32, 8, 128, 100, 100, 10, 1.0, 2, A, 1 << 30, A, None) == ERR_INVALID_ARG
    at = ad.lib().adamas_cp_attend
    ok = [A, A, A, A, BF16, 1, 32, 8, 128, 100, 100, 300, 100, 10, 1.0, 0, A, 2, 1, A, 1 << 30,
          None, A, None]
    for i, bad in [(12, -1), (11, 150), (11, 1 << 31), (16, None), (22, None), (17, 0), (18, 2),
                   (18, -1)]:
        args = list(ok); args[i] = bad
        assert at(*args) == ERR_INVALID_ARG, (i, bad)
    c = ad.lib().adamas_cp_combine
    assert c(A, 0, 1, 32, A, None) == ERR_INVALID_ARG
    assert c(None, 2, 1, 32, A, None) == ERR_INVALID_ARG


def test_context_parallel_workspace_size():
    # the error word plus, per CTA, its distances (u16 per key and selection head) and
    # cumulative histograms
    # (a context-parallel slice always runs on thread-block clusters)
    n = ad.lib().adamas_cp_workspace_bytes(1, 32, 8, 128, 16384, 128, 0)
    ad.set_decode_policy(ad.POLICY_CLUSTER)
    try:
        p = ad.decode_plan(1, 32, 8, 16384, 128)
    finally:
        ad.set_decode_policy(ad.POLICY_AUTO)
    per_cta = 4 * ((p["tokens_per_cta"] + 7) // 8 * 8) * 2 + 4 * 388 * 4
    assert n == 256 + p["ctas"] * per_cta
    assert ad.lib().adamas_cp_workspace_bytes(1, 32, 8, 128, 16384, 128, 2) == 0
    assert ad.lib().adamas_cp_workspace_bytes(1, 32, 8, 64, 16384, 128, 0) == 0


def test_scratch_distance_plan_workspace():
    # many units over a long context: the plan keeps each CTA's distances (u16 per key
    # and head) in the workspace, so fewer, longer CTAs run in one wave
    # (check the size rule whichever plan is chosen)
    for B, Hq, Hkv, L, k in [(4, 32, 8, 131072, 1024), (8, 32, 8, 131072, 256),
                             (2, 64, 8, 131072, 512)]:
        p = ad.decode_plan(B, Hq, Hkv, L, k)
        n = ad.decode_workspace_bytes(B, Hq, Hkv, L, k)
        stride = (p["tokens_per_cta"] + 7) // 8 * 8
        assert n in (256, 256 + p["ctas"] * (Hq // Hkv) * stride * 2)
        # a plan without scratch must fit its distances in shared memory
        if n == 256:
            assert (Hq // Hkv) * stride * 2 < p["smem_bytes"]
    ad.set_decode_policy(ad.POLICY_CLUSTER)
    try:
        assert ad.decode_workspace_bytes(1, 32, 8, 32768, 128) == 256   # fits on chip
    finally:
        ad.set_decode_policy(ad.POLICY_AUTO)


def test_copy_fault_hook_rejects_bad_arguments():
    # the bounded-wait test hook: byte counts must be multiples of 16 in [0, 2^20]
    # (host-side checks only)
    assert ad.lib().adamas_test_set_copy_fault(8) == ERR_INVALID_ARG
    assert ad.lib().adamas_test_set_copy_fault(-16) == ERR_INVALID_ARG
    assert ad.lib().adamas_test_set_copy_fault((1 << 20) + 16) == ERR_INVALID_ARG
    assert ad.lib().adamas_test_set_copy_fault(0) == OK

"""The bounded-wait error path of the decode kernel on the GPU, without a fault.

Every wait of the kernel on a bulk copy into shared memory is bounded; when one gives
up, the kernel records it in the workspace error word, stops issuing copies, waits
(bounded again) for the ones in flight and returns.  The test hook
adamas_test_set_copy_fault arms the first code chunk's barrier for 16 bytes the copy
never delivers, so the wait runs into its 1 s limit on purpose; the host must then read
ADAMAS_ERR_TIMEOUT, and the next, normal launch on the same device must be correct."""
import numpy as np
import pytest
import torch

import token_level_sparse_fwht_b200 as ad
from gpu_helpers import check_decode_head, f64, oracle_codes, upload
from workloads import WORKLOADS, generate

pytestmark = pytest.mark.gpu


def test_copy_wait_timeout_is_reported_and_device_stays_usable():
    w = WORKLOADS[2].scaled(L=3000, Hq=8, Hkv=2)
    inp = generate(w, "cpu")
    kc = oracle_codes(inp.k_cache, inp.t)
    q, kcache, vcache, codes = inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(), upload(kc)
    ad.set_decode_policy(ad.POLICY_CLUSTER)
    try:
        ws = ad.decode_workspace(w.B, w.Hq, w.Hkv, w.L, 64)
        ad.test_set_copy_fault(16)
        try:
            ad.decode_step(q, kcache, vcache, codes, w.L, 64, inp.t, ws)
            torch.cuda.synchronize()
        finally:
            ad.test_set_copy_fault(0)
        with pytest.raises(ad.AdamasError) as e:
            ad.check_workspace(ws)
        assert e.value.status == ad.ERR_TIMEOUT
        # the same shape again, normal operation: a fresh workspace reports no error and
        # the results match the oracle
        ws2 = ad.decode_workspace(w.B, w.Hq, w.Hkv, w.L, 64)
        idx = torch.empty((w.B, w.Hq, 64), dtype=torch.int32, device="cuda")
        out = ad.decode_step(q, kcache, vcache, codes, w.L, 64, inp.t, ws2, idx_out=idx)
        torch.cuda.synchronize()
        ad.check_workspace(ws2)
    finally:
        ad.set_decode_policy(ad.POLICY_AUTO)
    idx, out, qq = idx.cpu().numpy(), out.cpu().numpy(), f64(inp.q)
    for h in range(w.Hq):
        check_decode_head(idx[0, h], out[0, h], qq[0, h], f64(inp.k_cache[0, h // 4]),
                          f64(inp.v_cache[0, h // 4]), kc[0, h // 4], 64, inp.t)

"""Context-parallel decode protocol on CPU (gloo, world sizes 2 and 3).

Each process is one rank holding a contiguous slice of the context and runs
token_level_sparse_fwht_b200.context_parallel.ContextParallelDecode with a float64
numpy model of the kernel steps written from the step's definition (cumulative
histograms of the slice's distances; the slice's share of the global top-k from the
other and the lower ranks' counts, ties to lower positions; a log2-domain softmax
partial; the log-sum-exp merge).  The merged output and positions must
equal oracle.decode_step (or decode_step_shared) over the whole context: this
checks the protocol, the collective order and the phase split on the host; the
CUDA kernels of each step are checked on the GPU (tests/test_gpu_context_parallel.py).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

LOG2E = 1.4426950408889634


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class NumpyOps:
    """Float64 model of the kernel steps (CPU tensors in, CPU tensors out)."""

    def __init__(self, oracle):
        self.o = oracle

    def _dist(self, q, codes, L, t, shared):
        o = self.o
        qn = q.double().numpy()
        cq = o.unpack_codes(o.encode(qn, t))
        ck = o.unpack_codes(codes.numpy()[:, :, :L])
        B, Hq, _ = qn.shape
        Hkv = ck.shape[1]
        G = Hq // Hkv
        d = np.stack([np.stack([o.manhattan(cq[b, h], ck[b, h // G]) for h in range(Hq)])
                      for b in range(B)])                      # [B, Hq, L]
        if shared:
            d = d.reshape(B, Hkv, G, L).sum(2)
        return d

    def histograms(self, q, codes, L, k, t, ws, shared):
        d = self._dist(q, codes, L, t, shared)
        G = q.shape[1] // codes.shape[1]
        bins = 384 * G + 1 if shared else 385
        h = np.zeros(d.shape[:2] + (bins,), np.int64)
        for b in range(d.shape[0]):
            for r in range(d.shape[1]):
                h[b, r] = np.cumsum(np.bincount(d[b, r], minlength=bins))
        return torch.from_numpy(h.astype(np.int32))

    def attend(self, q, K, V, codes, L, L_total, pos_offset, k, t, hist_all, rank, ws, shared,
               idx_out):
        d = self._dist(q, codes, L, t, shared)
        cum = hist_all.numpy().astype(np.int64)                  # [W, B, rows, bins]
        ext = np.stack([cum.sum(0) - cum[rank], cum[:rank].sum(0)])
        qn = q.double().numpy()
        Kn, Vn = K.double().numpy(), V.double().numpy()
        B, Hq, _ = qn.shape
        Hkv = Kn.shape[1]
        G = Hq // Hkv
        keff = min(k, L_total)
        part = np.zeros((B, Hq, 132))
        sel_of = {}
        for b in range(B):
            for r in range(d.shape[1]):
                own = np.cumsum(np.bincount(d[b, r], minlength=ext.shape[-1]))
                tot = own + ext[0, b, r]
                dstar = int(np.argmax(tot >= keff))
                below = lambda c: int(c[dstar - 1]) if dstar > 0 else 0
                less = below(tot)
                need = keff - less
                eq_lower = int(ext[1, b, r, dstar]) - below(ext[1, b, r])
                take = min(max(need - eq_lower, 0), int(own[dstar]) - below(own))
                lt = np.nonzero(d[b, r] < dstar)[0]
                eq = np.nonzero(d[b, r] == dstar)[0][:take]
                sel = np.sort(np.concatenate([lt, eq]))
                base = below(ext[1, b, r]) + min(eq_lower, need)
                if idx_out is not None and len(sel):
                    idx_out[b, r, base:base + len(sel)] = torch.from_numpy(
                        (sel + pos_offset).astype(np.int32))
                sel_of[(b, r)] = sel
        for b in range(B):
            for h in range(Hq):
                sel = sel_of[(b, h // G if shared else h)]
                if len(sel) == 0:
                    part[b, h, 0] = -np.inf
                    continue
                s = Kn[b, h // G, sel] @ qn[b, h] / np.sqrt(128) * LOG2E
                m = s.max()
                p = np.exp2(s - m)
                part[b, h, 0], part[b, h, 1] = m, p.sum()
                part[b, h, 4:] = p @ Vn[b, h // G, sel]
        return torch.from_numpy(part)

    def combine(self, partials_all):
        p = partials_all.numpy()                                  # [W, B, Hq, 132]
        live = p[..., 1] > 0
        M = np.where(live, p[..., 0], -np.inf).max(0)
        e = np.where(live, np.exp2(p[..., 0] - M), 0.0)
        Ls = (p[..., 1] * e).sum(0)
        A = (p[..., 4:] * e[..., None]).sum(0)
        return torch.from_numpy(np.where(Ls[..., None] > 0, A / Ls[..., None], 0.0))


def _inputs():
    import workloads
    w = workloads.WORKLOADS[2].scaled(B=2, Hq=8, Hkv=2, L=300)
    inp = workloads.generate(w, "cpu")
    return w, inp


def _worker(rank, world, port, cuts, k, shared, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    import oracle
    from token_level_sparse_fwht_b200.context_parallel import ContextParallelDecode
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, inp = _inputs()
        codes = torch.from_numpy(oracle.encode(inp.k_cache.double().numpy(), inp.t))
        lo, hi = cuts[rank], cuts[rank + 1]
        step = ContextParallelDecode(ops=NumpyOps(oracle))
        o, idx = step(inp.q, inp.k_cache[:, :, lo:hi], inp.v_cache[:, :, lo:hi],
                      codes[:, :, lo:hi].contiguous(), hi - lo, w.L, lo, k, inp.t, None,
                      shared=shared, want_idx=True)
        out[rank] = (o.numpy(), idx.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cuts,k,shared", [
    ([0, 150, 300], 37, False),
    ([0, 40, 260, 300], 64, False),       # uneven slices, three ranks
    ([0, 100, 300], 50, True),            # shared selection
    ([0, 290, 300], 200, False),          # a slice shorter than its share of the budget
])
def test_context_parallel_matches_whole_context(cuts, k, shared):
    import oracle
    world = len(cuts) - 1
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), cuts, k, shared, out), nprocs=world, join=True)
    w, inp = _inputs()
    q, K, V = (x.double().numpy() for x in (inp.q, inp.k_cache, inp.v_cache))
    step = oracle.decode_step_shared if shared else oracle.decode_step
    want_idx, want_out = step(q, K, V, k, inp.t)
    for r in range(world):
        got_out, got_idx = out[r]
        assert np.array_equal(got_idx, want_idx), r
        assert np.abs(got_out - want_out).max() < 1e-9, r

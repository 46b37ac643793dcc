"""Context-parallel decode step: one rank per GPU, each holding a contiguous slice of
the context (lower ranks hold lower positions).

The step (see include/adamas.h, adamas_cp_*):
  1. cumulative histograms of the slice's distances (fused decode kernel, phase 1),
  2. all-gather of the histograms,
  3. selection of this slice's share of the global top-k (the other ranks' counts
     added at the bins the search reads), attention over it and one softmax partial
     per query head (fused decode kernel, phase 2),
  4. all-gather of the partials,
  5. the log-sum-exp merge of the partials into the output.
Optionally the selected positions are merged by an all-reduce (max) of -1-filled
index arrays.  Every rank takes the same collective steps in the same order.

The kernel calls and the process group are parameters, so the protocol can be run
by CPU processes (gloo) with a stand-in for the kernels; the default `ops` is the
CUDA library.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


class CudaOps:
    """The kernel steps of the library (token_level_sparse_fwht_b200)."""

    def __init__(self):
        import token_level_sparse_fwht_b200 as ad
        self.ad = ad

    def histograms(self, q, codes, L, k, t, ws, shared):
        return self.ad.cp_histograms(q, codes, L, k, t, ws, shared=shared)

    def attend(self, q, k_cache, v_cache, codes, L, L_total, pos_offset, k, t, hist_all, rank,
               ws, shared, idx_out):
        return self.ad.cp_attend(q, k_cache, v_cache, codes, L, L_total, pos_offset, k, t,
                                 hist_all, rank, ws, shared=shared, idx_out=idx_out)

    def combine(self, partials_all):
        return self.ad.cp_combine(partials_all)


class ContextParallelDecode:
    """One rank's side of a context-parallel decode step."""

    def __init__(self, group=None, ops=None):
        self.group = group
        self.ops = ops if ops is not None else CudaOps()
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def _all_gather(self, x: torch.Tensor) -> torch.Tensor:
        parts = [torch.empty_like(x) for _ in range(self.world)]
        dist.all_gather(parts, x.contiguous(), group=self.group)
        return torch.stack(parts)

    def __call__(self, q, k_cache, v_cache, codes, L: int, L_total: int, pos_offset: int, k: int,
                 t: float, ws, shared: bool = False, want_idx: bool = False):
        """Returns out [B, Hq, 128] float32 (and, with want_idx, the merged positions
        [B, rows, min(k, L_total)] int32, -1 past the selection)."""
        B, Hq, _ = q.shape
        Hkv = k_cache.shape[1]
        hist = self.ops.histograms(q, codes, L, k, t, ws, shared)
        hist_all = self._all_gather(hist)
        idx = None
        if want_idx:
            rows = Hkv if shared else Hq
            idx = torch.full((B, rows, min(k, L_total)), -1, dtype=torch.int32, device=q.device)
        partial = self.ops.attend(q, k_cache, v_cache, codes, L, L_total, pos_offset, k, t,
                                  hist_all, self.rank, ws, shared, idx)
        partials_all = self._all_gather(partial)
        out = self.ops.combine(partials_all)
        if want_idx:
            dist.all_reduce(idx, op=dist.ReduceOp.MAX, group=self.group)
            return out, idx
        return out

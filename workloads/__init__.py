"""Seeded synthetic inputs for the Adamas decode workloads.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no Hadamard transform, no codes, no distances, no softmax).
Both the CUDA path's tests / bench and the float64 oracle consume its tensors.

Recipe (stands in for the real-model workloads the pages evaluate on: Llama-3.1-8B
and Yarn-Llama-2-7B-128K, whose weights and datasets are not available here):

* torch generator seeded with ``1000 * config + layer`` on the requested device;
* K, V and q drawn i.i.d. N(0, 1) in float32, then cast to the stored dtype
  (round-to-nearest-even bf16, or kept float32 for the single-head case);
* "outlier channels": 4 distinct channel indices per layer, the same for K, V and
  q, multiplied by 10 (the blog's section 2.1 motivates H by such outliers);
* planted keys: k_j = q_h + 0.1 * N(0, 1) at distinct seeded positions, for the
  kv head that query head h reads.

The bucket threshold is t = 0.5 * sigma, sigma the per-coordinate standard
deviation of H x under this recipe: 1 without outliers, sqrt((124 + 4*100)/128)
with four x10 channels.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch

HEAD_DIM = 128
N_OUTLIER = 4
OUTLIER_SCALE = 10.0


def sigma_of(outliers: bool) -> float:
    if not outliers:
        return 1.0
    return math.sqrt((HEAD_DIM - N_OUTLIER + N_OUTLIER * OUTLIER_SCALE ** 2) / HEAD_DIM)


@dataclass(frozen=True)
class Workload:
    name: str
    config: int
    B: int
    Hq: int
    Hkv: int
    L: int
    budgets: tuple
    dtype: torch.dtype
    outliers: bool
    planted: int = 0            # planted keys per query head
    layers: int = 1
    append: int = 0             # tokens per sequence encoded inside the timed step
    d: int = HEAD_DIM

    @property
    def t(self) -> float:
        return 0.5 * sigma_of(self.outliers)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == torch.float32 else 2

    def algorithmic_bytes(self, k: int, shared: bool = False) -> int:
        """Bytes one decode step must move per layer: codes scanned, selected K+V
        rows per query head (per kv head when the selection is shared by the
        group), q read and fp32 output written."""
        k_eff = min(k, self.L)
        e = self.elem_bytes
        sel_rows = self.B * (self.Hkv if shared else self.Hq) * k_eff
        return (self.B * self.Hkv * self.L * (self.d // 4)
                + sel_rows * 2 * self.d * e
                + self.B * self.Hq * self.d * e
                + self.B * self.Hq * self.d * 4)

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    1: Workload("single-head d128 L1024 fp32, 4 planted keys", 1, B=1, Hq=1, Hkv=1, L=1024,
                budgets=(64,), dtype=torch.float32, outliers=False, planted=4),
    2: Workload("llama3.1-8b-layer B1 32q/8kv L32768 bf16", 2, B=1, Hq=32, Hkv=8, L=32768,
                budgets=(64, 128, 256, 1024), dtype=torch.bfloat16, outliers=True),
    3: Workload("llama3.1-8b-layer B8 32q/8kv L32768 bf16 +512 append", 3, B=8, Hq=32, Hkv=8,
                L=32768, budgets=(256, 1024), dtype=torch.bfloat16, outliers=True, append=512),
    4: Workload("llama2-7b-mha B1 32x128 L131072 bf16, 16 needles", 4, B=1, Hq=32, Hkv=32,
                L=131072, budgets=(128, 1024), dtype=torch.bfloat16, outliers=True, planted=16),
    5: Workload("llama3.1-8b 32 layers B4 32q/8kv L131072 bf16", 5, B=4, Hq=32, Hkv=8,
                L=131072, budgets=(1024,), dtype=torch.bfloat16, outliers=True, layers=32),
}


@dataclass
class Inputs:
    q: torch.Tensor            # [B, Hq, d]
    k_cache: torch.Tensor      # [B, Hkv, Lmax, d]
    v_cache: torch.Tensor      # [B, Hkv, Lmax, d]
    t: float
    outlier_channels: torch.Tensor
    planted: torch.Tensor = field(default=None)   # [B, Hq, n] positions, or None


def seed_of(config: int, layer: int = 0) -> int:
    return 1000 * config + layer


def _normal(shape, gen, device, chunk_elems=1 << 27):
    """float32 N(0,1) of `shape`, drawn in chunks along dim 0 to bound memory."""
    out = torch.empty(shape, dtype=torch.float32, device=device)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, chunk_elems):
        e = min(n, s + chunk_elems)
        flat[s:e] = torch.randn(e - s, generator=gen, device=device, dtype=torch.float32)
    return out


def _filled(shape, gen, device, dtype, scale_ch, chunk_rows=1 << 20):
    """N(0,1) cast to `dtype`, outlier channels scaled, built in row chunks so that a
    64 GiB cache never needs a float32 copy of itself."""
    out = torch.empty(shape, dtype=dtype, device=device)
    rows = out.view(-1, shape[-1])
    for s in range(0, rows.shape[0], chunk_rows):
        e = min(rows.shape[0], s + chunk_rows)
        blk = torch.randn((e - s, shape[-1]), generator=gen, device=device,
                          dtype=torch.float32)
        if scale_ch is not None:
            blk[:, scale_ch] *= OUTLIER_SCALE
        rows[s:e] = blk.to(dtype)
    return out


def generate(w: Workload, device="cpu", layer: int = 0, Lmax: int | None = None) -> Inputs:
    """Seeded inputs of workload `w` (one layer) on `device`."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed_of(w.config, layer))
    Lmax = w.L if Lmax is None else Lmax
    if Lmax < w.L:
        raise ValueError("Lmax < L")
    d = w.d
    ch = None
    if w.outliers:
        ch = torch.randperm(d, generator=gen, device=device)[:N_OUTLIER].sort().values
    q = _filled((w.B, w.Hq, d), gen, device, w.dtype, ch)
    k = _filled((w.B, w.Hkv, Lmax, d), gen, device, w.dtype, ch)
    v = _filled((w.B, w.Hkv, Lmax, d), gen, device, w.dtype, ch)
    planted = None
    if w.planted:
        G = w.G
        planted = torch.empty((w.B, w.Hq, w.planted), dtype=torch.int64, device=device)
        for b in range(w.B):
            for kvh in range(w.Hkv):
                # distinct positions across the whole group, so the planted keys of
                # one query head never overwrite another head's
                pos = torch.randperm(w.L, generator=gen, device=device)[: G * w.planted]
                for gi in range(G):
                    h = kvh * G + gi
                    p = pos[gi * w.planted:(gi + 1) * w.planted].sort().values
                    planted[b, h] = p
                    noise = torch.randn((w.planted, d), generator=gen, device=device,
                                        dtype=torch.float32)
                    rows = q[b, h].float()[None, :] + 0.1 * noise
                    k[b, kvh, p] = rows.to(w.dtype)
    return Inputs(q=q, k_cache=k, v_cache=v, t=float(w.t), outlier_channels=ch,
                  planted=planted)


def replicas_for_l2(bytes_per_replica: int, l2_bytes: int, factor: float = 2.0) -> int:
    """How many independent replicas make the rotated working set >= factor x L2."""
    if bytes_per_replica <= 0:
        return 1
    return max(1, math.ceil(factor * l2_bytes / bytes_per_replica))

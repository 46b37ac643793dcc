"""Shared helpers of the GPU parity tests (the CUDA path vs the float64 oracle).

Inputs come from the seeded generators in `workloads`; expected values come from
`oracle` only.  Oracle outputs may be uploaded to the GPU as inputs (for example
the oracle's key codes), never the other way round.
"""
from __future__ import annotations

import itertools

import numpy as np
import torch

import oracle

ATOL_OUT = 2e-3          # attention output tolerance (max-abs)
NEAR = 1e-4              # a coordinate this close to a threshold may take either code
MAX_MISMATCH_FRACTION = 1e-4


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def oracle_codes(x: torch.Tensor, t: float) -> np.ndarray:
    return oracle.encode(f64(x), t)


def encoder_mismatch(gpu_codes: np.ndarray, x: torch.Tensor, t: float):
    """Compares GPU packed codes with the oracle's.  Returns (n_mismatch_far,
    mismatch_fraction, near_fraction): mismatches at coordinates farther than NEAR
    from a threshold (must be 0), the fraction of coordinates whose code differs
    (must stay below MAX_MISMATCH_FRACTION), and, for the report, the fraction of
    coordinates that lie within NEAR of a threshold (a property of the data)."""
    y = oracle.hadamard_rotate(f64(x))
    want = oracle.bucketize(y, t)
    got = oracle.unpack_codes(gpu_codes)
    near = oracle.threshold_margin(y, t) < NEAR
    diff = got != want
    return int((diff & ~near).sum()), float(diff.mean()), float(near.mean())


def query_alternatives(q_vec: np.ndarray, t: float, max_alts: int = 16):
    """Packed query codes the kernel may legitimately compute: the oracle's code,
    with every coordinate within NEAR of a threshold taking either neighbouring
    bucket.  Returns a list of packed codes (the oracle's own first)."""
    y = oracle.hadamard_rotate(q_vec)
    base = oracle.bucketize(y, t)
    margin = oracle.threshold_margin(y, t)
    amb = np.nonzero(margin < NEAR)[0]
    tt = float(np.float32(t))
    options = []
    for i in amb:
        thr = min((-tt, 0.0, tt), key=lambda th: abs(y[i] - th))
        lo = oracle.bucketize(np.array([thr - 1e-9]), t)[0]
        hi = oracle.bucketize(np.array([thr]), t)[0]
        options.append((int(i), [int(lo), int(hi)]))
    alts = [oracle.pack_codes(base)]
    for combo in itertools.product(*[o[1] for o in options]):
        c = base.copy()
        for (i, _), v in zip(options, combo):
            c[i] = v
        p = oracle.pack_codes(c)
        if not any(np.array_equal(p, a) for a in alts):
            alts.append(p)
        if len(alts) >= max_alts:
            break
    return alts


def check_decode_head(gpu_idx, gpu_out, q_vec, K_rows, V_rows, key_codes_rows, k, t):
    """One (batch, query head) of a decode step: the GPU selection must equal the
    oracle's for one admissible query code, and the output must be within ATOL_OUT
    of the oracle's attention over that selection.  Returns max-abs error."""
    errs = []
    for qc in query_alternatives(q_vec, t):
        sel, out, _ = oracle.decode_head(q_vec, K_rows, V_rows, k, t,
                                         key_codes_rows=key_codes_rows, query_code=qc)
        if gpu_idx is not None and not np.array_equal(np.asarray(gpu_idx, np.int64), sel):
            continue
        err = float(np.abs(np.asarray(gpu_out, np.float64) - out).max())
        errs.append(err)
        if err <= ATOL_OUT:
            return err
    raise AssertionError(
        f"no admissible oracle selection matches (errors of matching selections: {errs})")


def upload(x, device="cuda"):
    if isinstance(x, np.ndarray):
        x = torch.from_numpy(np.ascontiguousarray(x))
    return x.to(device).contiguous()


def group_alternatives(qg: np.ndarray, t: float, cap: int = 64):
    """Packed query codes [G, 32] the kernel may compute for one group qg [G, 128]:
    every combination of the heads' admissible codes (at most `cap`)."""
    per_head = [query_alternatives(qg[g], t) for g in range(qg.shape[0])]
    for combo in itertools.islice(itertools.product(*per_head), cap):
        yield np.stack(combo)


def check_decode_unit_shared(gpu_idx, gpu_out, qg, Kg, Vg, kcg, k, t):
    """One (batch, kv head) of a shared-selection step, given the group's queries qg
    [G, 128], the unit's rows Kg, Vg [L, 128] and key codes kcg [L, 32]: the GPU's
    selection must equal the oracle's for one admissible combination of the group's
    query codes, and its outputs [G, 128] must be within ATOL_OUT of that selection's
    attention.  Returns the max-abs error."""
    errs = []
    for qcg in group_alternatives(qg, t):
        idx, out = oracle.decode_step_shared(qg[None], Kg[None, None], Vg[None, None], k, t,
                                             key_codes=kcg[None, None], query_codes=qcg[None])
        if not np.array_equal(np.asarray(gpu_idx, np.int64), idx[0, 0]):
            continue
        err = float(np.abs(np.asarray(gpu_out, np.float64) - out[0]).max())
        errs.append(err)
        if err <= ATOL_OUT:
            return err
    raise AssertionError(f"no admissible oracle selection matches: {errs}")

"""Plant plausible mistakes in the oracle (CPU only) and check the pins catch each.

Every mutation replaces one oracle function for the duration of one test; at least
one of the pin checks in tests/pins.py must then fail.
"""
import numpy as np
import pytest

import oracle.adamas_ref as ref
from pins import ALL_CHECKS

_orig = {name: getattr(ref, name) for name in (
    "sylvester_hadamard", "hadamard_rotate", "bucketize", "pack_codes", "unpack_codes",
    "manhattan", "select_topk", "sparse_attention", "decode_step", "decode_step_shared",
    "decode_step_varlen", "absmax_thresholds", "bucketize_per_vector", "encode_absmax",
    "decode_step_absmax", "threshold_margin", "decode_head")}


def _h_or(n=128):                      # popcount(i | j) instead of i & j
    idx = np.arange(n)
    o = np.bitwise_or.outer(idx, idx)
    par = np.zeros_like(o)
    for b in range(int(n).bit_length()):
        par ^= (o >> b) & 1
    return np.where(par == 1, -1, 1).astype(np.int64)


def _rotate_unscaled(x):               # forgot the 1/sqrt(d)
    x = np.asarray(x, np.float64)
    return x @ _orig["sylvester_hadamard"](x.shape[-1]).T.astype(np.float64)


def _rotate_reversed(x):               # output coordinates in reversed order
    return _orig["hadamard_rotate"](x)[..., ::-1]


def _bucket_le(y, t):                  # "<=" instead of "<"
    y = np.asarray(y, np.float64)
    t = float(np.float32(t))
    c = np.full(y.shape, 3, np.uint8)
    c[y <= t] = 2
    c[y <= 0] = 1
    c[y <= -t] = 0
    return c


def _bucket_swapped(y, t):             # buckets 1 and 2 swapped
    c = _orig["bucketize"](y, t)
    out = c.copy()
    out[c == 1] = 2
    out[c == 2] = 1
    return out


def _pack_msb_first(codes):            # first coordinate in the top bits
    c = np.asarray(codes, np.uint8)
    c = c.reshape(c.shape[:-1] + (c.shape[-1] // 4, 4)).astype(np.uint16)
    return (c[..., 3] | (c[..., 2] << 2) | (c[..., 1] << 4) | (c[..., 0] << 6)).astype(np.uint8)


def _manhattan_sq(cq, ck):             # squared instead of absolute difference
    a = np.asarray(cq, np.int64)
    b = np.asarray(ck, np.int64)
    return ((b - a[..., None, :]) ** 2).sum(-1)


def _manhattan_dropped(cq, ck):        # dropped the last coordinate
    a = np.asarray(cq, np.int64)[..., :-1]
    b = np.asarray(ck, np.int64)[..., :-1]
    return np.abs(b - a[..., None, :]).sum(-1)


def _topk_high_pos(dist, k):           # ties go to the HIGHER position
    dist = np.asarray(dist)
    L = dist.shape[-1]
    order = np.lexsort((-np.arange(L), dist))
    return np.sort(order[:min(k, L)])


def _topk_largest(dist, k):            # largest distance taken as most relevant
    return _orig["select_topk"](-np.asarray(dist), k)


def _attn_noscale(q, K, V, idx):       # forgot 1/sqrt(d)
    q = np.asarray(q, np.float64)
    s = np.asarray(K, np.float64)[idx] @ q
    p = np.exp(s - s.max())
    return (p / p.sum()) @ np.asarray(V, np.float64)[idx]


def _attn_uses_k(q, K, V, idx):        # transposed operand: K rows used as values
    return _orig["sparse_attention"](q, K, K, idx)


def _decode_mod_gqa(q, K, V, k, t, key_codes=None, query_codes=None):
    # query head h reads kv head h % Hkv instead of h // G
    B, Hq, d = q.shape
    Hkv = K.shape[1]
    perm = [h % Hkv for h in range(Hq)]
    G = Hq // Hkv
    # reorder q so that the original routine's h // G lands on h % Hkv
    inv = sorted(range(Hq), key=lambda h: (perm[h], h))
    idx, out = _orig["decode_step"](q[:, inv], K, V, k, t)
    back = np.argsort(inv)
    return idx[:, back], out[:, back]


def _shared_first_head_only(q, K, V, k, t, key_codes=None, query_codes=None):
    # shared selection scored by the group's first query head alone
    B, Hq, d = q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    qq = np.repeat(np.asarray(q)[:, ::G], G, axis=1)
    idx, _ = _orig["decode_step_shared"](qq, K, V, k, t)
    _, out = _orig["decode_step_shared"](q, K, V, k, t)
    return idx, out


def _varlen_full_cache(q, K, V, seq_lens, k, t, key_codes=None, query_codes=None,
                      shared=False):
    # every non-empty sequence scanned over the whole cache instead of its length
    lens = [K.shape[2] if int(x) else 0 for x in seq_lens]
    return _orig["decode_step_varlen"](q, K, V, lens, k, t, shared=shared)


def _varlen_zero_pad(q, K, V, seq_lens, k, t, key_codes=None, query_codes=None, shared=False):
    # unused index slots padded with 0 instead of -1
    idx, out = _orig["decode_step_varlen"](q, K, V, seq_lens, k, t, shared=shared)
    return np.where(idx < 0, 0, idx), out


def _varlen_off_by_one(q, K, V, seq_lens, k, t, key_codes=None, query_codes=None,
                       shared=False):
    # one slot past the length scanned as well
    lens = [min(int(x) + 1, K.shape[2]) if int(x) else 0 for x in seq_lens]
    return _orig["decode_step_varlen"](q, K, V, lens, k, t, shared=shared)


def _absmax_unrotated(x, ratio=0.5):
    # absmax of the raw vector instead of the rotated one
    return float(ratio) * np.abs(np.asarray(x, np.float64)).max(axis=-1)


def _absmax_global(x, ratio=0.5):
    # one absmax over the whole tensor instead of per vector
    y = _orig["hadamard_rotate"](x)
    return np.full(y.shape[:-1], float(ratio) * np.abs(y).max())


def _absmax_inverse_ratio(x, ratio=0.5):
    return _orig["absmax_thresholds"](x, 1.0 / ratio)


def _per_vector_le(y, t):
    # "<=" instead of "<"
    y = np.asarray(y, np.float64)
    tt = np.asarray(t, np.float64)[..., None]
    c = np.full(y.shape, 3, np.uint8)
    c[y <= tt] = 2
    c[y <= 0] = 1
    c[y <= -tt] = 0
    return c


def _decode_absmax_fixed_query(q, K, V, k, ratio=0.5, shared=False):
    # queries encoded with a fixed t = ratio instead of their own absmax threshold
    step = _orig["decode_step_shared"] if shared else _orig["decode_step"]
    return step(q, K, V, k, ratio, key_codes=_orig["encode_absmax"](K, ratio))


def _margin_scaled(y, t):               # margin in unscaled units (x sqrt(d))
    return _orig["threshold_margin"](y, t) * np.sqrt(128)


def _margin_no_zero(y, t):              # the 0 threshold forgotten
    y = np.asarray(y, np.float64)
    tt = float(np.float32(t))
    return np.minimum(np.abs(y + tt), np.abs(y - tt))


def _margin_f64_t(y, t):                # t kept in float64, not the kernels' float32
    y = np.asarray(y, np.float64)
    t = float(t)
    return np.minimum(np.minimum(np.abs(y + t), np.abs(y)), np.abs(y - t))


def _head_ignores_query_code(q_vec, K_rows, V_rows, k, t, key_codes_rows=None,
                             query_code=None):
    return _orig["decode_head"](q_vec, K_rows, V_rows, k, t, key_codes_rows=key_codes_rows)


def _head_ignores_key_codes(q_vec, K_rows, V_rows, k, t, key_codes_rows=None,
                            query_code=None):
    return _orig["decode_head"](q_vec, K_rows, V_rows, k, t, query_code=query_code)


def _head_kv_swapped(q_vec, K_rows, V_rows, k, t, key_codes_rows=None, query_code=None):
    # V rows used as keys in the attention (the codes still come from the keys)
    if key_codes_rows is None:
        key_codes_rows = ref.encode(K_rows, t)
    return _orig["decode_head"](q_vec, V_rows, K_rows, k, t, key_codes_rows=key_codes_rows,
                                query_code=query_code)


MUTATIONS = {
    "hadamard_or": ("sylvester_hadamard", _h_or),
    "rotate_unscaled": ("hadamard_rotate", _rotate_unscaled),
    "rotate_reversed": ("hadamard_rotate", _rotate_reversed),
    "bucket_le": ("bucketize", _bucket_le),
    "bucket_swapped": ("bucketize", _bucket_swapped),
    "pack_msb_first": ("pack_codes", _pack_msb_first),
    "manhattan_squared": ("manhattan", _manhattan_sq),
    "manhattan_dropped_term": ("manhattan", _manhattan_dropped),
    "topk_ties_high": ("select_topk", _topk_high_pos),
    "topk_largest": ("select_topk", _topk_largest),
    "attention_noscale": ("sparse_attention", _attn_noscale),
    "attention_k_as_v": ("sparse_attention", _attn_uses_k),
    "decode_gqa_modulo": ("decode_step", _decode_mod_gqa),
    "shared_first_head_only": ("decode_step_shared", _shared_first_head_only),
    "varlen_full_cache": ("decode_step_varlen", _varlen_full_cache),
    "varlen_zero_pad": ("decode_step_varlen", _varlen_zero_pad),
    "varlen_off_by_one": ("decode_step_varlen", _varlen_off_by_one),
    "absmax_unrotated": ("absmax_thresholds", _absmax_unrotated),
    "absmax_global": ("absmax_thresholds", _absmax_global),
    "absmax_inverse_ratio": ("absmax_thresholds", _absmax_inverse_ratio),
    "absmax_bucket_le": ("bucketize_per_vector", _per_vector_le),
    "absmax_fixed_query": ("decode_step_absmax", _decode_absmax_fixed_query),
    "margin_scaled": ("threshold_margin", _margin_scaled),
    "margin_no_zero_threshold": ("threshold_margin", _margin_no_zero),
    "margin_float64_t": ("threshold_margin", _margin_f64_t),
    "head_ignores_query_code": ("decode_head", _head_ignores_query_code),
    "head_ignores_key_codes": ("decode_head", _head_ignores_key_codes),
    "head_kv_swapped": ("decode_head", _head_kv_swapped),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(ref, attr, fn)
    failed = []
    for check in ALL_CHECKS:
        try:
            check()
        except AssertionError:
            failed.append(check.__name__)
        except Exception as e:          # a crash in a pin is a test bug, not a catch
            raise AssertionError(f"{check.__name__} crashed under {name}: {e!r}")
    assert failed, f"mutation {name} passed every pin"

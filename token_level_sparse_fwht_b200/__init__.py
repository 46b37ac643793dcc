"""Adamas decode hot path on B200: thin Python binding of libadamas.so.

Every step of the path runs in the library's CUDA kernels; this module only
marshals torch tensors (device memory, streams) into the C ABI declared in
include/adamas.h.  There is no CPU fallback: if the library is missing or a call
fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libadamas.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "adamas.h")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_INTERNAL = range(6)
F32, BF16 = 0, 1
HEAD_DIM = 128


class AdamasError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


_lib = None

_c_i = ctypes.c_int
_c_i64 = ctypes.c_int64
_c_f = ctypes.c_float
_c_sz = ctypes.c_size_t
_c_p = ctypes.c_void_p

_SIGNATURES = {
    "adamas_status_string": (ctypes.c_char_p, [_c_i]),
    "adamas_abi_version": (_c_i, []),
    "adamas_set_decode_policy": (_c_i, [_c_i]),
    "adamas_test_set_copy_fault": (_c_i, [_c_i]),
    "adamas_encode_keys": (_c_i, [_c_p, _c_i, _c_i, _c_i, _c_i, _c_i64, _c_i64, _c_i64, _c_f,
                                  _c_p, _c_p]),
    "adamas_encode_queries": (_c_i, [_c_p, _c_i, _c_i, _c_i, _c_i, _c_f, _c_p, _c_p]),
    "adamas_decode_workspace_bytes": (_c_sz, [_c_i, _c_i, _c_i, _c_i, _c_i64, _c_i]),
    "adamas_workspace_init": (_c_i, [_c_p, _c_sz, _c_p]),
    "adamas_check_workspace": (_c_i, [_c_p, _c_sz, _c_p]),
    "adamas_decode_step": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i64,
                                  _c_i64, _c_i, _c_f, _c_p, _c_sz, _c_p, _c_p, _c_p]),
    "adamas_decode_step_host": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i,
                                       _c_i, _c_i64, _c_i64, _c_i, _c_f, _c_p, _c_sz, _c_p,
                                       _c_p, _c_p, _c_p]),
    "adamas_select_topk": (_c_i, [_c_p, _c_p, _c_i, _c_i, _c_i, _c_i64, _c_i64, _c_i, _c_p,
                                  _c_sz, _c_p, _c_p]),
    "adamas_decode_step_shared": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_i,
                                         _c_i64, _c_i64, _c_i, _c_f, _c_p, _c_sz, _c_p, _c_p,
                                         _c_p]),
    "adamas_decode_step_shared_host": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i,
                                              _c_i, _c_i, _c_i64, _c_i64, _c_i, _c_f, _c_p,
                                              _c_sz, _c_p, _c_p, _c_p, _c_p]),
    "adamas_select_topk_shared": (_c_i, [_c_p, _c_p, _c_i, _c_i, _c_i, _c_i64, _c_i64, _c_i,
                                         _c_p, _c_sz, _c_p, _c_p]),
    "adamas_decode_step_varlen": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_i,
                                         _c_i64, _c_p, _c_i, _c_f, _c_i, _c_p, _c_sz, _c_p, _c_p,
                                         _c_p]),
    "adamas_decode_step_paged": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_i,
                                        _c_i, _c_i64, _c_p, _c_i, _c_p, _c_i64, _c_i, _c_f, _c_i,
                                        _c_p, _c_sz, _c_p, _c_p, _c_p]),
    "adamas_select_topk_paged": (_c_i, [_c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_i64, _c_p, _c_i,
                                        _c_p, _c_i64, _c_i, _c_i, _c_p, _c_sz, _c_p, _c_p]),
    "adamas_encode_pages": (_c_i, [_c_p, _c_i, _c_i, _c_i, _c_i, _c_i64, _c_p, _c_i64, _c_f,
                                   _c_p, _c_p]),
    "adamas_encode_keys_absmax": (_c_i, [_c_p, _c_i, _c_i, _c_i, _c_i, _c_i64, _c_i64, _c_i64,
                                         _c_f, _c_p, _c_p]),
    "adamas_encode_queries_absmax": (_c_i, [_c_p, _c_i, _c_i, _c_i, _c_i, _c_f, _c_p, _c_p]),
    "adamas_encode_pages_absmax": (_c_i, [_c_p, _c_i, _c_i, _c_i, _c_i, _c_i64, _c_p, _c_i64,
                                          _c_f, _c_p, _c_p]),
    "adamas_decode_step_paged_host": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i,
                                             _c_i, _c_i, _c_i64, _c_p, _c_i, _c_p, _c_i64, _c_i,
                                             _c_f, _c_i, _c_p, _c_sz, _c_p, _c_p, _c_p, _c_p]),
    "adamas_decode_step_absmax_host": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i,
                                              _c_i, _c_i, _c_i64, _c_i64, _c_i, _c_f, _c_i, _c_p,
                                              _c_sz, _c_p, _c_p, _c_p, _c_p]),
    "adamas_decode_step_absmax": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_i,
                                         _c_i64, _c_i64, _c_i, _c_f, _c_i, _c_p, _c_sz, _c_p,
                                         _c_p, _c_p]),
    "adamas_cp_hist_elems": (_c_sz, [_c_i, _c_i, _c_i, _c_i]),
    "adamas_cp_workspace_bytes": (_c_sz, [_c_i, _c_i, _c_i, _c_i, _c_i64, _c_i, _c_i]),
    "adamas_cp_histograms": (_c_i, [_c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i64, _c_i64,
                                    _c_i, _c_f, _c_i, _c_p, _c_sz, _c_p, _c_p]),
    "adamas_cp_attend": (_c_i, [_c_p, _c_p, _c_p, _c_p, _c_i, _c_i, _c_i, _c_i, _c_i, _c_i64,
                                _c_i64, _c_i64, _c_i64, _c_i, _c_f, _c_i, _c_p, _c_i, _c_i,
                                _c_p, _c_sz, _c_p, _c_p, _c_p]),
    "adamas_cp_combine": (_c_i, [_c_p, _c_i, _c_i, _c_i, _c_p, _c_p]),
    "adamas_sparse_attention_workspace_bytes": (_c_sz, [_c_i, _c_i, _c_i]),
    "adamas_sparse_attention": (_c_i, [_c_p, _c_p, _c_p, _c_i, _c_p, _c_i, _c_i, _c_i, _c_i,
                                       _c_i64, _c_i, _c_p, _c_sz, _c_p, _c_p]),
    "adamas_sparse_attention_noalloc": (_c_i, [_c_p, _c_p, _c_p, _c_i, _c_p, _c_i, _c_i, _c_i,
                                               _c_i, _c_i64, _c_i, _c_p, _c_p]),
    "adamas_decode_plan": (_c_i, [_c_i, _c_i, _c_i, _c_i, _c_i64, _c_i,
                                  ctypes.POINTER(_c_i), ctypes.POINTER(_c_i),
                                  ctypes.POINTER(_c_i64), ctypes.POINTER(_c_i)]),
    "adamas_decode_plan_shared": (_c_i, [_c_i, _c_i, _c_i, _c_i, _c_i64, _c_i,
                                         ctypes.POINTER(_c_i), ctypes.POINTER(_c_i),
                                         ctypes.POINTER(_c_i64), ctypes.POINTER(_c_i)]),
}


def lib():
    """The loaded libadamas.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m token_level_sparse_fwht_b200.build` (there is no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def header_symbols():
    """Entry points declared in include/adamas.h."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return sorted(set(re.findall(r"\b(adamas_[a-z_0-9]+)\s*\(", text)))


POLICY_AUTO, POLICY_CLUSTER, POLICY_FLAT = 0, 1, 2


def set_decode_policy(policy: int):
    """Which decode kernel the planner may use (adamas_set_decode_policy): POLICY_AUTO,
    POLICY_CLUSTER (thread-block clusters only) or POLICY_FLAT (the grid-wide kernel
    wherever it applies).  Process-wide; results are the same either way."""
    _check(lib().adamas_set_decode_policy(int(policy)), "adamas_set_decode_policy")


def test_set_copy_fault(extra_tx_bytes: int):
    """adamas_test_set_copy_fault: make the next decode launches' first copy wait run
    out (test hook of the bounded-wait error path); 0 restores normal operation."""
    _check(lib().adamas_test_set_copy_fault(int(extra_tx_bytes)), "adamas_test_set_copy_fault")


def status_string(s: int) -> str:
    return lib().adamas_status_string(int(s)).decode()


def _check(status: int, what: str):
    if status != OK:
        raise AdamasError(status, what)


def _stream(stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype} (bfloat16 or float32)")


def _dev(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


# ------------------------------------------------------------------ encoders
def encode_keys(k_cache: torch.Tensor, codes: torch.Tensor, pos0: int, n_new: int, t: float,
                stream=None):
    """Encodes positions [pos0, pos0+n_new) of k_cache [B,Hkv,Lmax,128] into codes
    [B,Hkv,Lmax,32] (uint8)."""
    B, Hkv, Lmax, d = k_cache.shape
    if codes.dtype != torch.uint8 or tuple(codes.shape) != (B, Hkv, Lmax, d // 4):
        raise ValueError("codes must be uint8 [B, Hkv, Lmax, d/4]")
    _check(lib().adamas_encode_keys(_dev(k_cache, "k_cache"), _dtype_code(k_cache), B, Hkv, d,
                                    Lmax, pos0, n_new, float(t), _dev(codes, "codes"),
                                    _stream(stream)), "adamas_encode_keys")
    return codes


def encode_queries(q: torch.Tensor, t: float, qcodes: torch.Tensor | None = None, stream=None):
    B, Hq, d = q.shape
    if qcodes is None:
        qcodes = torch.empty((B, Hq, d // 4), dtype=torch.uint8, device=q.device)
    _check(lib().adamas_encode_queries(_dev(q, "q"), _dtype_code(q), B, Hq, d, float(t),
                                       _dev(qcodes, "qcodes"), _stream(stream)),
           "adamas_encode_queries")
    return qcodes


# ---------------------------------------------------------------- workspace
def decode_workspace_bytes(B: int, Hq: int, Hkv: int, L: int, k: int) -> int:
    n = lib().adamas_decode_workspace_bytes(B, Hq, Hkv, HEAD_DIM, L, k)
    if n == 0:
        raise AdamasError(ERR_INVALID_ARG, "adamas_decode_workspace_bytes")
    return int(n)


def _plan(name: str, B: int, Hq: int, Hkv: int, L: int, k: int) -> dict:
    ctas, cluster, smem = _c_i(), _c_i(), _c_i()
    rng = _c_i64()
    _check(getattr(lib(), name)(B, Hq, Hkv, HEAD_DIM, L, k, ctypes.byref(ctas),
                                ctypes.byref(cluster), ctypes.byref(rng), ctypes.byref(smem)),
           name)
    return {"ctas": ctas.value, "cluster": cluster.value, "tokens_per_cta": rng.value,
            "smem_bytes": smem.value}


def decode_plan(B: int, Hq: int, Hkv: int, L: int, k: int) -> dict:
    """Launch plan of decode_step (host only): ctas, cluster, tokens_per_cta, smem_bytes."""
    return _plan("adamas_decode_plan", B, Hq, Hkv, L, k)


def decode_plan_shared(B: int, Hq: int, Hkv: int, L: int, k: int) -> dict:
    """Launch plan of decode_step_shared / select_topk_shared."""
    return _plan("adamas_decode_plan_shared", B, Hq, Hkv, L, k)


def init_workspace(ws: torch.Tensor, stream=None):
    _check(lib().adamas_workspace_init(_dev(ws, "workspace"), ws.numel(), _stream(stream)),
           "adamas_workspace_init")
    return ws


def decode_workspace(B: int, Hq: int, Hkv: int, L: int, k: int, device="cuda", stream=None):
    """A zero-initialised decode workspace (torch allocates, the library zero-fills)."""
    n = decode_workspace_bytes(B, Hq, Hkv, L, k)
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    return init_workspace(ws, stream)


def check_workspace(ws: torch.Tensor, stream=None):
    """Synchronizes the stream; raises AdamasError(ERR_TIMEOUT) if a device wait gave up."""
    _check(lib().adamas_check_workspace(_dev(ws, "workspace"), ws.numel(), _stream(stream)),
           "adamas_check_workspace")


# -------------------------------------------------------------- decode step
def _decode(name, q, k_cache, v_cache, codes, L, k, t, ws, idx_out, out, stream):
    B, Hq, d = q.shape
    _, Hkv, Lmax, _ = k_cache.shape
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    idx_ptr = None if idx_out is None else _dev(idx_out, "idx_out")
    _check(getattr(lib(), name)(_dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                                _dev(codes, "codes"), _dtype_code(k_cache), B, Hq, Hkv, d, Lmax,
                                L, k, float(t), _dev(ws, "workspace"), ws.numel(), idx_ptr,
                                _dev(out, "out"), _stream(stream)), name)
    return out


def decode_step(q, k_cache, v_cache, codes, L: int, k: int, t: float, ws, idx_out=None,
                out=None, stream=None):
    """One decode step (fused kernel).  Returns out [B,Hq,128] fp32 (and fills idx_out
    [B,Hq,min(k,L)] int32 if given)."""
    return _decode("adamas_decode_step", q, k_cache, v_cache, codes, L, k, t, ws, idx_out, out,
                   stream)


def decode_step_shared(q, k_cache, v_cache, codes, L: int, k: int, t: float, ws, idx_out=None,
                       out=None, stream=None):
    """Decode step with one selection per kv head shared by its query heads (scores
    summed over the group).  Returns out [B,Hq,128] fp32; idx_out, if given, is
    [B,Hkv,min(k,L)] int32."""
    return _decode("adamas_decode_step_shared", q, k_cache, v_cache, codes, L, k, t, ws,
                   idx_out, out, stream)


def decode_step_host(q_host, q_dev, k_cache, v_cache, codes, L: int, k: int, t: float, ws,
                     out_dev, out_host, idx_out=None, stream=None):
    """decode_step with host-resident q and output: one C call queues the host->device
    copy of q, the fused kernel and the device->host copy of out on `stream`."""
    return _decode_host("adamas_decode_step_host", q_host, q_dev, k_cache, v_cache, codes, L,
                        k, t, ws, out_dev, out_host, idx_out, stream)


def decode_step_shared_host(q_host, q_dev, k_cache, v_cache, codes, L: int, k: int, t: float,
                            ws, out_dev, out_host, idx_out=None, stream=None):
    """decode_step_host for the shared selection (idx_out [B,Hkv,min(k,L)])."""
    return _decode_host("adamas_decode_step_shared_host", q_host, q_dev, k_cache, v_cache,
                        codes, L, k, t, ws, out_dev, out_host, idx_out, stream)


def _decode_host(name, q_host, q_dev, k_cache, v_cache, codes, L, k, t, ws, out_dev, out_host,
                 idx_out, stream):
    B, Hq, d = q_dev.shape
    _, Hkv, Lmax, _ = k_cache.shape
    if q_host.is_cuda or out_host.is_cuda:
        raise ValueError("q_host and out_host must be host tensors")
    idx_ptr = None if idx_out is None else _dev(idx_out, "idx_out")
    _check(getattr(lib(), name)(q_host.data_ptr(), _dev(q_dev, "q_dev"),
                                _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                                _dev(codes, "codes"), _dtype_code(k_cache), B, Hq, Hkv, d, Lmax,
                                L, k, float(t), _dev(ws, "workspace"), ws.numel(), idx_ptr,
                                _dev(out_dev, "out_dev"), out_host.data_ptr(), _stream(stream)),
           name)
    return out_host


class PreparedDecodeHost:
    """A decode step bound to fixed buffers, for serving loops that reuse them every
    step: all pointers and sizes are resolved once, so each call is one C call with
    no per-call Python checks.  Same semantics as decode_step_host (shared=True:
    decode_step_shared_host)."""

    def __init__(self, q_host, q_dev, k_cache, v_cache, codes, L: int, k: int, t: float, ws,
                 out_dev, out_host, idx_out=None, stream=None, shared: bool = False):
        B, Hq, d = q_dev.shape
        _, Hkv, Lmax, _ = k_cache.shape
        if q_host.is_cuda or out_host.is_cuda:
            raise ValueError("q_host and out_host must be host tensors")
        if tuple(q_host.shape) != (B, Hq, d) or tuple(out_host.shape) != (B, Hq, d):
            raise ValueError("q_host / out_host shapes must be [B, Hq, d]")
        self._keep = (q_host, q_dev, k_cache, v_cache, codes, ws, out_dev, out_host, idx_out)
        self._name = "adamas_decode_step_shared_host" if shared else "adamas_decode_step_host"
        self._fn = getattr(lib(), self._name)
        self._args = (
            _c_p(q_host.data_ptr()), _c_p(_dev(q_dev, "q_dev")), _c_p(_dev(k_cache, "k_cache")),
            _c_p(_dev(v_cache, "v_cache")), _c_p(_dev(codes, "codes")),
            _c_i(_dtype_code(k_cache)), _c_i(B), _c_i(Hq), _c_i(Hkv), _c_i(d), _c_i64(Lmax),
            _c_i64(L), _c_i(k), _c_f(t), _c_p(_dev(ws, "workspace")), _c_sz(ws.numel()),
            _c_p(None if idx_out is None else _dev(idx_out, "idx_out")),
            _c_p(_dev(out_dev, "out_dev")), _c_p(out_host.data_ptr()), _c_p(_stream(stream)))

    def __call__(self):
        status = self._fn(*self._args)
        if status != OK:
            raise AdamasError(status, self._name)


def _select(name, rows_per_batch, qcodes, codes, L, k, ws, idx_out, stream):
    B, Hq, _ = qcodes.shape
    _, Hkv, Lmax, _ = codes.shape
    k_eff = min(k, L)
    if idx_out is None:
        rows = Hq if rows_per_batch == "Hq" else Hkv
        idx_out = torch.empty((B, rows, k_eff), dtype=torch.int32, device=qcodes.device)
    _check(getattr(lib(), name)(_dev(qcodes, "qcodes"), _dev(codes, "codes"), B, Hq, Hkv, Lmax,
                                L, k, _dev(ws, "workspace"), ws.numel(),
                                _dev(idx_out, "idx_out"), _stream(stream)), name)
    return idx_out


def select_topk(qcodes, codes, L: int, k: int, ws, idx_out=None, stream=None):
    """Distance scan + per-head top-k from query codes: idx [B,Hq,min(k,L)] int32."""
    return _select("adamas_select_topk", "Hq", qcodes, codes, L, k, ws, idx_out, stream)


def select_topk_shared(qcodes, codes, L: int, k: int, ws, idx_out=None, stream=None):
    """Shared selection from query codes: idx [B,Hkv,min(k,L)] int32."""
    return _select("adamas_select_topk_shared", "Hkv", qcodes, codes, L, k, ws, idx_out, stream)


# ------------------------------------ per-sequence lengths and paged caches
def _i32(t: torch.Tensor, name: str):
    if t.dtype != torch.int32:
        raise TypeError(f"{name} must be int32")
    return _dev(t, name)


def decode_step_varlen(q, k_cache, v_cache, codes, seq_lens, k: int, t: float, ws,
                       shared: bool = False, idx_out=None, out=None, stream=None):
    """Decode step with per-sequence lengths seq_lens [B] int32 (device) over
    contiguous caches [B,Hkv,Lmax,128].  Returns out [B,Hq,128]; idx_out, if given,
    is [B, Hq (Hkv if shared), min(k, Lmax)] int32, -1 past a sequence's count."""
    B, Hq, d = q.shape
    _, Hkv, Lmax, _ = k_cache.shape
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    idx_ptr = None if idx_out is None else _dev(idx_out, "idx_out")
    _check(lib().adamas_decode_step_varlen(
        _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"), _dev(codes, "codes"),
        _dtype_code(k_cache), B, Hq, Hkv, d, Lmax, _i32(seq_lens, "seq_lens"), k, float(t),
        int(bool(shared)), _dev(ws, "workspace"), ws.numel(), idx_ptr, _dev(out, "out"),
        _stream(stream)), "adamas_decode_step_varlen")
    return out


def decode_step_paged(q, k_pages, v_pages, code_pages, block_table, seq_lens,
                      max_seq_len: int, k: int, t: float, ws, shared: bool = False,
                      idx_out=None, out=None, stream=None):
    """Decode step over paged caches: k_pages, v_pages [P,Hkv,page,128], code_pages
    [P,Hkv,page,32], block_table [B,max_blocks] int32, seq_lens [B] int32."""
    B, Hq, d = q.shape
    P, Hkv, page, _ = k_pages.shape
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    idx_ptr = None if idx_out is None else _dev(idx_out, "idx_out")
    _check(lib().adamas_decode_step_paged(
        _dev(q, "q"), _dev(k_pages, "k_pages"), _dev(v_pages, "v_pages"),
        _dev(code_pages, "code_pages"), _dtype_code(k_pages), B, Hq, Hkv, d, page, P,
        _i32(block_table, "block_table"), block_table.shape[1], _i32(seq_lens, "seq_lens"),
        max_seq_len, k, float(t), int(bool(shared)), _dev(ws, "workspace"), ws.numel(), idx_ptr,
        _dev(out, "out"), _stream(stream)), "adamas_decode_step_paged")
    return out


def select_topk_paged(qcodes, code_pages, block_table, seq_lens, max_seq_len: int, k: int, ws,
                      shared: bool = False, idx_out=None, stream=None):
    B, Hq, _ = qcodes.shape
    P, Hkv, page, _ = code_pages.shape
    if idx_out is None:
        idx_out = torch.empty((B, Hkv if shared else Hq, min(k, max_seq_len)), dtype=torch.int32,
                              device=qcodes.device)
    _check(lib().adamas_select_topk_paged(
        _dev(qcodes, "qcodes"), _dev(code_pages, "code_pages"), B, Hq, Hkv, page, P,
        _i32(block_table, "block_table"), block_table.shape[1], _i32(seq_lens, "seq_lens"),
        max_seq_len, k, int(bool(shared)), _dev(ws, "workspace"), ws.numel(),
        _dev(idx_out, "idx_out"), _stream(stream)), "adamas_select_topk_paged")
    return idx_out


def encode_pages(k_pages, code_pages, t: float, page_ids=None, stream=None):
    """Encodes all rows of the listed pages (int32 device tensor; None: every page)."""
    P, Hkv, page, d = k_pages.shape
    if code_pages.dtype != torch.uint8 or tuple(code_pages.shape) != (P, Hkv, page, d // 4):
        raise ValueError("code_pages must be uint8 [P, Hkv, page, d/4]")
    ids = None if page_ids is None else _i32(page_ids, "page_ids")
    n = 0 if page_ids is None else page_ids.numel()
    _check(lib().adamas_encode_pages(_dev(k_pages, "k_pages"), _dtype_code(k_pages), Hkv, d, page,
                                     P, ids, n, float(t), _dev(code_pages, "code_pages"),
                                     _stream(stream)), "adamas_encode_pages")
    return code_pages


# --------------------------------------------- per-vector absmax thresholds
def encode_keys_absmax(k_cache: torch.Tensor, codes: torch.Tensor, pos0: int, n_new: int,
                       ratio: float = 0.5, stream=None):
    """encode_keys with each key's threshold ratio * max |H k / sqrt(d)|."""
    B, Hkv, Lmax, d = k_cache.shape
    if codes.dtype != torch.uint8 or tuple(codes.shape) != (B, Hkv, Lmax, d // 4):
        raise ValueError("codes must be uint8 [B, Hkv, Lmax, d/4]")
    _check(lib().adamas_encode_keys_absmax(_dev(k_cache, "k_cache"), _dtype_code(k_cache), B, Hkv,
                                           d, Lmax, pos0, n_new, float(ratio),
                                           _dev(codes, "codes"), _stream(stream)),
           "adamas_encode_keys_absmax")
    return codes


def encode_queries_absmax(q: torch.Tensor, ratio: float = 0.5, qcodes=None, stream=None):
    B, Hq, d = q.shape
    if qcodes is None:
        qcodes = torch.empty((B, Hq, d // 4), dtype=torch.uint8, device=q.device)
    _check(lib().adamas_encode_queries_absmax(_dev(q, "q"), _dtype_code(q), B, Hq, d,
                                              float(ratio), _dev(qcodes, "qcodes"),
                                              _stream(stream)), "adamas_encode_queries_absmax")
    return qcodes


def encode_pages_absmax(k_pages, code_pages, ratio: float = 0.5, page_ids=None, stream=None):
    P, Hkv, page, d = k_pages.shape
    if code_pages.dtype != torch.uint8 or tuple(code_pages.shape) != (P, Hkv, page, d // 4):
        raise ValueError("code_pages must be uint8 [P, Hkv, page, d/4]")
    ids = None if page_ids is None else _i32(page_ids, "page_ids")
    n = 0 if page_ids is None else page_ids.numel()
    _check(lib().adamas_encode_pages_absmax(_dev(k_pages, "k_pages"), _dtype_code(k_pages), Hkv, d,
                                            page, P, ids, n, float(ratio),
                                            _dev(code_pages, "code_pages"), _stream(stream)),
           "adamas_encode_pages_absmax")
    return code_pages


def decode_step_absmax(q, k_cache, v_cache, codes, L: int, k: int, ratio: float, ws,
                       shared: bool = False, idx_out=None, out=None, stream=None):
    """Decode step whose fused query encode uses per-vector absmax thresholds (codes
    from encode_keys_absmax with the same ratio)."""
    B, Hq, d = q.shape
    _, Hkv, Lmax, _ = k_cache.shape
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    idx_ptr = None if idx_out is None else _dev(idx_out, "idx_out")
    _check(lib().adamas_decode_step_absmax(
        _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"), _dev(codes, "codes"),
        _dtype_code(k_cache), B, Hq, Hkv, d, Lmax, L, k, float(ratio), int(bool(shared)),
        _dev(ws, "workspace"), ws.numel(), idx_ptr, _dev(out, "out"), _stream(stream)),
        "adamas_decode_step_absmax")
    return out


class _PreparedCall:
    """One C call bound to fixed buffers (pointers and sizes resolved once)."""

    def __init__(self, name, args, keep):
        self._name = name
        self._fn = getattr(lib(), name)
        self._args = args
        self._keep = keep

    def __call__(self):
        status = self._fn(*self._args)
        if status != OK:
            raise AdamasError(status, self._name)


def _host_pair(q_host, out_host, B, Hq, d):
    if q_host.is_cuda or out_host.is_cuda:
        raise ValueError("q_host and out_host must be host tensors")
    if tuple(q_host.shape) != (B, Hq, d) or tuple(out_host.shape) != (B, Hq, d):
        raise ValueError("q_host / out_host shapes must be [B, Hq, d]")


class PreparedPagedDecodeHost(_PreparedCall):
    """adamas_decode_step_paged_host bound to fixed buffers: host q in, host fp32 out
    (mapped page-locked buffers in place, else through q_dev / out_dev)."""

    def __init__(self, q_host, q_dev, k_pages, v_pages, code_pages, block_table, seq_lens,
                 max_seq_len: int, k: int, t: float, ws, out_dev, out_host, shared: bool = False,
                 idx_out=None, stream=None):
        B, Hq, d = q_dev.shape
        P, Hkv, page, _ = k_pages.shape
        _host_pair(q_host, out_host, B, Hq, d)
        args = (_c_p(q_host.data_ptr()), _c_p(_dev(q_dev, "q_dev")), _c_p(_dev(k_pages, "k_pages")),
                _c_p(_dev(v_pages, "v_pages")), _c_p(_dev(code_pages, "code_pages")),
                _c_i(_dtype_code(k_pages)), _c_i(B), _c_i(Hq), _c_i(Hkv), _c_i(d), _c_i(page),
                _c_i64(P), _c_p(_i32(block_table, "block_table")), _c_i(block_table.shape[1]),
                _c_p(_i32(seq_lens, "seq_lens")), _c_i64(max_seq_len), _c_i(k), _c_f(t),
                _c_i(int(bool(shared))), _c_p(_dev(ws, "workspace")), _c_sz(ws.numel()),
                _c_p(None if idx_out is None else _dev(idx_out, "idx_out")),
                _c_p(_dev(out_dev, "out_dev")), _c_p(out_host.data_ptr()), _c_p(_stream(stream)))
        super().__init__("adamas_decode_step_paged_host", args,
                         (q_host, q_dev, k_pages, v_pages, code_pages, block_table, seq_lens, ws,
                          out_dev, out_host, idx_out))


class PreparedAbsmaxDecodeHost(_PreparedCall):
    """adamas_decode_step_absmax_host bound to fixed buffers."""

    def __init__(self, q_host, q_dev, k_cache, v_cache, codes, L: int, k: int, ratio: float, ws,
                 out_dev, out_host, shared: bool = False, idx_out=None, stream=None):
        B, Hq, d = q_dev.shape
        _, Hkv, Lmax, _ = k_cache.shape
        _host_pair(q_host, out_host, B, Hq, d)
        args = (_c_p(q_host.data_ptr()), _c_p(_dev(q_dev, "q_dev")), _c_p(_dev(k_cache, "k_cache")),
                _c_p(_dev(v_cache, "v_cache")), _c_p(_dev(codes, "codes")),
                _c_i(_dtype_code(k_cache)), _c_i(B), _c_i(Hq), _c_i(Hkv), _c_i(d), _c_i64(Lmax),
                _c_i64(L), _c_i(k), _c_f(ratio), _c_i(int(bool(shared))),
                _c_p(_dev(ws, "workspace")), _c_sz(ws.numel()),
                _c_p(None if idx_out is None else _dev(idx_out, "idx_out")),
                _c_p(_dev(out_dev, "out_dev")), _c_p(out_host.data_ptr()), _c_p(_stream(stream)))
        super().__init__("adamas_decode_step_absmax_host", args,
                         (q_host, q_dev, k_cache, v_cache, codes, ws, out_dev, out_host, idx_out))


# ------------------------------------------------ context-parallel steps
PART_STRIDE = 132      # floats per exported softmax partial: m, l, 0, 0, acc[128]


def cp_hist_shape(B: int, Hq: int, Hkv: int, shared: bool = False):
    n = int(lib().adamas_cp_hist_elems(B, Hq, Hkv, int(bool(shared))))
    if n == 0:
        raise AdamasError(ERR_INVALID_ARG, "adamas_cp_hist_elems")
    rows = B * (Hkv if shared else Hq)
    return (B, rows // B, n // rows)


def cp_workspace(B: int, Hq: int, Hkv: int, L: int, k: int, shared: bool = False, device="cuda",
                 stream=None):
    """A zero-filled workspace for one rank's context-parallel steps (L: its positions)."""
    n = int(lib().adamas_cp_workspace_bytes(B, Hq, Hkv, HEAD_DIM, L, k, int(bool(shared))))
    if n == 0:
        raise AdamasError(ERR_INVALID_ARG, "adamas_cp_workspace_bytes")
    return init_workspace(torch.empty(n, dtype=torch.uint8, device=device), stream)


def cp_histograms(q, codes, L: int, k: int, t: float, ws, shared: bool = False, hist_out=None,
                  stream=None):
    """Phase 1 on this rank's slice: cumulative hist [B, rows, bins] int32 (uint32
    counts of distances <= bin)."""
    B, Hq, d = q.shape
    _, Hkv, Lmax, _ = codes.shape
    if hist_out is None:
        hist_out = torch.empty(cp_hist_shape(B, Hq, Hkv, shared), dtype=torch.int32,
                               device=q.device)
    _check(lib().adamas_cp_histograms(_dev(q, "q"), _dev(codes, "codes"), _dtype_code(q), B, Hq,
                                      Hkv, d, Lmax, L, k, float(t), int(bool(shared)),
                                      _dev(ws, "workspace"), ws.numel(), _dev(hist_out, "hist"),
                                      _stream(stream)), "adamas_cp_histograms")
    return hist_out


def cp_attend(q, k_cache, v_cache, codes, L: int, L_total: int, pos_offset: int, k: int,
              t: float, hist_all, rank: int, ws, shared: bool = False, idx_out=None,
              partial_out=None, stream=None):
    """Phase 2 on this rank's slice, given every rank's cumulative histograms
    hist_all [world, B, rows, bins]: partial [B, Hq, 132] float32."""
    B, Hq, d = q.shape
    _, Hkv, Lmax, _ = k_cache.shape
    if partial_out is None:
        partial_out = torch.empty((B, Hq, PART_STRIDE), dtype=torch.float32, device=q.device)
    idx_ptr = None if idx_out is None else _dev(idx_out, "idx_out")
    _check(lib().adamas_cp_attend(_dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                                  _dev(codes, "codes"), _dtype_code(k_cache), B, Hq, Hkv, d, Lmax,
                                  L, L_total, pos_offset, k, float(t), int(bool(shared)),
                                  _dev(hist_all, "hist_all"), hist_all.shape[0], rank,
                                  _dev(ws, "workspace"), ws.numel(), idx_ptr,
                                  _dev(partial_out, "partial"), _stream(stream)),
           "adamas_cp_attend")
    return partial_out


def cp_combine(partials_all, out=None, stream=None):
    """partials_all [world, B, Hq, 132] -> out [B, Hq, 128] float32."""
    world, B, Hq, _ = partials_all.shape
    if out is None:
        out = torch.empty((B, Hq, HEAD_DIM), dtype=torch.float32, device=partials_all.device)
    _check(lib().adamas_cp_combine(_dev(partials_all, "partials"), world, B, Hq, _dev(out, "out"),
                                   _stream(stream)), "adamas_cp_combine")
    return out


def sparse_attention_workspace(B: int, Hq: int, k_eff: int, device="cuda", stream=None):
    n = int(lib().adamas_sparse_attention_workspace_bytes(B, Hq, k_eff))
    if n == 0:
        raise AdamasError(ERR_INVALID_ARG, "adamas_sparse_attention_workspace_bytes")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    return init_workspace(ws, stream)


def sparse_attention(q, k_cache, v_cache, idx, ws=None, out=None, stream=None):
    B, Hq, d = q.shape
    _, Hkv, Lmax, _ = k_cache.shape
    k_eff = idx.shape[-1]
    if idx.dtype != torch.int32:
        raise TypeError("idx must be int32")
    if ws is None:
        ws = sparse_attention_workspace(B, Hq, k_eff, q.device, stream)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    _check(lib().adamas_sparse_attention(_dev(q, "q"), _dev(k_cache, "k_cache"),
                                         _dev(v_cache, "v_cache"), _dtype_code(k_cache),
                                         _dev(idx, "idx"), B, Hq, Hkv, d, Lmax, k_eff,
                                         _dev(ws, "workspace"), ws.numel(), _dev(out, "out"),
                                         _stream(stream)), "adamas_sparse_attention")
    return out


def sparse_attention_noalloc(q, k_cache, v_cache, idx, out=None, stream=None):
    """adamas_sparse_attention without a workspace (library-held scratch; see
    include/adamas.h for the size limit and the first-call set-up)."""
    B, Hq, d = q.shape
    _, Hkv, Lmax, _ = k_cache.shape
    if idx.dtype != torch.int32:
        raise TypeError("idx must be int32")
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    _check(lib().adamas_sparse_attention_noalloc(_dev(q, "q"), _dev(k_cache, "k_cache"),
                                                 _dev(v_cache, "v_cache"), _dtype_code(k_cache),
                                                 _dev(idx, "idx"), B, Hq, Hkv, d, Lmax,
                                                 idx.shape[-1], _dev(out, "out"),
                                                 _stream(stream)),
           "adamas_sparse_attention_noalloc")
    return out


__all__ = ["lib", "header_symbols", "status_string", "AdamasError", "encode_keys",
           "decode_step_host", "PreparedDecodeHost",
           "encode_queries", "decode_workspace_bytes", "decode_plan", "init_workspace",
           "decode_workspace", "check_workspace", "decode_step", "select_topk",
           "sparse_attention_workspace", "sparse_attention", "sparse_attention_noalloc"]

"""Float64 CPU oracle of the Adamas decode hot path (test infrastructure only).

See adamas_ref.py for what each function follows and how it is pinned.
"""
from .adamas_ref import (D, CODE_BYTES, MAX_DIST, sylvester_hadamard, hadamard_rotate,
                         bucketize, threshold_margin, pack_codes, unpack_codes, encode,
                         manhattan, select_topk, sparse_attention, decode_step,
                         decode_head, decode_step_shared, decode_step_varlen,
                         absmax_thresholds, bucketize_per_vector, encode_absmax,
                         decode_step_absmax)

__all__ = ["D", "CODE_BYTES", "MAX_DIST", "sylvester_hadamard", "hadamard_rotate",
           "bucketize", "threshold_margin", "pack_codes", "unpack_codes", "encode",
           "manhattan", "select_topk", "sparse_attention", "decode_step", "decode_head",
           "decode_step_shared", "decode_step_varlen", "absmax_thresholds",
           "bucketize_per_vector", "encode_absmax", "decode_step_absmax"]

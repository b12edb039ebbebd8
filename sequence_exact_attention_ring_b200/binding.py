"""ctypes binding of libringattn.so: the C entry points under the same names.

Argument marshalling only. Every step of the computation runs in the library's
CUDA kernels; nothing here computes attention. If the library is missing the
binding raises: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libringattn.so")

OK = 0
EINVAL = -1
EALIGN = -2
EUNSUPPORTED = -3
EWORKSPACE = -4
ECUDA = -5
ETIMEOUT = -6

LAYOUT_CONTIGUOUS = 0
LAYOUT_STRIPED = 1
LAYOUT_ZIGZAG = 2
DTYPE_FP32 = 0
DTYPE_BF16 = 1
ALGO_AUTO = 0
ALGO_SIMT = 1
ALGO_TCGEN05 = 2
ALGO_TCGEN05_1SM = 3
STEP_FIRST = 1
STEP_LAST = 2
BWD_PART_KV = 1
BWD_PART_Q = 2

_c_int, _c_i64, _c_size, _vp, _c_float = ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_float

# name -> (restype, argtypes); mirrors include/ringattn.h
SIGNATURES = {
    "ring_attn_version": (_c_int, []),
    "ring_attn_strerror": (ctypes.c_char_p, [_c_int]),
    "ring_attn_fwd_workspace_bytes": (_c_size, [_c_int, _c_int, _c_int, _c_i64, _c_int, _c_int, _c_int, _c_int,
                                                _c_int]),
    "ring_attn_fwd": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_i64, _c_int, _c_int, _c_int,
                               _c_int, _c_float, _c_int, _vp, _c_size, _vp]),
    "ring_attn_fwd_algo": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_i64, _c_int, _c_int,
                                    _c_int, _c_int, _c_float, _c_int, _vp, _c_size, _vp, _c_int]),
    "ring_attn_fwd_step": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_i64, _c_int, _c_int,
                                    _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _c_int, _vp, _c_size, _vp]),
    "ring_attn_fwd_ring_step": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_i64, _c_int,
                                         _c_int, _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _c_int, _vp,
                                         _c_size, _vp]),
    "ring_attn_merge": (_c_int, [_vp, _vp, _c_int, _c_i64, _c_int, _vp, _vp, _c_int, _vp]),
    "ring_attn_status": (_c_int, [_vp, _vp]),
    "ring_attn_bwd_workspace_bytes": (_c_size, [_c_int, _c_int, _c_int, _c_i64, _c_int, _c_int, _c_int, _c_int,
                                                _c_int]),
    "ring_attn_bwd": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_i64, _c_int,
                               _c_int, _c_int, _c_int, _c_float, _c_int, _vp, _c_size, _vp]),
    "ring_attn_bwd_ring_workspace_bytes": (_c_size, [_c_int, _c_int, _c_int, _c_i64, _c_int, _c_int, _c_int,
                                                     _c_int, _c_int]),
    "ring_attn_bwd_ring_prep": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _c_int, _c_i64, _c_int, _c_int, _c_int,
                                         _c_int, _c_int, _c_int, _vp, _c_size, _vp]),
    "ring_attn_bwd_ring_step": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int,
                                         _c_i64, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_float, _c_int,
                                         _c_int, _c_int, _vp, _c_size, _vp]),
    "ring_attn_decode_workspace_bytes": (_c_size, [_c_int, _c_int, _c_int, _c_i64, _c_int, _c_int, _c_int, _c_int]),
    "ring_attn_decode": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_i64, _c_int, _c_int, _c_int,
                                  _c_float, _c_int, _vp, _c_size, _vp]),
    "ring_attn_debug_bwd_visit_counts": (_c_i64, [_c_i64, _c_int, _c_int, _c_int, _c_int, _vp]),
    "ring_attn_fwd_noalloc": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_i64, _c_int, _c_int,
                                       _c_int, _c_int, _c_float, _c_int, _vp, ctypes.POINTER(_vp)]),
    "ring_attn_debug_visit_counts": (_c_i64, [_c_i64, _c_int, _c_int, _c_int, _c_int, _c_int, _vp]),
    "ring_attn_debug_decode_units": (_c_int, [_c_int, _c_int, _c_int, _c_i64, _c_int, _c_int, _c_int, _c_int,
                                              _vp, _c_i64]),
    "ring_attn_debug_unit_walk": (_c_i64, [_c_int, _c_int, _c_int, _c_i64, _c_int, _c_int, _c_int, _c_int,
                                           _c_int, _c_i64, _vp, _c_i64]),
    "ring_attn_debug_schedule_info": (_c_int, [_c_int, _c_int, _c_int, _c_i64, _c_int, _c_int, _c_int, _c_int,
                                               _vp]),
    "ring_attn_debug_watchdog": (_c_int, [_c_int, _vp, _c_size, _vp]),
    "ring_attn_debug_exp2": (_c_int, [_vp, _vp, _c_i64, _vp]),
}

_lib = None


class RingAttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {strerror(code)} ({code})")


def load() -> ctypes.CDLL:
    """Load the in-tree library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m sequence_exact_attention_ring_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def strerror(code: int) -> str:
    try:
        return load().ring_attn_strerror(code).decode()
    except Exception:  # pragma: no cover - only when the library itself is missing
        return f"error {code}"


def check(code: int, where: str) -> int:
    if code < 0:
        raise RingAttnError(code, where)
    return code


# Raw entry points with the C names (pointers and sizes as Python ints).

def ring_attn_version() -> int:
    return load().ring_attn_version()


def ring_attn_fwd_workspace_bytes(B, Hq, Hkv, S, D, P, causal, layout, dtype) -> int:
    return load().ring_attn_fwd_workspace_bytes(B, Hq, Hkv, S, D, P, causal, layout, dtype)


def ring_attn_fwd(q, k, v, out, lse, B, Hq, Hkv, S, D, P, causal, layout, scale, dtype, workspace,
                  workspace_bytes, stream) -> int:
    return load().ring_attn_fwd(q, k, v, out, lse, B, Hq, Hkv, S, D, P, causal, layout, scale, dtype, workspace,
                                workspace_bytes, stream)


def ring_attn_fwd_algo(q, k, v, out, lse, B, Hq, Hkv, S, D, P, causal, layout, scale, dtype, workspace,
                       workspace_bytes, stream, algo) -> int:
    return load().ring_attn_fwd_algo(q, k, v, out, lse, B, Hq, Hkv, S, D, P, causal, layout, scale, dtype,
                                     workspace, workspace_bytes, stream, algo)


def ring_attn_fwd_step(q, k, v, o_part, lse_part, B, Hq, Hkv, S, D, P, q_shard, kv_shard, causal, layout, scale,
                       dtype, algo, workspace, workspace_bytes, stream) -> int:
    return load().ring_attn_fwd_step(q, k, v, o_part, lse_part, B, Hq, Hkv, S, D, P, q_shard, kv_shard, causal,
                                     layout, scale, dtype, algo, workspace, workspace_bytes, stream)


def ring_attn_fwd_ring_step(q_shard, k_shard, v_shard, o_acc, lse_acc, out, lse_out, B, Hq, Hkv, S, D, P, q_index,
                            kv_index, causal, layout, scale, dtype, flags, workspace, workspace_bytes, stream) -> int:
    return load().ring_attn_fwd_ring_step(q_shard, k_shard, v_shard, o_acc, lse_acc, out, lse_out, B, Hq, Hkv, S, D,
                                          P, q_index, kv_index, causal, layout, scale, dtype, flags, workspace,
                                          workspace_bytes, stream)


def ring_attn_merge(o_parts, lse_parts, n_parts, rows, D, out, lse_out, out_dtype, stream) -> int:
    return load().ring_attn_merge(o_parts, lse_parts, n_parts, rows, D, out, lse_out, out_dtype, stream)


def ring_attn_status(workspace, stream) -> int:
    return load().ring_attn_status(workspace, stream)


def ring_attn_bwd_workspace_bytes(B, Hq, Hkv, S, D, P, causal, layout, dtype) -> int:
    return load().ring_attn_bwd_workspace_bytes(B, Hq, Hkv, S, D, P, causal, layout, dtype)


def ring_attn_bwd(q, k, v, out, lse, dout, dq, dk, dv, B, Hq, Hkv, S, D, P, causal, layout, scale, dtype, workspace,
                  workspace_bytes, stream) -> int:
    return load().ring_attn_bwd(q, k, v, out, lse, dout, dq, dk, dv, B, Hq, Hkv, S, D, P, causal, layout, scale,
                                dtype, workspace, workspace_bytes, stream)


def ring_attn_bwd_ring_workspace_bytes(B, Hq, Hkv, S, D, P, causal, layout, dtype) -> int:
    return load().ring_attn_bwd_ring_workspace_bytes(B, Hq, Hkv, S, D, P, causal, layout, dtype)


def ring_attn_bwd_ring_prep(out_shard, lse_shard, dout_shard, B, Hq, Hkv, S, D, P, q_index, causal, layout, dtype,
                            workspace, workspace_bytes, stream) -> int:
    return load().ring_attn_bwd_ring_prep(out_shard, lse_shard, dout_shard, B, Hq, Hkv, S, D, P, q_index, causal,
                                          layout, dtype, workspace, workspace_bytes, stream)


def ring_attn_bwd_ring_step(q_shard, dout_shard, k_shard, v_shard, dq_acc, dk_acc, dv_acc, dq, dk, dv, B, Hq, Hkv, S,
                            D, P, q_index, kv_index, causal, layout, scale, dtype, parts, flags, workspace,
                            workspace_bytes, stream) -> int:
    return load().ring_attn_bwd_ring_step(q_shard, dout_shard, k_shard, v_shard, dq_acc, dk_acc, dv_acc, dq, dk, dv,
                                          B, Hq, Hkv, S, D, P, q_index, kv_index, causal, layout, scale, dtype, parts,
                                          flags, workspace, workspace_bytes, stream)


def ring_attn_decode_workspace_bytes(B, Hq, Hkv, S, D, P, layout, dtype) -> int:
    return load().ring_attn_decode_workspace_bytes(B, Hq, Hkv, S, D, P, layout, dtype)


def ring_attn_decode(q, k, v, out, lse, B, Hq, Hkv, S, D, P, layout, scale, dtype, workspace, workspace_bytes,
                     stream) -> int:
    return load().ring_attn_decode(q, k, v, out, lse, B, Hq, Hkv, S, D, P, layout, scale, dtype, workspace,
                                   workspace_bytes, stream)


def ring_attn_debug_bwd_visit_counts(S, P, causal, layout, pass_, counts) -> int:
    return load().ring_attn_debug_bwd_visit_counts(S, P, causal, layout, pass_, counts)


def ring_attn_fwd_noalloc(q, k, v, out, lse, B, Hq, Hkv, S, D, P, causal, layout, scale, dtype, stream):
    """Returns (code, device address of the library's scratch for this device or None)."""
    scratch = _vp()
    rc = load().ring_attn_fwd_noalloc(q, k, v, out, lse, B, Hq, Hkv, S, D, P, causal, layout, scale, dtype, stream,
                                      ctypes.byref(scratch))
    return rc, scratch.value


def ring_attn_debug_visit_counts(S, P, causal, layout, tile_q, tile_k, counts_ptr) -> int:
    return load().ring_attn_debug_visit_counts(S, P, causal, layout, tile_q, tile_k, counts_ptr)


def ring_attn_debug_decode_units(B, Hq, Hkv, S, P, causal, layout, tile_q, units_ptr, max_units) -> int:
    return load().ring_attn_debug_decode_units(B, Hq, Hkv, S, P, causal, layout, tile_q, units_ptr, max_units)


def ring_attn_debug_unit_walk(B, Hq, Hkv, S, P, causal, layout, tile_q, tile_k, unit, pairs_ptr, max_pairs) -> int:
    return load().ring_attn_debug_unit_walk(B, Hq, Hkv, S, P, causal, layout, tile_q, tile_k, unit, pairs_ptr,
                                            max_pairs)


def ring_attn_debug_schedule_info(B, Hq, Hkv, S, D, P, causal, layout, info_ptr) -> int:
    return load().ring_attn_debug_schedule_info(B, Hq, Hkv, S, D, P, causal, layout, info_ptr)


def ring_attn_debug_watchdog(timeout_us, workspace, workspace_bytes, stream) -> int:
    return load().ring_attn_debug_watchdog(timeout_us, workspace, workspace_bytes, stream)


def ring_attn_debug_exp2(x, y, n, stream) -> int:
    return load().ring_attn_debug_exp2(x, y, n, stream)

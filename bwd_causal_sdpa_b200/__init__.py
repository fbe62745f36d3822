"""Python binding of libattn.so: causal SDPA forward/backward on B200.

Argument marshalling only. Every function here has the name and the argument
order of the C entry point it calls (include/attn.h); tensors may be passed as
torch tensors (their data_ptr() is used), plain integers (device addresses) or
None (NULL). All computation happens in the library's CUDA kernels; there is
no Python or CPU fallback, and importing this package fails if the library has
not been built (``python bwd_causal_sdpa_b200/build.py``).
"""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libattn.so")

ATTN_BF16 = 0
ATTN_F32 = 1

ATTN_OK = 0
ATTN_EINVAL = -1
ATTN_EUNSUPPORTED = -2
ATTN_EALIGN = -3
ATTN_EWORKSPACE = -4
ATTN_ECUDA = -5
ATTN_EDEVICE_INPUT = -6
ATTN_ETIMEOUT = -7
ATTN_ESCRATCH = -8
ATTN_NOALLOC_SCRATCH_BYTES = 8 << 20

# Every symbol include/attn.h declares, with its ctypes signature.
_P = ctypes.c_void_p
_I = ctypes.c_int
_SIGNATURES = {
    "attn_fwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, ctypes.c_float, _I, _P,
                      ctypes.c_size_t, _P]),
    "attn_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, ctypes.c_float, _I,
                      _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "attn_fwd_gqa": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, ctypes.c_float, _I,
                          _P, ctypes.c_size_t, _P]),
    "attn_bwd_gqa": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, ctypes.c_float,
                          _I, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "attn_saved_bytes": (ctypes.c_size_t, [_I, _I, _I, _I, _I, _I, _I]),
    "attn_fwd_save": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, ctypes.c_float, _I,
                           _P, ctypes.c_size_t, _P, ctypes.c_size_t, _P]),
    "attn_bwd_saved": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I,
                            ctypes.c_float, _I, _P, _P, _P, _P, ctypes.c_size_t, _P,
                            ctypes.c_size_t, _P]),
    "attn_decode": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, ctypes.c_float, _I,
                         _P, ctypes.c_size_t, _P]),
    "attn_decode_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I, _I, _I]),
    "attn_bwd_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, ctypes.c_float,
                              _I, _P, _P, _P, _P]),
    "attn_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I, _I, _I]),
    "attn_proj_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I, _I]),
    "attn_proj_gemm_plan": (_I, [_I, _I, _I, _I, ctypes.POINTER(_I)]),
    "attn_qkv_proj": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P,
                           ctypes.c_size_t, _P]),
    "attn_qkv_proj_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I,
                               _P, ctypes.c_size_t, _P]),
    "attn_out_proj": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "attn_out_proj_bwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "attn_workspace_bytes_gqa": (ctypes.c_size_t, [_I, _I, _I, _I, _I, _I, _I]),
    "attn_get_status": (_I, [_P]),
    "attn_error_string": (ctypes.c_char_p, [_I]),
    "attn_exp2_selftest": (_I, [_P, _P, _I, _P]),
    "attn_debug_withhold": (_I, [_I]),
    "attn_set_backward_route": (_I, [_I]),
    "attn_launch_count": (ctypes.c_ulonglong, []),
    "attn_tile_counts": (_I, [ctypes.POINTER(ctypes.c_ulonglong)] * 3),
    "attn_profile_enable": (_I, [_I]),
    "attn_profile_kinds": (_I, []),
    "attn_profile_read": (_I, [_I, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(_I),
                               ctypes.POINTER(ctypes.c_double)]),
}


class AttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {error_string(code)} (code {code})")
        self.code = code


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python bwd_causal_sdpa_b200/build.py` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream  # torch.cuda.Stream


def error_string(code: int) -> str:
    return _lib.attn_error_string(int(code)).decode()


def attn_workspace_bytes(B, H, T, D, dtype, is_bwd) -> int:
    return int(_lib.attn_workspace_bytes(B, H, T, D, dtype, int(is_bwd)))


def attn_workspace_bytes_gqa(B, H, H_kv, T, D, dtype, is_bwd) -> int:
    return int(_lib.attn_workspace_bytes_gqa(B, H, H_kv, T, D, dtype, int(is_bwd)))


def attn_fwd(q, k, v, rope_cos, rope_sin, cu_seqlens, o, lse, B, H, T, D, scale, dtype,
             workspace, ws_bytes, stream=None) -> int:
    return int(_lib.attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(rope_cos), _ptr(rope_sin),
                             _ptr(cu_seqlens), _ptr(o), _ptr(lse), B, H, T, D, float(scale),
                             dtype, _ptr(workspace), int(ws_bytes), _stream(stream)))


def attn_bwd(q, k, v, o, dO, lse, rope_cos, rope_sin, cu_seqlens, B, H, T, D, scale, dtype,
             dq, dk, dv, workspace, ws_bytes, stream=None) -> int:
    return int(_lib.attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dO), _ptr(lse),
                             _ptr(rope_cos), _ptr(rope_sin), _ptr(cu_seqlens), B, H, T, D,
                             float(scale), dtype, _ptr(dq), _ptr(dk), _ptr(dv),
                             _ptr(workspace), int(ws_bytes), _stream(stream)))


def attn_fwd_gqa(q, k, v, rope_cos, rope_sin, cu_seqlens, o, lse, B, H, H_kv, T, D, scale,
                 dtype, workspace, ws_bytes, stream=None) -> int:
    """attn_fwd with k, v of H_kv heads (grouped-query attention)."""
    return int(_lib.attn_fwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(rope_cos), _ptr(rope_sin),
                                 _ptr(cu_seqlens), _ptr(o), _ptr(lse), B, H, H_kv, T, D,
                                 float(scale), dtype, _ptr(workspace), int(ws_bytes),
                                 _stream(stream)))


def attn_bwd_gqa(q, k, v, o, dO, lse, rope_cos, rope_sin, cu_seqlens, B, H, H_kv, T, D, scale,
                 dtype, dq, dk, dv, workspace, ws_bytes, stream=None) -> int:
    """attn_bwd with k, v, dk, dv of H_kv heads (grouped-query attention)."""
    return int(_lib.attn_bwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dO), _ptr(lse),
                                 _ptr(rope_cos), _ptr(rope_sin), _ptr(cu_seqlens), B, H, H_kv,
                                 T, D, float(scale), dtype, _ptr(dq), _ptr(dk), _ptr(dv),
                                 _ptr(workspace), int(ws_bytes), _stream(stream)))


def attn_saved_bytes(B, H, H_kv, T, D, dtype, has_rope) -> int:
    """Bytes of the buffer attn_fwd_save keeps the rotated operands in (0: none)."""
    return int(_lib.attn_saved_bytes(B, H, H_kv, T, D, dtype, int(bool(has_rope))))


def attn_fwd_save(q, k, v, rope_cos, rope_sin, cu_seqlens, o, lse, B, H, H_kv, T, D, scale,
                  dtype, workspace, ws_bytes, saved, saved_bytes, stream=None) -> int:
    """attn_fwd_gqa that also leaves its rotated q, k in `saved` for attn_bwd_saved."""
    return int(_lib.attn_fwd_save(_ptr(q), _ptr(k), _ptr(v), _ptr(rope_cos), _ptr(rope_sin),
                                  _ptr(cu_seqlens), _ptr(o), _ptr(lse), B, H, H_kv, T, D,
                                  float(scale), dtype, _ptr(workspace), int(ws_bytes),
                                  _ptr(saved), int(saved_bytes), _stream(stream)))


def attn_bwd_saved(q, k, v, o, dO, lse, rope_cos, rope_sin, cu_seqlens, B, H, H_kv, T, D, scale,
                   dtype, dq, dk, dv, workspace, ws_bytes, saved, saved_bytes, stream=None) -> int:
    """attn_bwd_gqa reading the rotated q, k attn_fwd_save left in `saved`."""
    return int(_lib.attn_bwd_saved(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dO), _ptr(lse),
                                   _ptr(rope_cos), _ptr(rope_sin), _ptr(cu_seqlens), B, H, H_kv,
                                   T, D, float(scale), dtype, _ptr(dq), _ptr(dk), _ptr(dv),
                                   _ptr(workspace), int(ws_bytes), _ptr(saved), int(saved_bytes),
                                   _stream(stream)))


def attn_decode(q, k_cache, v_cache, cache_lens, rope_cos, rope_sin, o, lse, B, H, H_kv, T_max,
                D, scale, dtype, workspace, ws_bytes, stream=None) -> int:
    """One new token per sequence against a key/value cache (see include/attn.h)."""
    return int(_lib.attn_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(cache_lens),
                                _ptr(rope_cos), _ptr(rope_sin), _ptr(o), _ptr(lse), B, H, H_kv,
                                T_max, D, float(scale), dtype, _ptr(workspace), int(ws_bytes),
                                _stream(stream)))


def attn_decode_workspace_bytes(B, H, H_kv, T_max, D, dtype) -> int:
    return int(_lib.attn_decode_workspace_bytes(B, H, H_kv, T_max, D, dtype))


def attn_bwd_noalloc(q, k, v, o, dO, lse, rope_cos, rope_sin, cu_seqlens, B, H, T, D, scale,
                     dtype, dq, dk, dv, stream=None) -> int:
    """attn_bwd without a workspace: the library's fixed device scratch array
    is used instead (see include/attn.h for who needs this and its limits)."""
    return int(_lib.attn_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dO), _ptr(lse),
                                     _ptr(rope_cos), _ptr(rope_sin), _ptr(cu_seqlens), B, H, T,
                                     D, float(scale), dtype, _ptr(dq), _ptr(dk), _ptr(dv),
                                     _stream(stream)))


def attn_proj_workspace_bytes(B, T, H, H_kv, D) -> int:
    return int(_lib.attn_proj_workspace_bytes(B, T, H, H_kv, D))


def attn_proj_gemm_plan(M, N, K, f32_out):
    """(code, {bn, tiles_m, tiles_n, splits, kb_per_split, ctas}) of one
    projection GEMM; host arithmetic only."""
    out = (ctypes.c_int * 6)()
    code = int(_lib.attn_proj_gemm_plan(int(M), int(N), int(K), int(bool(f32_out)), out))
    keys = ("bn", "tiles_m", "tiles_n", "splits", "kb_per_split", "ctas")
    return code, dict(zip(keys, list(out)))


def attn_qkv_proj(x, w_qkv, rope_cos, rope_sin, cu_seqlens, q, k, v, B, T, C, H, H_kv, D,
                  workspace, ws_bytes, stream=None) -> int:
    """q, k, v = heads of x W_qkv^T, q and k rotated when tables are given."""
    return int(_lib.attn_qkv_proj(_ptr(x), _ptr(w_qkv), _ptr(rope_cos), _ptr(rope_sin),
                                  _ptr(cu_seqlens), _ptr(q), _ptr(k), _ptr(v), B, T, C, H, H_kv,
                                  D, _ptr(workspace), int(ws_bytes), _stream(stream)))


def attn_qkv_proj_bwd(dq, dk, dv, x, w_qkv, rope_cos, rope_sin, cu_seqlens, dx, dw_qkv, B, T, C,
                      H, H_kv, D, workspace, ws_bytes, stream=None) -> int:
    """dx and dw_qkv (float32) from the gradients of attn_qkv_proj's outputs."""
    return int(_lib.attn_qkv_proj_bwd(_ptr(dq), _ptr(dk), _ptr(dv), _ptr(x), _ptr(w_qkv),
                                      _ptr(rope_cos), _ptr(rope_sin), _ptr(cu_seqlens), _ptr(dx),
                                      _ptr(dw_qkv), B, T, C, H, H_kv, D, _ptr(workspace),
                                      int(ws_bytes), _stream(stream)))


def attn_out_proj(o, w_o, y, B, T, C, H, D, stream=None) -> int:
    """y = o W_o^T, o in the attention's [B, H, T, D] layout."""
    return int(_lib.attn_out_proj(_ptr(o), _ptr(w_o), _ptr(y), B, T, C, H, D, _stream(stream)))


def attn_out_proj_bwd(dy, o, w_o, d_o, dw_o, B, T, C, H, D, stream=None) -> int:
    """d_o = dy W_o ([B, H, T, D]) and dw_o = dy^T o (float32)."""
    return int(_lib.attn_out_proj_bwd(_ptr(dy), _ptr(o), _ptr(w_o), _ptr(d_o), _ptr(dw_o), B, T,
                                      C, H, D, _stream(stream)))


def attn_get_status(stream=None) -> int:
    return int(_lib.attn_get_status(_stream(stream)))


def attn_error_string(code: int) -> str:
    return error_string(code)


def attn_exp2_selftest(x, y, n, stream=None) -> int:
    return int(_lib.attn_exp2_selftest(_ptr(x), _ptr(y), int(n), _stream(stream)))


def attn_debug_withhold(what) -> int:
    """Watchdog test hook; ATTN_EUNSUPPORTED in this (hook-free) library."""
    return int(_lib.attn_debug_withhold(int(what)))


def attn_launch_count() -> int:
    return int(_lib.attn_launch_count())


def attn_set_backward_route(route: int) -> int:
    """0 default, 1 key-tile dK/dV + query-tile dQ pass, 2 CTA-pair dK/dV
    (D = 128) + query-tile dQ pass (see include/attn.h)."""
    return int(_lib.attn_set_backward_route(int(route)))


def attn_tile_counts():
    """(code, fwd_tiles, bwd_tiles, dq_tiles): tile products the tensor-core
    kernels executed since the previous read (counted on the device; resets
    them)."""
    f, b, q = ctypes.c_ulonglong(), ctypes.c_ulonglong(), ctypes.c_ulonglong()
    code = int(_lib.attn_tile_counts(ctypes.byref(f), ctypes.byref(b), ctypes.byref(q)))
    return code, int(f.value), int(b.value), int(q.value)


def attn_profile_enable(on) -> int:
    return int(_lib.attn_profile_enable(int(bool(on))))


def attn_profile_kinds() -> int:
    return int(_lib.attn_profile_kinds())


def attn_profile_read(kind: int):
    """Returns (code, name, launches, total_ms) for one kernel kind."""
    name = ctypes.c_char_p()
    n = ctypes.c_int()
    ms = ctypes.c_double()
    code = int(_lib.attn_profile_read(int(kind), ctypes.byref(name), ctypes.byref(n),
                                      ctypes.byref(ms)))
    return code, (name.value or b"").decode(), int(n.value), float(ms.value)


def profile_summary() -> dict:
    """{kernel name: (timed launches, total ms)} for every kind with launches."""
    out = {}
    for kind in range(attn_profile_kinds()):
        code, name, n, ms = attn_profile_read(kind)
        check(code, "attn_profile_read")
        if n:
            out[name] = (n, ms)
    return out


def check(code: int, where: str = "attn") -> None:
    """Raise AttnError for a non-zero return code."""
    if code != ATTN_OK:
        raise AttnError(code, where)


__all__ = [name for name in list(globals()) if name.startswith(("attn_", "ATTN_"))] + [
    "AttnError", "check", "error_string", "profile_summary", "LIB_PATH"]

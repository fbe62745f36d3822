"""The C ABI surface, on the CPU: the library loads, exports every function
include/attn.h declares, and rejects bad arguments on the host before any
CUDA call (no kernel is launched by these tests)."""

import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^[A-Za-z_][\w \*]*?\b(attn_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    import ctypes

    import bwd_causal_sdpa_b200 as A

    names = _declared_functions()
    assert {"attn_fwd", "attn_bwd", "attn_workspace_bytes", "attn_get_status",
            "attn_error_string"} <= set(names)
    lib = ctypes.CDLL(A.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
        assert hasattr(A, n), f"{n} has no Python binding of the same name"


def test_error_strings_and_codes():
    import bwd_causal_sdpa_b200 as A

    for code in (A.ATTN_OK, A.ATTN_EINVAL, A.ATTN_EUNSUPPORTED, A.ATTN_EALIGN,
                 A.ATTN_EWORKSPACE, A.ATTN_ECUDA, A.ATTN_EDEVICE_INPUT, A.ATTN_ETIMEOUT):
        s = A.attn_error_string(code)
        assert s and "unknown" not in s
    assert "unknown" in A.attn_error_string(12345)


def test_workspace_bytes():
    import bwd_causal_sdpa_b200 as A

    for dtype in (A.ATTN_BF16, A.ATTN_F32):
        for D in (64, 128):
            f = A.attn_workspace_bytes(2, 3, 200, D, dtype, 0)
            b = A.attn_workspace_bytes(2, 3, 200, D, dtype, 1)
            assert f > 0 and b > 0 and f % 256 == 0 and b % 256 == 0
    assert A.attn_workspace_bytes(1, 1, 128, 96, A.ATTN_BF16, 1) == 0
    assert A.attn_workspace_bytes(0, 1, 128, 64, A.ATTN_BF16, 1) == 0
    assert A.attn_workspace_bytes(1, 1, 128, 64, 7, 1) == 0


# Fake, aligned addresses: every call below fails validation on the host, so
# nothing is dereferenced and no CUDA call is made.
P = 1 << 20


def _fwd(**kw):
    import bwd_causal_sdpa_b200 as A

    a = dict(q=P, k=P, v=P, rope_cos=None, rope_sin=None, cu_seqlens=None, o=P, lse=P, B=1, H=1,
             T=128, D=64, scale=0.125, dtype=A.ATTN_BF16, workspace=P, ws_bytes=1 << 30)
    a.update(kw)
    return A.attn_fwd(**a)


def _bwd(**kw):
    import bwd_causal_sdpa_b200 as A

    a = dict(q=P, k=P, v=P, o=P, dO=P, lse=P, rope_cos=None, rope_sin=None, cu_seqlens=None,
             B=1, H=1, T=128, D=64, scale=0.125, dtype=A.ATTN_BF16, dq=P, dk=P, dv=P,
             workspace=P, ws_bytes=1 << 30)
    a.update(kw)
    return A.attn_bwd(**a)


@pytest.mark.parametrize("call", [_fwd, _bwd])
def test_host_validation(call):
    import bwd_causal_sdpa_b200 as A

    assert call(q=None) == A.ATTN_EINVAL
    assert call(B=0) == A.ATTN_EINVAL
    assert call(T=-3) == A.ATTN_EINVAL
    assert call(scale=float("nan")) == A.ATTN_EINVAL
    assert call(dtype=5) == A.ATTN_EINVAL
    assert call(rope_cos=P) == A.ATTN_EINVAL          # sin missing
    assert call(D=96) == A.ATTN_EUNSUPPORTED
    assert call(B=1 << 16, H=1 << 10, T=1 << 10) == A.ATTN_EUNSUPPORTED
    assert call(k=P + 8) == A.ATTN_EALIGN
    assert call(workspace=P + 4) == A.ATTN_EALIGN
    assert call(cu_seqlens=P + 2) == A.ATTN_EALIGN
    assert call(rope_cos=P + 4, rope_sin=P) == A.ATTN_EALIGN
    assert call(workspace=None) == A.ATTN_EWORKSPACE
    assert call(ws_bytes=16) == A.ATTN_EWORKSPACE


def test_bwd_specific_validation():
    import bwd_causal_sdpa_b200 as A

    assert _bwd(dO=None) == A.ATTN_EINVAL
    assert _bwd(dv=P + 8) == A.ATTN_EALIGN
    assert _fwd(lse=None) == A.ATTN_EINVAL
    assert _fwd(o=P + 2) == A.ATTN_EALIGN


def _fwd_gqa(**kw):
    import bwd_causal_sdpa_b200 as A

    a = dict(q=P, k=P, v=P, rope_cos=None, rope_sin=None, cu_seqlens=None, o=P, lse=P, B=1, H=4,
             H_kv=2, T=128, D=64, scale=0.125, dtype=A.ATTN_BF16, workspace=P, ws_bytes=1 << 30)
    a.update(kw)
    return A.attn_fwd_gqa(**a)


def _bwd_gqa(**kw):
    import bwd_causal_sdpa_b200 as A

    a = dict(q=P, k=P, v=P, o=P, dO=P, lse=P, rope_cos=None, rope_sin=None, cu_seqlens=None,
             B=1, H=4, H_kv=2, T=128, D=64, scale=0.125, dtype=A.ATTN_BF16, dq=P, dk=P, dv=P,
             workspace=P, ws_bytes=1 << 30)
    a.update(kw)
    return A.attn_bwd_gqa(**a)


@pytest.mark.parametrize("call", [_fwd_gqa, _bwd_gqa])
def test_grouped_query_host_validation(call):
    import bwd_causal_sdpa_b200 as A

    assert call(H_kv=0) == A.ATTN_EINVAL
    assert call(H_kv=-2) == A.ATTN_EINVAL
    assert call(H_kv=3) == A.ATTN_EINVAL       # 4 query heads do not split into 3 groups
    assert call(H_kv=8) == A.ATTN_EINVAL       # more key/value heads than query heads
    assert call(q=None) == A.ATTN_EINVAL
    assert call(D=96) == A.ATTN_EUNSUPPORTED
    assert call(v=P + 8) == A.ATTN_EALIGN
    assert call(ws_bytes=16) == A.ATTN_EWORKSPACE


def test_grouped_query_workspace_bytes():
    import bwd_causal_sdpa_b200 as A

    # G = 1 is the plain call's plan
    for is_bwd in (0, 1):
        assert (A.attn_workspace_bytes_gqa(2, 4, 4, 300, 128, A.ATTN_BF16, is_bwd)
                == A.attn_workspace_bytes(2, 4, 300, 128, A.ATTN_BF16, is_bwd))
    # a small grid splits the bf16 backward's groups: two fp32 [B*H_kv*T*D] accumulators more
    base = A.attn_workspace_bytes(1, 16, 4096, 128, A.ATTN_BF16, 1)
    split = A.attn_workspace_bytes_gqa(1, 16, 1, 4096, 128, A.ATTN_BF16, 1)
    assert split >= base + 2 * 4096 * 128 * 4
    # enough key/value heads x key tiles: no split, no extra room
    assert (A.attn_workspace_bytes_gqa(4, 16, 8, 1280, 128, A.ATTN_BF16, 1)
            <= A.attn_workspace_bytes(4, 16, 1280, 128, A.ATTN_BF16, 1))
    assert A.attn_workspace_bytes_gqa(1, 4, 3, 128, 64, A.ATTN_BF16, 1) == 0
    assert A.attn_workspace_bytes_gqa(1, 4, 0, 128, 64, A.ATTN_BF16, 1) == 0


def _decode(**kw):
    import bwd_causal_sdpa_b200 as A

    a = dict(q=P, k_cache=P, v_cache=P, cache_lens=P, rope_cos=None, rope_sin=None, o=P, lse=P,
             B=2, H=8, H_kv=2, T_max=1000, D=128, scale=0.088, dtype=A.ATTN_BF16, workspace=P,
             ws_bytes=1 << 30)
    a.update(kw)
    return A.attn_decode(**a)


def test_decode_host_validation_and_workspace():
    import bwd_causal_sdpa_b200 as A

    assert _decode(q=None) == A.ATTN_EINVAL
    assert _decode(cache_lens=None) == A.ATTN_EINVAL
    assert _decode(H_kv=3) == A.ATTN_EINVAL
    assert _decode(T_max=0) == A.ATTN_EINVAL
    assert _decode(dtype=9) == A.ATTN_EINVAL
    assert _decode(rope_sin=P) == A.ATTN_EINVAL
    assert _decode(D=96) == A.ATTN_EUNSUPPORTED
    assert _decode(H=130, H_kv=2) == A.ATTN_EUNSUPPORTED   # 65 query heads per cached head
    assert _decode(v_cache=P + 8) == A.ATTN_EALIGN
    assert _decode(cache_lens=P + 2) == A.ATTN_EALIGN
    assert _decode(workspace=None) == A.ATTN_EWORKSPACE
    assert _decode(ws_bytes=64) == A.ATTN_EWORKSPACE
    # partial sums f32 [B*H][chunks][D] plus two f32 [B*H][chunks], chunks of 128 tokens
    nb = A.attn_decode_workspace_bytes(2, 8, 2, 1000, 128, A.ATTN_BF16)
    assert nb >= 2 * 8 * 8 * (128 + 2) * 4
    assert A.attn_decode_workspace_bytes(2, 8, 3, 1000, 128, A.ATTN_BF16) == 0
    assert A.attn_decode_workspace_bytes(2, 8, 2, 1000, 80, A.ATTN_BF16) == 0


def test_projection_validation_on_host():
    import bwd_causal_sdpa_b200 as A

    def qkv(**kw):
        a = dict(x=P, w_qkv=P, rope_cos=None, rope_sin=None, cu_seqlens=None, q=P, k=P, v=P, B=1,
                 T=128, C=64, H=2, H_kv=1, D=64, workspace=None, ws_bytes=0)
        a.update(kw)
        return A.attn_qkv_proj(**a)

    def qkv_bwd(**kw):
        a = dict(dq=P, dk=P, dv=P, x=P, w_qkv=P, rope_cos=None, rope_sin=None, cu_seqlens=None,
                 dx=P, dw_qkv=P, B=1, T=128, C=64, H=2, H_kv=1, D=64, workspace=None, ws_bytes=0)
        a.update(kw)
        return A.attn_qkv_proj_bwd(**a)

    def out(**kw):
        a = dict(o=P, w_o=P, y=P, B=1, T=128, C=64, H=2, D=64)
        a.update(kw)
        return A.attn_out_proj(**a)

    def out_bwd(**kw):
        a = dict(dy=P, o=P, w_o=P, d_o=P, dw_o=P, B=1, T=128, C=64, H=2, D=64)
        a.update(kw)
        return A.attn_out_proj_bwd(**a)

    for call in (qkv, qkv_bwd):
        assert call(x=None) == A.ATTN_EINVAL
        assert call(H_kv=0) == A.ATTN_EINVAL
        assert call(rope_cos=P) == A.ATTN_EINVAL  # one table without the other
        assert call(D=96) == A.ATTN_EUNSUPPORTED
        assert call(T=200) == A.ATTN_EUNSUPPORTED  # not a multiple of 128
        assert call(C=60) == A.ATTN_EUNSUPPORTED   # rows not 16-byte strided
        assert call(B=0) == A.ATTN_EUNSUPPORTED
        assert call(x=P + 8) == A.ATTN_EALIGN
    # RoPE with packed documents needs the workspace (document positions);
    # the backward with RoPE needs it for the rotated-back gradients
    assert qkv(rope_cos=P, rope_sin=P, cu_seqlens=P) == A.ATTN_EWORKSPACE
    assert qkv_bwd(rope_cos=P, rope_sin=P) == A.ATTN_EWORKSPACE
    for call in (out, out_bwd):
        assert call(o=None) == A.ATTN_EINVAL
        assert call(D=32) == A.ATTN_EUNSUPPORTED
        assert call(T=64) == A.ATTN_EUNSUPPORTED
        assert call(o=P + 4) == A.ATTN_EALIGN
    assert out(y=None) == A.ATTN_EINVAL
    assert out_bwd(dw_o=None) == A.ATTN_EINVAL
    ws = A.attn_proj_workspace_bytes(2, 256, 3, 1, 64)
    assert ws >= 2 * 256 * 4 * 2 + 2 * 256 * 4 * 64 * 2 and ws % 256 == 0
    assert A.attn_proj_workspace_bytes(2, 200, 3, 1, 64) == 0


def test_debug_hook_is_absent_from_the_product_library():
    import ctypes

    import bwd_causal_sdpa_b200 as A

    # the product library has no hooks compiled in; the call touches no CUDA
    assert A.attn_debug_withhold(1) == A.ATTN_EUNSUPPORTED
    debug = os.path.join(ROOT, "bwd_causal_sdpa_b200", "libattn_debug.so")
    if os.path.exists(debug):
        lib = ctypes.CDLL(debug)
        for n in _declared_functions():
            assert hasattr(lib, n), f"{n} missing from the watchdog build"


def test_projection_gemm_plan():
    """The tile width and K split of the projection GEMM (host arithmetic)."""
    import bwd_causal_sdpa_b200 as A

    def plan(M, N, K, f32):
        code, p = A.attn_proj_gemm_plan(M, N, K, f32)
        assert code == A.ATTN_OK
        return p

    # bf16 outputs never split K; a persistent grid of at most 148 CTAs
    p = plan(8192, 3072, 2048, False)
    assert (p["bn"], p["tiles_m"], p["tiles_n"], p["splits"], p["ctas"]) == (256, 64, 12, 1, 148)
    assert p["kb_per_split"] == 32
    assert plan(8192, 200, 768, False)["bn"] == 128
    # fp32 weight gradients of the 8K layer: 192 tiles fill 1.3 rounds of 148
    # SMs; two K parts of 64 blocks make 384 units
    p = plan(3072, 2048, 8192, True)
    assert (p["splits"], p["kb_per_split"], p["ctas"]) == (2, 64, 148)
    # 128 tiles: the extra reduce traffic of a split costs more than it saves
    assert plan(2048, 2048, 8192, True)["splits"] == 1
    # few tiles with a long K (the 237M layer's weights): split
    assert plan(2304, 768, 8192, True)["splits"] == 2
    p = plan(768, 768, 8192, True)
    assert (p["splits"], p["kb_per_split"], p["ctas"]) == (8, 16, 144)
    # every part gets at least one K block, and no more than K holds
    for M, N, K in [(128, 8, 64), (320, 200, 512), (192, 8, 128), (100, 100, 100000)]:
        p = plan(M, N, K, True)
        nkb = -(-K // 64)
        assert 1 <= p["splits"] <= nkb and (p["splits"] - 1) * p["kb_per_split"] < nkb
        assert p["splits"] * p["kb_per_split"] >= nkb
        assert p["kb_per_split"] % 2 == 0  # the kernel's stages hold two K blocks
    assert A.attn_proj_gemm_plan(0, 8, 8, True)[0] == A.ATTN_EINVAL


def test_noalloc_counts_document_ranges_only_when_packed():
    """attn_bwd_noalloc's scratch holds Delta (4*B*H*T bytes) and, only when
    documents are packed, the document ranges (8*B*T more): a problem whose
    Delta alone fits the 8 MiB array is rejected with packing and passes the
    size check without it (on a machine without a GPU the call then stops at
    the device query, before any launch)."""
    import bwd_causal_sdpa_b200 as A

    P = 1 << 20  # fake aligned addresses, never dereferenced
    B, H, T = 1, 1, (1 << 21) - 256  # 4*T bytes: just under 8 MiB
    args = (P, P, P, P, P, P, None, None)
    tail = (B, H, T, 64, 0.125, A.ATTN_BF16, P, P, P, None)
    assert A.attn_bwd_noalloc(*args, P, *tail) == A.ATTN_ESCRATCH
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("the unpacked call would launch kernels on fake addresses")
    assert A.attn_bwd_noalloc(*args, None, *tail) == A.ATTN_ECUDA


def test_saved_operand_buffer_size_and_validation():
    import bwd_causal_sdpa_b200 as A

    up = lambda x: (x + 255) // 256 * 256
    B, H, Hkv, T, D = 2, 8, 2, 300, 128
    nt = (T + 127) // 128
    want = (up(B * H * T * D * 2) + up(B * Hkv * T * D * 2) + up(B * H * nt * 16)
            + up(B * Hkv * nt * 4) + up(2 * B * T * 4))  # rotated q, k, factors, document ranges
    assert A.attn_saved_bytes(B, H, Hkv, T, D, A.ATTN_BF16, 1) == want
    # nothing to keep: float32 storage, no RoPE, invalid sizes
    assert A.attn_saved_bytes(B, H, Hkv, T, D, A.ATTN_F32, 1) == 0
    assert A.attn_saved_bytes(B, H, Hkv, T, D, A.ATTN_BF16, 0) == 0
    assert A.attn_saved_bytes(B, H, 3, T, D, A.ATTN_BF16, 1) == 0
    assert A.attn_saved_bytes(B, H, Hkv, T, 96, A.ATTN_BF16, 1) == 0

    common = dict(q=P, k=P, v=P, rope_cos=P, rope_sin=P, cu_seqlens=None, B=B, H=H, H_kv=Hkv,
                  T=T, D=D, scale=0.088, dtype=A.ATTN_BF16, workspace=P, ws_bytes=1 << 30)
    fwd = lambda **kw: A.attn_fwd_save(**{**common, "o": P, "lse": P, "saved": P,
                                          "saved_bytes": want, **kw})
    bwd = lambda **kw: A.attn_bwd_saved(**{**common, "o": P, "dO": P, "lse": P, "dq": P,
                                           "dk": P, "dv": P, "saved": P, "saved_bytes": want,
                                           **kw})
    for call in (fwd, bwd):
        assert call(saved=P + 8) == A.ATTN_EALIGN
        assert call(saved_bytes=want - 1) == A.ATTN_EWORKSPACE
        assert call(q=None) == A.ATTN_EINVAL  # the plain call's checks still apply


def test_backward_route_argument_checked():
    import bwd_causal_sdpa_b200 as A

    assert A.attn_set_backward_route(3) == A.ATTN_EINVAL
    assert A.attn_set_backward_route(-1) == A.ATTN_EINVAL
    assert A.attn_set_backward_route(0) == A.ATTN_OK

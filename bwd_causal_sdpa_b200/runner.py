"""Device buffers for one attention problem, and the two C-ABI calls on them.

PyTorch is used here only to own device memory and streams; every step of the
attention runs in libattn.so through the ctypes binding.
"""

from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

from . import (ATTN_BF16, ATTN_F32, attn_bwd, attn_bwd_gqa, attn_bwd_saved, attn_fwd,
               attn_fwd_gqa, attn_fwd_save, attn_get_status, attn_saved_bytes,
               attn_workspace_bytes, attn_workspace_bytes_gqa, check)


def torch_dtype(dtype: int):
    return torch.bfloat16 if dtype == ATTN_BF16 else torch.float32


def to_device(x: np.ndarray, dtype: int, device) -> torch.Tensor:
    """float32 numpy (already bf16-representable for bf16) -> device tensor."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(device=device, dtype=torch_dtype(dtype)).contiguous()


@dataclass
class Problem:
    B: int
    H: int
    T: int
    D: int
    scale: float
    dtype: int
    H_kv: int


class AttnRunner:
    """Holds q, k, v, dO (inputs), o, lse, dq, dk, dv (outputs), the RoPE
    tables, cu_seqlens and one workspace sized for the larger of the two
    calls, all on one device. With H_kv < H (grouped-query attention) k, v,
    dk, dv have H_kv heads and the *_gqa entry points are called.

    save=True (a training step's usual pattern) also holds the buffer in
    which attn_fwd_save keeps the forward's rotated q, k, and runs the pair
    attn_fwd_save / attn_bwd_saved; backward() then needs the forward() of
    the same inputs before it. save=False runs the plain calls."""

    def __init__(self, B, H, T, D, *, dtype=ATTN_BF16, scale=None, rope=None, cu_seqlens=None,
                 device="cuda", stream: Optional[torch.cuda.Stream] = None, H_kv=None,
                 save: bool = False):
        H_kv = H if H_kv is None else H_kv
        self.p = Problem(B, H, T, D, 1.0 / math.sqrt(D) if scale is None else scale, dtype, H_kv)
        self.device = torch.device(device)
        self.stream = stream
        td = torch_dtype(dtype)
        mk = lambda h: torch.empty((B, h, T, D), dtype=td, device=self.device)
        self.q, self.k, self.v, self.do = mk(H), mk(H_kv), mk(H_kv), mk(H)
        self.o, self.dq, self.dk, self.dv = mk(H), mk(H), mk(H_kv), mk(H_kv)
        self.lse = torch.empty((B, H, T), dtype=torch.float32, device=self.device)
        self.rope_cos = self.rope_sin = None
        if rope is not None:
            c, s = rope
            self.rope_cos = torch.from_numpy(np.ascontiguousarray(c, np.float32)).to(self.device)
            self.rope_sin = torch.from_numpy(np.ascontiguousarray(s, np.float32)).to(self.device)
        self.cu = None
        if cu_seqlens is not None:
            self.cu = torch.from_numpy(np.asarray(cu_seqlens, dtype=np.int32)).to(self.device)
        if H_kv == H:
            self.ws_bytes = max(attn_workspace_bytes(B, H, T, D, dtype, 0),
                                attn_workspace_bytes(B, H, T, D, dtype, 1))
        else:
            self.ws_bytes = max(attn_workspace_bytes_gqa(B, H, H_kv, T, D, dtype, 0),
                                attn_workspace_bytes_gqa(B, H, H_kv, T, D, dtype, 1))
        self.ws = torch.empty(max(self.ws_bytes, 16), dtype=torch.uint8, device=self.device)
        self.saved_bytes = attn_saved_bytes(B, H, H_kv, T, D, dtype, rope is not None) if save else 0
        self.saved = (torch.empty(self.saved_bytes, dtype=torch.uint8, device=self.device)
                      if self.saved_bytes else None)

    @classmethod
    def from_workload(cls, w, device="cuda", stream=None, save: bool = False) -> "AttnRunner":
        dtype = ATTN_BF16 if w.dtype == "bf16" else ATTN_F32
        rope = None if w.rope_cos is None else (w.rope_cos, w.rope_sin)
        r = cls(w.B, w.H, w.T, w.D, dtype=dtype, scale=w.scale, rope=rope,
                cu_seqlens=w.cu_seqlens, device=device, stream=stream, H_kv=w.kv_heads, save=save)
        r.load_inputs(w.q, w.k, w.v, w.do)
        return r

    def load_inputs(self, q, k, v, do):
        for dst, src in ((self.q, q), (self.k, k), (self.v, v), (self.do, do)):
            dst.copy_(to_device(src, self.p.dtype, self.device))

    def forward(self) -> None:
        p = self.p
        if self.saved is not None:
            check(attn_fwd_save(self.q, self.k, self.v, self.rope_cos, self.rope_sin, self.cu,
                                self.o, self.lse, p.B, p.H, p.H_kv, p.T, p.D, p.scale, p.dtype,
                                self.ws, self.ws_bytes, self.saved, self.saved_bytes,
                                self.stream), "attn_fwd_save")
            return
        if p.H_kv != p.H:
            check(attn_fwd_gqa(self.q, self.k, self.v, self.rope_cos, self.rope_sin, self.cu,
                               self.o, self.lse, p.B, p.H, p.H_kv, p.T, p.D, p.scale, p.dtype,
                               self.ws, self.ws_bytes, self.stream), "attn_fwd_gqa")
            return
        check(attn_fwd(self.q, self.k, self.v, self.rope_cos, self.rope_sin, self.cu, self.o,
                       self.lse, p.B, p.H, p.T, p.D, p.scale, p.dtype, self.ws, self.ws_bytes,
                       self.stream), "attn_fwd")

    def backward(self) -> None:
        p = self.p
        if self.saved is not None:
            check(attn_bwd_saved(self.q, self.k, self.v, self.o, self.do, self.lse, self.rope_cos,
                                 self.rope_sin, self.cu, p.B, p.H, p.H_kv, p.T, p.D, p.scale,
                                 p.dtype, self.dq, self.dk, self.dv, self.ws, self.ws_bytes,
                                 self.saved, self.saved_bytes, self.stream), "attn_bwd_saved")
            return
        if p.H_kv != p.H:
            check(attn_bwd_gqa(self.q, self.k, self.v, self.o, self.do, self.lse, self.rope_cos,
                               self.rope_sin, self.cu, p.B, p.H, p.H_kv, p.T, p.D, p.scale,
                               p.dtype, self.dq, self.dk, self.dv, self.ws, self.ws_bytes,
                               self.stream), "attn_bwd_gqa")
            return
        check(attn_bwd(self.q, self.k, self.v, self.o, self.do, self.lse, self.rope_cos,
                       self.rope_sin, self.cu, p.B, p.H, p.T, p.D, p.scale, p.dtype, self.dq,
                       self.dk, self.dv, self.ws, self.ws_bytes, self.stream), "attn_bwd")

    def status(self) -> int:
        return attn_get_status(self.stream)

    def results(self) -> dict:
        """Outputs as float64 numpy arrays (synchronises)."""
        torch.cuda.synchronize(self.device)
        f = lambda t: t.detach().to(torch.float64).cpu().numpy()
        return {"o": f(self.o), "lse": f(self.lse), "dq": f(self.dq), "dk": f(self.dk),
                "dv": f(self.dv)}


class DecodeRunner:
    """Device buffers for one decode step (q, the key/value cache, the cache
    lengths, o, lse, the RoPE tables and the workspace) and the attn_decode
    call on them."""

    def __init__(self, w, device="cuda", stream: Optional[torch.cuda.Stream] = None):
        from . import attn_decode_workspace_bytes

        self.w = w
        self.device = torch.device(device)
        self.stream = stream
        self.dtype = ATTN_BF16 if w.dtype == "bf16" else ATTN_F32
        self.q = to_device(w.q, self.dtype, self.device)
        self.k = to_device(w.k_cache, self.dtype, self.device)
        self.v = to_device(w.v_cache, self.dtype, self.device)
        self.lens = torch.from_numpy(np.asarray(w.cache_lens, np.int32)).to(self.device)
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((w.B, w.H), dtype=torch.float32, device=self.device)
        self.rope_cos = self.rope_sin = None
        if w.rope_cos is not None:
            self.rope_cos = torch.from_numpy(np.ascontiguousarray(w.rope_cos, np.float32)).to(self.device)
            self.rope_sin = torch.from_numpy(np.ascontiguousarray(w.rope_sin, np.float32)).to(self.device)
        self.ws_bytes = attn_decode_workspace_bytes(w.B, w.H, w.H_kv, w.T_max, w.D, self.dtype)
        self.ws = torch.empty(max(self.ws_bytes, 16), dtype=torch.uint8, device=self.device)

    def run(self) -> None:
        from . import attn_decode

        w = self.w
        check(attn_decode(self.q, self.k, self.v, self.lens, self.rope_cos, self.rope_sin, self.o,
                          self.lse, w.B, w.H, w.H_kv, w.T_max, w.D, w.scale, self.dtype, self.ws,
                          self.ws_bytes, self.stream), "attn_decode")

    def status(self) -> int:
        return attn_get_status(self.stream)

    def results(self) -> dict:
        torch.cuda.synchronize(self.device)
        f = lambda t: t.detach().to(torch.float64).cpu().numpy()
        return {"o": f(self.o), "lse": f(self.lse)}


class ProjRunner:
    """Device buffers for the projections around one attention layer (x, the
    weights, q, k, v, o, the output and the gradients) and the four
    projection calls on them."""

    def __init__(self, w, device="cuda", stream: Optional[torch.cuda.Stream] = None,
                 rope: bool = True):
        from . import attn_proj_workspace_bytes

        c = w.cfg
        self.w = w
        self.device = torch.device(device)
        self.stream = stream
        dev = lambda a: to_device(a, ATTN_BF16, self.device)
        self.x, self.w_qkv, self.w_o, self.o = dev(w.x), dev(w.w_qkv), dev(w.w_o), dev(w.o)
        self.gq, self.gk, self.gv, self.dy = dev(w.dq), dev(w.dk), dev(w.dv), dev(w.dy)
        bf = dict(dtype=torch.bfloat16, device=self.device)
        self.q = torch.empty((c.B, c.H, c.T, c.D), **bf)
        self.k = torch.empty((c.B, c.H_kv, c.T, c.D), **bf)
        self.v = torch.empty((c.B, c.H_kv, c.T, c.D), **bf)
        self.y = torch.empty((c.B, c.T, c.C), **bf)
        self.dx = torch.empty((c.B, c.T, c.C), **bf)
        self.d_o = torch.empty((c.B, c.H, c.T, c.D), **bf)
        self.dw_qkv = torch.empty(tuple(w.w_qkv.shape), dtype=torch.float32, device=self.device)
        self.dw_o = torch.empty(tuple(w.w_o.shape), dtype=torch.float32, device=self.device)
        self.rope_cos = self.rope_sin = None
        if rope and w.rope_cos is not None:
            self.rope_cos = torch.from_numpy(np.ascontiguousarray(w.rope_cos, np.float32)).to(self.device)
            self.rope_sin = torch.from_numpy(np.ascontiguousarray(w.rope_sin, np.float32)).to(self.device)
        self.cu = None
        if w.cu_seqlens is not None:
            self.cu = torch.from_numpy(np.asarray(w.cu_seqlens, dtype=np.int32)).to(self.device)
        self.ws_bytes = attn_proj_workspace_bytes(c.B, c.T, c.H, c.H_kv, c.D)
        self.ws = torch.empty(max(self.ws_bytes, 16), dtype=torch.uint8, device=self.device)

    def qkv(self) -> None:
        from . import attn_qkv_proj

        c = self.w.cfg
        check(attn_qkv_proj(self.x, self.w_qkv, self.rope_cos, self.rope_sin, self.cu, self.q,
                            self.k, self.v, c.B, c.T, c.C, c.H, c.H_kv, c.D, self.ws,
                            self.ws_bytes, self.stream), "attn_qkv_proj")

    def qkv_bwd(self) -> None:
        from . import attn_qkv_proj_bwd

        c = self.w.cfg
        check(attn_qkv_proj_bwd(self.gq, self.gk, self.gv, self.x, self.w_qkv, self.rope_cos,
                                self.rope_sin, self.cu, self.dx, self.dw_qkv, c.B, c.T, c.C, c.H,
                                c.H_kv, c.D, self.ws, self.ws_bytes, self.stream),
              "attn_qkv_proj_bwd")

    def out(self) -> None:
        from . import attn_out_proj

        c = self.w.cfg
        check(attn_out_proj(self.o, self.w_o, self.y, c.B, c.T, c.C, c.H, c.D, self.stream),
              "attn_out_proj")

    def out_bwd(self) -> None:
        from . import attn_out_proj_bwd

        c = self.w.cfg
        check(attn_out_proj_bwd(self.dy, self.o, self.w_o, self.d_o, self.dw_o, c.B, c.T, c.C,
                                c.H, c.D, self.stream), "attn_out_proj_bwd")

    def status(self) -> int:
        return attn_get_status(self.stream)

    def results(self) -> dict:
        torch.cuda.synchronize(self.device)
        f = lambda t: t.detach().to(torch.float64).cpu().numpy()
        return {n: f(getattr(self, n)) for n in
                ("q", "k", "v", "y", "dx", "d_o", "dw_qkv", "dw_o")}

"""Python binding of libtq (include/tq.h): TurboQuant encode, scores and
compressed-cache decode attention on B200.

Argument marshalling only -- every step of the method runs in libtq's CUDA
kernels.  PyTorch supplies device memory and the current stream.  Packed code
and sign words are returned as torch.int32 tensors holding the uint32 bit
patterns of the C ABI.
"""
from __future__ import annotations

import ctypes as C
from typing import Optional

import numpy as np

from . import _lib as L
from ._lib import (BF16, F16, F32, LAYOUT_BLOCK32, LAYOUT_ROW, MODE_MSE, MODE_MSE_UNBIASED, MODE_PROD,  # noqa: F401
                   ROT_DENSE, ROT_HADAMARD, STORE_RNORM_F16, TQError)

__all__ = [
    "TQParams", "tq_build_codebook", "tq_make_rotation", "tq_params_create", "tq_encode_mse", "tq_encode_prod",
    "tq_decode", "tq_scores", "tq_decode_attention", "tq_decode_attention_workspace_size",
    "tq_decode_attention_noalloc", "tq_decode_step", "tq_decode_step_workspace_size",
    "tq_check_wait_expiry", "tq_sync_check", "tq_version", "lib_path", "TQError",
    "F32", "F16", "BF16", "LAYOUT_ROW", "LAYOUT_BLOCK32", "MODE_MSE", "MODE_PROD", "MODE_MSE_UNBIASED",
    "STORE_RNORM_F16", "ROT_HADAMARD", "ROT_DENSE",
]


def _torch():
    import torch

    return torch


def lib_path() -> str:
    return L.LIB_PATH


def tq_version() -> str:
    return L.lib().tq_version().decode()


def _stream(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _ptr(t) -> C.c_void_p:
    return C.c_void_p(0 if t is None else t.data_ptr())


def _dtype_code(t) -> int:
    torch = _torch()
    return {torch.float32: F32, torch.float16: F16, torch.bfloat16: BF16}[t.dtype]


def _ws(nbytes: int, device):
    torch = _torch()
    if nbytes == 0:
        return None
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def tq_build_codebook(d: int, bits: int):
    """(centroids [2^bits], boundaries [2^bits - 1]) as float32 numpy arrays."""
    n = 1 << bits
    c = np.zeros(n, np.float32)
    b = np.zeros(max(n - 1, 1), np.float32)
    L.check("tq_build_codebook", L.lib().tq_build_codebook(
        d, bits, c.ctypes.data_as(C.POINTER(C.c_float)), b.ctypes.data_as(C.POINTER(C.c_float))))
    return c, b[: n - 1]


def tq_make_rotation(G):
    """Dense rotation Pi (float32 [d, d], y = Pi x) from a Gaussian draw G."""
    G = np.ascontiguousarray(G, dtype=np.float64)
    d = G.shape[0]
    pi = np.zeros((d, d), np.float32)
    L.check("tq_make_rotation", L.lib().tq_make_rotation(
        d, G.ctypes.data_as(C.c_void_p), pi.ctypes.data_as(C.POINTER(C.c_float))))
    return pi


class TQParams:
    """Handle of one quantizer (tq_params_create / tq_params_destroy)."""

    def __init__(self, d: int, bits: int, mode: int, rot: int = ROT_HADAMARD, m: int = 0,
                 signs=None, S=None, G=None):
        self._h = C.c_void_p()
        sg = None if signs is None else np.ascontiguousarray(signs, dtype=np.int8)
        Sm = None if S is None else np.ascontiguousarray(S, dtype=np.float32)
        Gm = None if G is None else np.ascontiguousarray(G, dtype=np.float64)
        L.check("tq_params_create", L.lib().tq_params_create(
            d, bits, mode, rot, m,
            None if sg is None else sg.ctypes.data_as(C.c_void_p),
            None if Sm is None else Sm.ctypes.data_as(C.c_void_p),
            None if Gm is None else Gm.ctypes.data_as(C.c_void_p),
            C.byref(self._h)))
        vals = [C.c_int() for _ in range(5)]
        L.check("tq_params_info", L.lib().tq_params_info(self._h, *[C.byref(v) for v in vals]))
        self.d, self.bits, self.mode, self.rot = d, bits, mode & 0xFF, rot
        # residual norms stored as fp16 (torch.float16 tensors) instead of fp32
        self.rnorm_dtype = "float16" if mode & STORE_RNORM_F16 else "float32"
        self.d_pad, self.k, self.code_words, self.sign_words, self.m = [v.value for v in vals]

    @property
    def handle(self):
        return self._h

    def tables(self):
        """Host copies of (centroids, boundaries, Pi or None) used by the kernels."""
        n = 1 << self.k
        c = np.zeros(n, np.float32)
        b = np.zeros(max(n - 1, 1), np.float32)
        pi = np.zeros((self.d, self.d), np.float32) if self.rot == ROT_DENSE else None
        fp = C.POINTER(C.c_float)
        L.check("tq_params_tables", L.lib().tq_params_tables(
            self._h, c.ctypes.data_as(fp), b.ctypes.data_as(fp),
            None if pi is None else pi.ctypes.data_as(fp)))
        return c, b[: n - 1], pi

    def close(self):
        if self._h:
            L.lib().tq_params_destroy(self._h)
            self._h = C.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def tq_params_create(d, bits, mode, rot=ROT_HADAMARD, m=0, signs=None, S=None, G=None) -> TQParams:
    return TQParams(d, bits, mode, rot, m, signs, S, G)


def _rows(x, d):
    if x.dim() == 1:
        x = x.view(1, -1)
    x2 = x.reshape(-1, x.shape[-1])
    if x2.shape[-1] != d:
        raise ValueError(f"last dimension {x2.shape[-1]} != d {d}")
    if x2.stride(-1) != 1:
        x2 = x2.contiguous()
    return x2, x2.stride(0)


def _segments(n_vec, seg_len, seg_cap, block):
    sl = seg_len or n_vec
    if sl == 0:
        return 0, 0, 0
    sc = seg_cap or ((sl + 31) // 32 * 32 if block else sl)
    return sl, sc, n_vec // sl


def tq_encode_mse(p: TQParams, x, layout: int = LAYOUT_ROW, seg_len: int = 0, seg_cap: int = 0,
                  codes=None, norms=None, stream=None):
    """Q_MSE encode of the rows of x (any leading shape, last dim d).
    Returns (codes int32, norms float32)."""
    torch = _torch()
    x2, ld = _rows(x, p.d)
    n = x2.shape[0]
    sl, sc, ns = _segments(n, seg_len, seg_cap, layout == LAYOUT_BLOCK32)
    if codes is None:
        shape = (ns * sc // 32, p.k * p.d_pad) if layout == LAYOUT_BLOCK32 else (ns * sc, p.code_words)
        codes = torch.zeros(shape, dtype=torch.int32, device=x2.device)
    if norms is None:
        norms = torch.zeros(ns * sc, dtype=torch.float32, device=x2.device)
    need = C.c_size_t()
    L.check("tq_encode_workspace_size", L.lib().tq_encode_workspace_size(p.handle, n, C.byref(need)))
    ws = _ws(need.value, x2.device)
    L.check("tq_encode_mse", L.lib().tq_encode_mse(
        p.handle, _ptr(x2), _dtype_code(x2), n, ld, sl, sc, layout, _ptr(codes), _ptr(norms),
        _ptr(ws), need.value, _stream(stream)))
    return codes, norms


def tq_encode_prod(p: TQParams, x, seg_len: int = 0, seg_cap: int = 0, out=None, stream=None):
    """Q_prod encode.  Returns (codes, signs, norms, rnorms)."""
    torch = _torch()
    x2, ld = _rows(x, p.d)
    n = x2.shape[0]
    sl, sc, ns = _segments(n, seg_len, seg_cap, False)
    if out is None:
        dev = x2.device
        out = (torch.zeros((ns * sc, p.code_words), dtype=torch.int32, device=dev),
               torch.zeros((ns * sc, p.sign_words), dtype=torch.int32, device=dev),
               torch.zeros(ns * sc, dtype=torch.float32, device=dev),
               torch.zeros(ns * sc, dtype=getattr(torch, p.rnorm_dtype), device=dev))
    codes, signs, norms, rnorms = out
    need = C.c_size_t()
    L.check("tq_encode_workspace_size", L.lib().tq_encode_workspace_size(p.handle, n, C.byref(need)))
    ws = _ws(need.value, x2.device)
    L.check("tq_encode_prod", L.lib().tq_encode_prod(
        p.handle, _ptr(x2), _dtype_code(x2), n, ld, sl, sc, _ptr(codes), _ptr(signs), _ptr(norms),
        _ptr(rnorms), _ptr(ws), need.value, _stream(stream)))
    return codes, signs, norms, rnorms


def tq_decode(p: TQParams, codes, norms, n_vec: int, signs=None, rnorms=None,
              layout: int = LAYOUT_ROW, seg_len: int = 0, seg_cap: int = 0, stream=None):
    """Reconstruct n_vec vectors [n_vec, d] (fp32)."""
    torch = _torch()
    sl, sc, _ = _segments(n_vec, seg_len, seg_cap, layout == LAYOUT_BLOCK32)
    out = torch.empty((n_vec, p.d), dtype=torch.float32, device=codes.device)
    L.check("tq_decode", L.lib().tq_decode(
        p.handle, layout, _ptr(codes), _ptr(signs), _ptr(norms), _ptr(rnorms), n_vec, sl, sc,
        _ptr(out), p.d, _stream(stream)))
    return out


def tq_scores(p: TQParams, q, codes, signs, norms, rnorms, n_vec: Optional[int] = None,
              topk: int = 0, want_scores: bool = True, stream=None):
    """Inner-product estimates [nq, n_vec]; with topk > 0 also (top_s, top_i)."""
    torch = _torch()
    q2, ldq = _rows(q.float() if q.dtype != torch.float32 else q, p.d)
    nq = q2.shape[0]
    n = norms.shape[0] if n_vec is None else n_vec
    dev = q2.device
    scores = torch.empty((nq, n), dtype=torch.float32, device=dev) if want_scores else None
    top_s = torch.empty((nq, topk), dtype=torch.float32, device=dev) if topk else None
    top_i = torch.empty((nq, topk), dtype=torch.int64, device=dev) if topk else None
    need = C.c_size_t()
    L.check("tq_scores_workspace_size", L.lib().tq_scores_workspace_size(p.handle, nq, n, topk, C.byref(need)))
    ws = _ws(max(need.value, 256), dev)
    L.check("tq_scores", L.lib().tq_scores(
        p.handle, _ptr(q2), nq, ldq, _ptr(codes), _ptr(signs), _ptr(norms), _ptr(rnorms), n,
        _ptr(scores), topk, _ptr(top_s), _ptr(top_i), _ptr(ws), need.value, _stream(stream)))
    if topk:
        return scores, top_s, top_i
    return scores


def tq_decode_attention_workspace_size(kp: TQParams, vp: TQParams, L_: int, B: int, Hq: int,
                                       Hkv: int, seq: int) -> int:
    need = C.c_size_t()
    L.check("tq_decode_attention_workspace_size", L.lib().tq_decode_attention_workspace_size(
        kp.handle, vp.handle, L_, B, Hq, Hkv, seq, C.byref(need)))
    return need.value


def tq_decode_attention(kp: TQParams, vp: TQParams, q, kcache, vcache, seq: int, cap: int,
                        scale: float, out=None, ws=None, stream=None):
    """One decode step.  q [L, B, Hq, d] fp32; kcache = (codes, signs, norms,
    rnorms) in ROW layout with cap slots per (layer, batch, kv-head); vcache =
    (codes, norms) in BLOCK32 layout.  Returns out [L, B, Hq, d] fp32."""
    torch = _torch()
    Ln, B, Hq, d = q.shape
    kcodes, ksigns, knorms, krnorms = kcache
    vcodes, vnorms = vcache
    Hkv = knorms.numel() // (Ln * B * cap)
    if out is None:
        out = torch.empty((Ln, B, Hq, d), dtype=torch.float32, device=q.device)
    need = tq_decode_attention_workspace_size(kp, vp, Ln, B, Hq, Hkv, seq)
    if ws is None:
        ws = _ws(need, q.device)
    qc = q.contiguous()
    L.check("tq_decode_attention", L.lib().tq_decode_attention(
        kp.handle, vp.handle, _ptr(qc), Ln, B, Hq, Hkv, seq, cap, float(scale),
        _ptr(kcodes), _ptr(ksigns), _ptr(knorms), _ptr(krnorms), _ptr(vcodes), _ptr(vnorms),
        _ptr(out), _ptr(ws), ws.numel() if ws is not None else 0, _stream(stream)))
    return out


def tq_decode_attention_noalloc(kp: TQParams, vp: TQParams, q, kcache, vcache, seq: int, cap: int,
                                scale: float, out=None, stream=None):
    """tq_decode_attention without a workspace: the library's fixed device
    scratch array is used instead (see include/tq.h for its size limit and for
    why overlapping calls must be serialized)."""
    torch = _torch()
    Ln, B, Hq, d = q.shape
    kcodes, ksigns, knorms, krnorms = kcache
    vcodes, vnorms = vcache
    Hkv = knorms.numel() // (Ln * B * cap)
    if out is None:
        out = torch.empty((Ln, B, Hq, d), dtype=torch.float32, device=q.device)
    qc = q.contiguous()
    # the scratch array used is the current device's: make q's device current
    with torch.cuda.device(q.device):
        L.check("tq_decode_attention_noalloc", L.lib().tq_decode_attention_noalloc(
            kp.handle, vp.handle, _ptr(qc), Ln, B, Hq, Hkv, seq, cap, float(scale),
            _ptr(kcodes), _ptr(ksigns), _ptr(knorms), _ptr(krnorms), _ptr(vcodes), _ptr(vnorms),
            _ptr(out), _stream(stream)))
    return out


def tq_decode_step_workspace_size(kp: TQParams, vp: TQParams, L_: int, B: int, Hq: int, Hkv: int,
                                  pos: int) -> int:
    need = C.c_size_t()
    L.check("tq_decode_step_workspace_size", L.lib().tq_decode_step_workspace_size(
        kp.handle, vp.handle, L_, B, Hq, Hkv, pos, C.byref(need)))
    return need.value


def tq_decode_step(kp: TQParams, vp: TQParams, q, k_new, v_new, kcache, vcache, pos: int, cap: int,
                   scale: float, out=None, ws=None, stream=None):
    """One serving decode step: append k_new / v_new [L, B, Hkv, d] (fp32, fp16
    or bf16) at slot pos of the caches (updated in place), then attend q
    [L, B, Hq, d] over the pos + 1 cached tokens.  Returns out [L, B, Hq, d]."""
    torch = _torch()
    Ln, B, Hq, d = q.shape
    kcodes, ksigns, knorms, krnorms = kcache
    vcodes, vnorms = vcache
    Hkv = k_new.shape[2]
    if k_new.dtype != v_new.dtype or k_new.shape != v_new.shape or k_new.shape != (Ln, B, Hkv, d):
        raise ValueError("k_new and v_new must be [L, B, Hkv, d] of one dtype")
    kn, vn = k_new.contiguous(), v_new.contiguous()
    if out is None:
        out = torch.empty((Ln, B, Hq, d), dtype=torch.float32, device=q.device)
    need = tq_decode_step_workspace_size(kp, vp, Ln, B, Hq, Hkv, pos)
    if ws is None or ws.numel() < need:
        ws = _ws(need, q.device)
    qc = q.contiguous()
    L.check("tq_decode_step", L.lib().tq_decode_step(
        kp.handle, vp.handle, _ptr(qc), _ptr(kn), _ptr(vn), _dtype_code(kn), Ln, B, Hq, Hkv, pos, cap,
        float(scale), _ptr(kcodes), _ptr(ksigns), _ptr(knorms), _ptr(krnorms), _ptr(vcodes),
        _ptr(vnorms), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)))
    return out


def tq_check_wait_expiry(budget_cycles: int, stream=None):
    """Run the bounded-wait expiry path once (the status shows at tq_sync_check)."""
    L.check("tq_check_wait_expiry", L.lib().tq_check_wait_expiry(int(budget_cycles), _stream(stream)))


def tq_sync_check(stream=None):
    """Synchronize and raise if a kernel flagged a device-side error."""
    L.check("tq_sync_check", L.lib().tq_sync_check(_stream(stream)))

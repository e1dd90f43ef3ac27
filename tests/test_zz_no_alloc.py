"""tq_decode_attention_noalloc: decode attention for callers that cannot
allocate device memory (for example a plugin inside an inference engine that
owns the whole device memory pool).  It must give the same result as
tq_decode_attention with a caller workspace, on two calls in a row -- the
second call finds the first call's leftovers in the shared scratch array.

Called through the C ABI with ctypes.  Collected last on purpose (file name),
and self-contained, so it passes alone in a fresh process or after the rest."""
import ctypes as C
import math

import numpy as np
import pytest
import torch

import synth
import vector_compression_b200 as tq
from vector_compression_b200 import _lib as L
from tests.parity import REL_TOL

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _case(seed, seq, cap, G, d=128, Ln=2, B=1, Hkv=2):
    kd = synth.method_draws(d, synth.next_pow2(d), seed, stream=1)
    vd = synth.method_draws(d, synth.next_pow2(d), seed, stream=2)
    kp = tq.TQParams(d, 3, tq.MODE_PROD, tq.ROT_HADAMARD, m=synth.next_pow2(d), signs=kd["signs"], S=kd["S"])
    vp = tq.TQParams(d, 3, tq.MODE_MSE, tq.ROT_HADAMARD, signs=vd["signs"])
    n = Ln * B * Hkv * seq
    K = synth.gaussian_vectors(n, d, seed=seed + 1, dtype="float16", device=DEV, n_outliers=4, outlier_scale=20.0)
    V = synth.gaussian_vectors(n, d, seed=seed + 2, dtype="float16", device=DEV)
    q = synth.gaussian_vectors(Ln * B * Hkv * G, d, seed=seed + 3, device=DEV).view(Ln, B, Hkv * G, d)
    kc = tq.tq_encode_prod(kp, K, seg_len=seq, seg_cap=cap)
    vc = tq.tq_encode_mse(vp, V, layout=tq.LAYOUT_BLOCK32, seg_len=seq, seg_cap=cap)
    return kp, vp, q, kc, vc, (Ln, B, Hkv * G, Hkv)


def _call_noalloc(kp, vp, q, kc, vc, dims, seq, cap, scale):
    Ln, B, Hq, Hkv = dims
    out = torch.full((Ln, B, Hq, q.shape[-1]), float("nan"), device=DEV)
    p = lambda t: C.c_void_p(t.data_ptr())
    st = L.lib().tq_decode_attention_noalloc(
        kp.handle, vp.handle, p(q), Ln, B, Hq, Hkv, seq, cap, C.c_float(scale),
        p(kc[0]), p(kc[1]), p(kc[2]), p(kc[3]), p(vc[0]), p(vc[1]), p(out),
        C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, L.STATUS.get(st, st)
    return out


def test_noalloc_matches_workspace_entry_point_twice():
    results = []
    for seed, seq, cap, G in ((11, 700, 704, 8), (12, 257, 288, 4)):
        kp, vp, q, kc, vc, dims = _case(seed, seq, cap, G)
        scale = 1 / math.sqrt(128)
        got = _call_noalloc(kp, vp, q, kc, vc, dims, seq, cap, scale)
        want = tq.tq_decode_attention(kp, vp, q, kc, vc, seq, cap, scale)
        torch.cuda.synchronize()
        g, w = got.cpu().numpy(), want.cpu().numpy()
        assert np.all(np.isfinite(g))
        err = np.linalg.norm(g - w, axis=-1) / np.linalg.norm(w, axis=-1)
        assert err.max() <= REL_TOL, err.max()
        results.append(err.max())
    tq.tq_sync_check()


def test_noalloc_python_wrapper_matches_workspace_entry_point():
    # the binding's wrapper (which makes q's device current around the call)
    kp, vp, q, kc, vc, dims = _case(14, 500, 512, 4)
    scale = 1 / math.sqrt(128)
    got = tq.tq_decode_attention_noalloc(kp, vp, q, kc, vc, 500, 512, scale)
    want = tq.tq_decode_attention(kp, vp, q, kc, vc, 500, 512, scale)
    torch.cuda.synchronize()
    g, w = got.cpu().numpy(), want.cpu().numpy()
    assert np.all(np.isfinite(g))
    err = np.linalg.norm(g - w, axis=-1) / np.linalg.norm(w, axis=-1)
    assert err.max() <= REL_TOL, err.max()
    tq.tq_sync_check()


def test_noalloc_rejects_oversized_requests():
    kp, vp, q, kc, vc, dims = _case(13, 64, 64, 4)
    need = tq.tq_decode_attention_workspace_size(kp, vp, 4096, 64, 32, 8, 32768)
    assert need > (32 << 20)
    st = L.lib().tq_decode_attention_noalloc(
        kp.handle, vp.handle, C.c_void_p(q.data_ptr()), 4096, 64, 32, 8, 32768, 32768, C.c_float(1.0),
        *[C.c_void_p(q.data_ptr())] * 7, C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert L.STATUS[st] == "TQ_ERR_WORKSPACE"

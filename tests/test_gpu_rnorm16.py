"""Q_prod with fp16 residual-norm storage (TQ_STORE_RNORM_F16) on the GPU.

* Every encoder path writes the same codes, signs and norms as the fp32
  variant, and residual norms equal to its own fp32 value rounded to fp16
  (bit-exact); against the oracle's fp16 residual norms within 1e-3
  (one fp16 step is at most 2^-10 relative).  Paths: tensor-core (d = 128
  fp16 rows, m = 128 and 64), thread-per-vector (fp32 rows), warp-per-vector
  (d = 64) and the dense rotation.
* Scores, reconstruction (Q_prod^-1) and decode attention on oracle codes
  with fp16 residual norms (m = 128 and 64; int8 attention kernel), and the
  serving decode step, against the oracle."""
import math

import numpy as np
import pytest
import torch

import synth
import vector_compression_b200 as tq
from oracle import tq_oracle as o
from tests.parity import REL_TOL, assert_close_rel, check_codes, u32

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def make(d, bits, m, seed, f16=True, dense=False, stream=0):
    dr = synth.method_draws(d, m, seed, dense=dense, stream=stream)
    ora = o.Quantizer(d, bits, prod=True, draws=dr, rnorm_f16=f16)
    mode = tq.MODE_PROD | (tq.STORE_RNORM_F16 if f16 else 0)
    lib = tq.TQParams(d, bits, mode, tq.ROT_DENSE if dense else tq.ROT_HADAMARD, m=m,
                      signs=None if dense else dr["signs"], S=dr["S"], G=dr["G"] if dense else None)
    return ora, lib


@pytest.mark.parametrize("d,m,dtype,n,dense", [
    (128, 128, "float16", 1000, False),   # tensor-core encoder
    (128, 64, "bfloat16", 512, False),
    (128, 128, "float32", 700, False),    # thread-per-vector
    (64, 64, "float32", 300, False),      # warp-per-vector
    (96, 96, "float32", 200, True),       # dense rotation
])
def test_encode_prod_rnorm16(d, m, dtype, n, dense):
    ora, lib16 = make(d, 3, m, seed=100 + d + m, dense=dense)
    _, lib32 = make(d, 3, m, seed=100 + d + m, f16=False, dense=dense)
    x = synth.gaussian_vectors(n, d, seed=m, dtype=dtype, device=DEV, n_outliers=4, outlier_scale=20.0)
    x[3] = 0
    c16, s16, n16, r16 = tq.tq_encode_prod(lib16, x)
    c32, s32, n32, r32 = tq.tq_encode_prod(lib32, x)
    torch.cuda.synchronize()
    tq.tq_sync_check()
    assert r16.dtype == torch.float16 and r32.dtype == torch.float32
    assert torch.equal(c16, c32) and torch.equal(s16, s32) and torch.equal(n16, n32)
    assert torch.equal(r16, r32.half())  # the kernels round their fp32 value to nearest
    e = ora.encode(x.detach().float().cpu().numpy().astype(np.float64))
    gi = o.unpack_row(u32(c16), ora.k, ora.d_pad)
    _, bad = check_codes(gi, e["idx"], e["y"], ora.boundaries, ora.d_pad)
    assert_close_rel(r16.float().cpu().numpy(), e["rnorms"].astype(np.float64), 1e-30,
                     what="fp16 residual norms", mask=~bad)


def upload(e):
    t = lambda a: torch.from_numpy(a.view(np.int32) if a.dtype == np.uint32 else a).to(DEV)
    return t(e["codes"]), t(e["signs"]), t(e["norms"]), t(e["rnorms"])


@pytest.mark.parametrize("m", [128, 64])
def test_scores_and_decode_rnorm16_on_oracle_codes(m):
    ora, lib = make(128, 3, m, seed=110)
    rng = np.random.default_rng(3)
    x = rng.standard_normal((300, 128)) * 2
    qv = rng.standard_normal((8, 128))
    e = ora.encode(x)
    codes, signs, norms, rnorms = upload(e)
    assert rnorms.dtype == torch.float16
    got = tq.tq_scores(lib, torch.from_numpy(qv).float().to(DEV), codes, signs, norms, rnorms).cpu().numpy()
    want = ora.scores(qv, e["idx"], e["norms"], e["signs"], e["rnorms"])
    floor = e["norms"][None, :] * np.linalg.norm(qv, axis=1)[:, None] / math.sqrt(128)
    assert_close_rel(got, want, floor, what="scores")
    out = tq.tq_decode(lib, codes, norms, 300, signs=signs, rnorms=rnorms).cpu().numpy()
    want = ora.decode(e["idx"], e["norms"], e["signs"], e["rnorms"])
    fl = np.linalg.norm(want, axis=1, keepdims=True) / math.sqrt(128)
    assert_close_rel(out, want, fl, tol=1e-5, what="decode")


@pytest.mark.parametrize("G,seq,cap,m", [(4, 1000, 1024, 128), (8, 333, 384, 64), (2, 64, 64, 128)])
def test_attention_rnorm16_on_oracle_cache(G, seq, cap, m):
    d, Ln, B, Hkv = 128, 2, 1, 2
    groups = Ln * B * Hkv
    kq, kl = make(d, 3, m, seed=120, stream=1)
    vdr = synth.method_draws(d, d, 120, stream=2)
    vq = o.Quantizer(d, 3, prod=False, draws=vdr)
    vl = tq.TQParams(d, 3, tq.MODE_MSE, tq.ROT_HADAMARD, signs=vdr["signs"])
    rng = np.random.default_rng(12)
    K = rng.standard_normal((groups, seq, d)) * rng.lognormal(0, 1, size=(1, 1, d))
    V = rng.standard_normal((groups, seq, d))
    q = rng.standard_normal((Ln, B, G * Hkv, d))
    kc = np.zeros((groups * cap, kq.k * 4), np.uint32)
    ks = np.zeros((groups * cap, m // 32), np.uint32)
    kn = np.zeros(groups * cap, np.float32)
    kr = np.zeros(groups * cap, np.float16)
    vc = np.zeros((groups * cap // 32, vq.k * 128), np.uint32)
    vn = np.zeros(groups * cap, np.float32)
    encs = []
    for g in range(groups):
        ke, ve = kq.encode(K[g]), vq.encode(V[g], layout="block32")
        sl = slice(g * cap, g * cap + seq)
        kc[sl], ks[sl], kn[sl], kr[sl] = ke["codes"], ke["signs"], ke["norms"], ke["rnorms"]
        vc[g * cap // 32: g * cap // 32 + ve["codes"].shape[0]] = ve["codes"]
        vn[sl] = ve["norms"]
        encs.append((ke, ve))
    t = lambda a: torch.from_numpy(a.view(np.int32) if a.dtype == np.uint32 else a).to(DEV)
    scale = 1 / math.sqrt(d)
    out = tq.tq_decode_attention(kl, vl, torch.from_numpy(q).float().to(DEV), (t(kc), t(ks), t(kn), t(kr)),
                                 (t(vc), t(vn)), seq, cap, scale).cpu().numpy()
    for g in range(groups):
        l, h = g // Hkv, g % Hkv
        ke, ve = encs[g]
        want = o.decode_attention(q[l, 0, h * G:(h + 1) * G], kq, vq, ke, ve, scale, G)
        got = out[l, 0, h * G:(h + 1) * G]
        err = np.linalg.norm(got - want, axis=1) / np.linalg.norm(want, axis=1)
        assert err.max() <= REL_TOL, err.max()


def test_decode_step_rnorm16():
    # append three tokens into fp16-residual-norm key caches and attend
    d, G, cap, prefill, steps = 128, 4, 96, 61, 3
    Ln, B, Hkv = 2, 1, 2
    groups = Ln * B * Hkv
    kq, kl = make(d, 3, 64, seed=130, stream=1)
    vdr = synth.method_draws(d, d, 130, stream=2)
    vq = o.Quantizer(d, 3, prod=False, draws=vdr)
    vl = tq.TQParams(d, 3, tq.MODE_MSE, tq.ROT_HADAMARD, signs=vdr["signs"])
    T = prefill + steps
    rng = np.random.default_rng(13)
    Kt = torch.from_numpy(rng.standard_normal((groups, T, d))).to(DEV).half()
    Vt = torch.from_numpy(rng.standard_normal((groups, T, d))).to(DEV).half()
    Kn, Vn = Kt.float().cpu().numpy().astype(np.float64), Vt.float().cpu().numpy().astype(np.float64)
    z = lambda *s, dt=torch.int32: torch.zeros(s, dtype=dt, device=DEV)
    kc = (z(groups * cap, kl.code_words), z(groups * cap, kl.sign_words), z(groups * cap, dt=torch.float32),
          z(groups * cap, dt=torch.float16))
    vc = (z(groups * cap // 32, vl.code_words * 32), z(groups * cap, dt=torch.float32))
    tq.tq_encode_prod(kl, Kt[:, :prefill].contiguous(), seg_len=prefill, seg_cap=cap, out=kc)
    tq.tq_encode_mse(vl, Vt[:, :prefill].contiguous(), layout=tq.LAYOUT_BLOCK32, seg_len=prefill, seg_cap=cap,
                     codes=vc[0], norms=vc[1])
    scale = 1 / math.sqrt(d)
    for s in range(steps):
        pos = prefill + s
        q = torch.from_numpy(rng.standard_normal((Ln, B, G * Hkv, d))).float().to(DEV)
        kn_ = Kt[:, pos].reshape(Ln, B, Hkv, d).contiguous()
        vn_ = Vt[:, pos].reshape(Ln, B, Hkv, d).contiguous()
        out = tq.tq_decode_step(kl, vl, q, kn_, vn_, kc, vc, pos, cap, scale).cpu().numpy()
        qn = q.cpu().numpy().astype(np.float64)
        for g in range(groups):
            l, h = g // Hkv, g % Hkv
            ke, ve = kq.encode(Kn[g, :pos + 1]), vq.encode(Vn[g, :pos + 1], layout="block32")
            want = o.decode_attention(qn[l, 0, h * G:(h + 1) * G], kq, vq, ke, ve, scale, G)
            err = np.linalg.norm(out[l, 0, h * G:(h + 1) * G] - want, axis=1) / np.linalg.norm(want, axis=1)
            assert err.max() <= REL_TOL, (pos, g, err.max())
    torch.cuda.synchronize()
    tq.tq_sync_check()
    # residual norms of every appended slot: the fp16 rounding of the oracle's within one step
    for g in range(groups):
        ke = kq.encode(Kn[g])
        got = kc[3][g * cap: g * cap + T].float().cpu().numpy()
        assert np.all(np.abs(got / ke["rnorms"].astype(np.float64) - 1.0) <= 2.0 ** -10)
        assert np.all(kc[3][g * cap + T:(g + 1) * cap].float().cpu().numpy() == 0)

"""Q_MSE with EDEN's unbiased per-vector scale (DRIVE at one bit) on the GPU
against the oracle: the codes equal Q_MSE's, and the stored scale
S = n / <y, C[idx]> is within 1e-3 of the oracle's.  Rows holding a code
inside the boundary window are left out of the scale comparison (moving one
coordinate across a boundary changes <y, C[idx]> by |y_j| (C_(i+1) - C_i),
about 1 %); for every row, the GPU's own codes and scale satisfy the exact
identity <x~, x> = ||x||^2 of the unbiased scale.  Every encoder path is
covered: tensor-core (d = 128, fp16 / bf16), thread-per-vector (fp32, and
d = 192 padded to 256), warp-per-vector (d = 64) and the dense rotation.
Then the decoder on oracle codes, and decode attention over values stored
with the unbiased scale."""
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


def make_unbiased(d, bits, seed, dense=False, stream=0):
    dr = synth.method_draws(d, d if dense else synth.next_pow2(d), seed, dense=dense, stream=stream)
    ora = o.Quantizer(d, bits, prod=False, draws=dr, unbiased=True)
    lib = tq.TQParams(d, bits, tq.MODE_MSE_UNBIASED, tq.ROT_DENSE if dense else tq.ROT_HADAMARD,
                      signs=None if dense else dr["signs"], G=dr["G"] if dense else None)
    return ora, lib


def x_np(x):
    return x.detach().float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("d,dtype,layout,n,bits,dense", [
    (128, "float16", tq.LAYOUT_ROW, 1000, 3, False),       # tensor-core encoder
    (128, "bfloat16", tq.LAYOUT_BLOCK32, 1024, 2, False),
    (128, "float16", tq.LAYOUT_BLOCK32, 4096, 4, False),
    (128, "float16", tq.LAYOUT_ROW, 256, 1, False),
    (128, "float32", tq.LAYOUT_ROW, 777, 3, False),        # thread-per-vector
    (192, "float16", tq.LAYOUT_BLOCK32, 555, 4, False),    # tensor-core encoder, d_pad 256
    (256, "bfloat16", tq.LAYOUT_ROW, 300, 2, False),       # tensor-core encoder, d_pad 256, ROW
    (192, "float32", tq.LAYOUT_BLOCK32, 100, 3, False),    # thread-per-vector, d_pad 256
    (128, "float32", tq.LAYOUT_BLOCK32, 300, 1, False),
    (64, "float32", tq.LAYOUT_ROW, 300, 3, False),         # warp-per-vector
    (96, "float32", tq.LAYOUT_BLOCK32, 224, 2, True),      # dense rotation (BLOCK32: 32-row segments)
    (96, "float32", tq.LAYOUT_ROW, 100, 4, True),
])
def test_encode_unbiased_parity(d, dtype, layout, n, bits, dense):
    ora, lib = make_unbiased(d, bits, seed=70 + d + bits, dense=dense)
    x = synth.gaussian_vectors(n, d, seed=bits + 5, dtype=dtype, device=DEV, n_outliers=4,
                               outlier_scale=20.0)
    x[min(5, n - 1)] = 0  # a zero vector stores scale 0
    codes, norms = tq.tq_encode_mse(lib, x, layout=layout)
    torch.cuda.synchronize()
    tq.tq_sync_check()
    xn = x_np(x)
    lay = "row" if layout == tq.LAYOUT_ROW else "block32"
    e = ora.encode(xn, layout=lay)
    if layout == tq.LAYOUT_ROW:
        gi = o.unpack_row(u32(codes), ora.k, ora.d_pad)
    else:
        gi = o.unpack_block32(u32(codes), ora.k, ora.d_pad, n)
    _, bad = check_codes(gi, e["idx"], e["y"], ora.boundaries, ora.d_pad)
    gs = norms.cpu().numpy()[:n]
    assert gs[min(5, n - 1)] == 0.0
    assert_close_rel(gs, e["norms"], 1e-30, what="unbiased scale", mask=~bad)
    # the GPU's codes and scale, decoded by the oracle: <x~, x> = ||x||^2 per row
    xt = ora.decode(gi, gs)
    got, want = np.sum(xt * xn, axis=1), np.sum(xn * xn, axis=1)
    nz = want > 0
    assert np.max(np.abs(got[nz] / want[nz] - 1.0)) < 1e-4


@pytest.mark.parametrize("d,layout,dense", [(128, tq.LAYOUT_ROW, False), (192, tq.LAYOUT_BLOCK32, False),
                                            (96, tq.LAYOUT_ROW, True)])
def test_decode_unbiased_on_oracle_codes(d, layout, dense):
    ora, lib = make_unbiased(d, 2, seed=80, dense=dense)
    x = np.random.default_rng(2).standard_normal((70, d)) * 3
    lay = "row" if layout == tq.LAYOUT_ROW else "block32"
    e = ora.encode(x, layout=lay)
    codes = torch.from_numpy(e["codes"].view(np.int32)).to(DEV)
    norms = torch.from_numpy(e["norms"]).to(DEV)
    out = tq.tq_decode(lib, codes, norms, 70, layout=layout).cpu().numpy()
    want = ora.decode(e["idx"], e["norms"])
    floor = np.linalg.norm(want, axis=1, keepdims=True) / math.sqrt(d)
    assert_close_rel(out, want, floor, tol=1e-5, what="decode")


@pytest.mark.parametrize("G,seq,cap,bits", [(4, 1000, 1024, 3), (8, 97, 128, 2)])
def test_attention_with_unbiased_values(G, seq, cap, bits):
    # keys Q_prod, values Q_MSE with the unbiased scale, both from the oracle
    d, Ln, B, Hkv = 128, 2, 1, 2
    groups = Ln * B * Hkv
    kdr = synth.method_draws(d, d, 90, stream=1)
    kq = o.Quantizer(d, bits, prod=True, draws=kdr)
    kl = tq.TQParams(d, bits, tq.MODE_PROD, tq.ROT_HADAMARD, m=d, signs=kdr["signs"], S=kdr["S"])
    vq, vl = make_unbiased(d, bits, seed=90, stream=2)
    rng = np.random.default_rng(9)
    K = rng.standard_normal((groups, seq, d)) * rng.lognormal(0, 1, size=(1, 1, d))
    V = rng.standard_normal((groups, seq, d))
    q = rng.standard_normal((Ln, B, G * Hkv, d))
    kc = np.zeros((groups * cap, kq.k * 4), np.uint32)
    ks = np.zeros((groups * cap, kq.m // 32), np.uint32)
    kn = np.zeros(groups * cap, np.float32)
    kr = np.zeros(groups * cap, np.float32)
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

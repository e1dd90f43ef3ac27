"""GPU (libtq through its C ABI) versus the CPU oracle, element by element, on
seeded synthetic inputs: encode (Q_MSE row / block layouts, Q_prod), decode,
scores and top-k, and fused decode attention; Hadamard (d = 128, 192 -> 256)
and dense rotations; ragged sizes, segments with spare capacity, zero vectors
and empty inputs."""
import math

import numpy as np
import pytest
import torch

import synth
import vector_compression_b200 as tq
from oracle import tq_oracle as o
from tests.parity import (REL_TOL, assert_close_rel, check_codes, check_signs, u32)

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def make_pair(d, bits, prod, seed, m=None, dense=False, stream=0):
    m = m if m is not None else (d if dense else synth.next_pow2(d))
    dr = synth.method_draws(d, m, seed, dense=dense, stream=stream)
    ora = o.Quantizer(d, bits, prod=prod, draws=dr)
    lib = tq.TQParams(d, bits, tq.MODE_PROD if prod else tq.MODE_MSE,
                      tq.ROT_DENSE if dense else tq.ROT_HADAMARD, m=m if prod else 0,
                      signs=dr["signs"] if not dense else None, S=dr["S"] if prod else None,
                      G=dr["G"] if dense else None)
    return ora, lib


def x_np(x):
    return x.detach().float().cpu().numpy().astype(np.float64)


# ------------------------------------------------------------------ encode


@pytest.mark.parametrize("d,dtype,layout,n", [
    (128, "float32", tq.LAYOUT_ROW, 4096),
    (128, "bfloat16", tq.LAYOUT_BLOCK32, 1000),
    (128, "float16", tq.LAYOUT_ROW, 77),
    (192, "float16", tq.LAYOUT_BLOCK32, 555),  # d_pad 256 on the tensor cores (H256 = [[H, H], [H, -H]])
    (256, "bfloat16", tq.LAYOUT_ROW, 300),
    (200, "float16", tq.LAYOUT_ROW, 129),      # d_pad 256 with 56 zero-filled columns
    (64, "float32", tq.LAYOUT_ROW, 300),
    (100, "float32", tq.LAYOUT_BLOCK32, 333),  # d_pad 128, 400-byte rows (thread-per-vector)
    (104, "float16", tq.LAYOUT_ROW, 129),      # d_pad 128 with 24 zero-filled columns (tensor core)
    (36, "float32", tq.LAYOUT_ROW, 70),        # d_pad 64: warp-per-vector
])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_encode_mse_parity(d, dtype, layout, n, bits):
    ora, lib = make_pair(d, bits, False, seed=10 + d + bits)
    x = synth.gaussian_vectors(n, d, seed=bits, dtype=dtype, device=DEV, n_outliers=4, outlier_scale=20.0)
    x[min(5, n - 1)] = 0  # a zero vector
    codes, norms = tq.tq_encode_mse(lib, x, layout=layout)
    torch.cuda.synchronize()
    e = ora.encode(x_np(x), layout="row" if layout == tq.LAYOUT_ROW else "block32")
    if layout == tq.LAYOUT_ROW:
        gi = o.unpack_row(u32(codes), ora.k, ora.d_pad)
    else:
        gi = o.unpack_block32(u32(codes), ora.k, ora.d_pad, n)
        # missing vectors of the ragged last block are zero bits
        tail = u32(codes)[-1].reshape(ora.k, ora.d_pad)
        if n % 32:
            assert np.all((tail >> np.uint32(n % 32)) == 0)
    check_codes(gi, e["idx"], e["y"], ora.boundaries, ora.d_pad)
    gn = norms.cpu().numpy()[:n]  # BLOCK32 keeps seg_cap (a multiple of 32) slots
    assert gn[min(5, n - 1)] == 0.0
    assert_close_rel(gn, e["norms"], 1e-30, what="norms")


@pytest.mark.parametrize("d,m,bits,dtype,n", [
    (128, 128, 3, "float32", 4096),
    (128, 64, 2, "bfloat16", 999),
    (192, 256, 4, "float16", 400),
    (128, 256, 5, "float16", 130),
])
def test_encode_prod_parity(d, m, bits, dtype, n):
    ora, lib = make_pair(d, bits, True, seed=20 + bits, m=m)
    x = synth.gaussian_vectors(n, d, seed=7, dtype=dtype, device=DEV, n_outliers=4, outlier_scale=20.0)
    x[3] = 0
    codes, signs, norms, rnorms = tq.tq_encode_prod(lib, x)
    torch.cuda.synchronize()
    e = ora.encode(x_np(x))
    gi = o.unpack_row(u32(codes), ora.k, ora.d_pad)
    _, bad = check_codes(gi, e["idx"], e["y"], ora.boundaries, ora.d_pad)
    ns = check_signs(u32(signs), e["signs"], e["z"], e["rho64"], m, skip_rows=bad)
    assert ns <= 1e-4 * n * m
    assert_close_rel(norms.cpu().numpy(), e["norms"], 1e-30, what="norms")
    assert_close_rel(rnorms.cpu().numpy(), e["rnorms"], 1e-30, what="rnorms", mask=~bad)


def test_encode_segments_with_capacity():
    # 3 segments of 45 vectors into slots of 64: rows >= 45 untouched
    ora, lib = make_pair(128, 3, False, seed=3)
    x = synth.gaussian_vectors(135, 128, seed=3, dtype="float16", device=DEV)
    codes, norms = tq.tq_encode_mse(lib, x, layout=tq.LAYOUT_BLOCK32, seg_len=45, seg_cap=64)
    torch.cuda.synchronize()
    assert codes.shape == (3 * 2, 3 * 128)
    w = u32(codes)
    for s in range(3):
        e = ora.encode(x_np(x[45 * s:45 * (s + 1)]), layout="block32")
        gi = o.unpack_block32(w[2 * s:2 * s + 2], 3, 128, 45)
        check_codes(gi, e["idx"], e["y"], ora.boundaries, 128)
        gn = norms[64 * s:64 * s + 45].cpu().numpy()
        assert_close_rel(gn, e["norms"], 1e-30)
        assert np.all(norms[64 * s + 45:64 * (s + 1)].cpu().numpy() == 0)


def test_empty_inputs():
    _, lib = make_pair(128, 3, True, seed=1)
    x = torch.zeros((0, 128), device=DEV)
    c, s, n, r = tq.tq_encode_prod(lib, x)
    assert c.numel() == 0
    _, mse = make_pair(128, 3, False, seed=1)
    c, n = tq.tq_encode_mse(mse, x, layout=tq.LAYOUT_BLOCK32)
    assert c.numel() == 0
    tq.tq_sync_check()


# ------------------------------------------------------------------ decode


@pytest.mark.parametrize("d,prod,layout", [(128, True, tq.LAYOUT_ROW), (192, False, tq.LAYOUT_BLOCK32),
                                           (128, False, tq.LAYOUT_ROW)])
def test_decode_parity_on_oracle_codes(d, prod, layout):
    ora, lib = make_pair(d, 3, prod, seed=30)
    x = np.random.default_rng(1).standard_normal((70, d)) * 3
    lay = "row" if layout == tq.LAYOUT_ROW else "block32"
    e = ora.encode(x, layout=lay)
    codes = torch.from_numpy(e["codes"].view(np.int32)).to(DEV)
    norms = torch.from_numpy(e["norms"]).to(DEV)
    kw = {}
    if prod:
        kw = dict(signs=torch.from_numpy(e["signs"].view(np.int32)).to(DEV),
                  rnorms=torch.from_numpy(e["rnorms"]).to(DEV))
    out = tq.tq_decode(lib, codes, norms, 70, layout=layout, **kw).cpu().numpy()
    want = ora.decode(e["idx"], e["norms"], e.get("signs") if prod else None, e.get("rnorms") if prod else None)
    floor = np.linalg.norm(want, axis=1, keepdims=True) / math.sqrt(d)
    assert_close_rel(out, want, floor, tol=1e-5, what="decode")


# ------------------------------------------------------------------ scores


def test_scores_on_oracle_codes_exact():
    cfg = synth.TINY
    ora, lib = make_pair(cfg["d"], cfg["bits"], True, seed=cfg["seed"], m=cfg["m"])
    x = x_np(synth.gaussian_vectors(1000, 128, seed=0, n_outliers=4, outlier_scale=20.0))
    q = x_np(synth.gaussian_vectors(40, 128, seed=99))
    e = ora.encode(x)
    dev = lambda a, dt=None: torch.from_numpy(a.view(np.int32) if a.dtype == np.uint32 else a).to(DEV)
    s = tq.tq_scores(lib, torch.from_numpy(q).float().to(DEV), dev(e["codes"]), dev(e["signs"]),
                     dev(e["norms"]), dev(e["rnorms"])).cpu().numpy()
    want = ora.scores(q, e["idx"], e["norms"], e["signs"], e["rnorms"])
    floor = e["norms"][None, :] * np.linalg.norm(q, axis=1)[:, None] / math.sqrt(128)
    assert_close_rel(s, want, floor, tol=1e-5, what="scores")


def test_tiny_end_to_end_scores_and_topk():
    # N=4096 fp32, d=128, 4 outlier channels x20, 64 queries, Q_prod b=3, m=128, seed 0
    cfg = synth.TINY
    ora, lib = make_pair(cfg["d"], cfg["bits"], True, seed=cfg["seed"], m=cfg["m"])
    x = synth.gaussian_vectors(cfg["n"], cfg["d"], seed=cfg["seed"], device=DEV,
                               n_outliers=cfg["n_outliers"], outlier_scale=cfg["outlier_scale"])
    q = synth.gaussian_vectors(cfg["n_queries"], cfg["d"], seed=cfg["seed"] + 1, device=DEV)
    codes, signs, norms, rnorms = tq.tq_encode_prod(lib, x)
    s, ts, ti = tq.tq_scores(lib, q, codes, signs, norms, rnorms, topk=10)
    torch.cuda.synchronize()
    e = ora.encode(x_np(x))
    gi = o.unpack_row(u32(codes), ora.k, ora.d_pad)
    _, bad = check_codes(gi, e["idx"], e["y"], ora.boundaries, ora.d_pad)
    nsig = check_signs(u32(signs), e["signs"], e["z"], e["rho64"], cfg["m"], skip_rows=bad)
    sig_bad = (o.unpack_signs(u32(signs), cfg["m"]) != o.unpack_signs(e["signs"], cfg["m"])).any(axis=1)
    want = ora.scores(x_np(q), e["idx"], e["norms"], e["signs"], e["rnorms"])
    qn = np.linalg.norm(x_np(q), axis=1)
    floor = e["norms"][None, :] * qn[:, None] / math.sqrt(128)
    ok = ~(bad | sig_bad)
    assert ok.mean() > 0.99
    assert_close_rel(s.cpu().numpy()[:, ok], want[:, ok], floor[:, ok], what="scores")
    # top-k of the GPU scores is the exact top-k of those scores
    sg = s.cpu().numpy()
    vs, vi = o.topk(sg, 10)
    assert np.array_equal(ti.cpu().numpy(), vi)
    assert np.array_equal(ts.cpu().numpy(), vs)


# ------------------------------------------------------------------ attention


def _pack_cache(ora_k, ora_v, K, V, seq, cap):
    """Oracle-encode K, V [groups, seq, d] into cache arrays with cap slots."""
    groups = K.shape[0]
    kq, vq = ora_k, ora_v
    kc = np.zeros((groups * cap, kq.k * kq.d_pad // 32), np.uint32)
    ks = np.zeros((groups * cap, kq.m // 32), np.uint32)
    kn = np.zeros(groups * cap, np.float32)
    kr = np.zeros(groups * cap, np.float32)
    vc = np.zeros((groups * cap // 32, vq.k * vq.d_pad), np.uint32)
    vn = np.zeros(groups * cap, np.float32)
    encs = []
    for g in range(groups):
        ke = kq.encode(K[g])
        ve = vq.encode(V[g], layout="block32")
        sl = slice(g * cap, g * cap + seq)
        kc[sl], ks[sl], kn[sl], kr[sl] = ke["codes"], ke["signs"], ke["norms"], ke["rnorms"]
        vc[g * cap // 32: g * cap // 32 + ve["codes"].shape[0]] = ve["codes"]
        vn[sl] = ve["norms"]
        encs.append((ke, ve))
    t = lambda a: torch.from_numpy(a.view(np.int32) if a.dtype == np.uint32 else a).to(DEV)
    return (t(kc), t(ks), t(kn), t(kr)), (t(vc), t(vn)), encs


@pytest.mark.parametrize("d,G,seq,cap,bits,m", [(128, 8, 300, 320, 3, None), (128, 4, 64, 64, 2, None),
                                                (192, 4, 1000, 1024, 4, None), (128, 1, 33, 64, 3, None),
                                                (128, 4, 1000, 1024, 3, 64), (128, 8, 97, 128, 2, 64),
                                                (128, 2, 413, 416, 4, 64),
                                                (128, 16, 100, 128, 3, None),  # G = 16: SIMT kernel
                                                (128, 4, 1, 32, 2, None),      # a single token
                                                (100, 4, 77, 96, 3, None)])    # d = 100 padded to 128
def test_attention_on_oracle_cache(d, G, seq, cap, bits, m):
    # m = 64: the QJL projection with d / 2 rows (a storage variant with
    # 8 bytes of signs per token instead of 16)
    Ln, B, Hkv = 2, 1, 2
    Hq = G * Hkv
    kq, kl = make_pair(d, bits, True, seed=40, m=m, stream=1)
    vq, vl = make_pair(d, bits, False, seed=40, stream=2)
    rng = np.random.default_rng(5)
    K = rng.standard_normal((Ln * B * Hkv, seq, d)) * rng.lognormal(0, 1, size=(1, 1, d))
    V = rng.standard_normal((Ln * B * Hkv, seq, d))
    q = rng.standard_normal((Ln, B, Hq, d))
    kc, vc, encs = _pack_cache(kq, vq, K, V, seq, cap)
    scale = 1 / math.sqrt(d)
    out = tq.tq_decode_attention(kl, vl, torch.from_numpy(q).float().to(DEV), kc, vc, seq, cap, scale)
    out = out.cpu().numpy()
    for l in range(Ln):
        for b in range(B):
            for h in range(Hkv):
                g = (l * B + b) * Hkv + h
                ke, ve = encs[g]
                want = o.decode_attention(q[l, b, h * G:(h + 1) * G], kq, vq, ke, ve, scale, G)
                got = out[l, b, h * G:(h + 1) * G]
                err = np.linalg.norm(got - want, axis=1) / np.linalg.norm(want, axis=1)
                print(f"attention rel err (G={G}, bits={bits}, m={kq.m}): {err.max():.2e}")
                assert err.max() <= REL_TOL, err.max()


def test_attention_end_to_end_qwen_shape_subset():
    # Qwen2.5-3B-shaped cache (bf16, d=128, 2 KV heads, 16 query heads, seq
    # 8192, keys lognormal x outliers), layers {0, 35}: GPU encode + GPU
    # attention vs oracle encode + oracle attention.
    cfg = synth.KV_CONFIGS["qwen2.5-3b_8k_b3"]
    layers = range(0, 36, 35)
    K, V = synth.kv_cache(cfg, device=DEV, layers=layers)
    q = synth.decode_queries(cfg, device=DEV, layers=layers)
    kq, kl = make_pair(cfg.head_dim, cfg.key_bits, True, seed=cfg.seed, stream=1)
    vq, vl = make_pair(cfg.head_dim, cfg.value_bits, False, seed=cfg.seed, stream=2)
    seq = cap = cfg.seq
    kc = tq.tq_encode_prod(kl, K, seg_len=seq, seg_cap=cap)
    vc = tq.tq_encode_mse(vl, V, layout=tq.LAYOUT_BLOCK32, seg_len=seq, seg_cap=cap)
    scale = synth.softmax_scale(cfg.head_dim)
    out = tq.tq_decode_attention(kl, vl, q, kc, vc, seq, cap, scale).cpu().numpy()
    Kn, Vn, qn = x_np(K), x_np(V), q.cpu().numpy().astype(np.float64)
    G = cfg.group
    for li in range(len(layers)):
        for h in range(cfg.kv_heads):
            ke = kq.encode(Kn[li, 0, h])
            ve = vq.encode(Vn[li, 0, h], layout="block32")
            want = o.decode_attention(qn[li, 0, h * G:(h + 1) * G], kq, vq, ke, ve, scale, G)
            got = out[li, 0, h * G:(h + 1) * G]
            err = np.linalg.norm(got - want, axis=1) / np.linalg.norm(want, axis=1)
            assert err.max() <= REL_TOL, err.max()


# ------------------------------------------------------------------ dense rotation


@pytest.mark.parametrize("d,m,bits,prod,dtype,layout,n,seg,cap", [
    (256, 0, 3, False, "float16", tq.LAYOUT_ROW, 1000, 0, 0),
    (256, 0, 2, False, "float32", tq.LAYOUT_BLOCK32, 288, 96, 128),    # 3 segments with a spare block each
    (256, 512, 3, True, "bfloat16", tq.LAYOUT_ROW, 700, 0, 0),         # m = 2 d
    (512, 256, 2, True, "float32", tq.LAYOUT_ROW, 450, 150, 160),      # m = d / 2, 3 segments
])
def test_dense_tensor_core_encode(d, m, bits, prod, dtype, layout, n, seg, cap):
    # d and m multiples of 256 run the split-precision tensor-core products;
    # ragged row counts leave a partial last tile of 128 rows
    ora, lib = make_pair(d, bits, prod, seed=60 + d + bits, m=m if prod else None, dense=True)
    x = synth.gaussian_vectors(n, d, seed=61, dtype=dtype, device=DEV, n_outliers=4, outlier_scale=20.0)
    x[7] = 0  # a zero vector
    seg = seg or n
    cap = cap or seg
    ns = n // seg
    lay = "row" if layout == tq.LAYOUT_ROW else "block32"
    if prod:
        codes, signs, norms, rnorms = tq.tq_encode_prod(lib, x, seg_len=seg, seg_cap=cap)
    else:
        codes, norms = tq.tq_encode_mse(lib, x, layout=layout, seg_len=seg, seg_cap=cap)
    torch.cuda.synchronize()
    tq.tq_sync_check()
    wc = u32(codes)
    for s_ in range(ns):
        xs = x_np(x[seg * s_:seg * (s_ + 1)])
        e = ora.encode(xs, layout=lay)
        if layout == tq.LAYOUT_ROW:
            gi = o.unpack_row(wc[cap * s_:cap * s_ + seg], ora.k, ora.d_pad)
        else:
            blocks = cap // 32
            gi = o.unpack_block32(wc[blocks * s_:blocks * (s_ + 1)], ora.k, ora.d_pad, seg)
        _, bad = check_codes(gi, e["idx"], e["y"], ora.boundaries, ora.d_pad)
        gn = norms.cpu().numpy()[cap * s_:cap * s_ + seg]
        assert_close_rel(gn, e["norms"], 1e-30, what="norms")
        if cap > seg:
            assert np.all(norms.cpu().numpy()[cap * s_ + seg:cap * (s_ + 1)] == 0)
        if prod:
            nsg = check_signs(u32(signs)[cap * s_:cap * s_ + seg], e["signs"], e["z"], e["rho64"], m,
                              skip_rows=bad)
            assert nsg <= 1e-4 * seg * m
            gr = rnorms.cpu().numpy()[cap * s_:cap * s_ + seg]
            assert_close_rel(gr, e["rnorms"], 1e-30, what="rnorms", mask=~bad)
    assert norms.cpu().numpy()[7] == 0.0



@pytest.mark.parametrize("bits", [2, 4])
def test_dense_rotation_encode_scores(bits):
    d = 256
    ora, lib = make_pair(d, bits, True, seed=50, dense=True)
    pi = lib.tables()[2]
    assert np.max(np.abs(pi - ora.rot.Pi)) < 2e-7
    x = synth.gaussian_vectors(2000, d, seed=4, device=DEV, n_outliers=8, outlier_scale=10.0, normalize=True)
    q = synth.gaussian_vectors(16, d, seed=5, device=DEV, normalize=True)
    codes, signs, norms, rnorms = tq.tq_encode_prod(lib, x)
    s = tq.tq_scores(lib, q, codes, signs, norms, rnorms)
    torch.cuda.synchronize()
    e = ora.encode(x_np(x))
    gi = o.unpack_row(u32(codes), ora.k, ora.d_pad)
    _, bad = check_codes(gi, e["idx"], e["y"], ora.boundaries, d)
    check_signs(u32(signs), e["signs"], e["z"], e["rho64"], d, skip_rows=bad)
    sig_bad = (o.unpack_signs(u32(signs), d) != o.unpack_signs(e["signs"], d)).any(axis=1)
    want = ora.scores(x_np(q), e["idx"], e["norms"], e["signs"], e["rnorms"])
    floor = e["norms"][None, :] * np.linalg.norm(x_np(q), axis=1)[:, None] / math.sqrt(d)
    ok = ~(bad | sig_bad)
    assert_close_rel(s.cpu().numpy()[:, ok], want[:, ok], floor[:, ok], what="dense scores")

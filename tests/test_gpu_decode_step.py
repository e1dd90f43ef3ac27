"""tq_decode_step (append one token per (layer, batch, kv-head), then attend)
against the oracle: after each step the attention output equals the oracle's
attention over the grown sequence, and at the end every cache slot holds
the oracle's codes of the original key/value rows (slots past the sequence
untouched).  Covers a prefill of 70 tokens plus three steps, block
boundaries (pos 31, 32), the first token of an empty cache and the last slot,
m = 64 QJL rows, d = 192 (256-point rotation) with 8 query heads per KV head, and argument
errors."""
import math

import numpy as np
import pytest
import torch

import synth
import vector_compression_b200 as tq
from oracle import tq_oracle as o
from tests.parity import REL_TOL, assert_close_rel, check_codes, check_signs, u32

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def make_pair(d, bits, prod, seed, stream, m=None):
    m = m or synth.next_pow2(d)
    dr = synth.method_draws(d, m, seed, stream=stream)
    ora = o.Quantizer(d, bits, prod=prod, draws=dr)
    lib = tq.TQParams(d, bits, tq.MODE_PROD if prod else tq.MODE_MSE, tq.ROT_HADAMARD,
                      m=m if prod else 0, signs=dr["signs"], S=dr["S"] if prod else None)
    return ora, lib


def empty_cache(kl, vl, groups, cap):
    z = lambda *s, dt=torch.int32: torch.zeros(s, dtype=dt, device=DEV)
    kc = (z(groups * cap, kl.code_words), z(groups * cap, kl.sign_words),
          z(groups * cap, dt=torch.float32), z(groups * cap, dt=torch.float32))
    vc = (z(groups * cap // 32, vl.code_words * 32), z(groups * cap, dt=torch.float32))
    return kc, vc


def check_cache(kq, vq, K, V, kc, vc, n_tok, cap):
    """Slots 0 .. n_tok-1 of every group equal the oracle's codes; later slots are zero."""
    groups = K.shape[0]
    for g in range(groups):
        ke = kq.encode(K[g, :n_tok])
        ve = vq.encode(V[g, :n_tok], layout="block32")
        rows = slice(g * cap, g * cap + n_tok)
        gi = o.unpack_row(u32(kc[0][rows]), kq.k, kq.d_pad)
        _, bad = check_codes(gi, ke["idx"], ke["y"], kq.boundaries, kq.d_pad)
        check_signs(u32(kc[1][rows]), ke["signs"], ke["z"], ke["rho64"], kq.m, skip_rows=bad)
        assert_close_rel(kc[2][rows].cpu().numpy(), ke["norms"], 1e-30, what="key norms")
        assert_close_rel(kc[3][rows].cpu().numpy(), ke["rnorms"], 1e-30, what="rnorms", mask=~bad)
        blocks = u32(vc[0][g * cap // 32:(g + 1) * cap // 32])
        gv = o.unpack_block32(blocks, vq.k, vq.d_pad, n_tok)
        check_codes(gv, ve["idx"], ve["y"], vq.boundaries, vq.d_pad)
        assert_close_rel(vc[1][rows].cpu().numpy(), ve["norms"], 1e-30, what="value norms")
        assert np.all(u32(kc[0][g * cap + n_tok:(g + 1) * cap]) == 0)
        assert np.all(vc[1][g * cap + n_tok:(g + 1) * cap].cpu().numpy() == 0)
        tail = blocks.reshape(cap // 32, vq.k, vq.d_pad)
        for t in range(n_tok, cap):  # bits of the tokens not yet appended
            assert np.all((tail[t // 32] >> np.uint32(t % 32)) & 1 == 0)


def run_steps(d, G, bits, cap, prefill, steps, dtype="float16", seed=7, m=None):
    Ln, B, Hkv = 2, 1, 2
    groups = Ln * B * Hkv
    kq, kl = make_pair(d, bits, True, seed, 1, m=m)
    vq, vl = make_pair(d, bits, False, seed, 2)
    T = prefill + steps
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((groups, T, d)) * rng.lognormal(0, 1, size=(1, 1, d))
    V = rng.standard_normal((groups, T, d))
    tdt = getattr(torch, dtype)
    Kt = torch.from_numpy(K).to(DEV).to(tdt)
    Vt = torch.from_numpy(V).to(DEV).to(tdt)
    Kn = Kt.float().cpu().numpy().astype(np.float64)  # the rows the GPU sees
    Vn = Vt.float().cpu().numpy().astype(np.float64)
    kc, vc = empty_cache(kl, vl, groups, cap)
    if prefill:
        tq.tq_encode_prod(kl, Kt[:, :prefill].contiguous(), seg_len=prefill, seg_cap=cap, out=kc)
        tq.tq_encode_mse(vl, Vt[:, :prefill].contiguous(), layout=tq.LAYOUT_BLOCK32, seg_len=prefill,
                         seg_cap=cap, codes=vc[0], norms=vc[1])
    scale = 1 / math.sqrt(d)
    for s in range(steps):
        pos = prefill + s
        q = torch.from_numpy(rng.standard_normal((Ln, B, G * Hkv, d))).float().to(DEV)
        kn = Kt[:, pos].reshape(Ln, B, Hkv, d).contiguous()
        vn = Vt[:, pos].reshape(Ln, B, Hkv, d).contiguous()
        out = tq.tq_decode_step(kl, vl, q, kn, vn, kc, vc, pos, cap, scale).cpu().numpy()
        qn = q.cpu().numpy().astype(np.float64)
        for g in range(groups):
            l, h = g // Hkv, g % Hkv
            ke = kq.encode(Kn[g, :pos + 1])
            ve = vq.encode(Vn[g, :pos + 1], layout="block32")
            want = o.decode_attention(qn[l, 0, h * G:(h + 1) * G], kq, vq, ke, ve, scale, G)
            got = out[l, 0, h * G:(h + 1) * G]
            err = np.linalg.norm(got - want, axis=1) / np.linalg.norm(want, axis=1)
            assert err.max() <= REL_TOL, (pos, g, err.max())
    torch.cuda.synchronize()
    tq.tq_sync_check()
    check_cache(kq, vq, Kn, Vn, kc, vc, prefill + steps, cap)


def test_decode_steps_after_prefill():
    run_steps(128, 4, 3, cap=96, prefill=70, steps=3)


def test_decode_steps_cross_block_boundary():
    run_steps(128, 4, 3, cap=64, prefill=31, steps=2, dtype="bfloat16")


def test_decode_steps_from_empty_to_last_slot():
    run_steps(128, 1, 2, cap=32, prefill=0, steps=3, dtype="float32")
    run_steps(128, 2, 4, cap=32, prefill=29, steps=3)


def test_decode_steps_qjl_half_rows():
    # QJL with m = d / 2 = 64 projection rows
    run_steps(128, 4, 3, cap=96, prefill=62, steps=3, m=64)


def test_decode_steps_d192_gqa8():
    run_steps(192, 8, 4, cap=64, prefill=40, steps=2)


def test_decode_step_argument_errors():
    kq, kl = make_pair(128, 3, True, 1, 1)
    vq, vl = make_pair(128, 3, False, 1, 2)
    kc, vc = empty_cache(kl, vl, 1, 32)
    q = torch.zeros((1, 1, 4, 128), device=DEV)
    kn = torch.zeros((1, 1, 1, 128), device=DEV, dtype=torch.float16)
    with pytest.raises(tq.TQError, match="INVALID_ARG"):
        tq.tq_decode_step(kl, vl, q, kn, kn, kc, vc, 32, 32, 1.0)  # pos == cap
    with pytest.raises(tq.TQError, match="INVALID_ARG"):
        tq.tq_decode_step(vl, kl, q, kn, kn, kc, vc, 0, 32, 1.0)  # key/value handles swapped

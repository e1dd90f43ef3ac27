"""GPU encode versus the CPU oracle on the shapes the tensor-core encoder
takes (Hadamard rotation with d_pad = 128, fp16/bf16 rows, segments of a
multiple of 32 vectors): every code width, both layouts, Q_prod with m = 64
and 128, padded d, segments with spare capacity, ragged last tiles, zero
vectors, and enough tiles that every CTA cycles its input ring and its TMEM
buffers several times."""
import numpy as np
import pytest
import torch

import synth
import vector_compression_b200 as tq
from oracle import tq_oracle as o
from tests.parity import assert_close_rel, check_codes, check_signs, u32

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def make_pair(d, bits, prod, seed, m=None):
    m = m if m is not None else synth.next_pow2(d)
    dr = synth.method_draws(d, m, seed)
    ora = o.Quantizer(d, bits, prod=prod, draws=dr)
    lib = tq.TQParams(d, bits, tq.MODE_PROD if prod else tq.MODE_MSE, tq.ROT_HADAMARD,
                      m=m if prod else 0, signs=dr["signs"], S=dr["S"] if prod else None)
    return ora, lib


def x_np(x):
    return x.detach().float().cpu().numpy().astype(np.float64)


def vectors(n, d, dtype, seed):
    x = synth.gaussian_vectors(n, d, seed=seed, dtype=dtype, device=DEV, n_outliers=4,
                               outlier_scale=20.0)
    x[min(5, n - 1)] = 0  # a zero vector
    return x


@pytest.mark.parametrize("d,dtype,layout,n", [
    (128, "float16", tq.LAYOUT_ROW, 2080),      # 16 full tiles + a 32-row tail
    (128, "bfloat16", tq.LAYOUT_BLOCK32, 2080),
    (96, "float16", tq.LAYOUT_BLOCK32, 640),    # zero-padded columns 96..127
    (120, "bfloat16", tq.LAYOUT_ROW, 4096),
])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_tc_encode_mse(d, dtype, layout, n, bits):
    ora, lib = make_pair(d, bits, False, seed=40 + d + bits)
    x = vectors(n, d, dtype, seed=bits + 3)
    codes, norms = tq.tq_encode_mse(lib, x, layout=layout)
    torch.cuda.synchronize()
    e = ora.encode(x_np(x), layout="row" if layout == tq.LAYOUT_ROW else "block32")
    if layout == tq.LAYOUT_ROW:
        gi = o.unpack_row(u32(codes), ora.k, ora.d_pad)
    else:
        gi = o.unpack_block32(u32(codes), ora.k, ora.d_pad, n)
    check_codes(gi, e["idx"], e["y"], ora.boundaries, ora.d_pad)
    gn = norms.cpu().numpy()[:n]
    assert gn[5] == 0.0
    assert_close_rel(gn, e["norms"], 1e-30, what="norms")


@pytest.mark.parametrize("d,m,bits,dtype,n", [
    (128, 128, 3, "float16", 4128),
    (128, 128, 2, "bfloat16", 1024),
    (128, 64, 4, "float16", 2080),
    (104, 128, 3, "bfloat16", 640),
])
def test_tc_encode_prod(d, m, bits, dtype, n):
    ora, lib = make_pair(d, bits, True, seed=60 + bits, m=m)
    x = vectors(n, d, dtype, seed=9)
    codes, signs, norms, rnorms = tq.tq_encode_prod(lib, x)
    torch.cuda.synchronize()
    e = ora.encode(x_np(x))
    gi = o.unpack_row(u32(codes), ora.k, ora.d_pad)
    _, bad = check_codes(gi, e["idx"], e["y"], ora.boundaries, ora.d_pad)
    ns = check_signs(u32(signs), e["signs"], e["z"], e["rho64"], m, skip_rows=bad)
    assert ns <= 1e-4 * n * m
    assert_close_rel(norms.cpu().numpy(), e["norms"], 1e-30, what="norms")
    assert_close_rel(rnorms.cpu().numpy(), e["rnorms"], 1e-30, what="rnorms", mask=~bad)


@pytest.mark.parametrize("layout,seg,cap,ns", [(tq.LAYOUT_ROW, 96, 160, 5),
                                               (tq.LAYOUT_BLOCK32, 96, 160, 5),
                                               (tq.LAYOUT_ROW, 1184, 1216, 9),
                                               (tq.LAYOUT_BLOCK32, 32, 64, 70)])
def test_tc_encode_segments_with_capacity(layout, seg, cap, ns):
    # ns segments of seg vectors into slots of cap: slots >= seg untouched
    ora, lib = make_pair(128, 3, False, seed=5)
    x = synth.gaussian_vectors(seg * ns, 128, seed=11, dtype="float16", device=DEV)
    codes, norms = tq.tq_encode_mse(lib, x, layout=layout, seg_len=seg, seg_cap=cap)
    torch.cuda.synchronize()
    w = u32(codes)
    for s in range(ns):
        e = ora.encode(x_np(x[seg * s:seg * (s + 1)]), layout="row")
        if layout == tq.LAYOUT_ROW:
            gi = o.unpack_row(w[cap * s:cap * s + seg], 3, 128)
            assert np.all(w[cap * s + seg:cap * (s + 1)] == 0)
        else:
            blocks = w[(cap // 32) * s:(cap // 32) * (s + 1)]
            gi = o.unpack_block32(blocks[:seg // 32], 3, 128, seg)
            assert np.all(blocks[seg // 32:] == 0)
        check_codes(gi, e["idx"], e["y"], ora.boundaries, 128)
        assert_close_rel(norms[cap * s:cap * s + seg].cpu().numpy(), e["norms"], 1e-30)
        assert np.all(norms[cap * s + seg:cap * (s + 1)].cpu().numpy() == 0)


def test_tc_encode_prod_segments():
    # Q_prod rows land in slot s * cap + pos of their segment
    ora, lib = make_pair(128, 3, True, seed=6)
    seg, cap, ns = 160, 192, 7
    x = synth.gaussian_vectors(seg * ns, 128, seed=13, dtype="bfloat16", device=DEV)
    codes, signs, norms, rnorms = tq.tq_encode_prod(lib, x, seg_len=seg, seg_cap=cap)
    torch.cuda.synchronize()
    w, sg = u32(codes), u32(signs)
    for s in range(ns):
        e = ora.encode(x_np(x[seg * s:seg * (s + 1)]))
        gi = o.unpack_row(w[cap * s:cap * s + seg], ora.k, 128)
        _, bad = check_codes(gi, e["idx"], e["y"], ora.boundaries, 128)
        nsg = check_signs(sg[cap * s:cap * s + seg], e["signs"], e["z"], e["rho64"], ora.m, skip_rows=bad)
        assert nsg <= 1e-4 * seg * ora.m
        assert_close_rel(norms[cap * s:cap * s + seg].cpu().numpy(), e["norms"], 1e-30)
        assert_close_rel(rnorms[cap * s:cap * s + seg].cpu().numpy(), e["rnorms"], 1e-30, mask=~bad)
        assert np.all(w[cap * s + seg:cap * (s + 1)] == 0)
        assert np.all(sg[cap * s + seg:cap * (s + 1)] == 0)


def test_tc_encode_many_tiles_per_cta():
    # 6 tiles per SM and a ragged tail: the input ring (4 stages) and both TMEM
    # buffers wrap several times in every CTA
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    n = n_sm * 128 * 6 + 96
    for prod in (False, True):
        ora, lib = make_pair(128, 3, prod, seed=77)
        x = synth.gaussian_vectors(n, 128, seed=12, dtype="float16", device=DEV)
        if prod:
            codes, signs, norms, rnorms = tq.tq_encode_prod(lib, x)
        else:
            codes, norms = tq.tq_encode_mse(lib, x, layout=tq.LAYOUT_ROW)
        torch.cuda.synchronize()
        tq.tq_sync_check()
        e = ora.encode(x_np(x))
        gi = o.unpack_row(u32(codes), ora.k, ora.d_pad)
        _, bad = check_codes(gi, e["idx"], e["y"], ora.boundaries, ora.d_pad)
        assert_close_rel(norms.cpu().numpy(), e["norms"], 1e-30, what="norms")
        if prod:
            nsg = check_signs(u32(signs), e["signs"], e["z"], e["rho64"], ora.m, skip_rows=bad)
            assert nsg <= 1e-4 * n * ora.m
            assert_close_rel(rnorms.cpu().numpy(), e["rnorms"], 1e-30, what="rnorms", mask=~bad)

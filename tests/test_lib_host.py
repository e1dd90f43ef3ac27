"""Host-side checks of libtq that need no GPU: the shared library loads and
exports every entry point declared in include/tq.h, its own codebook solver
and QR agree with the oracle, and argument validation rejects bad calls
before any launch."""
import ctypes as C
import os
import re

import numpy as np
import pytest

from oracle import tq_oracle as o
import vector_compression_b200 as tq
from vector_compression_b200 import _lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "tq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    syms = declared_symbols()
    assert len(syms) >= 15
    lib = C.CDLL(L.LIB_PATH)
    for s in syms:
        assert hasattr(lib, s), s
        assert s in L.SIGNATURES, f"binding misses {s}"


def test_status_strings_and_version():
    lib = L.lib()
    for code, name in L.STATUS.items():
        assert lib.tq_status_string(code).decode() == name
    assert "sm_100a" in tq.tq_version()


@pytest.mark.parametrize("d", [32, 64, 128, 256, 1536])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_codebook_matches_oracle(d, bits):
    c, b = tq.tq_build_codebook(d, bits)
    co, bo = o.codebook(d, bits)
    # the library solves in double with its own quadrature and rounds to fp32
    assert np.all(np.abs(c - co) <= 2 * np.spacing(np.abs(co).astype(np.float32)) + 1e-12)
    assert np.all(np.abs(b - bo) <= 2 * np.spacing(np.maximum(np.abs(bo), 1e-30).astype(np.float32)) + 1e-12)
    assert np.all(c == -c[::-1]) and np.all(b == -b[::-1])


@pytest.mark.parametrize("d", [32, 96, 256])
def test_rotation_matches_oracle(d):
    G = np.random.default_rng(d).standard_normal((d, d))
    pi = tq.tq_make_rotation(G)
    assert np.max(np.abs(pi - o.haar_rotation(G))) < 2e-7


def test_codebook_rejects_bad_args():
    lib = L.lib()
    c = (C.c_float * 16)()
    assert lib.tq_build_codebook(128, 0, c, c) == 1
    assert lib.tq_build_codebook(128, 5, c, c) == 1
    assert lib.tq_build_codebook(2, 2, c, c) == 1
    assert lib.tq_build_codebook(128, 2, None, c) == 1


def _mse_handle(d=128, bits=3):
    dr = {"signs": np.ones(128 if d <= 128 else 256, np.int8)}
    return tq.TQParams(d, bits, tq.MODE_MSE, tq.ROT_HADAMARD, signs=dr["signs"][: max(32, 1 << (d - 1).bit_length())])


def test_params_validation():
    lib = L.lib()
    h = C.c_void_p()
    sg = np.ones(128, np.int8)
    p = sg.ctypes.data_as(C.c_void_p)
    assert lib.tq_params_create(0, 3, 0, 0, 0, p, None, None, C.byref(h)) == 1      # d
    assert lib.tq_params_create(128, 5, 0, 0, 0, p, None, None, C.byref(h)) == 1    # MSE bits
    assert lib.tq_params_create(128, 1, 1, 0, 128, p, None, None, C.byref(h)) == 1  # PROD bits
    assert lib.tq_params_create(128, 3, 0, 0, 0, None, None, None, C.byref(h)) == 1  # no signs
    assert lib.tq_params_create(512, 3, 0, 0, 0, p, None, None, C.byref(h)) == 2    # d_pad 512
    assert lib.tq_params_create(100, 3, 0, 1, 0, None, None, None, C.byref(h)) == 2  # dense d%32
    bad = np.ones(128, np.int8)
    bad[5] = 0
    assert lib.tq_params_create(128, 3, 0, 0, 0, bad.ctypes.data_as(C.c_void_p), None, None, C.byref(h)) == 1
    S = np.full((100, 128), 0.5, np.float32)  # m not a multiple of 32
    assert lib.tq_params_create(128, 3, 1, 0, 100, p, S.ctypes.data_as(C.c_void_p), None, C.byref(h)) == 1
    S = np.full((128, 128), 0.1, np.float32)  # not fp16-representable
    assert lib.tq_params_create(128, 3, 1, 0, 128, p, S.ctypes.data_as(C.c_void_p), None, C.byref(h)) == 1
    assert lib.tq_params_create(128, 3, 3, 0, 0, p, None, None, C.byref(h)) == 1    # no mode 3
    assert lib.tq_params_create(128, 3, 0x100, 0, 0, p, None, None, C.byref(h)) == 1  # fp16 rho needs PROD
    assert lib.tq_params_create(128, 3, 0x201, 0, 128, p, None, None, C.byref(h)) == 1  # unknown flag


def test_wait_expiry_check_validates_budget():
    lib = L.lib()
    assert lib.tq_check_wait_expiry(0, None) == 1
    assert lib.tq_check_wait_expiry((1 << 31) + 1, None) == 1


def test_unbiased_mode_handle():
    # Q_MSE with the unbiased (EDEN) scale: same code geometry as Q_MSE, and
    # accepted by the Q_MSE entry points' validation (a Q_prod call is not)
    u = tq.TQParams(128, 2, tq.MODE_MSE_UNBIASED, tq.ROT_HADAMARD, signs=np.ones(128, np.int8))
    assert (u.d_pad, u.k, u.code_words, u.sign_words, u.m) == (128, 2, 8, 0, 0)
    lib = L.lib()
    fake = C.c_void_p(0x10000)
    assert lib.tq_encode_mse(u.handle, fake, 0, 0, 128, 0, 0, 0, None, None, None, 0, None) == 0  # empty
    assert lib.tq_encode_mse(u.handle, None, 0, 10, 128, 0, 0, 0, fake, fake, None, 0, None) == 1
    assert lib.tq_encode_prod(u.handle, fake, 0, 10, 128, 0, 0, fake, fake, fake, fake, None, 0, None) == 1


def test_encode_and_attention_validation_before_launch():
    # a Q_MSE Hadamard handle allocates no device tables, so it can be made
    # without a GPU; every call below must fail validation before any launch.
    lib = L.lib()
    mse = tq.TQParams(128, 3, tq.MODE_MSE, tq.ROT_HADAMARD, signs=np.ones(128, np.int8))
    assert (mse.d_pad, mse.k, mse.code_words, mse.sign_words) == (128, 3, 12, 0)
    h = mse.handle
    fake = C.c_void_p(0x10000)  # aligned, never dereferenced
    mis = C.c_void_p(0x10008)
    # null input / bad dtype / bad layout / misaligned / bad segments
    assert lib.tq_encode_mse(h, None, 0, 10, 128, 0, 0, 0, fake, fake, None, 0, None) == 1
    assert lib.tq_encode_mse(h, fake, 7, 10, 128, 0, 0, 0, fake, fake, None, 0, None) == 1
    assert lib.tq_encode_mse(h, fake, 0, 10, 128, 0, 0, 5, fake, fake, None, 0, None) == 1
    assert lib.tq_encode_mse(h, mis, 0, 10, 128, 0, 0, 0, fake, fake, None, 0, None) == 1
    assert lib.tq_encode_mse(h, fake, 0, 10, 100, 0, 0, 0, fake, fake, None, 0, None) == 1  # ld < d
    h100 = _mse_handle(100)
    assert lib.tq_encode_mse(h100.handle, fake, 1, 10, 100, 0, 0, 0, fake, fake, None, 0, None) == 1  # 200-B rows
    assert lib.tq_encode_mse(h, fake, 0, 10, 128, 3, 0, 0, fake, fake, None, 0, None) == 1  # 10 % 3
    assert lib.tq_encode_mse(h, fake, 0, 10, 128, 10, 5, 0, fake, fake, None, 0, None) == 1  # cap < len
    assert lib.tq_encode_mse(h, fake, 0, 10, 128, 10, 40, 1, fake, fake, None, 0, None) == 1  # cap % 32
    assert lib.tq_encode_mse(h, fake, 0, 0, 128, 0, 0, 0, None, None, None, 0, None) == 0   # empty
    # a Q_MSE handle cannot encode Q_prod nor score
    assert lib.tq_encode_prod(h, fake, 0, 10, 128, 0, 0, fake, fake, fake, fake, None, 0, None) == 1
    assert lib.tq_scores(h, fake, 1, 128, fake, fake, fake, fake, 10, fake, 0, None, None, fake, 1 << 20, None) == 1
    # attention: wrong handle kinds, bad shapes, missing workspace
    f = C.c_float(1.0)
    args = [fake] * 7
    assert lib.tq_decode_attention(h, h, fake, 1, 1, 8, 2, 64, 64, f, *args, None, 0, None) == 1
    sz = C.c_size_t()
    assert lib.tq_decode_attention_workspace_size(h, h, 1, 1, 7, 2, 64, C.byref(sz)) == 1  # Hq % Hkv

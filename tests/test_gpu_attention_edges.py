"""Decode-attention edge cases against the oracle (turboquant-pytorch
Pattern 1: scores from the compressed keys, softmax, weighted sum of the
Q_MSE-reconstructed values).

One dominant key among hundreds of much smaller softmax weights, all inside
one short run of the cache: identical keys and values make every small
weight identical, so any rounding of the weights adds up coherently instead
of averaging out.  The query scale sweeps the weight ratio across several
values so that no fixed-point grid happens to represent it exactly.  The
caches hold the oracle's own codes, so the comparison isolates the
attention arithmetic."""
import math

import numpy as np
import pytest
import torch

import vector_compression_b200 as tq
from oracle import tq_oracle as o
from tests.parity import REL_TOL
from tests.test_gpu_parity import _pack_cache, make_pair

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.mark.parametrize("d,G,bits", [(128, 4, 3), (192, 4, 4)])
def test_attention_dominant_key_among_tiny_weights(d, G, bits):
    seq = cap = 32768
    kq, kl = make_pair(d, bits, True, seed=61, stream=1)
    vq, vl = make_pair(d, bits, False, seed=61, stream=2)
    rng = np.random.default_rng(62)
    q0 = rng.standard_normal((G, d))
    qhat = q0[0] / np.linalg.norm(q0[0])
    K = 0.3 * rng.standard_normal((1, seq, d))
    V = rng.standard_normal((1, seq, d))
    run = slice(384 * 5, 384 * 6)          # one run of 384 consecutive tokens
    dom = 384 * 5 + 17
    K[0, run] = 2.0 * qhat                 # identical small-weight keys ...
    V[0, run] = V[0, 384 * 5 + 3]          # ... with identical values
    K[0, dom] = 3.0 * qhat                 # the dominant key
    V[0, dom] = rng.standard_normal(d)
    kc, vc, encs = _pack_cache(kq, vq, K, V, seq, cap)
    ke, ve = encs[0]
    worst = 0.0
    # the logit gap between the dominant and the small keys grows with the
    # query scale: small-to-dominant weight ratios from about 7e-3 to 3e-4,
    # and the 383 small weights together from about 2.6 to 0.13 of the
    # dominant one
    for lam in (5.0, 5.6, 6.2, 6.8, 7.4, 8.0):
        q = (lam * q0)[None, None]
        scale = 1 / math.sqrt(d)
        out = tq.tq_decode_attention(kl, vl, torch.from_numpy(q).float().to(DEV), kc, vc, seq, cap, scale)
        got = out.cpu().numpy()[0, 0]
        want = o.decode_attention(q[0, 0], kq, vq, ke, ve, scale, G)
        err = np.linalg.norm(got - want, axis=1) / np.linalg.norm(want, axis=1)
        worst = max(worst, float(err.max()))
        assert err.max() <= REL_TOL, (lam, err.max())
    print(f"dominant-key attention: worst relative error {worst:.2e}")


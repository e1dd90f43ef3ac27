"""The turboquant-pytorch page's two synthetic reports (Pattern 2, attention
fidelity; Pattern 3, needle in a haystack), run on the GPU path with the
page's settings (d = 128, b = 3, proj_dim m = 64, unit vectors) and checked
against the same reports computed from the oracle's estimates.

* Fidelity: softmax of the exact scores <k, q> against softmax of the
  estimated scores, per query: cosine similarity of the two distributions
  and whether their argmax agree; 2048 keys, 100 queries.
* Needle: a haystack of random unit vectors with one vector close to the
  query (query + 0.1 noise, normalized); success when the estimated argmax
  is the true nearest neighbour; 20 trials at seq 8192."""
import numpy as np
import pytest
import torch

import synth
import vector_compression_b200 as tq
from oracle import tq_oracle as o

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
D, BITS, M = 128, 3, 64


def pair(seed):
    dr = synth.method_draws(D, M, seed, stream=1)
    ora = o.Quantizer(D, BITS, prod=True, draws=dr)
    lib = tq.TQParams(D, BITS, tq.MODE_PROD, tq.ROT_HADAMARD, m=M, signs=dr["signs"], S=dr["S"])
    return ora, lib


def unit(rng, *shape):
    x = rng.standard_normal(shape)
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def gpu_scores(lib, keys, queries):
    kt = torch.from_numpy(keys).float().to(DEV)
    codes, signs, norms, rnorms = tq.tq_encode_prod(lib, kt)
    s = tq.tq_scores(lib, torch.from_numpy(queries).float().to(DEV), codes, signs, norms, rnorms)
    torch.cuda.synchronize()
    tq.tq_sync_check()
    return s.cpu().numpy().astype(np.float64)


def oracle_scores(ora, keys, queries):
    e = ora.encode(keys.astype(np.float32).astype(np.float64))
    return ora.scores(queries.astype(np.float32).astype(np.float64), e["idx"], e["norms"], e["signs"], e["rnorms"])


def softmax(s):
    e = np.exp(s - s.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def fidelity(true_s, est_s):
    pt, pe = softmax(true_s), softmax(est_s)
    cos = np.sum(pt * pe, axis=1) / (np.linalg.norm(pt, axis=1) * np.linalg.norm(pe, axis=1))
    return cos, pt.argmax(axis=1) == pe.argmax(axis=1)


def test_attention_fidelity_report():
    rng = np.random.default_rng(2048)
    keys, queries = unit(rng, 2048, D), unit(rng, 100, D)
    ora, lib = pair(5)
    true_s = queries.astype(np.float32).astype(np.float64) @ keys.astype(np.float32).astype(np.float64).T
    cos_g, top_g = fidelity(true_s, gpu_scores(lib, keys, queries))
    cos_o, top_o = fidelity(true_s, oracle_scores(ora, keys, queries))
    print(f"fidelity: mean cosine {cos_g.mean():.4f} (oracle {cos_o.mean():.4f}), "
          f"top-1 {top_g.mean():.2%} (oracle {top_o.mean():.2%})")
    np.testing.assert_allclose(cos_g, cos_o, rtol=0, atol=1e-5)
    assert np.array_equal(top_g, top_o)
    # unit keys and queries give scores within [-1, 1]: the softmax is
    # nearly flat and the estimate must keep it so
    assert cos_g.mean() > 0.99


def test_needle_in_haystack_report():
    ora, lib = pair(6)
    succ_g = succ_o = 0
    for trial in range(20):
        rng = np.random.default_rng([8192, trial])
        hay = unit(rng, 8192, D)
        q = unit(rng, D)
        needle = q + 0.1 * rng.standard_normal(D)
        idx = int(rng.integers(0, 8192))
        hay[idx] = needle / np.linalg.norm(needle)
        true_best = int(np.argmax(hay.astype(np.float32).astype(np.float64) @ q.astype(np.float32)))
        eg = gpu_scores(lib, hay, q[None])[0]
        eo = oracle_scores(ora, hay, q[None])[0]
        assert int(np.argmax(eg)) == int(np.argmax(eo))
        succ_g += int(np.argmax(eg)) == true_best
        succ_o += int(np.argmax(eo)) == true_best
    print(f"needle retrieval: {succ_g}/20 (oracle {succ_o}/20)")
    assert succ_g == succ_o >= 19

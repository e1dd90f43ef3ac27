"""Scores and fused top-k on the tensor cores versus the oracle: many query
blocks (a partial last block), ragged vector counts (a partial last group of
two 128-vector tiles), Hadamard and dense rotations, key codes of 1..3 bits,
top-k of 1..32 with and without the full score matrix, and more work items
than SMs.  The caches hold the
oracle's codes, so scores are compared element by element at 1e-5 relative;
the top-k must be the exact (score descending, index ascending) top-k of the
GPU's own scores."""
import math

import numpy as np
import pytest
import torch

import synth
import vector_compression_b200 as tq
from oracle import tq_oracle as o
from tests.parity import assert_close_rel
from tests.test_gpu_parity import make_pair, x_np

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _dev(a):
    return torch.from_numpy(a.view(np.int32) if a.dtype == np.uint32 else a).to(DEV)


@pytest.mark.parametrize("d,dense,bits,n,nq,topk", [
    (128, False, 3, 1000, 100, 10),   # 4 query blocks (last with 4 queries), 3 groups + 232 vectors
    (128, False, 2, 257, 33, 1),      # one vector past a group, a 1-query last block
    (128, False, 4, 777, 64, 32),     # the largest top-k
    (256, True, 4, 700, 40, 10),      # dense rotation, m = 256, k = 3 (four features)
    (256, True, 2, 513, 31, 5),       # dense, k = 1, one partial query block
    # 33 query blocks x 12 ranges of 2 groups: more items than SMs, so a CTA
    # runs consecutive items of one query block (its lists carry over) and
    # crosses into the next block
    (128, False, 3, 6000, 1050, 10),
])
def test_tc_scores_and_topk(d, dense, bits, n, nq, topk):
    ora, lib = make_pair(d, bits, True, seed=70 + bits, dense=dense)
    x = x_np(synth.gaussian_vectors(n, d, seed=71, n_outliers=4, outlier_scale=20.0, normalize=dense))
    q = x_np(synth.gaussian_vectors(nq, d, seed=72, normalize=dense))
    e = ora.encode(x)
    args = (_dev(e["codes"]), _dev(e["signs"]), _dev(e["norms"]), _dev(e["rnorms"]))
    qt = torch.from_numpy(q).float().to(DEV)
    s, ts, ti = tq.tq_scores(lib, qt, *args, topk=topk)
    _, ts2, ti2 = tq.tq_scores(lib, qt, *args, topk=topk, want_scores=False)
    torch.cuda.synchronize()
    tq.tq_sync_check()
    want = ora.scores(q, e["idx"], e["norms"], e["signs"], e["rnorms"])
    floor = e["norms"][None, :] * np.linalg.norm(q, axis=1)[:, None] / math.sqrt(d)
    sg = s.cpu().numpy()
    assert_close_rel(sg, want, floor, tol=1e-5, what="scores")
    vs, vi = o.topk(sg, topk)
    assert np.array_equal(ti.cpu().numpy(), vi)
    assert np.array_equal(ts.cpu().numpy(), vs)
    # the fused top-k (no score matrix) is the same
    assert np.array_equal(ti2.cpu().numpy(), vi)
    assert np.array_equal(ts2.cpu().numpy(), vs)


def test_tc_topk_ties_go_to_the_lower_index():
    # identical vectors score identically: the top-k must list them by index
    d, bits = 128, 3
    ora, lib = make_pair(d, bits, True, seed=80)
    base = x_np(synth.gaussian_vectors(40, d, seed=81))
    x = np.concatenate([base] * 13)[:500]          # each vector repeated every 40 rows
    q = x_np(synth.gaussian_vectors(35, d, seed=82))
    e = ora.encode(x)
    args = (_dev(e["codes"]), _dev(e["signs"]), _dev(e["norms"]), _dev(e["rnorms"]))
    qt = torch.from_numpy(q).float().to(DEV)
    s, ts, ti = tq.tq_scores(lib, qt, *args, topk=12)
    torch.cuda.synchronize()
    vs, vi = o.topk(s.cpu().numpy(), 12)
    assert np.array_equal(ti.cpu().numpy(), vi)
    assert np.array_equal(ts.cpu().numpy(), vs)

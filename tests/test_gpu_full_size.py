"""GPU versus the CPU oracle at the workloads' full sizes, on sampled outputs
the oracle can compute one by one: the whole cache (or database) is encoded
and attended on the GPU in one launch per kernel, as bench.py times it; the
oracle re-encodes the sampled rows from the same inputs (rows are
independent) and recomputes the sampled attention heads and scores.

* Llama-3.1-8B-shaped cache, all 32 layers (fp16, d = 128, seq 32768, G = 4),
  b = 3 (and b = 2, 4 on a smaller sample): groups from the first and last
  layer and from different batches and heads.
* Long-context cache, d = 192 padded to a 256-point Hadamard, seq 131072,
  b = 4, m = 256: two of the eight KV heads.
* Retrieval set, 1,000,000 unit vectors of d = 1536 with the dense rotation,
  b = 2 and 4: 512 sampled database vectors and 16 queries; the top-10 lists
  are checked against the GPU's own score rows (ties to the lower index)."""
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


def check_group(cfg, kq, vq, K, V, q, kc, vc, out, li, b, h):
    """Codes, norms and attention of KV group (layer li, batch b, head h)."""
    seq, G = cfg.seq, cfg.group
    Kg, Vg = x_np(K[li, b, h]), x_np(V[li, b, h])
    ke = kq.encode(Kg)
    ve = vq.encode(Vg, layout="block32")
    rows = slice(((li * cfg.batch + b) * cfg.kv_heads + h) * seq, ((li * cfg.batch + b) * cfg.kv_heads + h + 1) * seq)
    codes, signs, norms, rnorms = kc
    gi = o.unpack_row(u32(codes[rows]), kq.k, kq.d_pad)
    _, bad = check_codes(gi, ke["idx"], ke["y"], kq.boundaries, kq.d_pad, what="key codes")
    ns = check_signs(u32(signs[rows]), ke["signs"], ke["z"], ke["rho64"], kq.m, skip_rows=bad)
    assert ns <= 1e-4 * seq * kq.m
    assert_close_rel(norms[rows].cpu().numpy(), ke["norms"], 1e-30, what="key norms")
    assert_close_rel(rnorms[rows].cpu().numpy(), ke["rnorms"], 1e-30, what="residual norms", mask=~bad)
    vcodes, vnorms = vc
    blocks = slice(rows.start // 32, rows.stop // 32)
    gv = o.unpack_block32(u32(vcodes[blocks]), vq.k, vq.d_pad, seq)
    check_codes(gv, ve["idx"], ve["y"], vq.boundaries, vq.d_pad, what="value codes")
    assert_close_rel(vnorms[rows].cpu().numpy(), ve["norms"], 1e-30, what="value norms")
    qg = q[li, b, h * G:(h + 1) * G].cpu().numpy().astype(np.float64)
    want = o.decode_attention(qg, kq, vq, ke, ve, synth.softmax_scale(cfg.head_dim), G)
    got = out[li, b, h * G:(h + 1) * G].cpu().numpy()
    err = np.linalg.norm(got - want, axis=1) / np.linalg.norm(want, axis=1)
    assert err.max() <= REL_TOL, f"attention relative error {err.max():.3g}"


def run_cache(cfg):
    K, V = synth.kv_cache(cfg, device=DEV)
    q = synth.decode_queries(cfg, device=DEV)
    kq, kl = make_pair(cfg.head_dim, cfg.key_bits, True, seed=cfg.seed, stream=1)
    vq, vl = make_pair(cfg.head_dim, cfg.value_bits, False, seed=cfg.seed, stream=2)
    seq = cap = cfg.seq
    kc = tq.tq_encode_prod(kl, K, seg_len=seq, seg_cap=cap)
    vc = tq.tq_encode_mse(vl, V, layout=tq.LAYOUT_BLOCK32, seg_len=seq, seg_cap=cap)
    out = tq.tq_decode_attention(kl, vl, q, kc, vc, seq, cap, synth.softmax_scale(cfg.head_dim))
    torch.cuda.synchronize()
    tq.tq_sync_check()
    return kq, vq, K, V, q, kc, vc, out


@pytest.mark.parametrize("bits,groups", [
    (3, [(0, 0, 0), (0, 3, 7), (31, 1, 4), (31, 2, 2)]),
    (2, [(0, 1, 5)]),
    (4, [(31, 0, 6)]),
])
def test_llama_cache_full_size(bits, groups):
    cfg = synth.KV_CONFIGS["llama3.1-8b_32k_b3"].with_bits(bits)
    kq, vq, K, V, q, kc, vc, out = run_cache(cfg)
    for li, b, h in groups:
        check_group(cfg, kq, vq, K, V, q, kc, vc, out, li, b, h)


def test_longctx_d192_cache_full_size():
    cfg = synth.KV_CONFIGS["longctx-d192_128k_b4"]
    kq, vq, K, V, q, kc, vc, out = run_cache(cfg)
    for h in (0, 5):
        check_group(cfg, kq, vq, K, V, q, kc, vc, out, 0, 0, h)


@pytest.mark.parametrize("bits", [2, 4])
def test_retrieval_full_size(bits):
    R = synth.RETRIEVAL
    d, n = R["d"], R["n"]
    ora, lib = make_pair(d, bits, True, seed=R["seed"], m=R["m"], dense=True)
    x = synth.gaussian_vectors(n, d, seed=R["seed"], device=DEV, n_outliers=R["n_outliers"],
                               outlier_scale=R["outlier_scale"], normalize=True)
    qs = synth.gaussian_vectors(16, d, seed=R["seed"] + 1, device=DEV, normalize=True)
    codes, signs, norms, rnorms = tq.tq_encode_prod(lib, x)
    scores, top_s, top_i = tq.tq_scores(lib, qs, codes, signs, norms, rnorms, topk=R["topk"])
    torch.cuda.synchronize()
    tq.tq_sync_check()
    rng = np.random.default_rng(11)
    idx = np.sort(rng.choice(n, size=512, replace=False))
    e = ora.encode(x_np(x[torch.from_numpy(idx).to(DEV)]))
    gi = o.unpack_row(u32(codes[idx]), ora.k, ora.d_pad)
    _, bad = check_codes(gi, e["idx"], e["y"], ora.boundaries, d)
    check_signs(u32(signs[idx]), e["signs"], e["z"], e["rho64"], ora.m, skip_rows=bad)
    sig_bad = (o.unpack_signs(u32(signs[idx]), ora.m) != o.unpack_signs(e["signs"], ora.m)).any(axis=1)
    assert_close_rel(norms[idx].cpu().numpy(), e["norms"], 1e-30, what="norms")
    want = ora.scores(x_np(qs), e["idx"], e["norms"], e["signs"], e["rnorms"])
    floor = e["norms"][None, :] * np.linalg.norm(x_np(qs), axis=1)[:, None] / math.sqrt(d)
    ok = ~(bad | sig_bad)
    assert_close_rel(scores[:, idx].cpu().numpy()[:, ok], want[:, ok], floor[:, ok], what="scores")
    # top-10 of each GPU score row, ties to the lower index
    s = scores.cpu().numpy()
    for r in range(s.shape[0]):
        order = np.lexsort((np.arange(n), -s[r]))[:R["topk"]]
        assert np.array_equal(top_i[r].cpu().numpy(), order)
        assert np.array_equal(top_s[r].cpu().numpy(), s[r, order])


@pytest.mark.parametrize("bits", [2, 4])
def test_retrieval_1024_queries_fused_topk_and_recall(bits):
    # The retrieval workload at its stated size: 1e6 x 1536 unit vectors,
    # 1024 unit queries, top-10 of the unbiased estimator with the fused
    # top-k (no score matrix), and recall@10 against the exact fp32 products.
    R = synth.RETRIEVAL
    d, n = R["d"], R["n"]
    ora, lib = make_pair(d, bits, True, seed=R["seed"], m=R["m"], dense=True)
    x = synth.gaussian_vectors(n, d, seed=R["seed"], device=DEV, n_outliers=R["n_outliers"],
                               outlier_scale=R["outlier_scale"], normalize=True)
    qs = synth.gaussian_vectors(R["n_queries"], d, seed=R["seed"] + 1, device=DEV, normalize=True)
    codes, signs, norms, rnorms = tq.tq_encode_prod(lib, x)
    _, top_s, top_i = tq.tq_scores(lib, qs, codes, signs, norms, rnorms, topk=R["topk"], want_scores=False)
    # the first 64 queries again with their score rows
    sc, ts64, ti64 = tq.tq_scores(lib, qs[:64], codes, signs, norms, rnorms, topk=R["topk"])
    torch.cuda.synchronize()
    tq.tq_sync_check()
    assert np.array_equal(top_i[:64].cpu().numpy(), ti64.cpu().numpy())
    assert np.array_equal(top_s[:64].cpu().numpy(), ts64.cpu().numpy())
    s = sc.cpu().numpy()
    for r in range(0, 64, 9):
        order = np.lexsort((np.arange(n), -s[r]))[:R["topk"]]
        assert np.array_equal(ti64[r].cpu().numpy(), order)
    # sampled scores against the oracle (1e-3 of max(|s|, n |q| / sqrt(d)))
    rng = np.random.default_rng(13)
    idx = np.sort(rng.choice(n, size=256, replace=False))
    e = ora.encode(x_np(x[torch.from_numpy(idx).to(DEV)]))
    gi = o.unpack_row(u32(codes[idx]), ora.k, ora.d_pad)
    _, bad = check_codes(gi, e["idx"], e["y"], ora.boundaries, d)
    sig_bad = (o.unpack_signs(u32(signs[idx]), ora.m) != o.unpack_signs(e["signs"], ora.m)).any(axis=1)
    qn = x_np(qs[:64])
    want = ora.scores(qn, e["idx"], e["norms"], e["signs"], e["rnorms"])
    floor = e["norms"][None, :] * np.linalg.norm(qn, axis=1)[:, None] / math.sqrt(d)
    ok = ~(bad | sig_bad)
    assert_close_rel(s[:, idx][:, ok], want[:, ok], floor[:, ok], what="scores")
    # recall@10 of the estimator's top-10 against the exact fp32 top-10
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    hits = 0
    for a in range(0, qs.shape[0], 128):
        exact = torch.topk(qs[a:a + 128] @ x.T, R["topk"], dim=1).indices
        hits += int((exact.unsqueeze(2) == top_i[a:a + 128].unsqueeze(1)).any(dim=2).sum().item())
    torch.backends.cuda.matmul.allow_tf32 = prev
    recall = hits / (qs.shape[0] * R["topk"])
    print(f"retrieval b={bits}: recall@10 = {recall:.3f} over {qs.shape[0]} queries")
    assert recall > 0.05  # a random top-10 of 1e6 would score ~1e-5

"""The seeded input recipe stated in the design notes: method draws (sign
flips +-1, S rounded to fp16, a Gaussian G for the dense rotation), outlier
channels chosen per group without replacement and scaled, KV caches of the
workload shapes and dtypes, and determinism under the seed."""
import numpy as np
import torch

import synth


def test_method_draws_shapes_and_values():
    dr = synth.method_draws(192, 256, seed=3, stream=1)
    assert dr["d_pad"] == 256 and dr["signs"].shape == (256,) and dr["S"].shape == (256, 256)
    assert set(np.unique(dr["signs"])) == {-1, 1}
    assert np.array_equal(dr["S"], dr["S"].astype(np.float16).astype(np.float32))  # fp16 values
    assert abs(dr["S"].std() - 1.0) < 0.01 and dr["G"] is None
    again = synth.method_draws(192, 256, seed=3, stream=1)
    other = synth.method_draws(192, 256, seed=3, stream=2)
    assert np.array_equal(dr["S"], again["S"]) and not np.array_equal(dr["S"], other["S"])
    dense = synth.method_draws(96, 96, seed=3, dense=True)
    assert dense["d_pad"] == 96 and dense["G"].shape == (96, 96)


def test_outlier_channels_and_scales():
    x = synth.gaussian_vectors(20000, 128, seed=4, n_outliers=8, outlier_scale=10.0).numpy()
    std = x.std(axis=0)
    big = np.sort(np.argsort(std)[-8:])
    _, chans = synth.outlier_plan(4, 1, 128, 8, lognormal=False)
    assert np.array_equal(big, np.sort(chans[0]))  # the planned channels, distinct
    assert np.all(np.abs(std[big] / 10.0 - 1.0) < 0.05)
    assert np.all(np.abs(np.delete(std, big) - 1.0) < 0.05)
    u = synth.gaussian_vectors(64, 1536, seed=4, normalize=True)
    assert torch.allclose(u.norm(dim=1), torch.ones(64), atol=1e-5)


def test_kv_cache_shapes_dtypes_and_determinism():
    cfg = synth.KV_CONFIGS["llama3.1-8b_32k_b3"].scaled(layers=2, batch=1, seq=256)
    K, V = synth.kv_cache(cfg)
    assert K.shape == (2, 1, cfg.kv_heads, 256, 128) and K.dtype == torch.float16
    assert V.shape == K.shape and V.dtype == torch.float16
    K2, _ = synth.kv_cache(cfg)
    assert torch.equal(K, K2)
    q = synth.decode_queries(cfg)
    assert q.shape == (2, 1, cfg.q_heads, 128) and q.dtype == torch.float32
    qwen = synth.KV_CONFIGS["qwen2.5-3b_8k_b3"]
    assert (qwen.layers, qwen.kv_heads, qwen.q_heads, qwen.head_dim, qwen.seq, qwen.dtype) == \
        (36, 2, 16, 128, 8192, "bfloat16")
    long = synth.KV_CONFIGS["longctx-d192_128k_b4"]
    assert (long.head_dim, long.d_pad, long.seq, long.key_bits) == (192, 256, 131072, 4)

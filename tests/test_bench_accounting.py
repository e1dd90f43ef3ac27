"""The algorithmic bytes bench.py divides by (the roofline numerator):
per vector and per token-head at the Llama-3.1-8B cache shape, for the
default storage and its variants, against the sizes counted by hand from
the bit layout (codes k d_pad / 8 bytes, signs m / 8, fp32 or fp16 norms)."""
import bench
import synth


def test_llama_b3_bytes_per_unit():
    cfg = synth.KV_CONFIGS["llama3.1-8b_32k_b3"]
    n = cfg.layers * cfg.batch * cfg.kv_heads * cfg.seq            # token-heads
    nq = cfg.layers * cfg.batch * cfg.q_heads
    # keys: 2-bit codes (8 words) + 128 signs (4 words); values: 3-bit codes (12 words)
    nb = bench.workload_bytes(cfg, 8, 4, 12)
    assert nb["encode_prod"] == n * (256 + 32 + 16 + 8)             # 312 B per fp16 key
    assert nb["encode_mse"] == n * (256 + 48 + 4)                   # 308 B per fp16 value
    assert nb["attention"] == n * (56 + 52) + nq * 128 * 4 * 2      # 108 B per token-head + q, out
    assert nb["encode_prod"] + nb["encode_mse"] + nb["attention"] == 24_431_820_800


def test_storage_variants_bytes():
    cfg = synth.KV_CONFIGS["llama3.1-8b_32k_b3"]
    n = cfg.layers * cfg.batch * cfg.kv_heads * cfg.seq
    # m = 64 (2 sign words) with fp16 residual norms: 32 + 8 + 4 + 2 = 46 B of key row
    nb = bench.workload_bytes(cfg, 8, 2, 12, rnorm_bytes=2)
    assert nb["encode_prod"] == n * (256 + 46)
    nq = cfg.layers * cfg.batch * cfg.q_heads
    assert nb["attention"] == n * (46 + 52) + nq * 128 * 4 * 2


def test_job_throughput_counts_every_rank():
    assert bench.job_throughput(24_431_820_800, 1, 7.5) == 24_431_820_800 / 7.5e-3 / 1e9
    assert bench.job_throughput(10 ** 9, 4, 1.0) == 4000.0


def test_retrieval_accounting():
    # 1e6 x 1536 unit vectors, m = 1536, b = 4 (3 MSE bits): 3 x 48 code words,
    # 48 sign words; 1024 queries
    enc_bytes, enc_flop, sc_flop = bench.retrieval_accounting(10**6, 1536, 1536, 1024, 3 * 48, 48)
    assert enc_bytes == 10**6 * (1536 * 4 + 4 * 192 + 8)   # 6144 in, 776 out per vector
    assert enc_flop == 10**6 * 2 * 1536 * 1536 * 2           # Pi x and S r
    assert sc_flop == 1024 * 10**6 * 2 * 3072


def test_scores_stream_bytes():
    # 40 queries = two 32-query blocks, each streaming the 1e6 rows of codes
    # (48 words), signs (48 words), norm and residual norm once
    b = bench.scores_stream_bytes(10**6, 40, 48, 48, 1536)
    assert b == 2 * 10**6 * (4 * 96 + 8) + 40 * 1536 * 4 + 40 * 10 * 12

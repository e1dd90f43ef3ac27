"""Benchmark: TurboQuant encode + compressed-cache decode attention on B200.

One step = the whole hot path over one synthetic KV cache: Q_prod encode of
every key, Q_MSE encode of every value, then one fused decode-attention step
for every query head (all layers).  The metric is algorithmic bytes moved
(encode: raw K/V in + compressed rows out; attention: compressed rows in +
queries/outputs) per second, and its fraction of the measured HBM copy
bandwidth.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]
                    [--workload llama3.1-8b_32k_b3 | qwen2.5-3b_8k_b3 | longctx-d192_128k_b4]

Multi-GPU (torchrun): every rank processes its own full cache (weak scaling,
no collective on the data path); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

DEFAULT_WORKLOAD = "llama3.1-8b_32k_b3"
METRIC = "encode & compressed decode-attention GB/s (% of B200 HBM peak), d=128 b=3"
UNIT = "GB/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="tq", choices=["tq", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.KV_CONFIGS))
    ap.add_argument("--layers", type=int, default=0, help="use only the first N layers (0 = all)")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-sample-groups", type=int, default=6)
    ap.add_argument("--value-scale", default="norm", choices=["norm", "unbiased"],
                    help="per-vector scale stored with the values: the norm, or EDEN's unbiased scale")
    ap.add_argument("--rnorm-f16", action="store_true", help="store the keys' residual norms as fp16")
    ap.add_argument("--retrieval-queries", type=int, default=0,
                    help="instead of the KV-cache step, time the retrieval set (1e6 x 1536 unit vectors, dense "
                         "rotation): Q_prod encode of the whole set and scores + top-10 for this many queries")
    ap.add_argument("--retrieval-bits", type=int, default=2, choices=[2, 4])
    ap.add_argument("--retrieval-vectors", type=int, default=0,
                    help="size of the retrieval set (0 = the 1e6 of the workload; smaller sets are for profiler "
                         "captures)")
    ap.add_argument("--qjl-rows", type=int, default=0,
                    help="QJL projection rows m of the keys (0 = the padded head dim; d_pad / 2 is the half-size variant)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def workload_bytes(cfg, k_words, k_signs, v_words, rnorm_bytes=4):
    """Algorithmic bytes of one step, split per kernel family."""
    n = cfg.layers * cfg.batch * cfg.kv_heads * cfg.seq
    esz = 2 if cfg.dtype in ("float16", "bfloat16") else 4
    key_row = 4 * (k_words + k_signs) + 4 + rnorm_bytes   # codes + signs + norm + residual norm
    val_row = 4 * v_words + 4               # codes + norm
    nq = cfg.layers * cfg.batch * cfg.q_heads
    return {
        "encode_prod": n * (cfg.head_dim * esz + key_row),
        "encode_mse": n * (cfg.head_dim * esz + val_row),
        "attention": n * (key_row + val_row) + nq * cfg.head_dim * 4 * 2,
        "per_vector": {"encode_prod": cfg.head_dim * esz + key_row,
                       "encode_mse": cfg.head_dim * esz + val_row,
                       "attention_token_head": key_row + val_row},
        "n_vectors": n,
    }


class ClockSampler:
    """SM clock and clock-event reasons sampled through NVML every few ms
    during the timed region (read-only queries); falls back to nvidia-smi.
    Reports the median SM MHz under load, the maximum SM MHz and every
    slowdown reason seen active."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, index, period_s=0.005):
        self.index = index
        self.period = period_s
        self.sm, self.reasons = [], set()
        self.smax = None
        self.stop_evt = threading.Event()
        self.t = None
        self.err = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.smax = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            masks = [(nm, getattr(pynvml, attr)) for nm, attr in self.REASONS]

            def loop():
                while True:
                    try:
                        self.sm.append(float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)))
                        r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                        for nm, mk in masks:
                            if r & mk:
                                self.reasons.add(nm)
                    except Exception as e:  # keep the samples taken so far
                        self.err = str(e)
                        return
                    if self.stop_evt.wait(self.period):
                        return

            self.t = threading.Thread(target=loop, daemon=True)
            self.t.start()
        except Exception as e:
            self.err = f"nvml unavailable: {e}"

    def stop(self):
        if self.t is not None:
            self.stop_evt.set()
            self.t.join(timeout=5)
        out = {"sm_mhz": statistics.median(self.sm) if self.sm else None,
               "sm_max_mhz": self.smax, "reasons": sorted(self.reasons), "samples": len(self.sm)}
        if self.err and not self.sm:
            out["reasons"] = [self.err]
        return out


class OracleSample:
    """A bounded sample of the workload for the float64 oracle: `groups`
    (layer, batch, kv-head) groups of one layer, each fully encoded (keys
    Q_prod, values Q_MSE) and attended by its G query heads."""

    def __init__(self, cfg, groups: int, layer: int = 0, m: int = 0, unbiased: bool = False,
                 rnorm_f16: bool = False):
        import torch

        from oracle import tq_oracle as o

        self.o = o
        self.cfg = cfg
        torch.set_num_threads(max(1, os.cpu_count() or 1))
        self.cores = torch.get_num_threads()
        kd = synth.method_draws(cfg.head_dim, m or cfg.d_pad, cfg.seed, stream=1)
        vd = synth.method_draws(cfg.head_dim, cfg.d_pad, cfg.seed, stream=2)
        self.kq = o.Quantizer(cfg.head_dim, cfg.key_bits, prod=True, draws=kd, rnorm_f16=rnorm_f16)
        self.vq = o.Quantizer(cfg.head_dim, cfg.value_bits, prod=False, draws=vd, unbiased=unbiased)
        one = cfg.scaled(layers=1)
        K, V = synth.kv_cache(one, device="cpu", layers=range(layer, layer + 1))
        q = synth.decode_queries(one, device="cpu", layers=range(layer, layer + 1))
        self.groups = min(groups, cfg.batch * cfg.kv_heads)
        self.K = K.float().numpy().astype(np.float64).reshape(-1, cfg.seq, cfg.head_dim)[: self.groups]
        self.V = V.float().numpy().astype(np.float64).reshape(-1, cfg.seq, cfg.head_dim)[: self.groups]
        self.q = q.numpy().astype(np.float64).reshape(-1, cfg.group, cfg.head_dim)[: self.groups]
        nb = workload_bytes(cfg.scaled(layers=1, batch=1, kv_heads=1, q_heads=cfg.group),
                            self.kq.k * self.kq.d_pad // 32, self.kq.m // 32, self.vq.k * self.vq.d_pad // 32,
                            rnorm_bytes=2 if rnorm_f16 else 4)
        self.bytes = (nb["encode_prod"] + nb["encode_mse"] + nb["attention"]) * self.groups
        self.sample = f"{self.groups} (layer, batch, kv-head) groups x {cfg.seq} tokens of layer {layer}"

    def run(self):
        """Oracle pass over the sample; returns (GB/s, seconds)."""
        o, cfg = self.o, self.cfg
        scale = synth.softmax_scale(cfg.head_dim)
        t0 = time.perf_counter()
        for g in range(self.groups):
            ke = self.kq.encode(self.K[g])
            ve = self.vq.encode(self.V[g], layout="block32")
            o.decode_attention(self.q[g], self.kq, self.vq, ke, ve, scale, cfg.group)
        dt = time.perf_counter() - t0
        return self.bytes / dt / 1e9, dt


def max_over_ranks(value: float, device) -> float:
    """The largest `value` over all ranks (every rank calls this at the same
    point; a single process returns its own)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(step_bytes: int, world: int, ms: float) -> float:
    """Whole-job GB/s: every rank processes step_bytes per step (weak scaling),
    timed by the slowest rank's ms per step."""
    return world * step_bytes / (ms * 1e-3) / 1e9


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    sample = OracleSample(cfg, max(1, args.cpu_sample_groups // 3), m=args.qjl_rows,
                          unbiased=args.value_scale == "unbiased", rnorm_f16=args.rnorm_f16)
    for _ in range(args.warmup):
        sample.run()
    vals, secs = [], []
    for _ in range(args.steps):
        v, dt = sample.run()
        vals.append(v)
        secs.append(dt)
    cores, sample = sample.cores, sample.sample
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000 * statistics.median(secs), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "layers": cfg.layers, "batch": cfg.batch, "kv_heads": cfg.kv_heads,
                   "q_heads": cfg.q_heads, "head_dim": cfg.head_dim, "seq": cfg.seq},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def retrieval_accounting(n, d, m, nq, code_words, sign_words):
    """Algorithmic work of the retrieval line: bytes of the Q_prod encode
    (fp32 rows in; code and sign words, norm and residual norm out), its flop
    (y = Pi x and z = S r: 2 d^2 + 2 m d per vector) and the scores' flop
    (<q', C[idx]> and <S q', signs>: 2 (d + m) per (query, vector) pair)."""
    enc_bytes = n * (d * 4 + 4 * (code_words + sign_words) + 8)
    enc_flop = n * (2 * d * d + 2 * m * d)
    sc_flop = nq * n * 2 * (d + m)
    return enc_bytes, enc_flop, sc_flop


def scores_stream_bytes(n, nq, code_words, sign_words, d):
    """Bytes the scores stream from HBM: every block of 32 queries reads each
    vector's code words, sign words, norm and residual norm once, plus the
    fp32 queries and the top-10 lists out (the query operands stay in L2)."""
    blocks = (nq + 31) // 32
    return blocks * n * (4 * (code_words + sign_words) + 8) + nq * d * 4 + nq * 10 * 12


def run_retrieval(args):
    """Retrieval set timing (one GPU): Q_prod encode of 1e6 x 1536 fp32 unit
    vectors with the dense rotation (y = Pi x and z = S r are dense
    contractions, 2 d^2 + 2 m d flop per vector), then scores for the first
    `--retrieval-queries` queries and their top-10 (2 (d + m) flop per pair).
    Prints one JSON line with both parts."""
    import torch

    import vector_compression_b200 as tq

    R = synth.RETRIEVAL
    n, d, m, bits = args.retrieval_vectors or R["n"], R["d"], R["m"], args.retrieval_bits
    dr = synth.method_draws(d, m, R["seed"], dense=True)
    p = tq.TQParams(d, bits, tq.MODE_PROD, tq.ROT_DENSE, m=m, S=dr["S"], G=dr["G"])
    dev = torch.device("cuda", 0)
    x = synth.gaussian_vectors(n, d, seed=R["seed"], device=dev, n_outliers=R["n_outliers"],
                               outlier_scale=R["outlier_scale"], normalize=True)
    nq = args.retrieval_queries
    q = synth.gaussian_vectors(nq, d, seed=R["seed"] + 1, device=dev, normalize=True)
    out = (torch.empty((n, p.code_words), dtype=torch.int32, device=dev),
           torch.empty((n, p.sign_words), dtype=torch.int32, device=dev),
           torch.empty(n, dtype=torch.float32, device=dev), torch.empty(n, dtype=torch.float32, device=dev))
    stream = torch.cuda.current_stream()

    def timed(fn, reps):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    enc_ms = timed(lambda: tq.tq_encode_prod(p, x, out=out), args.steps)
    # top-10 only: the scores stay on the SM (no nq x n score matrix)
    sc_ms = timed(lambda: tq.tq_scores(p, q, *out, topk=R["topk"], want_scores=False), max(1, args.steps // 5))
    tq.tq_sync_check()
    # recall@10 of the estimator's top-10 against the exact fp32 inner products
    _, _, top_i = tq.tq_scores(p, q, *out, topk=R["topk"], want_scores=False)
    recall = recall_at_k(torch, x, q, top_i, R["topk"])
    enc_bytes, enc_flop, sc_flop = retrieval_accounting(n, d, m, nq, p.code_words, p.sign_words)
    sc_bytes = scores_stream_bytes(n, nq, p.code_words, p.sign_words, d)
    hbm = peaks()[0]
    peak_tf = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))["bf16_tflops"] \
        if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")) else 1590.0
    line = {
        "metric": "retrieval set: Q_prod encode and scores + top-10",
        "workload": f"retrieval {'1e6' if n == 1_000_000 else n} x {d}, dense",
        "bits": bits, "m": m, "queries": nq,
        "encode": {"ms": enc_ms, "GB/s": enc_bytes / (enc_ms * 1e-3) / 1e9,
                   "TFLOP/s": enc_flop / (enc_ms * 1e-3) / 1e12,
                   "frac_of_bf16_peak": enc_flop / (enc_ms * 1e-3) / 1e12 / peak_tf},
        "scores_topk": {"ms": sc_ms, "TFLOP/s": sc_flop / (sc_ms * 1e-3) / 1e12,
                        "frac_of_bf16_peak": sc_flop / (sc_ms * 1e-3) / 1e12 / peak_tf,
                        "pairs_per_s": nq * n / (sc_ms * 1e-3),
                        "GB/s": sc_bytes / (sc_ms * 1e-3) / 1e9,
                        "frac_of_hbm": sc_bytes / (sc_ms * 1e-3) / 1e9 / hbm},
        "recall_at_10": recall,
        "arithmetic": {"encode": "Pi x and S r as tcgen05 fp16 contractions of split operands (hi.lo + lo.hi + "
                                 "hi.hi and lo.S + hi.S, operands split into fp16 hi + lo), fp32 accumulation per "
                                 "128-wide K chunk, chunk sums added in fp32",
                       "scores": "exact integer tcgen05 contractions of the code and sign bits against 24-bit "
                                 "fixed-point q' and S q'; fused per-query top-10"},
        "peak": "measured bf16 tensor figure (algorithmic flop: 2 d^2 + 2 m d per encoded vector, "
                "2 (d + m) per scored pair)",
    }
    print(json.dumps(line), flush=True)


def recall_at_k(torch, x, q, top_i, k, block=128):
    """Mean |top-k of the estimator & top-k of the exact fp32 inner products| / k
    over the queries (exact products by fp32 matmul on the device, TF32 off)."""
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        hits = 0
        for a in range(0, q.shape[0], block):
            exact = torch.topk(q[a:a + block] @ x.T, k, dim=1).indices
            got = top_i[a:a + block]
            hits += int((exact.unsqueeze(2) == got.unsqueeze(1)).any(dim=2).sum().item())
        return hits / (q.shape[0] * k)
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev


def main():
    args = parse()
    if args.retrieval_queries:
        return run_retrieval(args)
    cfg = synth.KV_CONFIGS[args.workload]
    if args.layers:
        cfg = cfg.scaled(layers=min(args.layers, cfg.layers))
    if args.impl == "reference":
        return run_reference(args, cfg)

    import torch
    import torch.distributed as dist

    import vector_compression_b200 as tq

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    m = args.qjl_rows or cfg.d_pad
    kd = synth.method_draws(cfg.head_dim, m, cfg.seed, stream=1)
    vd = synth.method_draws(cfg.head_dim, cfg.d_pad, cfg.seed, stream=2)
    kmode = tq.MODE_PROD | (tq.STORE_RNORM_F16 if args.rnorm_f16 else 0)
    kp = tq.TQParams(cfg.head_dim, cfg.key_bits, kmode, tq.ROT_HADAMARD, m=m,
                     signs=kd["signs"], S=kd["S"])
    vmode = tq.MODE_MSE_UNBIASED if args.value_scale == "unbiased" else tq.MODE_MSE
    vp = tq.TQParams(cfg.head_dim, cfg.value_bits, vmode, tq.ROT_HADAMARD, signs=vd["signs"])
    K, V = synth.kv_cache(cfg, device=dev)
    q = synth.decode_queries(cfg, device=dev)
    seq = cap = cfg.seq
    n = cfg.layers * cfg.batch * cfg.kv_heads * seq
    kc = (torch.empty((n, kp.code_words), dtype=torch.int32, device=dev),
          torch.empty((n, kp.sign_words), dtype=torch.int32, device=dev),
          torch.empty(n, dtype=torch.float32, device=dev),
          torch.empty(n, dtype=getattr(torch, kp.rnorm_dtype), device=dev))
    vcodes = torch.empty((n // 32, vp.k * vp.d_pad), dtype=torch.int32, device=dev)
    vnorms = torch.empty(n, dtype=torch.float32, device=dev)
    out = torch.empty((cfg.layers, cfg.batch, cfg.q_heads, cfg.head_dim), dtype=torch.float32, device=dev)
    ws = torch.empty(tq.tq_decode_attention_workspace_size(kp, vp, cfg.layers, cfg.batch, cfg.q_heads,
                                                           cfg.kv_heads, seq), dtype=torch.uint8, device=dev)
    scale = synth.softmax_scale(cfg.head_dim)
    stream = torch.cuda.current_stream()
    nb = workload_bytes(cfg, kp.code_words, kp.sign_words, vp.k * vp.d_pad // 32,
                        rnorm_bytes=2 if args.rnorm_f16 else 4)

    ev = {k: [] for k in ("encode_prod", "encode_mse", "attention")}

    def step(record):
        if record:
            e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            e[0].record(stream)
        tq.tq_encode_prod(kp, K, seg_len=seq, seg_cap=cap, out=kc)
        if record:
            e[1].record(stream)
        tq.tq_encode_mse(vp, V, layout=tq.LAYOUT_BLOCK32, seg_len=seq, seg_cap=cap, codes=vcodes, norms=vnorms)
        if record:
            e[2].record(stream)
        tq.tq_decode_attention(kp, vp, q, kc, (vcodes, vnorms), seq, cap, scale, out=out, ws=ws)
        if record:
            e[3].record(stream)
            ev["encode_prod"].append((e[0], e[1]))
            ev["encode_mse"].append((e[1], e[2]))
            ev["attention"].append((e[2], e[3]))

    for _ in range(args.warmup):
        step(False)
    tq.tq_sync_check()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    try:
        nvml_index = torch.cuda._get_nvml_device_index(local)  # honours CUDA_VISIBLE_DEVICES
    except Exception:
        nvml_index = local
    clocks = ClockSampler(nvml_index)
    clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for _ in range(args.steps):
        step(True)
    t_end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    ms = max_over_ranks(t_start.elapsed_time(t_end) / args.steps, dev)
    tq.tq_sync_check()

    kern_ms = {k: statistics.mean(a.elapsed_time(b) for a, b in v) for k, v in ev.items()}
    step_bytes = nb["encode_prod"] + nb["encode_mse"] + nb["attention"]
    value = job_throughput(step_bytes, world, ms)
    peak, peak_kind = peaks()
    kernels = {}
    for k in ("encode_prod", "encode_mse", "attention"):
        gbs = nb[k] / (kern_ms[k] * 1e-3) / 1e9
        kernels[k] = {"ms": kern_ms[k], "GB/s": gbs, "frac_of_hbm": gbs / peak,
                      "bytes": nb[k], "share": kern_ms[k] / sum(kern_ms.values())}
    dom = max(kernels, key=lambda k: kernels[k]["ms"])
    traffic_file = os.path.join(ROOT, "profiles", "traffic.json")
    traffic = None
    if os.path.exists(traffic_file):
        tr = json.load(open(traffic_file))
        ent = tr.get(cfg.name, {}).get(dom)
        if ent and ent.get("source_hash") == source_hash():
            traffic = ent["bytes_per_launch"]

    # ---- serving decode step (outside the timed region): append the last
    # token of every (layer, batch, kv-head) at slot seq - 1 and attend
    step_info = decode_step_timing(tq, kp, vp, K, V, q, kc, vcodes, vnorms, out, seq, cap, scale, stream)

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, tq, kp, vp, K, V, q, kc, vcodes, vnorms, out, ws, seq, cap, scale, step_bytes)
    e2e_ms = max_over_ranks(e2e["ms"] if e2e else 0.0, dev)
    if e2e:
        e2e["ms"] = e2e_ms
        e2e["value"] = job_throughput(step_bytes, world, e2e_ms)

    cpu = None
    if rank == 0 and world == 1:
        s = OracleSample(cfg, args.cpu_sample_groups, m=args.qjl_rows, unbiased=args.value_scale == "unbiased",
                         rnorm_f16=args.rnorm_f16)
        v, dt = s.run()
        cpu = {"value": v, "unit": UNIT, "cores": s.cores, "kind": "oracle", "sample": s.sample, "seconds": dt}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": cfg.name, "layers": cfg.layers, "batch": cfg.batch, "kv_heads": cfg.kv_heads,
                       "q_heads": cfg.q_heads, "head_dim": cfg.head_dim, "seq": cfg.seq, "input_dtype": cfg.dtype,
                       "key_bits": cfg.key_bits, "value_bits": cfg.value_bits, "qjl_m": kp.m, "value_scale": args.value_scale,
                       "rnorm_dtype": kp.rnorm_dtype,
                       "rotation": "randomized Hadamard", "l2": "inputs larger than L2 (no flush)",
                       "arithmetic": ARITHMETIC,
                       "bytes_per_step": step_bytes, "parallelism": f"replica x{world}"},
            "roofline": {"bound": "hbm", "kernel": dom, "achieved": kernels[dom]["GB/s"], "peak": peak,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": kernels[dom]["frac_of_hbm"],
                         "traffic": traffic},
            "kernels": kernels,
            "gpu_launches": args.steps * 5,
            "clocks": clk,
            "e2e": None if e2e is None else {"value": e2e["value"], "unit": UNIT,
                                             "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"]},
            "cpu_baseline": cpu,
            "decode_step": step_info,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# What the path computes in, beside the line's "dtype" (the type of the
# stored norms, scores and outputs).
ARITHMETIC = {
    "encode": "fp32; rotation and S r as tcgen05 MMAs (exact +-1 fp16 rotation entries, fp16 S, "
              "residual split fp16 hi + lo), fp32 accumulation",
    "attention": "exact integer tensor-core contractions of code bits against fixed-point operands: "
                 "queries q' and S q' 24-bit per head, softmax weights p ||v|| 16-bit per head and "
                 "384-token sub-chunk; fp32 softmax, norms and folds",
}


def source_hash():
    import hashlib

    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "vector_compression_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def decode_step_timing(tq, kp, vp, K, V, q, kc, vcodes, vnorms, out, seq, cap, scale, stream, reps=10):
    """Latency of tq_decode_step on the full cache: the new token of every
    (layer, batch, kv-head) is the cache's last row, appended at slot seq - 1
    (rewriting it with the same codes), then attention over seq tokens."""
    import torch

    kn = K[:, :, :, seq - 1].contiguous()
    vn = V[:, :, :, seq - 1].contiguous()
    L_, B, Hkv = kn.shape[0], kn.shape[1], kn.shape[2]
    ws = torch.empty(tq.tq_decode_step_workspace_size(kp, vp, L_, B, q.shape[2], Hkv, seq - 1),
                     dtype=torch.uint8, device=q.device)
    for _ in range(3):
        tq.tq_decode_step(kp, vp, q, kn, vn, kc, (vcodes, vnorms), seq - 1, cap, scale, out=out, ws=ws)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        tq.tq_decode_step(kp, vp, q, kn, vn, kc, (vcodes, vnorms), seq - 1, cap, scale, out=out, ws=ws)
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    return {"ms": ms, "tokens_appended": int(L_ * B * Hkv), "context": seq, "launches": 6}


def run_e2e(args, tq, kp, vp, K, V, q, kc, vcodes, vnorms, out, ws, seq, cap, scale, step_bytes):
    """Same step through the public API with host inputs: pinned host K, V and
    queries are copied to the device inside the timed region and the attention
    output is read back."""
    import torch

    stream = torch.cuda.current_stream()
    try:
        Kh = torch.empty(K.shape, dtype=K.dtype, pin_memory=True)
        Vh = torch.empty(V.shape, dtype=V.dtype, pin_memory=True)
    except RuntimeError:
        return None
    Kh.copy_(K)
    Vh.copy_(V)
    qh = q.cpu().pin_memory()
    oh = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    Kd, Vd, qd = torch.empty_like(K), torch.empty_like(V), torch.empty_like(q)

    def step():
        Kd.copy_(Kh, non_blocking=True)
        Vd.copy_(Vh, non_blocking=True)
        qd.copy_(qh, non_blocking=True)
        tq.tq_encode_prod(kp, Kd, seg_len=seq, seg_cap=cap, out=kc)
        tq.tq_encode_mse(vp, Vd, layout=tq.LAYOUT_BLOCK32, seg_len=seq, seg_cap=cap, codes=vcodes, norms=vnorms)
        tq.tq_decode_attention(kp, vp, qd, kc, (vcodes, vnorms), seq, cap, scale, out=out, ws=ws)
        oh.copy_(out, non_blocking=True)

    step()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.e2e_steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / args.e2e_steps
    h2d = Kh.numel() * Kh.element_size() + Vh.numel() * Vh.element_size() + qh.numel() * 4
    d2h = oh.numel() * 4
    del Kd, Vd, Kh, Vh
    return {"ms": ms, "value": step_bytes / (ms * 1e-3) / 1e9, "h2d": h2d, "d2h": d2h}


if __name__ == "__main__":
    main()

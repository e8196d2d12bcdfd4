#!/usr/bin/env python
"""Benchmark of the B200 DSA lightning indexer (one JSON line on rank 0).

Default workload: the DSA indexer prefill layer the metric is quoted on,
batch 1, L = 131072 causal, H_I = 64, d = 128, top-k = 2048, bf16 q / k ~ N(0,1),
w ~ N(0, 1/64).  A step is one whole indexer layer (score -> causal mask ->
exact token top-k set, the library's default unordered output) through the
library's C ABI.  Inputs are larger than L2 (q alone is 2 GiB), so no explicit
flush is needed between steps.  The same run then times, on one GPU, the
metric's other configurations as secondary lines: the 32 x 131072-key e4m3
decode batch (us / query) and MISA, MISA-dagger, HISA and stacked MISA + HISA
at L = 131072 (ms / layer).  Other workloads run alone with --workload.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

N > 1 (torchrun): the layer is partitioned across the ranks (prefill: zigzag
query-row chunks, decode: sequences; sparse_attention_token_dsa_b200.partition)
with no collective on the data path; the reported time of a layer is the max
over ranks (strong scaling: the layer is fixed, the ranks share it).
--impl reference times the CPU oracle (the only reference this method has) on
a bounded sample of rows of the same workload, extrapolated to a full layer.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_attention_token_dsa_b200 import inputs as gen  # noqa: E402

METRIC = "indexer ms/layer @128K prefill; decode µs/query; % of tensor-pipe / HBM peak"

_L128 = 131072
WORKLOADS = {
    "dsa_prefill_1k_int": dict(
        desc="DSA indexer prefill, batch 1, L=1024 causal, H_I=64, d=128, top-k=128, "
             "integer q,k in [-3,3] and w in [-2,2] (bf16 storage, exact)",
        kind="prefill", batch=1, L=1024, H=64, topk=128, fp8=False, seed=1, needles=0,
        integer=True),
    "dsa_prefill_32k": dict(
        desc="DSA indexer prefill, batch 1, L=32768 causal, H_I=64, d=128, top-k=2048, "
             "bf16 q,k ~N(0,1), w ~N(0,1/64), 32 planted needles",
        kind="prefill", batch=1, L=32768, H=64, topk=2048, fp8=False, seed=2, needles=32),
    "dsa_prefill_32k_fp8": dict(
        desc="DSA indexer prefill, batch 1, L=32768 causal, H_I=64, d=128, top-k=2048, "
             "e4m3 q,k with per-token fp32 scales (quantised outside the timed region)",
        kind="prefill", batch=1, L=32768, H=64, topk=2048, fp8=True, seed=2, needles=32),
    "dsa_prefill_8k": dict(
        desc="DSA indexer prefill, batch 1, L=8192 causal, H_I=64, d=128, top-k=2048, bf16 "
             "(small case of the 32K workload, sized for ncu captures)",
        kind="prefill", batch=1, L=8192, H=64, topk=2048, fp8=False, seed=2, needles=8),
    "dsa_prefill_16k": dict(
        desc="DSA indexer prefill, batch 1, L=16384 causal, H_I=64, d=128, top-k=2048, bf16 "
             "(small case of the 128K workload, sized for ncu captures)",
        kind="prefill", batch=1, L=16384, H=64, topk=2048, fp8=False, seed=2, needles=0),
    "misa_dagger_prefill_16k": dict(
        desc="MISA-dagger prefill, batch 1, L=16384 causal, H_I=64, d=128, B=1024, h=8, "
             "k'=8192, top-k=2048, bf16 (small case of the 128K workload, sized for ncu "
             "captures)",
        kind="dagger", batch=1, L=16384, H=64, topk=2048, seed=4, block=1024, h=8,
        k_prime=8192),
    "dsa_decode_128k": dict(
        desc="DSA indexer decode, 32 sequences x 131072 cached keys, one query each, H_I=64, "
             "d=128, e4m3 K with per-token fp32 scale, bf16 q, fp32 w, top-k=2048",
        kind="decode", batch=32, L=131072, H=64, topk=2048, fp8=True, seed=3, needles=0),
    "dsa_decode_32k": dict(
        desc="DSA indexer decode, 32 sequences x 32768 cached keys, one query each, H_I=64, "
             "d=128, e4m3 K with per-token fp32 scale, bf16 q, fp32 w, top-k=2048 (small case "
             "of the 128K decode, sized for ncu captures)",
        kind="decode", batch=32, L=32768, H=64, topk=2048, fp8=True, seed=3, needles=0),
    "misa_prefill_16k": dict(
        desc="MISA prefill, batch 1, L=16384 causal, H_I=64, d=128, B=1024, h=8, top-k=2048, "
             "bf16 (small case of the 128K workload, sized for ncu captures)",
        kind="misa", batch=1, L=16384, H=64, topk=2048, seed=4, block=1024, h=8),
    "hisa_prefill_16k": dict(
        desc="HISA prefill, batch 1, L=16384 causal, H_I=64, d=128, b=64, r=128, top-k=2048, "
             "bf16, clustered keys (small case of the 128K workload, sized for ncu captures)",
        kind="hisa", batch=1, L=16384, H=64, topk=2048, seed=5, hb=64, r=128, h=0,
        block=1024, keys="clusters"),
    "dsa_prefill_128k": dict(
        desc="DSA indexer prefill, batch 1, L=131072 causal, H_I=64, d=128, top-k=2048, "
             "bf16 q,k ~N(0,1), w ~N(0,1/64) (the dense scan MISA and HISA reduce)",
        kind="prefill", batch=1, L=_L128, H=64, topk=2048, fp8=False, seed=4, needles=0),
    "misa_prefill_128k": dict(
        desc="MISA prefill, batch 1, L=131072 causal, H_I=64, d=128, B=1024 mean-pooled "
             "blocks, h=8 routed heads, top-k=2048, bf16 q,k ~N(0,1), w ~N(0,1/64)",
        kind="misa", batch=1, L=_L128, H=64, topk=2048, seed=4, block=1024, h=8),
    "misa_prefill_128k_h32": dict(
        desc="MISA prefill, batch 1, L=131072 causal, H_I=32, d=128, B=1024, h=8, "
             "top-k=2048, bf16 q,k ~N(0,1), w ~N(0,1/32)",
        kind="misa", batch=1, L=_L128, H=32, topk=2048, seed=6, block=1024, h=8),
    "misa_dagger_prefill_128k": dict(
        desc="MISA-dagger prefill, batch 1, L=131072 causal, H_I=64, d=128, B=1024, h=8, "
             "k'=8192 reranked by all heads, top-k=2048, bf16 q,k ~N(0,1)",
        kind="dagger", batch=1, L=_L128, H=64, topk=2048, seed=4, block=1024, h=8,
        k_prime=8192),
    "hisa_prefill_128k": dict(
        desc="HISA prefill, batch 1, L=131072 causal, H_I=64, d=128, b=64 mean-pooled "
             "blocks, r=128 kept (8192 candidates), top-k=2048, bf16, keys from 256 "
             "Gaussian centres in contiguous runs",
        kind="hisa", batch=1, L=_L128, H=64, topk=2048, seed=5, hb=64, r=128, h=0,
        block=1024, keys="clusters"),
    "lisa_prefill_128k": dict(
        desc="Indexer LISA prefill, batch 1, L=131072 causal, H_I=64, d=128, top-k=2048 by "
             "the linear term of the fused query, bf16 q,k ~N(0,1), w ~N(0,1/64)",
        kind="lisa", batch=1, L=_L128, H=64, topk=2048, seed=4, pool=0),
    "lisa_dagger_prefill_128k": dict(
        desc="LISA-dagger prefill, batch 1, L=131072 causal, H_I=64, d=128, pool M=8192 by "
             "the linear term reranked by all heads, top-k=2048, bf16 q,k ~N(0,1)",
        kind="lisa", batch=1, L=_L128, H=64, topk=2048, seed=4, pool=8192),
    "resmisa_prefill_128k": dict(
        desc="ResMiSA prefill, batch 1, L=131072 causal, H_I=64, d=128, shared linear term + "
             "r=7 residual heads routed by block bounds (B=1024), top-k=2048, bf16 q,k ~N(0,1)",
        kind="resmisa", batch=1, L=_L128, H=64, topk=2048, seed=4, block=1024, r=7),
    "dosa_prefill_128k": dict(
        desc="DoSA (exact bound pruning) over the DSA prefill scan, batch 1, L=131072 causal, "
             "H_I=64, d=128, top-k=2048, 1024-token bound blocks, bf16 q,k ~N(0,1), "
             "w ~N(0,1/64) (the headline problem: independent keys, loose bounds)",
        kind="prefill", batch=1, L=_L128, H=64, topk=2048, fp8=False, seed=4, needles=0,
        dosa=True),
    "dsa_locality_prefill_128k": dict(
        desc="DSA indexer prefill, batch 1, L=131072 causal, H_I=64, d=128, top-k=2048, bf16, "
             "keys with locality: 64 Gaussian centres in contiguous runs (mean 8192 tokens) "
             "+ 0.01 N(0,1) noise",
        kind="prefill", batch=1, L=_L128, H=64, topk=2048, fp8=False, seed=7, needles=0,
        keys="locality"),
    "dosa_locality_prefill_128k": dict(
        desc="DoSA (exact bound pruning) over the DSA prefill scan, batch 1, L=131072 causal, "
             "H_I=64, d=128, top-k=2048, 1024-token bound blocks, keys with locality (64 "
             "centres in runs of mean 8192 tokens + 0.01 noise)",
        kind="prefill", batch=1, L=_L128, H=64, topk=2048, fp8=False, seed=7, needles=0,
        keys="locality", dosa=True),
    "hisa_misa_prefill_128k": dict(
        desc="Stacked MISA (B=1024, h=8) + HISA (b=64, r=128) prefill, batch 1, L=131072 "
             "causal, H_I=64, d=128, top-k=2048, bf16, clustered keys",
        kind="hisa", batch=1, L=_L128, H=64, topk=2048, seed=5, hb=64, r=128, h=8,
        block=1024, keys="clusters"),
}
ROUTED = ("misa", "dagger", "hisa", "lisa", "resmisa")

KERNEL_SOURCES = ["common.cuh", "scan.cuh", "select.cuh"]
TRAFFIC_TABLE = os.path.join(ROOT, "profiles", "traffic_scan_kernel.txt")


def kernel_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "sparse_attention_token_dsa_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(workload: str):
    """dram__bytes_read.sum + dram__bytes_write.sum of one scan-kernel launch of
    `workload`, from the table of one-pass ncu captures in profiles/; None
    unless that capture was taken on the present kernel sources (their hash is
    recorded beside each row)."""
    if not os.path.exists(TRAFFIC_TABLE):
        return None
    src = kernel_hash()
    for line in open(TRAFFIC_TABLE):
        f = [x.strip().strip("`") for x in line.strip().strip("|").split("|")]
        if len(f) >= 5 and f[0] == workload and f[4] == src:
            try:
                return int(f[1].replace(",", "")) + int(f[2].replace(",", ""))
            except ValueError:
                return None
    return None


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            d = json.load(fh)
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"],
                    bf16_sustained=d["bf16_tflops_sustained"], src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, src="fallback")


def make_problem(w):
    if w.get("integer"):
        return gen.integer_problem(w["seed"], w["batch"], w["L"], w["L"], w["H"], 128, w["topk"],
                                   dtype=gen.BF16)
    if w["kind"] == "decode":
        p, _ = gen.decode_problem(w["seed"], w["batch"], w["L"], w["H"], 128, w["topk"])
        return p
    if w.get("keys") == "locality":
        return gen.normal_problem(w["seed"], w["batch"], w["L"], w["L"], w["H"], 128, w["topk"],
                                  key_structure="clusters", n_centres=64, mean_run=8192.0,
                                  noise=0.01)
    return gen.normal_problem(w["seed"], w["batch"], w["L"], w["L"], w["H"], 128, w["topk"],
                              n_needles=w.get("needles", 0),
                              key_structure=w.get("keys", "iid"))


def tile_pairs(p):
    """(query row, 128-key tile) pairs of the legal prefixes: what DoSA may skip."""
    return int(((legal_counts(p) + 127) // 128).sum())


def legal_counts(p):
    """|legal| of every query row (closed form for the causal layouts used here)."""
    out = []
    for b in range(p.batch):
        pos = p.pos0(b) + np.arange(p.n_q, dtype=np.int64)
        out.append(np.clip(np.minimum(pos + 1, p.klen(b)), 0, None))
    return np.concatenate(out)


def algorithmic_work(p, w=None):
    """Scored (query, key, head) dot products of the method and their FLOPs (2 d each).

    DSA: H |legal|.  MISA: H M_t + h |legal| (router + routed scan).  MISA-dagger:
    + H min(k', |legal|).  LISA: |legal| (one fused-query dot per key; LISA-dagger
    + H min(M, |legal|)).  ResMiSA: H M_t block bounds + (1 + r) |legal|.  HISA: hh M^b_t + hh min(r b, |legal|) (coarse + rerank;
    the rerank count is an upper bound, exact unless the kept set holds the
    partial boundary block), hh = h when stacked (+ H M_t for its router)."""
    n = legal_counts(p)
    kind = "prefill" if w is None else w["kind"]
    H = p.heads
    if kind in ("prefill", "decode"):
        dots = H * n
    elif kind in ("misa", "dagger"):
        m = (n + w["block"] - 1) // w["block"]
        dots = H * m + w["h"] * n
        if kind == "dagger":
            dots = dots + H * np.minimum(w["k_prime"], n)
    elif kind == "lisa":
        dots = n + (H * np.minimum(w["pool"], n) if w["pool"] else 0)
    elif kind == "resmisa":
        dots = H * ((n + w["block"] - 1) // w["block"]) + (1 + w["r"]) * n
    else:
        hh = w["h"] if w["h"] else H
        mb = (n + w["hb"] - 1) // w["hb"]
        dots = hh * mb + hh * np.minimum(w["r"] * w["hb"], n)
        if w["h"]:
            dots = dots + H * ((n + w["block"] - 1) // w["block"])
    dots = int(dots.sum())
    return int(n.sum()), dots, 2.0 * dots * p.dim


def decode_bytes(p):
    """Algorithmic HBM bytes of one decode scan: every cached key's e4m3 code row
    (d bytes) and fp32 scale, plus the bf16 query and fp32 weights of each row."""
    kbytes = p.batch * p.n_k * (p.dim + 4)
    qbytes = p.batch * p.n_q * p.heads * (p.dim * 2 + 4)
    return kbytes + qbytes


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"dsa_bench_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}",
                 "--query-gpu=index,clocks.sm,clocks.max.sm,power.draw,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return None
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ---------------------------------------------------------------- oracle legs --

def _oracle_inputs(p, w):
    import oracle
    if w.get("fp8") and w["kind"] == "decode":
        kc, ks = oracle.quantize_rows(p.k, gen.BF16)
        return oracle.Inputs(p, k=kc, k_dtype=gen.E4M3, k_scale=ks)
    if w.get("fp8"):
        qc, qs = oracle.quantize_rows(p.q.reshape(p.batch * p.n_q, -1), gen.BF16)
        kc, ks = oracle.quantize_rows(p.k, gen.BF16)
        return oracle.Inputs(p, q=qc.reshape(p.q.shape), k=kc, q_dtype=gen.E4M3,
                             k_dtype=gen.E4M3, q_scale=qs, k_scale=ks)
    return oracle.Inputs(p)


def _oracle_rows(inp, p, w, rows):
    """The oracle's own computation of the workload's method on the listed rows."""
    import oracle
    kind = w["kind"]
    if kind in ("prefill", "decode"):
        oracle.dsa(inp, p.topk, rows)
    elif kind == "misa":
        oracle.misa(inp, p.topk, w["block"], w["h"], rows=rows)
    elif kind == "dagger":
        oracle.misa(inp, p.topk, w["block"], w["h"], k_prime=w["k_prime"], rows=rows)
    elif kind == "lisa":
        oracle.lisa(inp, p.topk, pool_m=w["pool"], rows=rows)
    elif kind == "resmisa":
        oracle.resmisa(inp, p.topk, w["block"], w["r"], rows=rows)
    else:
        oracle.hisa(inp, p.topk, w["hb"], w["r"], route_h=w["h"], route_block=w["block"],
                    rows=rows)


def _sample_rows(p, n, seed):
    """A random sample of rows (uniform over the layer, fixed seed)."""
    total = p.batch * p.n_q
    r = np.random.Generator(np.random.PCG64(seed))
    return r.permutation(total)[: min(n, total)].astype(np.int64)


def cpu_baseline(p, w, seconds=12.0):
    """Oracle on a bounded random sample of rows (about `seconds` of CPU work),
    extrapolated to the whole layer by the causal-pair count."""
    import oracle
    oracle.build()
    inp = _oracle_inputs(p, w)
    legal = legal_counts(p)
    total_pairs = int(legal.sum())
    rows_all = _sample_rows(p, 1 << 16, 11)
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    done, pairs_done, t_used = 0, 0, 0.0
    for i in range(0, len(rows_all), cores):       # one row per core per call
        chunk = rows_all[i:i + cores]
        t0 = time.perf_counter()
        _oracle_rows(inp, p, w, chunk)
        t_used += time.perf_counter() - t0
        done += len(chunk)
        pairs_done += int(legal[chunk].sum())
        if t_used > seconds:
            break
    per_pair = t_used / max(pairs_done, 1)
    return dict(layer_ms=per_pair * total_pairs * 1e3, rows=done, pairs=pairs_done,
                wall_s=t_used, omp=cores)


def unit_of(w):
    return ("µs/query", 1e3 / (w["batch"])) if w["kind"] == "decode" else ("ms/layer", 1.0)


def run_reference(args, w, p):
    """Reference arm: the CPU oracle as it stands, K timed sample steps."""
    import oracle
    oracle.build()
    inp = _oracle_inputs(p, w)
    legal = legal_counts(p)
    total_pairs = int(legal.sum())
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    rows = _sample_rows(p, max(cores, 16), 13)
    unit, scale = unit_of(w)

    def step():
        t0 = time.perf_counter()
        _oracle_rows(inp, p, w, rows)
        dt = time.perf_counter() - t0
        return dt * total_pairs / max(int(legal[rows].sum()), 1) * 1e3   # ms per layer

    for _ in range(args.warmup):
        step()
    vals = [step() for _ in range(args.steps)]
    ms = statistics.mean(vals)
    value = ms * scale
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": unit,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w["desc"]},
            "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
                             "sample": f"{len(rows)} random query rows per step, "
                                       "extrapolated by causal pair count"},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm --

MLA_WORKLOAD = dict(
    desc="Sparse MLA prefill chunk: 4096 query tokens x 128 heads, 2048 selected positions "
         "each (causal, position order) from a 131072-row latent cache, d_qk 576 (512 latent "
         "+ 64 rope), d_v 512, bf16, softmax scale 1/sqrt(192)",
    n_q=4096, n_k=131072, heads=128, topk=2048, seed=5)


def mla_line(steps, warmup, dev):
    """Sparse MLA over fixed selected positions (the indexer's consumer), timed
    with CUDA events; tensor roofline by its algorithmic FLOPs (2 per
    multiply-add over the 576 logit and 512 value dimensions of every selected
    (token, head, position)), and the gathered bytes (each selected row once
    per token)."""
    import torch
    from sparse_attention_token_dsa_b200 import binding as B
    from sparse_attention_token_dsa_b200 import workloads
    w = MLA_WORKLOAD
    pr = workloads.mla_problem(w["n_q"], w["n_k"], w["heads"], w["topk"], seed=w["seed"])
    q = torch.from_numpy(pr["q"].view(np.int16)).to(dev).view(torch.bfloat16)
    kv = torch.from_numpy(pr["kv"].view(np.int16)).to(dev).view(torch.bfloat16)
    idx = torch.from_numpy(pr["idx"]).to(dev)
    out = torch.empty((w["n_q"], w["heads"], 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w["n_q"], w["heads"]), dtype=torch.float32, device=dev)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def call():
        B.sparse_mla(q, kv, idx, pr["scale"], tokens_per_seq=pr["tps"], out=out, out_lse=lse,
                     workspace=ws, stream=stream)

    for _ in range(max(warmup, 3)):
        call()
    st = B.dsa_read_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {st}: {B.status_string(st)}")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    nsel = int((pr["idx"] >= 0).sum())
    flops = 2.0 * w["heads"] * nsel * (576 + 512)
    nbytes = nsel * 576 * 2
    pk = peaks()
    tf = flops / (ms * 1e-3) / 1e12
    return {"workload": w["desc"], "value": ms, "unit": "ms/chunk", "ms_per_step": ms,
            "steps": steps, "warmup": max(warmup, 3),
            "roofline": {"bound": "tensor", "achieved": tf, "peak": pk["bf16"],
                         "unit": "TFLOP/s", "frac": tf / pk["bf16"],
                         "peak_source": f"{pk['src']} bf16 burst",
                         "work": f"{flops / 1e12:.3f} TFLOP per call",
                         "gathered_gb_per_s": nbytes / (ms * 1e-3) / 1e9,
                         "kernel": "sparse_mla_kernel", "kernel_ms": ms, "traffic": None},
            "gpu_launches": steps}


BWD_WORKLOAD = dict(
    desc="Indexer backward with score recompute (sparse stage): L=8192 prefill rows, H_I=64, "
         "d=128, 2048 selected causal positions per row, bf16 q,k ~N(0,1), upstream gradient "
         "N(0,1); dq, dk, dw in fp32",
    n_q=8192, heads=64, topk=2048, seed=7)


def backward_line(steps, warmup, dev):
    """Indexer backward timed with CUDA events; tensor roofline by its algorithmic
    FLOPs: three products (recomputed z, dq, dk) of 2 * 64 * 128 per selected
    (row, position)."""
    import torch
    from sparse_attention_token_dsa_b200 import binding as B
    from sparse_attention_token_dsa_b200 import workloads
    w = BWD_WORKLOAD
    p, sel, grad = workloads.backward_problem(w["n_q"], w["heads"], w["topk"], seed=w["seed"])
    q = torch.from_numpy(p.q.view(np.int16)).to(dev).view(torch.bfloat16)
    k = torch.from_numpy(p.k.view(np.int16)).to(dev).view(torch.bfloat16)
    wt = torch.from_numpy(p.w).to(dev)
    sd = torch.from_numpy(sel).to(dev).view(1, w["n_q"], w["topk"])
    gd = torch.from_numpy(grad).to(dev).view(1, w["n_q"], w["topk"])
    dk = torch.zeros(k.shape, dtype=torch.float32, device=dev)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def call():
        B.indexer_backward(q, k, wt, sd, gd, dk=dk, workspace=ws, stream=stream)

    for _ in range(max(warmup, 3)):
        call()
    st = B.dsa_read_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {st}: {B.status_string(st)}")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    nsel = int((sel >= 0).sum())
    flops = 3 * 2.0 * nsel * w["heads"] * 128
    pk = peaks()
    tf = flops / (ms * 1e-3) / 1e12
    return {"workload": w["desc"], "value": ms, "unit": "ms/layer", "ms_per_step": ms,
            "steps": steps, "warmup": max(warmup, 3),
            "roofline": {"bound": "tensor", "achieved": tf, "peak": pk["bf16"],
                         "unit": "TFLOP/s", "frac": tf / pk["bf16"],
                         "peak_source": f"{pk['src']} bf16 burst",
                         "work": f"{flops / 1e12:.3f} TFLOP per call",
                         "kernel": "indexer_backward_kernel", "kernel_ms": ms, "traffic": None},
            "gpu_launches": steps}


# in an order that reuses generated problems: DoSA, MISA and MISA-dagger share
# the headline problem, stacked HISA shares HISA's clustered keys, DoSA on keys
# with locality follows the unpruned scan of the same problem
SECONDARY = ["dosa_prefill_128k", "misa_prefill_128k", "misa_dagger_prefill_128k",
             "lisa_prefill_128k", "lisa_dagger_prefill_128k", "resmisa_prefill_128k",
             "hisa_prefill_128k", "hisa_misa_prefill_128k", "dsa_locality_prefill_128k",
             "dosa_locality_prefill_128k", "dsa_decode_128k"]


def max_over_ranks(x: float, device=None) -> float:
    """The largest value of x over all ranks (x itself without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _bf16(a):
    import torch
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)


class Case:
    """One workload on this rank: its share of the layer (partition.py) as a list
    of library calls on device-resident inputs, plus the same calls fed from
    pinned host buffers for the end-to-end measurement."""

    def __init__(self, w, p, dev, world, rank):
        import torch
        from sparse_attention_token_dsa_b200 import binding as B
        from sparse_attention_token_dsa_b200 import partition as part
        self.w, self.p, self.dev, self.B = w, p, dev, B
        self.kind = w["kind"]
        self.fp8 = w.get("fp8", False)
        self.stream = torch.cuda.current_stream()
        # this rank's share: (batch start, batch count, row start, row count) pieces
        if self.kind == "decode":
            b0, nb = part.decode_seq_range(p.batch, world, rank)
            self.pieces = [(b0, nb, 0, p.n_q)] if nb else []
        else:
            assert p.batch == 1 or world == 1, "prefill partition is per sequence (batch 1)"
            self.pieces = [(0, p.batch, r0, nr)
                           for r0, nr in part.prefill_row_ranges(p.n_q, world, rank)]
        self.qh, self.kh, self.wh = _bf16(p.q), _bf16(p.k), torch.from_numpy(p.w)
        self.q = self.qh.to(dev)
        self.k = self.kh.to(dev)
        self.wt = self.wh.to(dev)
        self.q_scale = self.k_scale = None
        if self.fp8:
            self.k, self.k_scale = B.dsa_quantize_e4m3(self.k)
            if self.kind == "prefill":
                q2, qs = B.dsa_quantize_e4m3(self.q.reshape(p.batch * p.n_q, -1))
                self.q, self.q_scale = q2.reshape(p.q.shape), qs.reshape(p.batch, p.n_q)
        self.idx = torch.full((p.batch, p.n_q, p.topk), -1, dtype=torch.int32, device=dev)
        self.sc = torch.empty((p.batch, p.n_q, p.topk), dtype=torch.float32, device=dev)
        self.calls = [self._piece(pc) for pc in self.pieces]
        nbytes = max([c["ws_bytes"] for c in self.calls] + [256])
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        self.launches = sum(c["launches"] for c in self.calls)
        torch.cuda.synchronize()

    def _piece(self, pc):
        """Argument views of one library call over rows [r0, r0 + nr) of sequences
        [b0, b0 + nb), with its causal position and key length made explicit."""
        import torch
        B, p, w = self.B, self.p, self.w
        b0, nb, r0, nr = pc
        pos0 = torch.tensor([p.pos0(b) + r0 for b in range(b0, b0 + nb)], dtype=torch.int32,
                            device=self.dev)
        klen = torch.tensor([p.klen(b) for b in range(b0, b0 + nb)], dtype=torch.int32,
                            device=self.dev)

        def view(t, seq_axis_rows=True):
            if t is None:
                return None
            t = t[b0:b0 + nb]
            return t[:, r0:r0 + nr] if seq_axis_rows else t

        c = dict(q=view(self.q), k=view(self.k, False), w=view(self.wt),
                 q_scale=view(self.q_scale), k_scale=view(self.k_scale, False),
                 idx=view(self.idx), sc=view(self.sc), pos0=pos0, klen=klen, rows=(b0, nb, r0, nr))
        for key in ("q", "w", "q_scale", "idx", "sc"):
            if c[key] is not None and not c[key].is_contiguous():
                raise ValueError("partitioned rows must be contiguous (batch 1 prefill)")
        c["prob"] = B.problem(c["q"], c["k"], p.topk, pos0, klen,
                              B.DSA_FLAG_DOSA if w.get("dosa") else 0)
        if self.kind in ROUTED:
            algo = {"misa": B.DSA_ALGO_MISA, "dagger": B.DSA_ALGO_MISA_DAGGER,
                    "hisa": B.DSA_ALGO_HISA, "lisa": B.DSA_ALGO_LISA,
                    "resmisa": B.DSA_ALGO_RESMISA}[self.kind]
            if self.kind == "hisa":
                rp = B.route_params(misa_block=w["block"] if w["h"] else 0, misa_h=w["h"],
                                    hisa_block=w["hb"], hisa_r=w["r"])
            elif self.kind == "lisa":
                rp = B.route_params(lisa_pool=w["pool"])
            elif self.kind == "resmisa":
                rp = B.route_params(res_block=w["block"], res_r=w["r"])
            else:
                rp = B.route_params(misa_block=w["block"], misa_h=w["h"],
                                    k_prime=w.get("k_prime", 0))
            c["ws_bytes"] = B.dsa_workspace_size(c["prob"], algo, rp)
            chunks = -(-nr // B.dsa_route_chunk_rows(c["prob"], algo, rp))
            c["chunks"] = chunks
            if self.kind == "misa":
                c["launches"] = 2 + 2 * chunks
            elif self.kind == "dagger":
                c["launches"] = 2 + 4 * chunks
            elif self.kind == "lisa":
                c["launches"] = 1 + (4 if w["pool"] else 2) * chunks
            elif self.kind == "resmisa":
                c["launches"] = (3 if w["r"] else 1) + 2 * chunks
            else:
                c["launches"] = (2 if w["h"] else 0) + 1 + 5 * chunks
        else:
            c["ws_bytes"] = B.dsa_workspace_size(c["prob"])
            c["launches"] = 2 + (1 if (self.fp8 and self.kind == "decode") else 0)
            if w.get("dosa"):
                c["launches"] += 3                   # key ranges, bounds, seeds
        return c

    def _routed(self, c, q, k, w_, out):
        B, p, w = self.B, self.p, self.w
        if self.kind == "misa":
            B.misa_index(q, k, w_, p.topk, w["block"], w["h"], q_pos0=c["pos0"],
                         k_len=c["klen"], out=out, workspace=self.ws)
        elif self.kind == "dagger":
            B.misa_dagger_index(q, k, w_, p.topk, w["block"], w["h"], w["k_prime"],
                                q_pos0=c["pos0"], k_len=c["klen"], out=out, workspace=self.ws)
        elif self.kind == "lisa":
            B.lisa_index(q, k, w_, p.topk, pool=w["pool"], q_pos0=c["pos0"], k_len=c["klen"],
                         out=out, workspace=self.ws)
        elif self.kind == "resmisa":
            B.resmisa_index(q, k, w_, p.topk, w["block"], w["r"], q_pos0=c["pos0"],
                            k_len=c["klen"], out=out, workspace=self.ws)
        else:
            B.hisa_index(q, k, w_, p.topk, w["hb"], w["r"], route_h=w["h"],
                         route_block=w["block"], q_pos0=c["pos0"], k_len=c["klen"], out=out,
                         workspace=self.ws)

    def step(self, ev=None):
        """One pass over this rank's share.  ev: a list of (start, end) event pairs
        that bracket the scan stage of each DSA call (the whole call when routed)."""
        B = self.B
        for i, c in enumerate(self.calls):
            if ev is not None:
                ev[i][0].record(self.stream)
            if self.kind in ROUTED:
                self._routed(c, c["q"], c["k"], c["w"], (c["idx"], c["sc"]))
                if ev is not None:
                    ev[i][1].record(self.stream)
            else:
                B.dsa_index_scan(c["prob"], c["q"], c["k"], c["w"], self.ws, q_scale=c["q_scale"],
                                 k_scale=c["k_scale"], stream=self.stream)
                if ev is not None:
                    ev[i][1].record(self.stream)
                B.dsa_index_select(c["prob"], c["idx"], c["sc"], self.ws, stream=self.stream)

    def status(self):
        return self.B.dsa_read_status(self.ws)

    # ---- end to end: this rank's inputs copied from pinned host buffers, its
    # outputs copied back, inside the timed region
    def e2e_setup(self):
        import torch
        p = self.p
        self.qp, self.kp, self.wp = (self.qh.pin_memory(), self.kh.pin_memory(),
                                     self.wh.pin_memory())
        self.e2e_bufs = []
        h2d = d2h = 0
        # bf16 prefill: the library's host-buffer call streams the query rows in
        # chunks, its copies overlapping the scan; the others copy whole inputs
        self.streamed = self.kind == "prefill" and not self.fp8
        for c in self.calls:
            b0, nb, r0, nr = c["rows"]
            hq = self.qp[b0:b0 + nb, r0:r0 + nr]
            hw = self.wp[b0:b0 + nb, r0:r0 + nr]
            hk = self.kp[b0:b0 + nb]
            bufs = dict(hq=hq, hw=hw, hk=hk,
                        dk=torch.empty(hk.shape, dtype=hk.dtype, device=self.dev),
                        hi=torch.empty(c["idx"].shape, dtype=torch.int32).pin_memory(),
                        hs=torch.empty(c["sc"].shape, dtype=torch.float32).pin_memory())
            if self.streamed:
                nbytes = self.B.dsa_host_staging_size(c["prob"], HOST_CHUNK_ROWS)
                bufs["stg"] = torch.empty(nbytes, dtype=torch.uint8, device=self.dev)
            else:
                bufs["dq"] = torch.empty(hq.shape, dtype=hq.dtype, device=self.dev)
                bufs["dw"] = torch.empty(hw.shape, dtype=hw.dtype, device=self.dev)
            h2d += sum(t.numel() * t.element_size() for t in (hq, hw, hk))
            d2h += c["idx"].numel() * 4 + c["sc"].numel() * 4
            self.e2e_bufs.append(bufs)
        return h2d, d2h

    def e2e_step(self):
        B, p = self.B, self.p
        for c, b in zip(self.calls, self.e2e_bufs):
            if self.streamed:
                b["dk"].copy_(b["hk"], non_blocking=True)
                B.dsa_index_host(b["hq"], b["dk"], b["hw"], p.topk, q_pos0=c["pos0"],
                                 k_len=c["klen"], flags=c["prob"].flags,
                                 chunk_rows=HOST_CHUNK_ROWS, out=(b["hi"], b["hs"]),
                                 staging=b["stg"], stream=self.stream)
                continue
            b["dq"].copy_(b["hq"], non_blocking=True)
            b["dk"].copy_(b["hk"], non_blocking=True)
            b["dw"].copy_(b["hw"], non_blocking=True)
            out = (c["idx"], c["sc"])
            if self.kind in ROUTED:
                self._routed(c, b["dq"], b["dk"], b["dw"], out)
            else:
                qq, kk, qs_, ks_ = b["dq"], b["dk"], None, None
                if self.fp8:
                    kk, ks_ = B.dsa_quantize_e4m3(b["dk"])
                    if self.kind == "prefill":
                        n = qq.shape[0] * qq.shape[1]
                        q2, qs_ = B.dsa_quantize_e4m3(qq.reshape(n, -1))
                        qq, qs_ = q2.reshape(b["dq"].shape), qs_.reshape(qq.shape[0], qq.shape[1])
                B.dsa_index(qq, kk, b["dw"], p.topk, q_scale=qs_, k_scale=ks_, q_pos0=c["pos0"],
                            k_len=c["klen"], flags=c["prob"].flags, out=out, workspace=self.ws,
                            stream=self.stream)
            b["hi"].copy_(c["idx"], non_blocking=True)
            b["hs"].copy_(c["sc"], non_blocking=True)


# rows per chunk of the streamed end-to-end call (16 chunks at 128K)
HOST_CHUNK_ROWS = 8192


def timed(case, steps, warmup, world, dev, sample_clocks=False, local=0):
    """W untimed steps, then K steps between barriers and device syncs, CUDA
    events on the launching stream.  Returns (ms per layer max over ranks,
    kernel ms per layer of this rank, clock summary)."""
    import torch
    import torch.distributed as dist
    for _ in range(max(warmup, 3)):
        case.step()
    st = case.status()
    if st != 0:
        raise RuntimeError(f"device status {st}: {case.B.status_string(st)}")
    torch.cuda.synchronize()
    n = len(case.calls)
    stage_ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(n)] for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk = ClockSampler(local) if sample_clocks else None
    if clk:
        clk.__enter__()
    try:
        t0.record(case.stream)
        for i in range(steps):
            case.step(stage_ev[i])
        t1.record(case.stream)
        torch.cuda.synchronize()
    finally:
        if clk:
            clk.__exit__(None, None, None)
    if world > 1:
        dist.barrier()
    st = case.status()
    if st != 0:
        raise RuntimeError(f"device status {st}: {case.B.status_string(st)}")
    elapsed = max_over_ranks(t0.elapsed_time(t1), dev)
    kernel_ms = (sum(a.elapsed_time(b) for evs in stage_ev for a, b in evs) / steps
                 if n else 0.0)
    return elapsed / steps, kernel_ms, (clk.summary() if clk else None)


def e2e_ms(case, steps, world, dev):
    import torch
    import torch.distributed as dist
    h2d, d2h = case.e2e_setup()
    case.e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(case.stream)
    for _ in range(steps):
        case.e2e_step()
    e1.record(case.stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    return max_over_ranks(e0.elapsed_time(e1) / steps, dev), h2d, d2h


def roofline(case, name, ms_per_step, kernel_ms, long_region):
    """Roofline of the dominant kernel: the scan (DSA prefill: tensor; decode: HBM)
    or, for routed methods, the whole call (all its launches) as a lower bound."""
    p, w, kind = case.p, case.w, case.kind
    pk = peaks()
    pairs, dots, flops = algorithmic_work(p, w)
    bf16_peak = pk["bf16_sustained"] if long_region else pk["bf16"]
    burst = "sustained" if long_region else "burst"
    if kind == "decode":
        nbytes = decode_bytes(p)
        gbs = nbytes / (kernel_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": gbs, "peak": pk["hbm"], "unit": "GB/s",
                "frac": gbs / pk["hbm"], "peak_source": f"{pk['src']} copy bandwidth",
                "work": f"{nbytes / 1e6:.1f} MB per launch (e4m3 K + scales + q + w)",
                "kernel": "scan_kernel", "kernel_ms": kernel_ms}
    elif kind == "prefill":
        tf = flops / (kernel_ms * 1e-3) / 1e12
        peak = 2.0 * bf16_peak if case.fp8 else bf16_peak
        roof = {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s",
                "frac": tf / peak,
                "peak_source": f"{pk['src']} bf16 {burst}"
                               + (" x2 (fp8 nominal ratio)" if case.fp8 else ""),
                "work": f"{flops / 1e12:.3f} TFLOP per launch (2*pairs*H*d)",
                "kernel": "scan_kernel", "kernel_ms": kernel_ms}
    else:
        tf = flops / (kernel_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": tf, "peak": bf16_peak, "unit": "TFLOP/s",
                "frac": tf / bf16_peak, "peak_source": f"{pk['src']} bf16 {burst}",
                "work": f"{flops / 1e12:.3f} TFLOP per call ({dots} scored "
                        "query-key-head dots x 2d, router and rerank included)",
                "kernel": f"whole {kind} call ({case.launches} launches: pooling, router, "
                          "scans, selects)", "kernel_ms": kernel_ms}
    roof["traffic"] = measured_traffic(name) if kind in ("prefill", "decode") else None
    return roof, dots


def iou_rows(a_idx, b_idx, rows):
    """Mean IoU of two top-k index sets over the listed rows (on the GPU)."""
    import torch
    topk = a_idx.shape[-1]
    a_ = a_idx.reshape(-1, topk)[rows].sort(dim=1).values
    b_ = b_idx.reshape(-1, topk)[rows].sort(dim=1).values
    inter = torch.zeros(len(rows), device=a_.device)
    for j in range(0, topk, 256):          # |A ∩ B| by membership of A's entries
        blk = a_[:, j:j + 256]
        pos = torch.searchsorted(b_, blk).clamp(max=topk - 1)
        inter += ((torch.gather(b_, 1, pos) == blk) & (blk >= 0)).sum(1).float()
    nv = (a_ >= 0).sum(1).float()
    return (inter / (2 * nv - inter)).mean().item()


def dense_reference(case):
    """The exact DSA top-k of the same problem (GPU) and its time, for a routed
    method's overlap and speed-up."""
    import torch
    B, p = case.B, case.p
    prob = B.problem(case.q, case.k, p.topk)
    dws = torch.empty(B.dsa_workspace_size(prob), dtype=torch.uint8, device=case.dev)
    didx = torch.empty_like(case.idx)
    dsc = torch.empty_like(case.sc)
    B.dsa_index(case.q, case.k, case.wt, p.topk, out=(didx, dsc), workspace=dws)
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0.record(case.stream)
    B.dsa_index(case.q, case.k, case.wt, p.topk, out=(didx, dsc), workspace=dws)
    d1.record(case.stream)
    torch.cuda.synchronize()
    del dws
    return didx, d0.elapsed_time(d1)


def cutoff_margin(case):
    """Top-k cut-off margin m = I_(k) - I_(k+1) per row ("PaperTrace 2.2.2",
    section 2.3: a score error E leaves the selected set unchanged while
    2E < m), from one sorted top-(k+1) call of the same layer outside the timed
    region.  Quantiles of m and of m / |I_(k)| over the rows with more than k
    legal keys, and the rows whose k-th and (k+1)-th scores tie exactly."""
    import torch
    B, p = case.B, case.p
    c = case.calls[0]
    kk = p.topk + 1
    prob = B.problem(c["q"], c["k"], kk, c["pos0"], c["klen"], B.DSA_FLAG_SORTED)
    ws = torch.empty(B.dsa_workspace_size(prob), dtype=torch.uint8, device=case.dev)
    _, sc = B.dsa_index(c["q"], c["k"], c["w"], kk, q_scale=c["q_scale"], k_scale=c["k_scale"],
                        q_pos0=c["pos0"], k_len=c["klen"], flags=B.DSA_FLAG_SORTED, workspace=ws)
    torch.cuda.synchronize()
    del ws
    sc = sc.reshape(-1, kk)
    full = torch.isfinite(sc[:, kk - 1])
    sk, sk1 = sc[full, kk - 2].double(), sc[full, kk - 1].double()
    m = sk - sk1
    rel = m / sk.abs().clamp_min(1e-30)
    qs = torch.tensor([0.01, 0.1, 0.5, 0.9], dtype=torch.float64, device=m.device)
    out = {"rows": int(full.sum().item()), "exact_ties": int((m == 0).sum().item()),
           "quantiles": [0.01, 0.1, 0.5, 0.9],
           "m": [float(x) for x in torch.quantile(m, qs).tolist()],
           "m_over_kth": [float(x) for x in torch.quantile(rel, qs).tolist()]} if m.numel() else {}
    del sc
    torch.cuda.empty_cache()
    return out


def quality(case, name, ms_per_step, dense=None):
    """Selection quality outside every timed region: needle recall at the probe
    rows; for routed methods the IoU with the exact DSA top-k of the same rows
    (both on the GPU) and the speed-up over that dense layer; for the dense
    layers the top-k cut-off margin."""
    import torch
    p = case.p
    out = {}
    if case.kind in ("prefill", "decode") and not case.w.get("dosa") and len(case.calls) == 1:
        out["cutoff_margin"] = cutoff_margin(case)
    gi = case.idx.reshape(p.batch * p.n_q, p.topk)
    if p.needles:
        found = 0
        for b, t, s_ in zip(p.needles["b"], p.needles["t"], p.needles["s"]):
            found += int((gi[b * p.n_q + t] == s_).any().item())
        out["needle_recall"] = found / len(p.needles["s"])
    if case.kind in ROUTED or case.w.get("dosa"):
        didx, dense_ms = dense if dense is not None else dense_reference(case)
        rows = torch.linspace(p.n_q // 16, p.n_q - 1, 512).long().to(case.dev)
        out.update({"iou_vs_dsa": iou_rows(case.idx, didx, rows), "dsa_ms": dense_ms,
                    "speedup_vs_dsa": dense_ms / ms_per_step})
    if case.w.get("dosa"):
        # exactness at full size: every row's set equals the unpruned scan's
        a_ = case.idx.reshape(-1, p.topk).sort(dim=1).values
        b_ = didx.reshape(-1, p.topk).sort(dim=1).values
        out["identical_to_dsa"] = bool(torch.equal(a_, b_))
        del a_, b_
        pruned = case.B.dsa_read_pruned(case.ws)
        out["dosa_pruned_pairs"] = pruned
        out["dosa_pruned_frac"] = pruned / tile_pairs(p)
    return out


def secondary_line(name, steps, warmup, dev, cache):
    """A secondary configuration timed in the same run (one GPU)."""
    import torch
    w = WORKLOADS[name]
    key = (w["seed"], w["L"], w["H"], w.get("keys", "iid"), w["kind"] == "decode")
    if key not in cache:
        cache.clear()
        torch.cuda.empty_cache()
        cache[key] = make_problem(w)
    p = cache[key]
    case = Case(w, p, dev, 1, 0)
    ms, kms, _ = timed(case, steps, warmup, 1, dev)
    unit, scale = unit_of(w)
    roof, dots = roofline(case, name, ms, kms, ms * steps > 1000.0)
    dense = cache.get(("dense",) + key)
    if (case.kind in ROUTED or w.get("dosa")) and dense is None:
        dense = dense_reference(case)
        cache[("dense",) + key] = dense
    q = quality(case, name, ms, dense)
    if case.kind == "prefill" and not case.fp8 and not w.get("dosa"):
        cache[("dense",) + key] = (case.idx.clone(), ms)   # exact DSA of this problem
    line = {"workload": w["desc"], "value": ms * scale, "unit": unit, "ms_per_step": ms,
            "steps": steps, "warmup": max(warmup, 3), "roofline": roof,
            "scored_dots_per_s": dots / (ms * 1e-3), "gpu_launches": steps * case.launches}
    if case.kind == "decode":
        line["select_ms"] = ms - kms
    else:
        line["row_chunks"] = sum(c.get("chunks", 1) for c in case.calls)
    line.update(q)
    del case
    torch.cuda.empty_cache()
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="dsa_prefill_128k", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="time only --workload (no secondary configurations)")
    args = ap.parse_args()
    w = WORKLOADS[args.workload]
    kind = w["kind"]

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            run_reference(args, w, make_problem(w))
        return

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)

    p = make_problem(w)
    case = Case(w, p, dev, world, rank)
    ms_per_step, kernel_ms, clocks = timed(case, args.steps, args.warmup, world, dev,
                                           sample_clocks=True, local=local)
    e2e_steps = max(3, min(args.steps, 10))
    e2e, h2d, d2h = e2e_ms(case, e2e_steps, world, dev)
    # every rank's own kernel share is timed; the slowest rank sets the roofline
    kernel_ms = max_over_ranks(kernel_ms, dev)
    launches = case.launches * args.steps
    qual = quality(case, args.workload, ms_per_step) if (rank == 0 and world == 1) else {}

    line = None
    if rank == 0:
        unit, scale = unit_of(w)
        roof, dots = roofline(case, args.workload, ms_per_step, kernel_ms,
                              ms_per_step * args.steps > 1000.0)
        par = (f"{world} ranks, one layer partitioned by "
               + ("sequences" if kind == "decode" else "zigzag query-row chunks")
               + ", no data-path collective") if world > 1 else "single GPU"
        cfg = {"workload": w["desc"], "l2": "inputs larger than L2 (no flush)",
               "parallelism": par, "scored_dots_per_s": dots / (ms_per_step * 1e-3)}
        if kind in ("prefill", "decode"):
            cfg["select_ms"] = ms_per_step - kernel_ms
        else:
            cfg["row_chunks"] = sum(c.get("chunks", 1) for c in case.calls)
        cfg.update(qual)
        line = {"metric": METRIC, "value": ms_per_step * scale, "unit": unit, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
                "higher_is_better": False, "scaling": "strong" if world > 1 else "weak",
                "vs_baseline": None, "dtype": "e4m3/f32" if case.fp8 else "bf16/f32",
                "data": "synthetic", "config": cfg, "roofline": roof,
                "e2e": {"value": e2e * scale, "unit": unit, "h2d_bytes_per_step": h2d,
                        "d2h_bytes_per_step": d2h,
                        "call": (f"dsa_index_host, rows streamed in {HOST_CHUNK_ROWS}-row chunks "
                                 "with the copies overlapping the scan") if case.streamed
                                else "whole-input copies, then the library call"},
                "gpu_launches": launches, "clocks": clocks}
    dense = None
    if world == 1 and case.kind == "prefill" and not case.fp8:
        dense = (case.idx.clone(), ms_per_step)     # exact DSA of this problem
    del case
    torch.cuda.empty_cache()

    if world == 1 and rank == 0:
        if not args.no_secondary and args.workload == "dsa_prefill_128k":
            cache = {(w["seed"], w["L"], w["H"], w.get("keys", "iid"), False): p}
            if dense is not None:
                cache[("dense", w["seed"], w["L"], w["H"], w.get("keys", "iid"), False)] = dense
            line["secondary"] = [secondary_line(n, min(args.steps, 5), args.warmup, dev, cache)
                                 for n in SECONDARY]
            cache.clear()
            torch.cuda.empty_cache()
            line["secondary"].append(mla_line(min(args.steps, 5), args.warmup, dev))
            line["secondary"].append(backward_line(min(args.steps, 5), args.warmup, dev))
            line["gpu_launches"] += sum(s["gpu_launches"] for s in line["secondary"])
            cache.clear()
        if not args.no_cpu_baseline:
            cb = cpu_baseline(p, w)
            unit, scale = unit_of(w)
            line["cpu_baseline"] = {"value": cb["layer_ms"] * scale, "unit": unit,
                                    "cores": cb["omp"], "kind": "oracle",
                                    "sample": f"{cb['rows']} random query rows "
                                              f"({cb['pairs']} causal pairs, {cb['wall_s']:.1f} s"
                                              "), extrapolated by causal pair count"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

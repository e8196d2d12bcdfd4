#!/usr/bin/env python
"""Benchmark of the B200 DSA lightning indexer (one JSON line on rank 0).

Default workload: DSA indexer prefill, batch 1, L = 32768 causal, H_I = 64,
d = 128, top-k = 2048, bf16 q / k ~ N(0,1), w ~ N(0, 1/64), 32 planted needles.
A step is one whole indexer layer (score -> causal mask -> exact token top-k
set, the library's default unordered output) through the library's C ABI.
Inputs are larger than L2 (q alone is 512 MiB), so no explicit flush is needed
between steps.  Other workloads: the 32K fp8 variant, the 128K-key decode
batch, and at L = 131072 the DSA layer, MISA, MISA-dagger, HISA and stacked
MISA + HISA (--workload).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

N > 1 (torchrun): every rank runs its own independent layer (weak scaling, no
collective on the data path); the reported time is the max over ranks.
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
    "dsa_decode_128k": dict(
        desc="DSA indexer decode, 32 sequences x 131072 cached keys, one query each, H_I=64, "
             "d=128, e4m3 K with per-token fp32 scale, bf16 q, fp32 w, top-k=2048",
        kind="decode", batch=32, L=131072, H=64, topk=2048, fp8=True, seed=3, needles=0),
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
    "hisa_misa_prefill_128k": dict(
        desc="Stacked MISA (B=1024, h=8) + HISA (b=64, r=128) prefill, batch 1, L=131072 "
             "causal, H_I=64, d=128, top-k=2048, bf16, clustered keys",
        kind="hisa", batch=1, L=_L128, H=64, topk=2048, seed=5, hb=64, r=128, h=8,
        block=1024, keys="clusters"),
}
ROUTED = ("misa", "dagger", "hisa")

# dram__bytes_read.sum + dram__bytes_write.sum of one scan-kernel launch, from the
# ncu captures summarised under profiles/, valid only while the kernel sources
# hash to `src`; otherwise the traffic is reported as null.
TRAFFIC = {
    # profiles/scan_kernel_dsa_prefill_32k.md: 601.29 MB read + 1.91 GB written
    "dsa_prefill_32k": {"bytes": 601_290_000 + 1_910_000_000, "src": "23b61bde9a857492"},
    # profiles/scan_kernel_dsa_decode_128k.md: 559.32 MB read + 26.36 MB written
    "dsa_decode_128k": {"bytes": 559_320_000 + 26_360_000, "src": "23b61bde9a857492"},
}

KERNEL_SOURCES = ["common.cuh", "scan.cuh", "select.cuh"]


def kernel_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "sparse_attention_token_dsa_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


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
    return gen.normal_problem(w["seed"], w["batch"], w["L"], w["L"], w["H"], 128, w["topk"],
                              n_needles=w.get("needles", 0),
                              key_structure=w.get("keys", "iid"))


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
    + H min(k', |legal|).  HISA: hh M^b_t + hh min(r b, |legal|) (coarse + rerank;
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
        self.path = os.path.join(ROOT, "gpurun_out", f"clocks_{os.getpid()}.csv")

    def __enter__(self):
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
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

def max_over_ranks(x: float, device=None) -> float:
    """The largest value of x over all ranks (x itself without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="dsa_prefill_32k", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
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
    from sparse_attention_token_dsa_b200 import binding as B

    p = make_problem(w)
    dev = torch.device("cuda", local)
    fp8 = w.get("fp8", False)

    qh = torch.from_numpy(p.q.view(np.int16)).view(torch.bfloat16)
    kh = torch.from_numpy(p.k.view(np.int16)).view(torch.bfloat16)
    wh = torch.from_numpy(p.w)
    q, k, wt = qh.to(dev), kh.to(dev), wh.to(dev)
    q_scale = k_scale = None
    if fp8:
        k, k_scale = B.dsa_quantize_e4m3(k)
        if kind == "prefill":
            q2, q_scale = B.dsa_quantize_e4m3(q.reshape(p.batch * p.n_q, -1))
            q = q2.reshape(p.q.shape)
            q_scale = q_scale.reshape(p.batch, p.n_q)
    torch.cuda.synchronize()
    prob = B.problem(q, k, p.topk)
    idx = torch.empty((p.batch, p.n_q, p.topk), dtype=torch.int32, device=dev)
    sc = torch.empty((p.batch, p.n_q, p.topk), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    if kind in ROUTED:
        algo = {"misa": B.DSA_ALGO_MISA, "dagger": B.DSA_ALGO_MISA_DAGGER,
                "hisa": B.DSA_ALGO_HISA}[kind]
        if kind == "hisa":
            rp = B.route_params(misa_block=w["block"] if w["h"] else 0, misa_h=w["h"],
                                hisa_block=w["hb"], hisa_r=w["r"])
        else:
            rp = B.route_params(misa_block=w["block"], misa_h=w["h"],
                                k_prime=w.get("k_prime", 0))
        ws = torch.empty(B.dsa_workspace_size(prob, algo, rp), dtype=torch.uint8, device=dev)
        chunks = -(-p.n_q // B.dsa_route_chunk_rows(prob, algo, rp))
        if kind == "misa":
            per_call = 2 + 2 * chunks
        elif kind == "dagger":
            per_call = 2 + 4 * chunks
        else:
            per_call = (2 if w["h"] else 0) + 1 + 5 * chunks

        def call(qq, kk, ww):
            if kind == "misa":
                B.misa_index(qq, kk, ww, p.topk, w["block"], w["h"], out=(idx, sc), workspace=ws)
            elif kind == "dagger":
                B.misa_dagger_index(qq, kk, ww, p.topk, w["block"], w["h"], w["k_prime"],
                                    out=(idx, sc), workspace=ws)
            else:
                B.hisa_index(qq, kk, ww, p.topk, w["hb"], w["r"], route_h=w["h"],
                             route_block=w["block"], out=(idx, sc), workspace=ws)

        def step(ev=None):
            if ev is not None:
                ev[0].record(stream)
            call(q, k, wt)
            if ev is not None:
                ev[1].record(stream)
    else:
        ws = torch.empty(B.dsa_workspace_size(prob), dtype=torch.uint8, device=dev)
        per_call = 2 + (1 if (fp8 and kind == "decode") else 0)

        def step(ev=None):
            if ev is not None:
                ev[0].record(stream)
            B.dsa_index_scan(prob, q, k, wt, ws, q_scale=q_scale, k_scale=k_scale, stream=stream)
            if ev is not None:
                ev[1].record(stream)
            B.dsa_index_select(prob, idx, sc, ws, stream=stream)

    for _ in range(max(args.warmup, 3)):
        step()
    st = B.dsa_read_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {st}: {B.status_string(st)}")
    torch.cuda.synchronize()

    stage_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t0.record(stream)
        for i in range(args.steps):
            step(stage_ev[i])
        t1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    elapsed = t0.elapsed_time(t1)
    stage_ms = statistics.mean(a.elapsed_time(b) for a, b in stage_ev)
    st = B.dsa_read_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {st}: {B.status_string(st)}")
    elapsed = max_over_ranks(elapsed, dev)

    # end to end through the public call with host buffers (pinned), copies inside
    qp, kp, wp = qh.pin_memory(), kh.pin_memory(), wh.pin_memory()
    idx_h = torch.empty(idx.shape, dtype=torch.int32).pin_memory()
    sc_h = torch.empty(sc.shape, dtype=torch.float32).pin_memory()
    q_d = torch.empty_like(qh, device=dev)
    k_d = torch.empty_like(kh, device=dev)
    w_d = torch.empty_like(wh, device=dev)

    def e2e_step():
        q_d.copy_(qp, non_blocking=True)
        k_d.copy_(kp, non_blocking=True)
        w_d.copy_(wp, non_blocking=True)
        if kind in ROUTED:
            call(q_d, k_d, w_d)
        else:
            qq, kk, qs_, ks_ = q_d, k_d, None, None
            if fp8:
                kk, ks_ = B.dsa_quantize_e4m3(k_d)
                if kind == "prefill":
                    q2, qs_ = B.dsa_quantize_e4m3(q_d.reshape(p.batch * p.n_q, -1))
                    qq, qs_ = q2.reshape(p.q.shape), qs_.reshape(p.batch, p.n_q)
            B.dsa_index(qq, kk, w_d, p.topk, q_scale=qs_, k_scale=ks_, out=(idx, sc), workspace=ws)
        idx_h.copy_(idx, non_blocking=True)
        sc_h.copy_(sc, non_blocking=True)

    e2e_steps = max(3, min(args.steps, 10))
    e2e_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, dev)
    h2d = qh.numel() * qh.element_size() + kh.numel() * kh.element_size() + wh.numel() * 4
    d2h = idx.numel() * 4 + sc.numel() * 4

    # quality of the selection (outside every timed region): needle recall at the
    # probe rows; for routed methods the overlap with the exact DSA top-k of the
    # same rows (both on the GPU) and the dense layer's time for the speed-up
    quality = {}
    if rank == 0:
        gi = idx.reshape(p.batch * p.n_q, p.topk)
        if p.needles:
            found = 0
            for b, t, s_ in zip(p.needles["b"], p.needles["t"], p.needles["s"]):
                found += int((gi[b * p.n_q + t] == s_).any().item())
            quality["needle_recall"] = found / len(p.needles["s"])
        if kind in ROUTED:
            dprob = B.problem(q, k, p.topk)
            dws = torch.empty(B.dsa_workspace_size(dprob), dtype=torch.uint8, device=dev)
            didx = torch.empty_like(idx)
            dsc = torch.empty_like(sc)
            B.dsa_index(q, k, wt, p.topk, out=(didx, dsc), workspace=dws)
            d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            d0.record(stream)
            B.dsa_index(q, k, wt, p.topk, out=(didx, dsc), workspace=dws)
            d1.record(stream)
            torch.cuda.synchronize()
            dense_ms = d0.elapsed_time(d1)
            rows = torch.linspace(p.n_q // 16, p.n_q - 1, 512).long().to(dev)
            a_ = gi[rows].sort(dim=1).values
            b_ = didx.reshape(-1, p.topk)[rows].sort(dim=1).values
            inter = torch.zeros(len(rows), device=dev)
            for j in range(0, p.topk, 256):          # |A ∩ B| by membership of A's entries
                blk = a_[:, j:j + 256]
                pos = torch.searchsorted(b_, blk).clamp(max=p.topk - 1)
                inter += ((torch.gather(b_, 1, pos) == blk) & (blk >= 0)).sum(1).float()
            nv = (a_ >= 0).sum(1).float()
            iou = (inter / (2 * nv - inter)).mean().item()
            quality.update({"iou_vs_dsa": iou, "dsa_ms": dense_ms,
                            "speedup_vs_dsa": dense_ms / (elapsed / args.steps)})
            del dws

    if rank == 0:
        unit, scale = unit_of(w)
        ms_per_step = elapsed / args.steps
        value = ms_per_step / world * scale
        pk = peaks()
        pairs, dots, flops = algorithmic_work(p, w)
        long_region = elapsed > 1000.0
        bf16_peak = pk["bf16_sustained"] if long_region else pk["bf16"]
        burst = "sustained" if long_region else "burst"
        if kind == "decode":
            nbytes = decode_bytes(p)
            gbs = nbytes / (stage_ms * 1e-3) / 1e9
            roof = {"bound": "hbm", "achieved": gbs, "peak": pk["hbm"], "unit": "GB/s",
                    "frac": gbs / pk["hbm"], "peak_source": f"{pk['src']} copy bandwidth",
                    "work": f"{nbytes / 1e6:.1f} MB per launch (e4m3 K + scales + q + w)",
                    "kernel": "scan_kernel", "kernel_ms": stage_ms}
        elif kind == "prefill":
            tf = flops / (stage_ms * 1e-3) / 1e12
            peak = 2.0 * bf16_peak if fp8 else bf16_peak
            roof = {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s",
                    "frac": tf / peak,
                    "peak_source": f"{pk['src']} bf16 {burst}"
                                   + (" x2 (fp8 nominal ratio)" if fp8 else ""),
                    "work": f"{flops / 1e12:.3f} TFLOP per launch (2*pairs*H*d)",
                    "kernel": "scan_kernel", "kernel_ms": stage_ms}
        else:
            tf = flops / (stage_ms * 1e-3) / 1e12
            roof = {"bound": "tensor", "achieved": tf, "peak": bf16_peak, "unit": "TFLOP/s",
                    "frac": tf / bf16_peak, "peak_source": f"{pk['src']} bf16 {burst}",
                    "work": f"{flops / 1e12:.3f} TFLOP per call ({dots} scored "
                            "query-key-head dots x 2d, router and rerank included)",
                    "kernel": f"whole {kind} call ({per_call} launches: pooling, router, "
                              "scans, selects)", "kernel_ms": stage_ms}
        tr = TRAFFIC.get(args.workload)
        roof["traffic"] = tr["bytes"] if tr and tr["src"] == kernel_hash() else None
        cfg = {"workload": w["desc"], "l2": "inputs larger than L2 (no flush)",
               "parallelism": f"replicas x{world}",
               "scored_dots_per_s": dots / (ms_per_step * 1e-3)}
        if kind in ("prefill", "decode"):
            cfg["select_ms"] = ms_per_step - stage_ms
        else:
            cfg["row_chunks"] = chunks
        cfg.update(quality)
        line = {"metric": METRIC, "value": value, "unit": unit, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
                "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
                "dtype": "e4m3/f32" if fp8 else "bf16/f32", "data": "synthetic",
                "config": cfg,
                "roofline": roof,
                "e2e": {"value": e2e_ms / world * scale, "unit": unit, "h2d_bytes_per_step": h2d,
                        "d2h_bytes_per_step": d2h},
                "gpu_launches": args.steps * per_call,
                "clocks": clk.summary()}
        if world == 1 and not args.no_cpu_baseline:
            cb = cpu_baseline(p, w)
            line["cpu_baseline"] = {"value": cb["layer_ms"] * scale, "unit": unit,
                                    "cores": cb["omp"], "kind": "oracle",
                                    "sample": f"{cb['rows']} random query rows "
                                              f"({cb['pairs']} causal pairs, {cb['wall_s']:.1f} s"
                                              "), extrapolated by causal pair count"}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

"""Multi-rank host logic on CPU (gloo, world size 2).

One indexer layer is partitioned across ranks with no collective on the data
path: prefill by zigzag query-row chunks, decode by sequences
(sparse_attention_token_dsa_b200.partition).  Each rank computes its own rows;
ranks only meet for the barrier around the timed region and the
max-over-ranks reduction of its time.  Here each rank runs the CPU oracle on
exactly the sub-problems the benchmark would give the library, and the rows
gathered from both ranks must equal the single-rank layer bit for bit.
CPU only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = 3.0 + 2.5 * rank                # each rank's own timed region (ms)
        dist.barrier()
        out[rank] = bench.max_over_ranks(local)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    port = _free_port()
    # spawn, not fork: the test process already runs torch and OpenMP threads
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        assert dict(out) == {0: 5.5, 1: 5.5}


def _sub_problem(p, start, count, gen):
    """Rows [start, start + count) of a one-sequence prefill problem as a problem
    of its own: the query / weight rows sliced, its query position start + pos0."""
    import numpy as np
    return gen.Problem(1, count, p.n_k, p.heads, p.dim, p.topk, p.q_dtype, p.k_dtype,
                       np.ascontiguousarray(p.q[:, start:start + count]), p.k,
                       np.ascontiguousarray(p.w[:, start:start + count]),
                       np.array([p.pos0(0) + start], np.int32), p.k_len)


def _partition_worker(rank, world, port, out):
    import numpy as np
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from sparse_attention_token_dsa_b200 import inputs as gen
    from sparse_attention_token_dsa_b200 import partition as part
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # prefill: 301 rows (not a multiple of 2 * world) over a 420-key cache
        p = gen.integer_problem(90, 1, 301, 420, 16, 128, 40, dtype=gen.BF16)
        mine = {}
        for start, count in part.prefill_row_ranges(p.n_q, world, rank):
            sub = _sub_problem(p, start, count, gen)
            idx, sc, _, _ = oracle.dsa(oracle.Inputs(sub), sub.topk)
            mine[start] = (idx, sc)
        # decode: 5 sequences, ragged prefixes, split by sequence
        d = gen.integer_problem(91, 5, 1, 700, 16, 128, 64, q_pos0=[699, 650, 500, 300, 10],
                                k_len=[700, 651, 501, 301, 11], dtype=gen.BF16)
        b0, nb = part.decode_seq_range(d.batch, world, rank)
        dsub = gen.Problem(nb, 1, d.n_k, d.heads, d.dim, d.topk, d.q_dtype, d.k_dtype,
                           d.q[b0:b0 + nb], np.ascontiguousarray(d.k[b0:b0 + nb]),
                           d.w[b0:b0 + nb], d.q_pos0[b0:b0 + nb], d.k_len[b0:b0 + nb])
        didx, dsc, _, _ = oracle.dsa(oracle.Inputs(dsub), dsub.topk) if nb else (None,) * 4
        gathered = [None] * world
        dist.all_gather_object(gathered, (mine, (b0, didx, dsc)))
        if rank == 0:
            out["gathered"] = gathered
    finally:
        dist.destroy_process_group()


def test_partitioned_layer_reassembles_the_single_rank_layer():
    """Every row computed once, on one rank, and identical to the whole layer."""
    import numpy as np
    sys.path.insert(0, ROOT)
    import oracle
    from sparse_attention_token_dsa_b200 import inputs as gen
    oracle.build()
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        os.environ.setdefault("OMP_NUM_THREADS", "2")
        mp.spawn(_partition_worker, args=(2, port, out), nprocs=2, join=True)
        gathered = out["gathered"]
    p = gen.integer_problem(90, 1, 301, 420, 16, 128, 40, dtype=gen.BF16)
    ri, rs, _, _ = oracle.dsa(oracle.Inputs(p), p.topk)
    gi = np.full_like(ri, -7)
    gs = np.full_like(rs, 7.0)
    seen = np.zeros(p.n_q, np.int32)
    for mine, _ in gathered:
        for start, (idx, sc) in mine.items():
            gi[start:start + len(idx)] = idx
            gs[start:start + len(idx)] = sc
            seen[start:start + len(idx)] += 1
    assert np.all(seen == 1)
    assert np.array_equal(gi, ri) and np.array_equal(gs, rs)
    d = gen.integer_problem(91, 5, 1, 700, 16, 128, 64, q_pos0=[699, 650, 500, 300, 10],
                            k_len=[700, 651, 501, 301, 11], dtype=gen.BF16)
    di, ds, _, _ = oracle.dsa(oracle.Inputs(d), d.topk)
    got_i = np.concatenate([g[1][1] for g in gathered if g[1][1] is not None])
    got_s = np.concatenate([g[1][2] for g in gathered if g[1][2] is not None])
    assert [g[1][0] for g in gathered] == [0, 2]
    assert np.array_equal(got_i, di) and np.array_equal(got_s, ds)


@pytest.mark.parametrize("n_q,world", [(131072, 2), (131072, 8), (32768, 4), (1001, 3), (7, 2)])
def test_zigzag_balances_causal_work(n_q, world):
    """Each rank scores the same number of causal pairs up to one row's length,
    and the ranks' rows cover the layer exactly once."""
    sys.path.insert(0, ROOT)
    from sparse_attention_token_dsa_b200 import partition as part
    pairs, rows = [], []
    for r in range(world):
        rg = part.prefill_row_ranges(n_q, world, r)
        pairs.append(part.causal_pairs(rg, 0, n_q))
        for start, count in rg:
            rows.extend(range(start, start + count))
    assert sorted(rows) == list(range(n_q))
    assert sum(pairs) == n_q * (n_q + 1) // 2
    assert max(pairs) - min(pairs) <= n_q


def test_decode_split_covers_every_sequence_once():
    sys.path.insert(0, ROOT)
    from sparse_attention_token_dsa_b200 import partition as part
    for batch, world in ((32, 8), (32, 3), (5, 2), (2, 4)):
        got = []
        for r in range(world):
            b0, nb = part.decode_seq_range(batch, world, r)
            got.extend(range(b0, b0 + nb))
        assert got == list(range(batch))


def test_max_over_ranks_without_group_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(1.25) == 1.25


def test_reference_arm_under_torchrun_prints_one_line():
    """bench.py --impl reference launched like the driver's N = 2 run: rank 0
    alone runs the oracle arm and prints one JSON line; every rank exits 0."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--workload", "dsa_prefill_1k_int", "--steps", "1",
           "--warmup", "1"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0

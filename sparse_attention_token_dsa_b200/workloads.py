"""Seeded synthetic inputs of the Sparse MLA consumer (no method arithmetic).

The pages give the step after the indexer as Sparse MLA reading the latent KV
at the selected positions ("PaperTrace 2.2.2 MISA, LISA and ResMiSA", section
2.2).  Shapes are the MLA read used here: 128 query heads, a 576-dimensional
absorbed query and cached row (512 latent + 64 rope), value = the 512 latent
dimensions, softmax scale 1/sqrt(128 + 64) (the per-head query-key width
before absorption).  Each query token at causal position p selects k distinct
positions in [0, p] (all of them when p < k), in ascending order as the
indexer's position-ordered output returns them.
"""
from __future__ import annotations

import numpy as np

from . import inputs as gen

DQK, DV = 576, 512
SCALE = 192 ** -0.5


def mla_problem(n_q: int, n_k: int, heads: int, topk: int, seed: int = 1, batch: int = 1):
    """q [batch * n_q, heads, 576] and kv [batch, n_k, 576] as bf16 words
    (N(0,1) rounded), idx [batch * n_q, topk] int32, tokens at positions
    n_k - n_q + i of each sequence."""
    r = np.random.Generator(np.random.PCG64(1000 * seed + 1))
    q = gen.f32_to_bf16_bits(r.standard_normal((batch * n_q, heads, DQK), dtype=np.float32))
    r = np.random.Generator(np.random.PCG64(1000 * seed + 2))
    kv = gen.f32_to_bf16_bits(r.standard_normal((batch, n_k, DQK), dtype=np.float32))
    r = np.random.Generator(np.random.PCG64(1000 * seed + 4))
    idx = np.full((batch * n_q, topk), -1, np.int32)
    for t in range(batch * n_q):
        pos = n_k - n_q + (t % n_q)
        if pos + 1 <= topk:
            sel = np.arange(pos + 1)
        else:
            # k distinct positions in [0, pos]: a random subset, ascending
            sel = np.sort(r.choice(pos + 1, size=topk, replace=False))
        idx[t, :len(sel)] = sel
    return dict(q=q, kv=kv, idx=idx, scale=SCALE, tps=n_q)


def backward_problem(n_q: int, heads: int, topk: int, seed: int = 1):
    """Indexer backward workload: one prefill sequence of n_q tokens (q, k bf16
    N(0,1), w N(0, 1/heads)), each row's topk distinct causal positions in
    ascending order (all of them when the prefix is shorter), upstream
    gradient N(0,1).  Returns (problem, sel, grad)."""
    p = gen.normal_problem(seed, 1, n_q, n_q, heads, 128, topk)
    r = np.random.Generator(np.random.PCG64(1000 * seed + 5))
    sel = np.full((n_q, topk), -1, np.int32)
    for t in range(n_q):
        if t + 1 <= topk:
            pick = np.arange(t + 1)
        else:
            pick = np.sort(r.choice(t + 1, size=topk, replace=False))
        sel[t, :len(pick)] = pick
    grad = r.standard_normal(sel.shape, dtype=np.float32)
    return p, sel, grad

"""GPU parity of dsa_sparse_mla (Sparse MLA over a fixed set of selected
positions) against the CPU oracle's naive gather attention ("PaperTrace 2.2.2
MISA, LISA and ResMiSA", section 2.3, acceptance step two: the same candidate
set through the naive gather attention and the kernel, checking the output
and the log-sum-exp of the row maximum and denominator).

Tolerance.  The kernel computes logits in fp32 from bf16 operands, rounds each
softmax weight to bf16 before the value product (fp32 accumulation) and writes
bf16 outputs.  A weight rounded by at most 2^-9 of itself moves o by at most
2^-9 sum_s w_s |v_s - o|; with the output's own bf16 rounding the bound used is
|o_gpu - o_ref| <= 2^-8 (sum_s w_s |v_s| + |o_ref|) per element, and
|lse_gpu - lse_ref| <= 2^-8 (the denominator sums the rounded weights).
Closed forms are checked exactly: one selected position returns its value,
q = 0 returns the mean of the selected values.
"""
import numpy as np
import pytest

import oracle
from sparse_attention_token_dsa_b200 import inputs as gen

pytestmark = pytest.mark.gpu

DQK, DV = 576, 512


@pytest.fixture(scope="module")
def B():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from sparse_attention_token_dsa_b200 import binding
    oracle.build()
    return binding


def _t(x):
    import torch
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def run(B, q, kv, idx, scale, tps, flags=0, rows=None):
    """GPU output rows (all, or the listed tokens) as fp64, and the kernel time."""
    import torch
    qd, kvd, idd = _t(q), _t(kv), _t(idx)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    out, lse = B.sparse_mla(qd, kvd, idd, scale, tokens_per_seq=tps, flags=flags | B.DSA_FLAG_CHECK)
    e1.record()
    torch.cuda.synchronize()
    print(f"sparse MLA call: {e0.elapsed_time(e1):.3f} ms for {q.shape[0]} tokens")
    if rows is not None:
        rr = torch.as_tensor(np.asarray(rows), device=out.device)
        out, lse = out[rr], lse[rr]
    o = out.view(torch.int16).cpu().numpy().view(np.uint16)
    return gen.bf16_bits_to_f32(o).astype(np.float64), lse.cpu().numpy().astype(np.float64)


def make(seed, batch, tps, n_k, heads, topk, empty_frac=0.1, q_scale=1.0):
    r = np.random.default_rng(seed)
    T = batch * tps
    q = gen.f32_to_bf16_bits((r.standard_normal((T, heads, DQK)) * q_scale).astype(np.float32))
    kv = gen.f32_to_bf16_bits(r.standard_normal((batch, n_k, DQK)).astype(np.float32))
    idx = np.stack([r.permutation(n_k)[:topk] for _ in range(T)]).astype(np.int32)
    idx[r.random(idx.shape) < empty_frac] = -1
    return q, kv, idx


def check(q, kv, idx, scale, tps, o, lse, rows=None):
    """The documented bound, with the oracle's own weights.  o / lse hold the
    GPU rows listed in `rows` (all tokens when None), in that order; only those
    rows and their selected keys are decoded on the host."""
    T, H, _ = q.shape
    rows = np.arange(T) if rows is None else np.asarray(rows)
    worst = 0.0
    for a, t in enumerate(rows):
        b = t // tps
        sel = idx[t][(idx[t] >= 0) & (idx[t] < kv.shape[1])]
        one = oracle.sparse_mla(q[t:t + 1], kv[b:b + 1], idx[t:t + 1], scale, DV, 1)
        if len(sel) == 0:
            assert np.all(o[a] == 0.0) and np.all(np.isneginf(lse[a]))
            continue
        qf = gen.bf16_bits_to_f32(q[t]).astype(np.float64)          # [H, DQK]
        kf = gen.bf16_bits_to_f32(kv[b, sel]).astype(np.float64)    # [n, DQK]
        x = scale * qf @ kf.T                                        # [H, n]
        w = np.exp(x - x.max(1, keepdims=True))
        w /= w.sum(1, keepdims=True)
        wabs = w @ np.abs(kf[:, :DV])                                # [H, DV]
        bound = 2.0 ** -8 * (wabs + np.abs(one["o"][0]))
        err = np.abs(o[a] - one["o"][0])
        assert np.all(err <= bound), f"token {t}: output error {np.max(err / bound):.3f} x bound"
        assert np.all(np.abs(lse[a] - one["lse"][0]) <= 2.0 ** -8), f"token {t}: lse"
        worst = max(worst, float(np.max(err / np.maximum(bound, 1e-30))))
    print(f"sparse MLA: {len(rows)} tokens, largest error / bound {worst:.3f}")


@pytest.mark.parametrize("heads,topk", [(128, 200), (128, 2048), (64, 130), (16, 64)])
def test_sparse_mla_matches_oracle(B, heads, topk):
    """Two sequences, ragged last tiles, empty entries, fewer than 128 heads."""
    scale = 192 ** -0.5
    q, kv, idx = make(200 + heads + topk, 2, 3, 3000, heads, topk)
    o, lse = run(B, q, kv, idx, scale, 3)
    check(q, kv, idx, scale, 3, o, lse)


def test_sparse_mla_closed_forms_exact(B):
    """One selected position: the output is that row's value, bit for bit.
    q = 0: uniform weights, the output is the mean of the selected values."""
    q, kv, idx = make(210, 1, 4, 400, 128, 96, empty_frac=0.0)
    one = np.full_like(idx, -1)
    one[:, 37] = idx[:, 37]
    o, lse = run(B, q, kv, one, 0.1, 4)
    kvf = gen.bf16_bits_to_f32(kv).astype(np.float64)
    for t in range(4):
        assert np.array_equal(o[t], np.repeat(kvf[0, one[t, 37], :DV][None], 128, 0))
    z = np.zeros_like(q)
    o, lse = run(B, z, kv, idx, 0.1, 4)
    for t in range(4):
        mean = kvf[0, idx[t], :DV].mean(0)
        np.testing.assert_allclose(o[t], np.repeat(mean[None], 128, 0), rtol=2.0 ** -8, atol=1e-6)
        np.testing.assert_allclose(lse[t], np.log(96), rtol=1e-6)


def test_sparse_mla_order_and_empty_sets(B):
    """Position order gives the same output as any order (within the bound);
    a token with no selected position returns zeros and lse = -inf."""
    scale = 192 ** -0.5
    q, kv, idx = make(211, 1, 5, 2000, 128, 512, empty_frac=0.0)
    srt = np.sort(idx, 1).astype(np.int32)
    o1, l1 = run(B, q, kv, idx, scale, 5)
    o2, l2 = run(B, q, kv, srt, scale, 5)
    check(q, kv, idx, scale, 5, o1, l1)
    check(q, kv, srt, scale, 5, o2, l2)
    idx[2] = -1
    o3, l3 = run(B, q, kv, idx, scale, 5)
    assert np.all(o3[2] == 0.0) and np.all(np.isneginf(l3[2]))
    check(q, kv, idx, scale, 5, o3, l3)


def test_sparse_mla_medium_sampled(B):
    """512 query tokens over a 16384-row cache (a smaller case of the full one)."""
    from sparse_attention_token_dsa_b200 import workloads
    w = workloads.mla_problem(512, 16384, 128, 2048, seed=6)
    rows = np.array([0, 255, 511])
    o, lse = run(B, w["q"], w["kv"], w["idx"], w["scale"], w["tps"], rows=rows)
    check(w["q"], w["kv"], w["idx"], w["scale"], w["tps"], o, lse, rows=rows)


def test_sparse_mla_full_size_sampled(B):
    """4096 query tokens over a 131072-row cache, 128 heads, k = 2048 causal
    positions each (position order), checked on sampled tokens."""
    from sparse_attention_token_dsa_b200 import workloads
    w = workloads.mla_problem(4096, 131072, 128, 2048, seed=5)
    rows = np.array([0, 1, 1000, 2047, 3000, 4095])
    o, lse = run(B, w["q"], w["kv"], w["idx"], w["scale"], w["tps"], rows=rows)
    check(w["q"], w["kv"], w["idx"], w["scale"], w["tps"], o, lse, rows=rows)

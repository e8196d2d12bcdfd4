"""GPU parity of lisa_index (indexer LISA, LISA-dagger) and resmisa_index
against the CPU oracle ("PaperTrace 2.2.2 MISA, LISA and ResMiSA", sections
3.1 and 3.2).

Exact on integer-valued inputs: the fused query g = sum_j w_j q_j is an
integer below 2^16, so its two bf16 parts hold it exactly; every dot product,
residual bound and score is an integer below 2^24 and fp32 is exact.  On
real-valued inputs the decisions upstream of the final top-k (the residual
heads, the LISA-dagger pool) must be correct up to near-ties, and the oracle
re-run with the GPU's decision forced must agree within the tolerance rule of
tests/parity.py (1e-3 of max(|I|, nu)).
"""
import numpy as np
import pytest

import oracle
import parity
from sparse_attention_token_dsa_b200 import inputs as gen

pytestmark = pytest.mark.gpu

TOL = 1e-3


@pytest.fixture(scope="module")
def B():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from sparse_attention_token_dsa_b200 import binding
    oracle.build()
    return binding


def dev(x):
    import torch
    if x is None:
        return None
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _flat(t, width):
    return t.cpu().numpy().reshape(-1, width)


def run(B, p, algo, pool=0, block=0, r=0, flags=None):
    import torch
    flags = B.DSA_FLAG_SORTED | B.DSA_FLAG_CHECK if flags is None else flags
    q, k, w = dev(p.q), dev(p.k), dev(p.w)
    pos0, klen = dev(p.q_pos0), dev(p.k_len)
    rows = (p.batch, p.n_q)
    out = {}
    if algo == "lisa":
        pl = torch.full((*rows, max(pool, 1)), -7, dtype=torch.int32, device="cuda")
        idx, sc = B.lisa_index(q, k, w, p.topk, pool=pool, q_pos0=pos0, k_len=klen, flags=flags,
                               out_pool=pl if pool else None)
        torch.cuda.synchronize()
        out["pool"] = _flat(pl, max(pool, 1)) if pool else None
    else:
        heads = torch.full((*rows, max(r, 1)), -7, dtype=torch.int32, device="cuda")
        S = torch.full((*rows, p.heads), -7.0, dtype=torch.float32, device="cuda")
        idx, sc = B.resmisa_index(q, k, w, p.topk, block, r, q_pos0=pos0, k_len=klen, flags=flags,
                                  out_heads=heads if r else None, out_S=S)
        torch.cuda.synchronize()
        out["heads"] = _flat(heads, max(r, 1))[:, :r]
        out["S"] = _flat(S, p.heads)
    gi, gs = _flat(idx, p.topk), _flat(sc, p.topk)
    if not flags & B.DSA_FLAG_SORTED:
        gi, gs = parity.order_rows(gi, gs)
    out["idx"], out["score"] = gi, gs
    return out


CASES = [
    # (batch, n_q, n_k, heads, q_pos0, k_len)
    (1, 700, 700, 64, None, None),
    (2, 300, 900, 32, [0, 600], [400, 900]),
]


# ------------------------------------------------------------------ exact ---

@pytest.mark.parametrize("case", CASES)
def test_lisa_integer_bit_exact(B, case):
    batch, nq, nk, H, pos0, klen = case
    p = gen.integer_problem(110, batch, nq, nk, H, 128, 128, q_pos0=pos0, k_len=klen,
                            dtype=gen.BF16)
    g = run(B, p, "lisa")
    ref = oracle.lisa(oracle.Inputs(p), p.topk)
    parity.exact(g["idx"], g["score"], ref["idx"], ref["score"])


@pytest.mark.parametrize("case", CASES)
def test_lisa_dagger_integer_bit_exact(B, case):
    """Pool of M = 256 by the linear term, reranked by the full score: the pool set
    and the final rows are the oracle's."""
    batch, nq, nk, H, pos0, klen = case
    p = gen.integer_problem(111, batch, nq, nk, H, 128, 128, q_pos0=pos0, k_len=klen,
                            dtype=gen.BF16)
    g = run(B, p, "lisa", pool=256)
    ref = oracle.lisa(oracle.Inputs(p), p.topk, pool_m=256)
    assert np.array_equal(np.sort(g["pool"], 1), np.sort(ref["pool"], 1))
    parity.exact(g["idx"], g["score"], ref["idx"], ref["score"])


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("r", [7, 1])
def test_resmisa_integer_bit_exact(B, case, r):
    """Block B = 128 (ragged last block, causal prefixes, k_len): residual heads, their
    bounds S, indices and scores identical to the oracle."""
    batch, nq, nk, H, pos0, klen = case
    p = gen.integer_problem(112, batch, nq, nk, H, 128, 128, q_pos0=pos0, k_len=klen,
                            dtype=gen.BF16)
    g = run(B, p, "resmisa", block=128, r=r)
    ref = oracle.resmisa(oracle.Inputs(p), p.topk, 128, r)
    assert np.array_equal(g["heads"], ref["heads"])
    assert np.array_equal(g["S"].astype(np.float64), ref["S"])
    parity.exact(g["idx"], g["score"], ref["idx"], ref["score"])


def test_resmisa_limits_are_dsa_and_lisa(B):
    """r = H recovers the DSA score and r = 0 the LISA score (all on the GPU)."""
    import torch
    p = gen.integer_problem(113, 1, 400, 400, 16, 128, 64, dtype=gen.BF16)
    full = run(B, p, "resmisa", block=64, r=16)
    idx, sc = B.dsa_index(dev(p.q), dev(p.k), dev(p.w), p.topk, flags=B.DSA_FLAG_SORTED)
    torch.cuda.synchronize()
    assert np.array_equal(full["idx"], _flat(idx, p.topk))
    assert np.array_equal(full["score"], _flat(sc, p.topk))
    none = run(B, p, "resmisa", block=64, r=0)
    lisa = run(B, p, "lisa")
    assert np.array_equal(none["idx"], lisa["idx"]) and np.array_equal(none["score"], lisa["score"])


def test_lisa_short_prefixes_pad(B):
    p = gen.integer_problem(114, 1, 200, 200, 64, 128, 128, dtype=gen.BF16)
    g = run(B, p, "lisa", pool=160, flags=0)
    ref = oracle.lisa(oracle.Inputs(p), p.topk, pool_m=160)
    assert np.array_equal(np.sort(g["pool"], 1), np.sort(ref["pool"], 1))
    parity.exact(g["idx"], g["score"], ref["idx"], ref["score"])


# ---------------------------------------------------- conditional (real) ---

@pytest.fixture(scope="module")
def real_small():
    return gen.normal_problem(115, 1, 2048, 2048, 64, 128, 256, key_structure="clusters",
                              mean_run=128.0)


def test_lisa_real(B, real_small):
    p = real_small
    inp = oracle.Inputs(p)
    rows = gen.stratified_rows(p, 48)
    g = run(B, p, "lisa")
    ref = oracle.lisa(inp, p.topk, rows=rows)
    r = parity.within_tolerance(inp, rows, g["idx"][rows], g["score"][rows], ref["idx"],
                                ref["score64"], TOL, label="LISA",
                                score_fn=lambda a, rr, ss: oracle.linear_pairs(inp, rr, ss))
    assert r.iou > 0.98


def test_lisa_dagger_real_conditional(B, real_small):
    p = real_small
    inp = oracle.Inputs(p)
    rows = gen.stratified_rows(p, 32)
    g = run(B, p, "lisa", pool=1024)
    # the pool: a correct top-1024 by the linear term up to near-ties at its cut-off
    for a, row in enumerate(rows):
        n = p.legal_count(int(row))
        nv = min(1024, n)
        gp = g["pool"][row]
        gset = gp[gp >= 0]
        assert len(gset) == nv and len(np.unique(gset)) == nv
        assert np.all((gset >= 0) & (gset < n))
        lin = oracle.linear_pairs(inp, np.full(n, row, np.int64), np.arange(n))
        order = np.lexsort((np.arange(n), -lin))
        cut = lin[order[nv - 1]]
        diff = np.setxor1d(gset, order[:nv])
        if len(diff):
            rr = np.full(len(diff), row, np.int64)
            e = TOL * np.maximum(np.abs(lin[diff]), oracle.nu_pairs(inp, rr, diff))
            e_cut = TOL * max(abs(cut), float(oracle.nu_pairs(
                inp, np.array([row], np.int64), np.array([order[nv - 1]], np.int64))[0]))
            assert np.all(np.abs(lin[diff] - cut) <= e + e_cut), f"row {row}: pool differs"
    ref = oracle.lisa(inp, p.topk, pool_m=1024, rows=rows, forced_pool=g["pool"][rows])
    r = parity.within_tolerance(inp, rows, g["idx"][rows], g["score"][rows], ref["idx"],
                                ref["score64"], TOL, label="LISA-dagger")
    assert r.iou > 0.98


def test_resmisa_real_conditional(B, real_small):
    p = real_small
    inp = oracle.Inputs(p)
    rows = gen.stratified_rows(p, 32)
    g = run(B, p, "resmisa", block=256, r=7)
    ref = oracle.resmisa(inp, p.topk, 256, 7, rows=rows)
    # heads: a correct top-7 of the oracle's S up to near-ties (scale: the row's largest S)
    for a, row in enumerate(rows):
        S = ref["S"][a]
        scale = TOL * max(float(np.max(np.abs(S))), 1e-30)
        np.testing.assert_array_less(np.abs(g["S"][row] - S), scale + 1e-30)
        order = np.lexsort((np.arange(len(S)), -S))
        cut = S[order[6]]
        gset = set(int(x) for x in g["heads"][row])
        assert len(gset) == 7 and list(g["heads"][row]) == sorted(gset)
        for j in gset ^ set(int(x) for x in order[:7]):
            assert abs(S[j] - cut) <= scale, f"row {row}: head {j} is not a near-tie"
    fh = g["heads"][rows]
    ref2 = oracle.resmisa(inp, p.topk, 256, 7, rows=rows, forced_heads=fh)
    r = parity.within_tolerance(
        inp, rows, g["idx"][rows], g["score"][rows], ref2["idx"], ref2["score64"], TOL,
        label="ResMiSA",
        score_fn=lambda a, rr, ss: oracle.resmisa_pairs(inp, rr, ss,
                                                        np.repeat(fh[a][None], len(rr), 0)))
    assert r.iou > 0.98

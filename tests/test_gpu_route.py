"""GPU parity of misa_index, misa_dagger_index and hisa_index against the CPU oracle.

Exact on segment-structured integer inputs (pooled keys, router sums, block
scores and token scores are all exactly representable, so heads, pools,
blocks, indices and scores must be bit-identical, ties to the lower index).

Real-valued inputs follow the tolerance rule of tests/parity.py in two steps
(conditional parity): every upstream decision of the GPU (routed heads, the
MISA-dagger pool, the kept HISA blocks) must be a correct one up to near-ties
at its cut-off, judged on the oracle's fp64 values; the oracle then re-runs
with that decision forced and the final top-k is compared within tolerance.
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


def run_route(B, p, algo, block=0, h=0, k_prime=0, hb=0, r=0, flags=None):
    """One routed call; returns host arrays (idx, score, heads, E, pool, blocks)."""
    import torch
    flags = B.DSA_FLAG_SORTED if flags is None else flags
    q, k, w = dev(p.q), dev(p.k), dev(p.w)
    pos0, klen = dev(p.q_pos0), dev(p.k_len)
    rows = (p.batch, p.n_q)
    out = dict(heads=None, E=None, pool=None, blocks=None)
    heads = torch.full((*rows, max(h, 1)), -7, dtype=torch.int32, device="cuda") if h else None
    if algo == "misa":
        E = torch.full((*rows, p.heads), -7.0, dtype=torch.float32, device="cuda")
        idx, sc = B.misa_index(q, k, w, p.topk, block, h, q_pos0=pos0, k_len=klen, flags=flags,
                               out_heads=heads, out_E=E)
        torch.cuda.synchronize()
        out["E"] = _flat(E, p.heads)
    elif algo == "dagger":
        pool = torch.full((*rows, k_prime), -7, dtype=torch.int32, device="cuda")
        idx, sc = B.misa_dagger_index(q, k, w, p.topk, block, h, k_prime, q_pos0=pos0,
                                      k_len=klen, flags=flags, out_heads=heads, out_pool=pool)
        torch.cuda.synchronize()
        out["pool"] = _flat(pool, k_prime)
    else:
        blocks = torch.full((*rows, r), -7, dtype=torch.int32, device="cuda")
        idx, sc = B.hisa_index(q, k, w, p.topk, hb, r, route_h=h, route_block=block,
                               q_pos0=pos0, k_len=klen, flags=flags, out_blocks=blocks,
                               out_heads=heads)
        torch.cuda.synchronize()
        out["blocks"] = _flat(blocks, r)
    if h:
        out["heads"] = _flat(heads, h)
    gi, gs = _flat(idx, p.topk), _flat(sc, p.topk)
    if not flags & B.DSA_FLAG_SORTED:
        gi, gs = parity.order_rows(gi, gs)
    out["idx"], out["score"] = gi, gs
    return out


def sorted_sets(a):
    return np.sort(np.asarray(a), axis=1)


# ------------------------------------------------------------------ exact ---

SEG_CASES = [
    # (batch, n_q, n_k, heads, q_pos0, k_len)
    (1, 1500, 1500, 64, None, None),
    (2, 600, 1500, 32, [0, 900], [500, 1500]),
]


@pytest.mark.parametrize("case", SEG_CASES)
def test_misa_integer_bit_exact(B, case):
    """MISA, B = 128, h = 8, k = 128 on segment-structured integers: heads, E, indices
    and scores identical to the oracle (ragged last block, causal prefixes, k_len)."""
    batch, nq, nk, H, pos0, klen = case
    p = gen.segment_integer_problem(70, batch, nq, nk, H, 128, 128, seg=128, q_pos0=pos0,
                                    k_len=klen)
    g = run_route(B, p, "misa", block=128, h=8)
    ref = oracle.misa(oracle.Inputs(p), p.topk, 128, 8)
    assert np.array_equal(g["heads"], ref["heads"])
    np.testing.assert_allclose(g["E"], ref["E"], rtol=2.0 ** -22, atol=0)
    parity.exact(g["idx"], g["score"], ref["idx"], ref["score"])


@pytest.mark.parametrize("H,h", [(16, 8), (128, 16)])
def test_misa_integer_head_counts(B, H, h):
    p = gen.segment_integer_problem(71, 1, 700, 700, H, 128, 64, seg=64)
    g = run_route(B, p, "misa", block=64, h=h)
    ref = oracle.misa(oracle.Inputs(p), p.topk, 64, h)
    assert np.array_equal(g["heads"], ref["heads"])
    parity.exact(g["idx"], g["score"], ref["idx"], ref["score"])


def test_misa_with_all_heads_matches_dsa(B):
    """h = H routes every head: the output is the DSA output (both on the GPU)."""
    p = gen.segment_integer_problem(72, 1, 520, 520, 8, 128, 64, seg=64)
    g = run_route(B, p, "misa", block=64, h=8)
    idx, sc = B.dsa_index(dev(p.q), dev(p.k), dev(p.w), p.topk, flags=B.DSA_FLAG_SORTED)
    assert np.array_equal(g["idx"], _flat(idx, p.topk))
    assert np.array_equal(g["score"], _flat(sc, p.topk))


@pytest.mark.parametrize("case", SEG_CASES)
def test_misa_dagger_integer_bit_exact(B, case):
    """MISA-dagger, k' = 512: the pool set and the reranked top-k are the oracle's."""
    batch, nq, nk, H, pos0, klen = case
    p = gen.segment_integer_problem(73, batch, nq, nk, H, 128, 128, seg=128, q_pos0=pos0,
                                    k_len=klen)
    g = run_route(B, p, "dagger", block=128, h=8, k_prime=512)
    ref = oracle.misa(oracle.Inputs(p), p.topk, 128, 8, k_prime=512)
    assert np.array_equal(g["heads"], ref["heads"])
    assert np.array_equal(sorted_sets(g["pool"]), sorted_sets(ref["pool"]))
    parity.exact(g["idx"], g["score"], ref["idx"], ref["score"])


@pytest.mark.parametrize("case", SEG_CASES)
@pytest.mark.parametrize("stacked", [False, True])
def test_hisa_integer_bit_exact(B, case, stacked):
    """HISA b = 64, r = 8 (and stacked with the B = 128, h = 8 router): kept blocks,
    indices and scores identical to the oracle."""
    batch, nq, nk, H, pos0, klen = case
    p = gen.segment_integer_problem(74, batch, nq, nk, H, 128, 128, seg=128, q_pos0=pos0,
                                    k_len=klen)
    h = 8 if stacked else 0
    g = run_route(B, p, "hisa", block=128, h=h, hb=64, r=8)
    ref = oracle.hisa(oracle.Inputs(p), p.topk, 64, 8, route_h=h, route_block=128)
    if stacked:
        assert np.array_equal(g["heads"], ref["heads"])
    assert np.array_equal(sorted_sets(g["blocks"]), sorted_sets(ref["blocks"]))
    parity.exact(g["idx"], g["score"], ref["idx"], ref["score"])


def test_hisa_small_blocks_and_unsorted_output(B):
    """b = 16 (eight block runs per 128-key tile), r = 40, default (unsorted) output."""
    p = gen.segment_integer_problem(75, 1, 900, 900, 64, 128, 200, seg=64)
    g = run_route(B, p, "hisa", hb=16, r=40, flags=0)
    ref = oracle.hisa(oracle.Inputs(p), p.topk, 16, 40)
    assert np.array_equal(sorted_sets(g["blocks"]), sorted_sets(ref["blocks"]))
    parity.exact(g["idx"], g["score"], ref["idx"], ref["score"])


def test_routed_short_prefixes_pad(B):
    """Rows whose prefix is shorter than one block, than k' or than r blocks pad with -1."""
    p = gen.segment_integer_problem(76, 1, 300, 300, 64, 128, 128, seg=64)
    for algo, kw in (("dagger", dict(block=64, h=8, k_prime=256)),
                     ("hisa", dict(hb=64, r=4))):
        g = run_route(B, p, algo, **kw)
        if algo == "dagger":
            ref = oracle.misa(oracle.Inputs(p), p.topk, 64, 8, k_prime=256)
            assert np.array_equal(sorted_sets(g["pool"]), sorted_sets(ref["pool"]))
        else:
            ref = oracle.hisa(oracle.Inputs(p), p.topk, 64, 4)
            assert np.array_equal(sorted_sets(g["blocks"]), sorted_sets(ref["blocks"]))
        parity.exact(g["idx"], g["score"], ref["idx"], ref["score"])


# ---------------------------------------------------- conditional (real) ---

def check_heads(inp, rows, g_heads, g_E, ref_E, h):
    """GPU head sets are a correct top-h of the oracle's E up to near-ties."""
    for a, row in enumerate(rows):
        e = ref_E[a]
        scale = TOL * max(float(np.max(np.abs(e))), 1e-30)
        np.testing.assert_array_less(np.abs(g_E[row] - e), scale + 1e-30)
        order = np.lexsort((np.arange(len(e)), -e))
        cut = e[order[h - 1]]
        gset = set(int(x) for x in g_heads[row])
        assert len(gset) == h and list(g_heads[row]) == sorted(gset)
        rset = set(int(x) for x in order[:h])
        for j in gset ^ rset:
            assert abs(e[j] - cut) <= scale, f"row {row}: head {j} is not a near-tie"


def check_pool(inp, rows, g_pool, g_heads, kp):
    for row in rows:
        heads = g_heads[row]
        v = oracle.score_row(inp, int(row), heads)
        n = len(v)
        nv = min(kp, n)
        gp = g_pool[row]
        gset = gp[gp >= 0]
        assert len(gset) == nv and len(np.unique(gset)) == nv
        assert np.all((gset >= 0) & (gset < n))
        order = np.lexsort((np.arange(n), -v))
        if nv == 0:
            continue
        cut = v[order[nv - 1]]
        diff = np.setxor1d(gset, order[:nv])
        if len(diff):
            rr = np.full(len(diff), row, np.int64)
            hh = np.repeat(np.asarray(heads)[None], len(diff), 0)
            e = TOL * np.maximum(np.abs(v[diff]), oracle.nu_pairs(inp, rr, diff, hh))
            kth = np.array([order[nv - 1]], np.int64)
            e_cut = TOL * max(abs(cut), float(oracle.nu_pairs(
                inp, np.array([row], np.int64), kth, np.asarray(heads)[None])[0]))
            assert np.all(np.abs(v[diff] - cut) <= e + e_cut), f"row {row}: pool differs"


def check_blocks(inp, rows, g_blocks, block, r, heads=None):
    for row in rows:
        hh = None if heads is None else heads[row]
        J = oracle.block_scores(inp, int(row), block, hh)
        m = len(J)
        nv = min(r, m)
        gb = g_blocks[row]
        gset = gb[gb >= 0]
        assert len(gset) == nv and len(np.unique(gset)) == nv
        assert np.all((gset >= 0) & (gset < m))
        if nv == 0:
            continue
        order = np.lexsort((np.arange(m), -J))
        cut = J[order[nv - 1]]
        scale = TOL * max(float(np.max(np.abs(J))), 1e-30)
        for x in np.setxor1d(gset, order[:nv]):
            assert abs(J[x] - cut) <= scale, f"row {row}: block {x} is not a near-tie"


@pytest.fixture(scope="module")
def real_small():
    return gen.normal_problem(80, 1, 2048, 2048, 64, 128, 256, key_structure="clusters",
                              mean_run=128.0)


def test_misa_real_conditional(B, real_small):
    p = real_small
    inp = oracle.Inputs(p)
    rows = gen.stratified_rows(p, 48)
    g = run_route(B, p, "misa", block=256, h=8)
    ref = oracle.misa(inp, p.topk, 256, 8, rows=rows)
    check_heads(inp, rows, g["heads"], g["E"], ref["E"], 8)
    fh = g["heads"][rows]
    ref2 = oracle.misa(inp, p.topk, 256, 8, rows=rows, forced_heads=fh)
    r = parity.within_tolerance(inp, rows, g["idx"][rows], g["score"][rows], ref2["idx"],
                                ref2["score64"], TOL, heads=fh)
    assert r.iou > 0.98


def test_misa_dagger_real_conditional(B, real_small):
    p = real_small
    inp = oracle.Inputs(p)
    rows = gen.stratified_rows(p, 32)
    g = run_route(B, p, "dagger", block=256, h=8, k_prime=1024)
    check_pool(inp, rows, g["pool"], g["heads"], 1024)
    ref = oracle.misa(inp, p.topk, 256, 8, k_prime=1024, rows=rows,
                      forced_heads=g["heads"][rows], forced_pool=g["pool"][rows])
    r = parity.within_tolerance(inp, rows, g["idx"][rows], g["score"][rows], ref["idx"],
                                ref["score64"], TOL)
    assert r.iou > 0.98


@pytest.mark.parametrize("stacked", [False, True])
def test_hisa_real_conditional(B, real_small, stacked):
    p = real_small
    inp = oracle.Inputs(p)
    rows = gen.stratified_rows(p, 32)
    h = 8 if stacked else 0
    g = run_route(B, p, "hisa", block=256, h=h, hb=64, r=16)
    heads = g["heads"] if stacked else None
    check_blocks(inp, rows, g["blocks"], 64, 16, heads)
    ref = oracle.hisa(inp, p.topk, 64, 16, route_h=h, route_block=256, rows=rows,
                      forced_heads=None if heads is None else heads[rows],
                      forced_blocks=g["blocks"][rows])
    r = parity.within_tolerance(inp, rows, g["idx"][rows], g["score"][rows], ref["idx"],
                                ref["score64"], TOL,
                                heads=None if heads is None else heads[rows])
    assert r.iou > 0.98


# ------------------------------------------------- full size, sampled rows ---

@pytest.fixture(scope="module")
def full128k():
    """L = 131072 causal, H_I = 64, d = 128, k = 2048, bf16, clustered keys."""
    return gen.normal_problem(5, 1, 131072, 131072, 64, 128, 2048, key_structure="clusters")


def test_full_size_misa_and_dagger_sampled(B, full128k):
    """MISA (B = 1024, h = 8) and MISA-dagger (k' = 8192) at 128K, sampled rows."""
    p = full128k
    inp = oracle.Inputs(p)
    rows = gen.stratified_rows(p, 6)
    g = run_route(B, p, "misa", block=1024, h=8)
    ref = oracle.misa(inp, p.topk, 1024, 8, rows=rows)
    check_heads(inp, rows, g["heads"], g["E"], ref["E"], 8)
    fh = g["heads"][rows]
    ref2 = oracle.misa(inp, p.topk, 1024, 8, rows=rows, forced_heads=fh)
    r = parity.within_tolerance(inp, rows, g["idx"][rows], g["score"][rows], ref2["idx"],
                                ref2["score64"], TOL, heads=fh, label="MISA 128K")
    assert r.iou > 0.98
    gd = run_route(B, p, "dagger", block=1024, h=8, k_prime=8192)
    assert np.array_equal(gd["heads"], g["heads"])
    check_pool(inp, rows, gd["pool"], gd["heads"], 8192)
    ref3 = oracle.misa(inp, p.topk, 1024, 8, k_prime=8192, rows=rows, forced_heads=fh,
                       forced_pool=gd["pool"][rows])
    r = parity.within_tolerance(inp, rows, gd["idx"][rows], gd["score"][rows], ref3["idx"],
                                ref3["score64"], TOL, label="MISA-dagger 128K")
    assert r.iou > 0.98


@pytest.mark.parametrize("stacked", [False, True])
def test_full_size_hisa_sampled(B, full128k, stacked):
    """HISA (b = 64, r = 128) and stacked MISA(h = 8, B = 1024) + HISA at 128K."""
    p = full128k
    inp = oracle.Inputs(p)
    rows = gen.stratified_rows(p, 6)
    h = 8 if stacked else 0
    g = run_route(B, p, "hisa", block=1024, h=h, hb=64, r=128)
    heads = g["heads"] if stacked else None
    check_blocks(inp, rows, g["blocks"], 64, 128, heads)
    ref = oracle.hisa(inp, p.topk, 64, 128, route_h=h, route_block=1024, rows=rows,
                      forced_heads=None if heads is None else heads[rows],
                      forced_blocks=g["blocks"][rows])
    r = parity.within_tolerance(inp, rows, g["idx"][rows], g["score"][rows], ref["idx"],
                                ref["score64"], TOL, heads=None if heads is None else heads[rows],
                                label="HISA 128K")
    assert r.iou > 0.98

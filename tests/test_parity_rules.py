"""The comparison rules of tests/parity.py reject wrong outputs.

The GPU parity tests pass when parity.exact / parity.within_tolerance accept
the CUDA path's rows.  Here the oracle's own rows stand in for a correct
output, and copies with one planted fault (a far token swapped in, a score off
by more than the tolerance, a duplicate, a wrong order, an illegal index, a
lost entry, a -0.0) must each be rejected.  CPU only; nothing runs on a GPU.
"""
import numpy as np
import pytest

import oracle
import parity
from sparse_attention_token_dsa_b200 import inputs as gen

TOL = 1e-3


@pytest.fixture(scope="module")
def case():
    oracle.build()
    p = gen.normal_problem(61, 1, 48, 200, 8, 128, 16)
    inp = oracle.Inputs(p)
    rows = np.arange(p.n_q)
    ri, rs, rs64, _ = oracle.dsa(inp, p.topk, rows)
    return inp, rows, ri, rs, rs64


def _row_with_room(case):
    """A row with more legal keys than k (so a non-selected token exists)."""
    inp, rows, ri, _, _ = case
    for a, row in enumerate(rows):
        if inp.prob.legal_count(int(row)) > inp.prob.topk + 4:
            return a
    raise AssertionError("no row with spare legal keys")


def test_reference_rows_pass(case):
    inp, rows, ri, rs, rs64 = case
    r = parity.within_tolerance(inp, rows, ri, rs, ri, rs64, TOL)
    assert r.iou == 1.0 and r.max_rel < 1e-6
    parity.exact(ri, rs, ri, rs)


def test_far_token_swapped_in_is_rejected(case):
    inp, rows, ri, rs, rs64 = case
    a = _row_with_room(case)
    row = int(rows[a])
    n = inp.prob.legal_count(row)
    outside = np.setdiff1d(np.arange(n), ri[a])
    sc = oracle.score_pairs(inp, np.full(len(outside), row, np.int64), outside)
    worst = int(outside[np.argmin(sc)])             # far below the k-th score
    gi, gs = ri.copy(), rs.copy()
    gi[a, 0] = worst                                 # replace the best token
    gs[a, 0] = np.float32(sc.min())
    gi[a], gs[a] = parity.order_rows(gi[a:a + 1], gs[a:a + 1])
    with pytest.raises(AssertionError, match="not near the cut-off"):
        parity.within_tolerance(inp, rows, gi, gs, ri, rs64, TOL)


def _nu_numpy(inp, row, s):
    """nu(t, s) = sum_j |w_tj| ||q_tj|| ||k_s|| / sqrt(d), from the bf16 operands."""
    p = inp.prob
    q = gen.bf16_bits_to_f32(p.q.reshape(p.batch * p.n_q, p.heads, p.dim)[row]).astype(np.float64)
    k = gen.bf16_bits_to_f32(p.k[row // p.n_q, s]).astype(np.float64)
    w = p.w.reshape(-1, p.heads)[row].astype(np.float64)
    return float(np.sum(np.abs(w) * np.linalg.norm(q, axis=1)) * np.linalg.norm(k)
                 / np.sqrt(p.dim))


@pytest.mark.parametrize("factor,rejected", [(2.0, True), (0.5, False)])
def test_score_error_against_the_tolerance(case, factor, rejected):
    """A last-place score moved by factor x tol x max(|I|, nu) (nu computed here
    from the operands, independently of the oracle) is rejected above the
    tolerance and accepted below it."""
    inp, rows, ri, rs, rs64 = case
    a = 3
    row = int(rows[a])
    nv = int(np.sum(ri[a] >= 0))
    scale = max(abs(float(rs64[a, nv - 1])), _nu_numpy(inp, row, int(ri[a, nv - 1])))
    gs = rs.copy()
    gs[a, nv - 1] = np.float32(rs64[a, nv - 1] - factor * TOL * scale)   # still last in order
    if rejected:
        with pytest.raises(AssertionError, match="score error"):
            parity.within_tolerance(inp, rows, ri, gs, ri, rs64, TOL)
    else:
        r = parity.within_tolerance(inp, rows, ri, gs, ri, rs64, TOL)
        assert 0.4 * TOL < r.max_rel < 0.6 * TOL


def test_nu_is_well_below_the_absolute_sum(case):
    """On N(0,1) operands nu is several times smaller than sum_j |w| sum_c |q_c k_c|
    (the scale an earlier rule used), so the tolerance rule is that much tighter."""
    inp, rows, ri, _, _ = case
    p = inp.prob
    row = int(rows[5])
    s = int(ri[5, 0])
    q = gen.bf16_bits_to_f32(p.q.reshape(-1, p.heads, p.dim)[row]).astype(np.float64)
    k = gen.bf16_bits_to_f32(p.k[0, s]).astype(np.float64)
    w = p.w.reshape(-1, p.heads)[row].astype(np.float64)
    absum = float(np.sum(np.abs(w) * np.sum(np.abs(q * k[None]), axis=1)))
    assert _nu_numpy(inp, row, s) < absum / 4


def test_duplicate_index_is_rejected(case):
    inp, rows, ri, rs, rs64 = case
    a = _row_with_room(case)
    gi = ri.copy()
    gi[a, 1] = gi[a, 0]
    with pytest.raises(AssertionError, match="duplicate"):
        parity.within_tolerance(inp, rows, gi, rs, ri, rs64, TOL)


def test_wrong_order_is_rejected(case):
    inp, rows, ri, rs, rs64 = case
    a = _row_with_room(case)
    gi, gs = ri.copy(), rs.copy()
    gi[a, [0, -1]] = gi[a, [-1, 0]]
    gs[a, [0, -1]] = gs[a, [-1, 0]]
    with pytest.raises(AssertionError, match="not ordered"):
        parity.within_tolerance(inp, rows, gi, gs, ri, rs64, TOL)


def test_illegal_index_is_rejected(case):
    inp, rows, ri, rs, rs64 = case
    a = 0
    row = int(rows[a])
    n = inp.prob.legal_count(row)
    nv = int(np.sum(ri[a] >= 0))
    gi = ri.copy()
    gi[a, nv - 1] = n                                # one past the causal position
    with pytest.raises(AssertionError, match="illegal"):
        parity.within_tolerance(inp, rows, gi, rs, ri, rs64, TOL)


def test_lost_entry_is_rejected(case):
    inp, rows, ri, rs, rs64 = case
    a = _row_with_room(case)
    gi, gs = ri.copy(), rs.copy()
    gi[a, -1], gs[a, -1] = -1, -np.inf
    with pytest.raises(AssertionError, match="valid entries"):
        parity.within_tolerance(inp, rows, gi, gs, ri, rs64, TOL)


def test_exact_rule_rejects_any_difference(case):
    _, _, ri, rs, _ = case
    gi, gs = ri.copy(), rs.copy()
    gi[2, 5] += 1
    with pytest.raises(AssertionError):
        parity.exact(gi, rs, ri, rs)
    gs[2, 5] = np.nextafter(gs[2, 5], np.float32(np.inf))
    with pytest.raises(AssertionError):
        parity.exact(ri, gs, ri, rs)
    zi = np.array([[0, -1]], np.int32)
    zs = np.array([[0.0, -np.inf]], np.float32)
    parity.exact(zi, zs, zi, zs)
    with pytest.raises(AssertionError):
        parity.exact(zi, np.array([[-0.0, -np.inf]], np.float32), zi, zs)

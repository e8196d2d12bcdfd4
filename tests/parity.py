"""Comparison rules between the CUDA path and the CPU oracle.

Exact rule (integer-valued inputs, where fp32 accumulation is exact in any
order): indices and scores must be bit-identical, padding included.

Tolerance rule (real-valued inputs).  The north star's "max relative error"
(1e-3 for bf16 operands with fp32 accumulation, 2e-2 for fp8) is taken
relative to max(|I_ref|, nu), with
    nu(t, s) = sum_j |w_tj| ||q_tj|| ||k_s|| / sqrt(d)
the typical magnitude of a score (the Cauchy-Schwarz bound of each dot product
scaled to unaligned d-vectors; oracle.nu_pairs).  A score near zero is then
judged against the size scores of that row have, not against itself.
  - every returned score satisfies |I_gpu - I_ref| <= tol * max(|I_ref|, nu);
  - the returned sets may differ only on tokens s whose reference score lies
    within e(s) + e(kth) of the reference k-th score, e(x) = tol * max(|I_ref(x)|,
    nu(x)): a swap of s with u needs gpu(s) >= gpu(u) while ref(s) <= ref(u), so
    ref(u) - ref(s) <= e(s) + e(u), and both lie that close to the cut-off;
  - the number of valid entries is exactly min(k, |legal|), indices are unique,
    legal, and ordered by (score desc, index asc);
  - the IoU against the reference set and the largest observed
    |I_gpu - I_ref| / max(|I_ref|, nu) are returned (and printed).
"""
from __future__ import annotations

from typing import NamedTuple

import numpy as np

import oracle


def order_rows(idx, score):
    """Order each row by (score desc, index asc), padding (-1, -inf) last."""
    idx = np.asarray(idx)
    score = np.asarray(score)
    oi = np.empty_like(idx)
    os_ = np.empty_like(score)
    for r in range(idx.shape[0]):
        valid = idx[r] >= 0
        order = np.lexsort((idx[r][valid], -score[r][valid].astype(np.float64)))
        nv = int(valid.sum())
        oi[r, :nv] = idx[r][valid][order]
        os_[r, :nv] = score[r][valid][order]
        oi[r, nv:] = -1
        os_[r, nv:] = -np.inf
    return oi, os_


def exact(gpu_idx, gpu_score, ref_idx, ref_score):
    gi, gs = np.asarray(gpu_idx), np.asarray(gpu_score)
    assert np.array_equal(gi, ref_idx), _first_diff(gi, ref_idx)
    both_inf = np.isneginf(gs) & np.isneginf(ref_score)
    assert np.array_equal(gs[~both_inf], ref_score[~both_inf])
    assert not np.any(np.signbit(gs[gs == 0]))


def _first_diff(a, b):
    d = np.argwhere(a != b)
    if len(d) == 0:
        return "shapes differ"
    r = tuple(d[0])
    return f"first difference at {r}: gpu {a[r]} ref {b[r]}"


class Agreement(NamedTuple):
    iou: float        # mean IoU of the GPU set against the reference set
    max_rel: float    # largest |I_gpu - I_ref| / max(|I_ref|, nu) over returned entries


def within_tolerance(inp: oracle.Inputs, rows, gpu_idx, gpu_score, ref_idx, ref_score64, tol,
                     heads=None, legal=None, label="", check_scores=True, score_fn=None):
    """Check the tolerance rule row by row; returns Agreement(iou, max_rel).

    heads: per-row head lists [n_rows, h] for routed scores (None: all heads).
    legal: per-row legal key counts (None: from the problem).
    check_scores=False measures without asserting the score and near-cut-off
    rules (a comparison against operands the GPU did not see, e.g. the
    unquantised values of an fp8 run, whose differences are the quantisation's);
    count, uniqueness, legality and order are still asserted.
    score_fn(a, rows_v, idx) -> fp64 reference scores of row a at the listed keys,
    for methods whose score is not the DSA score over `heads` (LISA's linear term,
    ResMiSA's I^); nu then stays the one of `heads` (None: every head)."""
    p = inp.prob
    ious = []
    max_rel = 0.0
    for a, row in enumerate(rows):
        gi = np.asarray(gpu_idx[a])
        gs = np.asarray(gpu_score[a])
        ri = np.asarray(ref_idx[a])
        nv = int(np.sum(ri >= 0))
        gv = int(np.sum(gi >= 0))
        assert gv == nv, f"row {row}: {gv} valid entries, reference {nv}"
        assert np.all(gi[nv:] == -1) and np.all(np.isneginf(gs[nv:]))
        if nv == 0:
            ious.append(1.0)
            continue
        g_set = gi[:nv]
        assert len(np.unique(g_set)) == nv, f"row {row}: duplicate indices"
        n_legal = p.legal_count(int(row)) if legal is None else int(legal[a])
        assert np.all((g_set >= 0) & (g_set < n_legal)), f"row {row}: illegal index"
        hrow = None if heads is None else np.repeat(np.asarray(heads[a])[None], nv, 0)
        rows_v = np.full(nv, row, np.int64)
        ref_at_g = (oracle.score_pairs(inp, rows_v, g_set, hrow) if score_fn is None
                    else score_fn(a, rows_v, g_set))
        scale_g = np.maximum(np.abs(ref_at_g), oracle.nu_pairs(inp, rows_v, g_set, hrow))
        err = np.abs(gs[:nv].astype(np.float64) - ref_at_g)
        rel = err / scale_g
        max_rel = max(max_rel, float(rel.max()))
        bad = np.argwhere(rel > tol) if check_scores else []
        assert len(bad) == 0, (f"row {row}: score error {err[bad[0][0]]:.3e} > "
                               f"{tol * scale_g[bad[0][0]]:.3e} at s={g_set[bad[0][0]]}")
        # order by (score desc, index asc) on the GPU's own scores
        s0, s1 = gs[: nv - 1], gs[1:nv]
        i0, i1 = g_set[:-1], g_set[1:]
        assert np.all((s0 > s1) | ((s0 == s1) & (i0 < i1))), f"row {row}: output not ordered"
        # set difference only near the reference cutoff
        cutoff = ref_score64[a, nv - 1]
        kth = np.array([ri[nv - 1]], np.int64)
        hk = None if heads is None else np.asarray(heads[a])[None]
        e_kth = tol * max(abs(cutoff), float(oracle.nu_pairs(inp, np.array([row], np.int64),
                                                             kth, hk)[0]))
        extra = np.setdiff1d(g_set, ri[:nv])
        missing = np.setdiff1d(ri[:nv], g_set)
        for group in (extra, missing):
            if len(group) == 0 or not check_scores:
                continue
            rr = np.full(len(group), row, np.int64)
            hh = None if heads is None else np.repeat(np.asarray(heads[a])[None], len(group), 0)
            v = (oracle.score_pairs(inp, rr, group, hh) if score_fn is None
                 else score_fn(a, rr, group))
            e_s = tol * np.maximum(np.abs(v), oracle.nu_pairs(inp, rr, group, hh))
            far = np.abs(v - cutoff) > e_s + e_kth
            assert not np.any(far), (f"row {row}: token {group[far][0]} differs from the "
                                     f"reference set but is not near the cut-off")
        inter = len(np.intersect1d(g_set, ri[:nv]))
        ious.append(inter / (2 * nv - inter))
    res = Agreement(float(np.mean(ious)) if ious else 1.0, max_rel)
    print(f"parity{(' ' + label) if label else ''}: {len(rows)} rows, IoU {res.iou:.4f}, "
          f"max |dI|/max(|I|, nu) {res.max_rel:.3e} (tol {tol:g})")
    return res

"""ctypes wrapper of the plain CPU oracle (dsa_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by the tests, the package smoke check and
the benchmark's CPU-baseline / reference leg, never by the product path.  The
C source shares nothing with the CUDA library.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "dsa_oracle.c")
# DSA_ORACLE_MUTANT=n builds and loads the oracle with planted mistake n (see
# the ORC_MUTANT switches in dsa_oracle.c); only tests/test_oracle_mutants.py
# sets it, to check that the pins reject every such mistake.
MUTANT = int(os.environ.get("DSA_ORACLE_MUTANT", "0"))
LIB = os.path.join(HERE, "libdsa_oracle.so" if MUTANT == 0 else f"libdsa_oracle_m{MUTANT}.so")

F32, BF16, E4M3 = 0, 1, 2
F64 = 3   # oracle-only operand type: values already decoded to fp64 (split_query)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (IEEE semantics: no fast-math, no FMA contraction)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off",
                               "-fno-fast-math", f"-DORC_MUTANT={MUTANT}", "-shared", "-fPIC",
                               SRC, "-o", tmp, "-lm"])
        os.replace(tmp, LIB)
    return LIB


class _Inputs(C.Structure):
    _fields_ = [("batch", C.c_int32), ("n_q", C.c_int32), ("n_k", C.c_int32),
                ("heads", C.c_int32), ("dim", C.c_int32), ("q_dtype", C.c_int32),
                ("k_dtype", C.c_int32), ("q_pos0", C.c_void_p), ("k_len", C.c_void_p),
                ("q", C.c_void_p), ("q_scale", C.c_void_p), ("k", C.c_void_p),
                ("k_scale", C.c_void_p), ("w", C.c_void_p)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        vp, i32, i64 = C.c_void_p, C.c_int32, C.c_int64
        _lib.orc_e4m3_decode.restype = C.c_double
        _lib.orc_e4m3_decode.argtypes = [C.c_uint8]
        _lib.orc_e4m3_encode.restype = C.c_uint8
        _lib.orc_e4m3_encode.argtypes = [C.c_float]
        _lib.orc_quantize_rows.argtypes = [vp, i32, i64, i32, vp, vp]
        _lib.orc_split_query.argtypes = [vp, i32, i64, i32, vp]
        _lib.orc_dsa_rows.argtypes = [vp, i32, vp, i64, vp, vp, vp, vp]
        _lib.orc_score_pairs.argtypes = [vp, vp, vp, i64, vp, i32, vp]
        _lib.orc_nu_pairs.argtypes = [vp, vp, vp, i64, vp, i32, vp]
        _lib.orc_pool.argtypes = [vp, i32, i64, i32, vp]
        _lib.orc_misa_rows.argtypes = [vp, i32, i32, i32, i32, vp, i64, vp, vp, vp, vp, vp, vp,
                                       vp, vp, vp]
        _lib.orc_hisa_rows.argtypes = [vp, i32, i32, i32, i32, i32, vp, i64, vp, vp, vp, vp, vp,
                                       vp, vp, vp, vp]
        _lib.orc_block_scores.restype = C.c_int64
        _lib.orc_block_scores.argtypes = [vp, i64, i32, vp, i32, vp]
        _lib.orc_lisa_rows.argtypes = [vp, i32, i32, vp, i64, vp, vp, vp, vp, vp, vp]
        _lib.orc_resmisa_rows.argtypes = [vp, i32, i32, i32, vp, i64, vp, vp, vp, vp, vp, vp, vp]
        _lib.orc_linear_pairs.argtypes = [vp, vp, vp, i64, vp]
        _lib.orc_resmisa_pairs.argtypes = [vp, vp, vp, i64, vp, i32, vp]
        _lib.orc_sparse_mla.argtypes = [vp, vp, vp, i64, i32, i32, i32, i32, i32, i32,
                                        C.c_double, vp, vp, vp, vp]
        _lib.orc_indexer_backward.argtypes = [vp, vp, vp, i32, vp, vp, vp]
        _lib.orc_residual_bounds.restype = C.c_int64
        _lib.orc_residual_bounds.argtypes = [vp, i64, i32, vp]
        _lib.orc_dosa_bounds.restype = C.c_int64
        _lib.orc_dosa_bounds.argtypes = [vp, i64, i32, vp, vp, vp]
        _lib.orc_dosa_seed.restype = C.c_double
        _lib.orc_dosa_seed.argtypes = [vp, i64, i32, i32]
        _lib.orc_score_row.restype = C.c_int64
        _lib.orc_score_row.argtypes = [vp, i64, vp, i32, vp]
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


class Inputs:
    """Host operands of one problem, pinned for the C calls.

    q / k are float32 (F32), uint16 bf16 words (BF16) or uint8 e4m3 codes (E4M3,
    with q_scale / k_scale)."""

    def __init__(self, prob, q=None, k=None, q_dtype=None, k_dtype=None, q_scale=None,
                 k_scale=None):
        self.prob = prob
        self.q = np.ascontiguousarray(prob.q if q is None else q)
        self.k = np.ascontiguousarray(prob.k if k is None else k)
        self.w = np.ascontiguousarray(prob.w, dtype=np.float32)
        self.q_dtype = prob.q_dtype if q_dtype is None else q_dtype
        self.k_dtype = prob.k_dtype if k_dtype is None else k_dtype
        self.q_scale = None if q_scale is None else np.ascontiguousarray(q_scale, np.float32)
        self.k_scale = None if k_scale is None else np.ascontiguousarray(k_scale, np.float32)
        self.q_pos0 = None if prob.q_pos0 is None else np.ascontiguousarray(prob.q_pos0, np.int32)
        self.k_len = None if prob.k_len is None else np.ascontiguousarray(prob.k_len, np.int32)
        self.s = _Inputs(prob.batch, prob.n_q, prob.n_k, prob.heads, prob.dim, self.q_dtype,
                         self.k_dtype, _p(self.q_pos0), _p(self.k_len), _p(self.q),
                         _p(self.q_scale), _p(self.k), _p(self.k_scale), _p(self.w))

    @property
    def ref(self):
        return C.byref(self.s)


def _rows(prob, rows):
    if rows is None:
        rows = np.arange(prob.batch * prob.n_q, dtype=np.int64)
    return np.ascontiguousarray(rows, dtype=np.int64)


def dsa(inp: Inputs, topk: int, rows=None):
    """Exact DSA top-k rows: (idx int32, score fp32, score fp64, dots int64)."""
    rows = _rows(inp.prob, rows)
    n = len(rows)
    idx = np.empty((n, topk), np.int32)
    sc = np.empty((n, topk), np.float32)
    sc64 = np.empty((n, topk), np.float64)
    dots = np.empty(n, np.int64)
    rc = lib().orc_dsa_rows(inp.ref, topk, _p(rows), n, _p(idx), _p(sc), _p(sc64), _p(dots))
    assert rc == 0
    return idx, sc, sc64, dots


def misa(inp: Inputs, topk: int, block: int, h: int, k_prime: int = 0, rows=None,
         forced_heads=None, forced_pool=None):
    """MISA (k_prime == 0) / MISA-dagger rows.

    Returns dict(idx, score, score64, heads, E, pool, dots)."""
    rows = _rows(inp.prob, rows)
    n, H = len(rows), inp.prob.heads
    out = dict(idx=np.empty((n, topk), np.int32), score=np.empty((n, topk), np.float32),
               score64=np.empty((n, topk), np.float64), heads=np.empty((n, h), np.int32),
               E=np.empty((n, H), np.float64), dots=np.empty(n, np.int64))
    out["pool"] = np.empty((n, k_prime), np.int32) if k_prime > 0 else None
    fh = None if forced_heads is None else np.ascontiguousarray(forced_heads, np.int32)
    fp = None if forced_pool is None else np.ascontiguousarray(forced_pool, np.int32)
    rc = lib().orc_misa_rows(inp.ref, topk, block, h, k_prime, _p(rows), n, _p(fh), _p(fp),
                             _p(out["idx"]), _p(out["score"]), _p(out["score64"]),
                             _p(out["heads"]), _p(out["E"]), _p(out["pool"]), _p(out["dots"]))
    assert rc == 0
    return out


def hisa(inp: Inputs, topk: int, block: int, r: int, route_h: int = 0, route_block: int = 1024,
         rows=None, forced_heads=None, forced_blocks=None):
    """HISA / stacked MISA+HISA rows.  Returns dict(idx, score, score64, blocks, J, heads, dots)."""
    rows = _rows(inp.prob, rows)
    n = len(rows)
    nh = route_h if route_h > 0 else inp.prob.heads
    out = dict(idx=np.empty((n, topk), np.int32), score=np.empty((n, topk), np.float32),
               score64=np.empty((n, topk), np.float64), blocks=np.empty((n, r), np.int32),
               J=np.empty((n, r), np.float64),
               heads=np.empty((n, nh), np.int32) if route_h > 0 else None,
               dots=np.empty(n, np.int64))
    fh = None if forced_heads is None else np.ascontiguousarray(forced_heads, np.int32)
    fb = None if forced_blocks is None else np.ascontiguousarray(forced_blocks, np.int32)
    rc = lib().orc_hisa_rows(inp.ref, topk, block, r, route_h, route_block, _p(rows), n, _p(fh),
                             _p(fb), _p(out["idx"]), _p(out["score"]), _p(out["score64"]),
                             _p(out["blocks"]), _p(out["J"]), _p(out["heads"]), _p(out["dots"]))
    assert rc == 0
    return out


def lisa(inp: Inputs, topk: int, pool_m: int = 0, rows=None, forced_pool=None):
    """Indexer LISA (pool_m == 0: tokens ranked by the linear term l = g . k) or
    LISA-dagger (pool_m > 0: top-pool_m by l reranked by the full I).
    Returns dict(idx, score, score64, pool, dots)."""
    rows = _rows(inp.prob, rows)
    n = len(rows)
    out = dict(idx=np.empty((n, topk), np.int32), score=np.empty((n, topk), np.float32),
               score64=np.empty((n, topk), np.float64), dots=np.empty(n, np.int64),
               pool=np.empty((n, pool_m), np.int32) if pool_m > 0 else None)
    fp = None if forced_pool is None else np.ascontiguousarray(forced_pool, np.int32)
    rc = lib().orc_lisa_rows(inp.ref, topk, pool_m, _p(rows), n, _p(fp), _p(out["idx"]),
                             _p(out["score"]), _p(out["score64"]), _p(out["pool"]),
                             _p(out["dots"]))
    assert rc == 0
    return out


def resmisa(inp: Inputs, topk: int, block: int, r: int, rows=None, forced_heads=None):
    """ResMiSA rows: returns dict(idx, score, score64, heads [n, r], S [n, H], dots)."""
    rows = _rows(inp.prob, rows)
    n, H = len(rows), inp.prob.heads
    out = dict(idx=np.empty((n, topk), np.int32), score=np.empty((n, topk), np.float32),
               score64=np.empty((n, topk), np.float64), heads=np.empty((n, max(r, 1)), np.int32),
               S=np.empty((n, H), np.float64), dots=np.empty(n, np.int64))
    fh = None if forced_heads is None else np.ascontiguousarray(forced_heads, np.int32)
    rc = lib().orc_resmisa_rows(inp.ref, topk, block, r, _p(rows), n, _p(fh), _p(out["idx"]),
                                _p(out["score"]), _p(out["score64"]), _p(out["heads"]),
                                _p(out["S"]), _p(out["dots"]))
    assert rc == 0
    out["heads"] = out["heads"][:, :r]
    return out


def linear_pairs(inp: Inputs, rows, s):
    """fp64 LISA linear terms l = g . k at (rows[a], s[a])."""
    rows = np.ascontiguousarray(rows, np.int64)
    s = np.ascontiguousarray(s, np.int64)
    out = np.empty(len(rows), np.float64)
    lib().orc_linear_pairs(inp.ref, _p(rows), _p(s), len(rows), _p(out))
    return out


def resmisa_pairs(inp: Inputs, rows, s, heads):
    """fp64 ResMiSA scores at (rows[a], s[a]) with residual heads heads[a] ([n, r])."""
    rows = np.ascontiguousarray(rows, np.int64)
    s = np.ascontiguousarray(s, np.int64)
    heads = np.ascontiguousarray(heads, np.int32).reshape(len(rows), -1)
    out = np.empty(len(rows), np.float64)
    lib().orc_resmisa_pairs(inp.ref, _p(rows), _p(s), len(rows), _p(heads), heads.shape[1],
                            _p(out))
    return out


def residual_bounds(inp: Inputs, row: int, block: int):
    """U^- [M_t, H] of one row (the ResMiSA router's per-block residual bounds)."""
    p = inp.prob
    m = (p.n_k + block - 1) // block + 1
    out = np.empty((m, p.heads), np.float64)
    got = lib().orc_residual_bounds(inp.ref, int(row), block, _p(out))
    return out[:got]


def dosa_bounds(inp: Inputs, row: int, shift: int):
    """DoSA block bounds of one row: ([nblk] UB, [nblk] LB, [nblk] rounding
    allowance), blocks of 2^shift keys over the whole sequence; -inf past the
    legal prefix."""
    p = inp.prob
    nblk = (p.n_k + (1 << shift) - 1) >> shift
    ub = np.empty(nblk, np.float64)
    lb = np.empty(nblk, np.float64)
    sl = np.empty(nblk, np.float64)
    got = lib().orc_dosa_bounds(inp.ref, int(row), shift, _p(ub), _p(lb), _p(sl))
    assert got == nblk
    return ub, lb, sl


def dosa_seed(inp: Inputs, row: int, shift: int, keep: int) -> float:
    """DoSA seed-set lower bound of one row's keep-th best score (-inf when the
    row has fewer than keep legal keys)."""
    return float(lib().orc_dosa_seed(inp.ref, int(row), shift, keep))


def score_pairs(inp: Inputs, rows, s, heads=None):
    """fp64 I at (rows[a], s[a]); heads [n, nh] restricts each pair to its head list."""
    rows = np.ascontiguousarray(rows, np.int64)
    s = np.ascontiguousarray(s, np.int64)
    out = np.empty(len(rows), np.float64)
    if heads is not None:
        heads = np.ascontiguousarray(heads, np.int32)
        nh = heads.shape[1]
    else:
        nh = 0
    lib().orc_score_pairs(inp.ref, _p(rows), _p(s), len(rows), _p(heads), nh, _p(out))
    return out


def nu_pairs(inp: Inputs, rows, s, heads=None):
    """nu(t, s) = sum_j |w_tj| ||q_tj|| ||k_s|| / sqrt(d) (fp64): the magnitude
    scale of each score, the denominator of the relative score tolerance."""
    rows = np.ascontiguousarray(rows, np.int64)
    s = np.ascontiguousarray(s, np.int64)
    out = np.empty(len(rows), np.float64)
    if heads is not None:
        heads = np.ascontiguousarray(heads, np.int32)
        nh = heads.shape[1]
    else:
        nh = 0
    lib().orc_nu_pairs(inp.ref, _p(rows), _p(s), len(rows), _p(heads), nh, _p(out))
    return out


def score_row(inp: Inputs, row: int, heads=None):
    """All legal fp64 scores of one row (index = key position)."""
    n = inp.prob.legal_count(row)
    out = np.empty(max(n, 1), np.float64)
    h = None if heads is None else np.ascontiguousarray(heads, np.int32)
    got = lib().orc_score_row(inp.ref, int(row), _p(h), 0 if h is None else len(h), _p(out))
    return out[:got]


def block_scores(inp: Inputs, row: int, block: int, heads=None):
    """HISA coarse scores J of every block of one row's legal prefix (fp64)."""
    n = inp.prob.legal_count(row)
    out = np.empty(max((n + block - 1) // block, 1), np.float64)
    h = None if heads is None else np.ascontiguousarray(heads, np.int32)
    got = lib().orc_block_scores(inp.ref, int(row), block, _p(h), 0 if h is None else len(h),
                                 _p(out))
    return out[:got]


def pool(inp: Inputs, b: int, n: int, block: int):
    m = (n + block - 1) // block
    out = np.empty((m, inp.prob.dim), np.float64)
    lib().orc_pool(inp.ref, b, n, block, _p(out))
    return out


def e4m3_decode(codes) -> np.ndarray:
    f = lib().orc_e4m3_decode
    return np.array([f(int(c)) for c in np.asarray(codes).ravel()], np.float64).reshape(np.shape(codes))


def e4m3_encode(values) -> np.ndarray:
    f = lib().orc_e4m3_encode
    v = np.asarray(values, np.float32)
    return np.array([f(float(x)) for x in v.ravel()], np.uint8).reshape(v.shape)


def quantize_rows(x: np.ndarray, x_dtype: int):
    """Per-row e4m3 quantisation: (codes uint8 [rows, cols], scale fp32 [rows])."""
    x = np.ascontiguousarray(x)
    cols = x.shape[-1]
    rows = x.size // cols
    out = np.empty(x.shape, np.uint8)
    sc = np.empty(x.shape[:-1], np.float32)
    rc = lib().orc_quantize_rows(_p(x), x_dtype, rows, cols, _p(out), _p(sc))
    assert rc == 0
    return out, sc


def split_query(x: np.ndarray, x_dtype: int) -> np.ndarray:
    """Two-part e4m3 value of each query head vector (last axis): s * (hi + lo), fp64."""
    x = np.ascontiguousarray(x)
    dim = x.shape[-1]
    out = np.empty(x.shape, np.float64)
    rc = lib().orc_split_query(_p(x), x_dtype, x.size // dim, dim, _p(out))
    assert rc == 0
    return out


def sparse_mla(q, kv, idx, scale, dv, tps):
    """Naive gather attention over fixed candidate sets (fp64).

    q [T, heads, dqk] and kv [batch, n_k, dqk] as uint16 bf16 words; idx [T, k]
    int32 (-1 empty); token t belongs to sequence t // tps.  Returns dict(o
    [T, heads, dv], lse, max, den [T, heads])."""
    q = np.ascontiguousarray(q, np.uint16)
    kv = np.ascontiguousarray(kv, np.uint16)
    idx = np.ascontiguousarray(idx, np.int32)
    T, H, dqk = q.shape
    n_k = kv.shape[1]
    topk = idx.shape[1]
    out = dict(o=np.empty((T, H, dv), np.float64), lse=np.empty((T, H), np.float64),
               max=np.empty((T, H), np.float64), den=np.empty((T, H), np.float64))
    rc = lib().orc_sparse_mla(_p(q), _p(kv), _p(idx), T, tps, n_k, H, dqk, dv, topk, float(scale),
                              _p(out["o"]), _p(out["lse"]), _p(out["max"]), _p(out["den"]))
    assert rc == 0
    return out


def indexer_backward(inp: Inputs, sel, grad):
    """Gradients of sum_{t, s in S_t} g_{t,s} I_{t,s}: dict(dq [rows, H, d],
    dk [batch, n_k, d], dw [rows, H]) in fp64."""
    p = inp.prob
    sel = np.ascontiguousarray(sel, np.int32).reshape(p.batch * p.n_q, -1)
    grad = np.ascontiguousarray(grad, np.float32).reshape(sel.shape)
    out = dict(dq=np.empty((p.batch * p.n_q, p.heads, p.dim)),
               dk=np.empty((p.batch, p.n_k, p.dim)), dw=np.empty((p.batch * p.n_q, p.heads)))
    rc = lib().orc_indexer_backward(inp.ref, _p(sel), _p(grad), sel.shape[1], _p(out["dq"]),
                                    _p(out["dk"]), _p(out["dw"]))
    assert rc == 0
    return out

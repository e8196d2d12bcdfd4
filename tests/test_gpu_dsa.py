"""GPU parity of dsa_index (and the FP8 quantiser) against the CPU oracle.

Exact on integer-valued inputs; within the tolerance rule of tests/parity.py on
real-valued inputs: 1e-3 of max(|I|, nu) against the oracle on the operands the
GPU computes with (bf16, or the same e4m3 codes and scales, or the two-part
e4m3 value of a bf16 query against e4m3 keys).  Against the unquantised values
an fp8 run differs by its quantisation error, which is measured and reported
(IoU floor, largest relative difference) rather than asserted.  Sizes span several 128-key tiles and query tiles with
ragged tails; full-size workloads are checked on sampled rows.
"""
import numpy as np
import pytest

import oracle
import parity
from sparse_attention_token_dsa_b200 import inputs as gen

pytestmark = pytest.mark.gpu

TOL_BF16 = 1e-3
TOL_FP8 = 2e-2


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


def run_dsa(B, p, q=None, k=None, q_scale=None, k_scale=None, flags=0):
    """GPU top-k rows; without DSA_FLAG_SORTED the set is ordered on the host."""
    q = dev(p.q) if q is None else q
    k = dev(p.k) if k is None else k
    idx, sc = B.dsa_index(q, k, dev(p.w), p.topk, q_scale=q_scale, k_scale=k_scale,
                          q_pos0=dev(p.q_pos0), k_len=dev(p.k_len), flags=flags)
    import torch
    torch.cuda.synchronize()
    gi = idx.cpu().numpy().reshape(-1, p.topk)
    gs = sc.cpu().numpy().reshape(-1, p.topk)
    if not flags & B.DSA_FLAG_SORTED:
        gi, gs = parity.order_rows(gi, gs)
    return gi, gs


# ------------------------------------------------------------------ exact ---

@pytest.mark.parametrize("dtype", [gen.F32, gen.BF16])
def test_integer_full_layer_bit_exact(B, dtype):
    """L = 1024 causal, H = 64, d = 128, k = 128, integer q, k, w: bit-exact,
    including the (score desc, index asc) order requested by DSA_FLAG_SORTED."""
    p = gen.integer_problem(1, 1, 1024, 1024, 64, 128, 128, dtype=dtype)
    gi, gs = run_dsa(B, p, flags=B.DSA_FLAG_CHECK | B.DSA_FLAG_SORTED)
    ri, rs, _, _ = oracle.dsa(oracle.Inputs(p), p.topk)
    parity.exact(gi, gs, ri, rs)


@pytest.mark.parametrize("heads", [8, 16, 32, 128])
def test_integer_heads_bit_exact(B, heads):
    p = gen.integer_problem(2, 1, 300, 700, heads, 128, 64, q_pos0=[400], dtype=gen.BF16)
    gi, gs = run_dsa(B, p)
    ri, rs, _, _ = oracle.dsa(oracle.Inputs(p), p.topk)
    parity.exact(gi, gs, ri, rs)


def test_integer_ragged_batches_bit_exact(B):
    """Several sequences, per-sequence query offsets and key lengths, rows with
    fewer legal keys than k (padding), tails in both tiles."""
    p = gen.integer_problem(3, 3, 150, 500, 64, 128, 200, q_pos0=[0, 100, 37],
                            k_len=[300, 500, 200], dtype=gen.BF16)
    gi, gs = run_dsa(B, p)
    ri, rs, _, _ = oracle.dsa(oracle.Inputs(p), p.topk)
    parity.exact(gi, gs, ri, rs)


def test_integer_topk_above_keys_pads(B):
    p = gen.integer_problem(4, 1, 40, 300, 64, 128, 512, dtype=gen.F32)
    gi, gs = run_dsa(B, p)
    ri, rs, _, _ = oracle.dsa(oracle.Inputs(p), p.topk)
    parity.exact(gi, gs, ri, rs)
    assert np.all(gi[:, 300:] == -1)


@pytest.mark.parametrize("flags", [0, 2])
def test_integer_many_ties_long_rows_bit_exact(B, flags):
    """Small value range => massive score ties; exact raises and the tie fallback."""
    p = gen.integer_problem(5, 1, 64, 20000, 64, 128, 1024, qk_max=1, w_max=1, dtype=gen.BF16)
    gi, gs = run_dsa(B, p, flags=flags)
    ri, rs, _, _ = oracle.dsa(oracle.Inputs(p), p.topk)
    parity.exact(gi, gs, ri, rs)


@pytest.mark.parametrize("topk", [2048, 4096, 8192])
def test_integer_sorted_large_topk_bit_exact(B, topk):
    """Ordered output with several keys per select thread: rows just below and
    just above topk legal keys (every candidate a winner / a real selection)."""
    p = gen.integer_problem(7, 1, 64, 12000, 64, 128, topk, q_pos0=[topk - 32], dtype=gen.BF16)
    gi, gs = run_dsa(B, p, flags=B.DSA_FLAG_SORTED)
    ri, rs, _, _ = oracle.dsa(oracle.Inputs(p), p.topk)
    parity.exact(gi, gs, ri, rs)


def test_single_key_and_single_query(B):
    p = gen.integer_problem(6, 2, 1, 1, 64, 128, 4, dtype=gen.F32)
    gi, gs = run_dsa(B, p)
    ri, rs, _, _ = oracle.dsa(oracle.Inputs(p), p.topk)
    parity.exact(gi, gs, ri, rs)


# -------------------------------------------------------------- real-valued --

def test_bf16_real_small(B):
    p = gen.normal_problem(20, 2, 1000, 1300, 64, 128, 256, q_pos0=[300, 0], k_len=[1300, 1000])
    gi, gs = run_dsa(B, p)
    inp = oracle.Inputs(p)
    rows = np.arange(p.batch * p.n_q)[::7]
    ri, _, rs64, _ = oracle.dsa(inp, p.topk, rows)
    r = parity.within_tolerance(inp, rows, gi[rows], gs[rows], ri, rs64, TOL_BF16)
    assert r.iou > 0.99


def test_bf16_needles_32k_sampled(B):
    """Full-size 32K prefill layer (H = 64, k = 2048) with planted needles."""
    p = gen.normal_problem(2, 1, 32768, 32768, 64, 128, 2048, n_needles=32)
    gi, gs = run_dsa(B, p)
    inp = oracle.Inputs(p)
    rows = gen.stratified_rows(p, 24)
    ri, _, rs64, _ = oracle.dsa(inp, p.topk, rows)
    r = parity.within_tolerance(inp, rows, gi[rows], gs[rows], ri, rs64, TOL_BF16)
    assert r.iou > 0.99
    for b, t, s in zip(p.needles["b"], p.needles["t"], p.needles["s"]):
        assert s in set(gi[b * p.n_q + t].tolist()), "needle not selected"


# ---------------------------------------------------------------------- FP8 --

def test_quantizer_matches_oracle_bit_exact(B):
    import torch
    rng = np.random.default_rng(3)
    x = rng.standard_normal((777, 128)).astype(np.float32)
    x[5] = 0.0
    x[6] *= 1e-6
    x[7] *= 1e4
    x[8, :5] = [448.0, -448.0, 1e-12, -0.0, 3.0]
    for dt, arr in ((gen.F32, x), (gen.BF16, gen.f32_to_bf16_bits(x))):
        codes, sc = B.dsa_quantize_e4m3(dev(arr))
        torch.cuda.synchronize()
        rc, rsc = oracle.quantize_rows(arr, dt)
        assert np.array_equal(sc.cpu().numpy(), rsc)
        assert np.array_equal(codes.cpu().numpy(), rc)


def _fp8_problem(p, B):
    """GPU-quantised operands (checked bit-exact against the oracle's quantiser)."""
    qd, kd = dev(p.q), dev(p.k)
    qc, qs = B.dsa_quantize_e4m3(qd.reshape(p.batch * p.n_q, p.heads * p.dim))
    kc, ks = B.dsa_quantize_e4m3(kd)
    rqc, rqs = oracle.quantize_rows(p.q.reshape(p.batch * p.n_q, -1), gen.BF16)
    rkc, rks = oracle.quantize_rows(p.k, gen.BF16)
    assert np.array_equal(qc.cpu().numpy(), rqc) and np.array_equal(kc.cpu().numpy(), rkc)
    return qc.reshape(p.q.shape), qs, kc, ks, rqc.reshape(p.q.shape), rqs, rkc, rks


def test_fp8_prefill(B):
    p = gen.normal_problem(21, 1, 2048, 2048, 64, 128, 256)
    qc, qs, kc, ks, rqc, rqs, rkc, rks = _fp8_problem(p, B)
    gi, gs = run_dsa(B, p, q=qc, k=kc, q_scale=qs, k_scale=ks, flags=B.DSA_FLAG_CHECK)
    rows = np.arange(p.n_q)[::5]
    # quantisation-faithful: oracle on the same e4m3 codes
    inq = oracle.Inputs(p, q=rqc, k=rkc, q_dtype=gen.E4M3, k_dtype=gen.E4M3, q_scale=rqs,
                        k_scale=rks)
    ri, _, rs64, _ = oracle.dsa(inq, p.topk, rows)
    r = parity.within_tolerance(inq, rows, gi[rows], gs[rows], ri, rs64, TOL_BF16,
                                label="same e4m3 operands")
    assert r.iou > 0.99
    # against the unquantised bf16 values: the quantisation's own effect
    inp = oracle.Inputs(p)
    ri, _, rs64, _ = oracle.dsa(inp, p.topk, rows)
    r = parity.within_tolerance(inp, rows, gi[rows], gs[rows], ri, rs64, TOL_FP8,
                                label="vs unquantised", check_scores=False)
    assert r.iou > 0.9 and r.max_rel < 0.05


def _check_split_decode(p, gi, gs, rkc, rks):
    """bf16 query against e4m3 keys: 1e-3 against the oracle on the operands the
    MMA sees (the query's two-part e4m3 value, oracle.split_query, and the same
    key codes and scales); the bf16 query itself differs by the split's own
    rounding (at most 2^-8 per value), reported against the 2e-2 fp8 figure."""
    rows = np.arange(p.batch * p.n_q)
    qsplit = oracle.split_query(p.q.reshape(-1, p.dim), gen.BF16).reshape(p.q.shape)
    ins = oracle.Inputs(p, q=qsplit, q_dtype=oracle.F64, k=rkc, k_dtype=gen.E4M3, k_scale=rks)
    ri, _, rs64, _ = oracle.dsa(ins, p.topk, rows)
    r = parity.within_tolerance(ins, rows, gi, gs, ri, rs64, TOL_BF16, label="split query")
    assert r.iou > 0.99
    inq = oracle.Inputs(p, k=rkc, k_dtype=gen.E4M3, k_scale=rks)
    ri, _, rs64, _ = oracle.dsa(inq, p.topk, rows)
    r = parity.within_tolerance(inq, rows, gi, gs, ri, rs64, TOL_FP8, label="bf16 query")
    assert r.iou > 0.95


@pytest.mark.parametrize("batch,n_k", [(4, 20000), (3, 5000)])
def test_fp8_decode_split_query(B, batch, n_k):
    """Decode: bf16 q (split into two e4m3 parts inside the library), e4m3 keys."""
    p, _ = gen.decode_problem(30 + batch, batch, n_k, 64, 128, 2048,
                              k_len=[n_k - 37 * b for b in range(batch)])
    kc, ks = B.dsa_quantize_e4m3(dev(p.k))
    gi, gs = run_dsa(B, p, k=kc, k_scale=ks)
    rkc, rks = oracle.quantize_rows(p.k, gen.BF16)
    assert np.array_equal(kc.cpu().numpy(), rkc)
    _check_split_decode(p, gi, gs, rkc, rks)


@pytest.mark.parametrize("batch,n_k", [(5, 9000), (3, 3001), (2, 200)])
def test_integer_e4m3_decode_bit_exact(B, batch, n_k):
    """Decode with e4m3 q and k holding small integers (exact codes, unit scales):
    the split-K scan and merge are bit-exact.  Ragged prefixes give key chunks
    with odd tile counts, so a pipeline unit of two key tiles ends half full."""
    k_len = [n_k - 131 * b for b in range(batch)]
    p = gen.integer_problem(40 + batch, batch, 1, n_k, 64, 128, 2048,
                            q_pos0=[n - 1 for n in k_len], k_len=k_len)
    qc = oracle.e4m3_encode(p.q)
    kc = oracle.e4m3_encode(p.k)
    assert np.array_equal(oracle.e4m3_decode(qc), p.q) and np.array_equal(oracle.e4m3_decode(kc), p.k)
    qs = np.ones((batch, 1), np.float32)
    ks = np.ones((batch, n_k), np.float32)
    gi, gs = run_dsa(B, p, q=dev(qc), k=dev(kc), q_scale=dev(qs), k_scale=dev(ks),
                     flags=B.DSA_FLAG_CHECK)
    inq = oracle.Inputs(p, q=qc, k=kc, q_dtype=gen.E4M3, k_dtype=gen.E4M3, q_scale=qs,
                        k_scale=ks)
    ri, rs, _, _ = oracle.dsa(inq, p.topk)
    parity.exact(gi, gs, ri, rs)


def test_fp8_decode_full_size(B):
    """32 sequences x 131072 cached keys, H = 64, k = 2048 (every row checked)."""
    p, _ = gen.decode_problem(3, 32, 131072, 64, 128, 2048)
    kc, ks = B.dsa_quantize_e4m3(dev(p.k))
    gi, gs = run_dsa(B, p, k=kc, k_scale=ks)
    rkc, rks = oracle.quantize_rows(p.k, gen.BF16)
    _check_split_decode(p, gi, gs, rkc, rks)


def test_check_flag_reports_bad_scale(B):
    import torch
    p = gen.normal_problem(22, 1, 64, 256, 64, 128, 16)
    qc, qs, kc, ks, *_ = _fp8_problem(p, B)
    ks[0, 3] = float("nan")
    with pytest.raises(B.DsaError) as e:
        B.dsa_index(qc, kc, dev(p.w), p.topk, q_scale=qs, k_scale=ks, flags=B.DSA_FLAG_CHECK)
    assert e.value.status == B.DSA_ERR_NONFINITE
    torch.cuda.synchronize()


# ------------------------------------------------------------ failure path --

def test_expired_wait_returns_timeout_then_next_call_is_exact(B):
    """DSA_FLAG_TEST_STALL makes the first CTA withhold one stage of keys and
    shortens every bounded wait to about a millisecond: the wait on that stage
    runs out, the call returns DSA_ERR_TIMEOUT within a fraction of a second,
    the select writes padding rows, and the next call on the same stream and
    workspace is bit-exact.  Nothing traps or hangs: every role drains its own
    copies and MMAs and exits."""
    import time
    import torch
    p = gen.integer_problem(8, 1, 1024, 1024, 64, 128, 128, dtype=gen.BF16)
    q, k, w = dev(p.q), dev(p.k), dev(p.w)
    prob = B.problem(q, k, p.topk)
    ws = torch.empty(B.dsa_workspace_size(prob), dtype=torch.uint8, device="cuda")
    idx = torch.full((1, p.n_q, p.topk), 7, dtype=torch.int32, device="cuda")
    sc = torch.full((1, p.n_q, p.topk), 7.0, dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    with pytest.raises(B.DsaError) as e:
        B.dsa_index(q, k, w, p.topk, flags=B.DSA_FLAG_CHECK | B.DSA_FLAG_TEST_STALL,
                    out=(idx, sc), workspace=ws)
    took = time.perf_counter() - t0
    assert e.value.status == B.DSA_ERR_TIMEOUT
    assert took < 1.0, f"the failed call took {took:.3f} s"
    assert B.dsa_read_status(ws) == B.DSA_ERR_TIMEOUT
    assert torch.all(idx == -1).item() and torch.all(torch.isneginf(sc)).item()
    # the same stream and workspace, a normal call: exact
    B.dsa_index(q, k, w, p.topk, flags=B.DSA_FLAG_CHECK | B.DSA_FLAG_SORTED, out=(idx, sc),
                workspace=ws)
    torch.cuda.synchronize()
    assert B.dsa_read_status(ws) == B.DSA_OK
    ri, rs, _, _ = oracle.dsa(oracle.Inputs(p), p.topk)
    parity.exact(idx.cpu().numpy().reshape(-1, p.topk), sc.cpu().numpy().reshape(-1, p.topk),
                 ri, rs)


@pytest.mark.parametrize("topk", [128, 2048])
def test_position_order_bit_exact(B, topk):
    """DSA_FLAG_BY_POSITION: each row is the oracle's top-k set in ascending token
    order, scores carried with their tokens, padding last."""
    p = gen.integer_problem(9, 2, 200, 3000, 64, 128, topk, q_pos0=[2800, 100],
                            k_len=[3000, 2500], dtype=gen.BF16)
    idx, sc = B.dsa_index(dev(p.q), dev(p.k), dev(p.w), p.topk, q_pos0=dev(p.q_pos0),
                          k_len=dev(p.k_len), flags=B.DSA_FLAG_BY_POSITION | B.DSA_FLAG_CHECK)
    import torch
    torch.cuda.synchronize()
    gi = idx.cpu().numpy().reshape(-1, p.topk)
    gs = sc.cpu().numpy().reshape(-1, p.topk)
    ri, rs, _, _ = oracle.dsa(oracle.Inputs(p), p.topk)
    for r in range(len(ri)):
        nv = int(np.sum(ri[r] >= 0))
        order = np.argsort(ri[r][:nv], kind="stable")
        assert np.array_equal(gi[r][:nv], ri[r][:nv][order])
        assert np.array_equal(gs[r][:nv], rs[r][:nv][order])
        assert np.all(gi[r][nv:] == -1) and np.all(np.isneginf(gs[r][nv:]))


@pytest.mark.parametrize("dosa", [False, True])
def test_integer_empty_cache_and_positions_past_the_cache(B, dosa):
    """A sequence with an empty cache (k_len = 0: every row pads), rows whose
    positions lie past their sequence's cache (all k_len keys legal), and an
    ordinary sequence, in one call; with and without DoSA."""
    p = gen.integer_problem(30, 3, 200, 900, 64, 128, 64, q_pos0=[0, 700, 100],
                            k_len=[0, 300, 900], dtype=gen.BF16)
    flags = B.DSA_FLAG_CHECK | B.DSA_FLAG_SORTED | (B.DSA_FLAG_DOSA if dosa else 0)
    gi, gs = run_dsa(B, p, flags=flags)
    ri, rs, _, _ = oracle.dsa(oracle.Inputs(p), p.topk)
    parity.exact(gi, gs, ri, rs)
    assert np.all(gi[:p.n_q] == -1) and np.all(np.isneginf(gs[:p.n_q]))

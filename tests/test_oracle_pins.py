"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test fixes the oracle to something the pages print (worked example, cost
arithmetic), to a closed form, to an identity between the definitions
(MISA with h = H is DSA, HISA keeping every block is DSA, MISA-dagger with
k' >= L is DSA), to brute-force ranking on tiny inputs, to the OCP E4M3
definition, or to the FP8 margin bound of the pages.  CPU only.
"""
import json
import math
import os

import numpy as np
import pytest

from sparse_attention_token_dsa_b200 import inputs as gen

GOLD = os.path.join(os.path.dirname(__file__), "golden")
F32, BF16, E4M3 = gen.F32, gen.BF16, gen.E4M3


def make(q, k, w, topk, q_pos0=None, k_len=None, dtype=F32):
    q = np.asarray(q, np.float32)
    k = np.asarray(k, np.float32)
    w = np.asarray(w, np.float32)
    B, nq, H, d = q.shape
    nk = k.shape[1]
    if dtype == BF16:
        q, k = gen.f32_to_bf16_bits(q), gen.f32_to_bf16_bits(k)
    return gen.Problem(B, nq, nk, H, d, topk, dtype, dtype, q, k, w,
                       None if q_pos0 is None else np.asarray(q_pos0, np.int32),
                       None if k_len is None else np.asarray(k_len, np.int32))


# ------------------------------------------------------------ worked example --

def test_worked_example_score(oracle_mod):
    g = json.load(open(os.path.join(GOLD, "worked_example.json")))
    p = make(np.array(g["q"])[None, None], np.array(g["k"])[None, None],
             np.array(g["w"])[None, None], topk=1)
    inp = oracle_mod.Inputs(p)
    idx, sc, sc64, _ = oracle_mod.dsa(inp, 1)
    assert idx[0, 0] == 0
    assert sc64[0, 0] == g["score"]
    assert sc[0, 0] == np.float32(g["score"])


# --------------------------------------------------------------- closed forms --

def _line_problem(nq, nk, coeffs, w, sign=+1.0, topk=8, q_pos0=None, k_len=None):
    """q_{t,j} = c_{t,j} e_0, k_s = sign * s * e_0 (d = 4).  Then
    I_{t,s} = s * sum_j w_{t,j} max(sign * c_{t,j}, 0) for s >= 0."""
    d = 4
    q = np.zeros((1, nq, len(coeffs[0]), d), np.float32)
    q[0, :, :, 0] = coeffs
    k = np.zeros((1, nk, d), np.float32)
    k[0, :, 0] = sign * np.arange(nk)
    return make(q, k, np.asarray(w, np.float32)[None], topk, q_pos0, k_len)


@pytest.mark.parametrize("sign", [+1.0, -1.0])
def test_closed_form_line(oracle_mod, sign):
    rng = np.random.default_rng(5)
    nq, nk, H, topk = 12, 40, 6, 8
    c = rng.integers(-3, 4, size=(nq, H)).astype(np.float32)
    w = rng.integers(-2, 3, size=(nq, H)).astype(np.float32)
    p = _line_problem(nq, nk, c, w, sign, topk)
    idx, sc, sc64, _ = oracle_mod.dsa(oracle_mod.Inputs(p), topk)
    for i in range(nq):
        pos = nk - nq + i
        A = float(np.sum(w[i] * np.maximum(sign * c[i], 0.0)))
        legal = np.arange(pos + 1)
        if A > 0:
            want = legal[::-1][:topk]            # largest positions
        else:
            want = legal[:topk]                  # A <= 0: s = 0 first, ties by index
        assert list(idx[i]) == list(want), (i, A)
        assert np.array_equal(sc64[i], want * A + 0.0)


def test_closed_form_causal_short_rows_and_padding(oracle_mod):
    # queries at positions 0..5 with topk 8: rows hold pos+1 entries then padding
    c = np.ones((6, 2), np.float32)
    w = np.ones((6, 2), np.float32)
    p = _line_problem(6, 6, c, w, +1.0, topk=8, q_pos0=[0])
    idx, sc, _, _ = oracle_mod.dsa(oracle_mod.Inputs(p), 8)
    for i in range(6):
        assert list(idx[i, : i + 1]) == list(range(i, -1, -1))
        assert np.all(idx[i, i + 1:] == -1)
        assert np.all(np.isneginf(sc[i, i + 1:]))
        assert np.array_equal(sc[i, : i + 1], 2.0 * np.arange(i, -1, -1))


def test_closed_form_k_len_limits_rows(oracle_mod):
    c = np.ones((4, 2), np.float32)
    w = np.ones((4, 2), np.float32)
    p = _line_problem(4, 20, c, w, +1.0, topk=5, k_len=[10])
    idx, _, _, dots = oracle_mod.dsa(oracle_mod.Inputs(p), 5)
    assert np.all(idx[:, 0] == 9)              # key 9 is the last legal one
    assert np.all(dots == 2 * 10)


def test_negative_zero_written_as_positive(oracle_mod):
    # w < 0 with ReLU = 0 gives -0.0 in IEEE arithmetic; the output is +0.0
    q = np.array([[[[1.0, 0, 0, 0]]]], np.float32)
    k = np.array([[[-1.0, 0, 0, 0], [-2.0, 0, 0, 0]]], np.float32)
    p = make(q, k, np.array([[[-1.0]]], np.float32), topk=2, q_pos0=[1])
    _, sc, _, _ = oracle_mod.dsa(oracle_mod.Inputs(p), 2)
    assert np.all(sc == 0.0) and not np.any(np.signbit(sc))


# ---------------------------------------------------------- brute-force ranks --

@pytest.mark.parametrize("seed", range(6))
def test_bruteforce_ranking_tiny(oracle_mod, seed):
    """n <= 32: rank(s) = #{s' beating s}; the top-k are the ranks < k in rank order."""
    rng = np.random.default_rng(seed)
    B, nq, nk, H, d = 2, 7, 23, 4, 8
    topk = int(rng.integers(1, 12))
    q = rng.integers(-2, 3, size=(B, nq, H, d)).astype(np.float32)
    k = rng.integers(-2, 3, size=(B, nk, d)).astype(np.float32)
    w = rng.integers(-2, 3, size=(B, nq, H)).astype(np.float32)
    p = make(q, k, w, topk, q_pos0=[3, 16], k_len=[nk, 19])
    inp = oracle_mod.Inputs(p)
    idx, sc, _, _ = oracle_mod.dsa(inp, topk)
    for row in range(B * nq):
        n = p.legal_count(row)
        s_all = np.arange(n)
        I = oracle_mod.score_pairs(inp, np.full(n, row), s_all)
        rank = np.array([np.sum((I > I[s]) | ((I == I[s]) & (s_all < s))) for s in s_all])
        want = [int(s_all[rank == r][0]) for r in range(min(topk, n))]
        assert list(idx[row, : len(want)]) == want
        assert np.all(idx[row, len(want):] == -1)


def test_invariants_random(oracle_mod):
    p = gen.normal_problem(90, 2, 33, 70, 8, 16, topk=16, q_pos0=[37, 0], k_len=[70, 20])
    inp = oracle_mod.Inputs(p)
    idx, sc, sc64, _ = oracle_mod.dsa(inp, 16)
    for row in range(p.batch * p.n_q):
        b, i = divmod(row, p.n_q)
        n = p.legal_count(row)
        valid = idx[row][idx[row] >= 0]
        assert len(valid) == min(16, n)
        assert len(set(valid.tolist())) == len(valid)
        assert np.all(valid <= p.pos0(b) + i) and np.all(valid < p.klen(b))
        v = sc64[row, : len(valid)]
        order_ok = np.all((v[:-1] > v[1:]) | ((v[:-1] == v[1:]) & (valid[:-1] < valid[1:])))
        assert order_ok


# -------------------------------------------------------- reduction identities --

def _real_problem(seed, nq=40, nk=300, H=8, d=16, topk=12, B=1):
    return gen.normal_problem(seed, B, nq, nk, H, d, topk)


def test_misa_with_all_heads_is_dsa(oracle_mod):
    p = _real_problem(11)
    inp = oracle_mod.Inputs(p)
    ref = oracle_mod.dsa(inp, p.topk)
    m = oracle_mod.misa(inp, p.topk, block=32, h=p.heads)
    assert np.array_equal(m["idx"], ref[0]) and np.array_equal(m["score64"], ref[2])
    assert np.all(m["heads"] == np.arange(p.heads))


def test_misa_dagger_with_full_pool_is_dsa(oracle_mod):
    p = _real_problem(12)
    inp = oracle_mod.Inputs(p)
    ref = oracle_mod.dsa(inp, p.topk)
    m = oracle_mod.misa(inp, p.topk, block=32, h=2, k_prime=p.n_k)
    assert np.array_equal(m["idx"], ref[0]) and np.array_equal(m["score64"], ref[2])


def test_misa_dagger_pool_of_k_keeps_misa_set(oracle_mod):
    p = _real_problem(13)
    inp = oracle_mod.Inputs(p)
    a = oracle_mod.misa(inp, p.topk, block=32, h=3)
    b = oracle_mod.misa(inp, p.topk, block=32, h=3, k_prime=p.topk)
    for r in range(p.n_q):
        assert set(a["idx"][r]) == set(b["idx"][r])
    full = oracle_mod.score_pairs(inp, np.repeat(np.arange(p.n_q), p.topk),
                                  np.where(b["idx"] < 0, 0, b["idx"]).ravel())
    mask = b["idx"].ravel() >= 0
    assert np.array_equal(b["score64"].ravel()[mask], full[mask])


@pytest.mark.parametrize("blk", [1, 8, 64])
def test_hisa_keeping_every_block_is_dsa(oracle_mod, blk):
    p = _real_problem(14)
    inp = oracle_mod.Inputs(p)
    ref = oracle_mod.dsa(inp, p.topk)
    r_all = -(-p.n_k // blk)
    h = oracle_mod.hisa(inp, p.topk, block=blk, r=r_all)
    assert np.array_equal(h["idx"], ref[0]) and np.array_equal(h["score64"], ref[2])


def test_hisa_block_one_rerank_is_dsa_on_kept_tokens(oracle_mod):
    # b = 1: representatives are the keys themselves (rounded to their own type,
    # a no-op), so the coarse score is I itself and keeping r >= k blocks returns the DSA top-k
    p = _real_problem(15)
    inp = oracle_mod.Inputs(p)
    ref = oracle_mod.dsa(inp, p.topk)
    h = oracle_mod.hisa(inp, p.topk, block=1, r=p.topk)
    assert np.array_equal(h["idx"], ref[0])


def test_stacked_with_all_heads_is_hisa(oracle_mod):
    p = _real_problem(16)
    inp = oracle_mod.Inputs(p)
    a = oracle_mod.hisa(inp, p.topk, block=16, r=6)
    b = oracle_mod.hisa(inp, p.topk, block=16, r=6, route_h=p.heads, route_block=64)
    assert np.array_equal(a["idx"], b["idx"]) and np.array_equal(a["score64"], b["score64"])


# ------------------------------------------------------------ pooling / router --

def test_pool_block_constant_keys_exact(oracle_mod):
    rng = np.random.default_rng(3)
    d, blk, nk = 8, 16, 100
    const = gen.bf16_bits_to_f32(gen.f32_to_bf16_bits(rng.standard_normal((7, d)).astype(np.float32)))
    k = np.repeat(const, blk, axis=0)[:nk][None]
    p = make(np.zeros((1, 1, 8, d)), k, np.ones((1, 1, 8)), 4, dtype=BF16)
    reps = oracle_mod.pool(oracle_mod.Inputs(p), 0, nk, blk)
    assert np.array_equal(reps, const[: reps.shape[0]].astype(np.float64))


def test_pool_ramp_mean_closed_form(oracle_mod):
    d, blk, n = 4, 8, 37
    k = np.zeros((1, 64, d), np.float32)
    k[0, :, 0] = np.arange(64)
    p = make(np.zeros((1, 1, 8, d)), k, np.ones((1, 1, 8)), 4)
    reps = oracle_mod.pool(oracle_mod.Inputs(p), 0, n, blk)
    for b in range(reps.shape[0]):
        lo, hi = b * blk, min((b + 1) * blk, n)
        assert reps[b, 0] == (lo + hi - 1) / 2.0
        assert np.all(reps[b, 1:] == 0.0)


def test_pool_rounds_the_mean_once_to_the_key_type(oracle_mod):
    """A representative is the exact block mean, rounded once (to nearest even)
    to the key storage type: bf16 keys 1 and 1 + 2^-7 average to 1 + 2^-8, a
    tie between bf16 neighbours that rounds to 1; 1 and 1 + 3 * 2^-7 average to
    1 + 1.5 * 2^-7, a tie that rounds up to the even 1 + 2^-6.  fp32 keys 1 and
    1 + 2^-23 average to a tie that rounds to 1."""
    d = 2
    k = np.array([[[1.0, 1.0], [1.0 + 2**-7, 1.0 + 3 * 2**-7]]], np.float32)
    p = make(np.zeros((1, 1, 8, d)), k, np.ones((1, 1, 8)), 1, dtype=BF16)
    reps = oracle_mod.pool(oracle_mod.Inputs(p), 0, 2, 2)
    assert reps[0, 0] == 1.0 and reps[0, 1] == 1.0 + 2**-6
    k = np.array([[[1.0, 3.0], [1.0 + 2**-23, 3.0]]], np.float32)
    p = make(np.zeros((1, 1, 8, d)), k, np.ones((1, 1, 8)), 1)
    reps = oracle_mod.pool(oracle_mod.Inputs(p), 0, 2, 2)
    assert reps[0, 0] == 1.0 and reps[0, 1] == 3.0


def test_misa_scores_tokens_with_the_routed_heads(oracle_mod):
    """MISA, closed form (d = 2, two heads, h = 1): the router keeps head 0
    (S_0 = 10.5 > S_1 = 2.5 over the two blocks of 2 keys), and the token
    scores use head 0 only: 10, 0, 10, 1 for keys (1, 0), (0, 5), (1, 0),
    (0.1, 0), so the top 3 are tokens 0, 2, 3 (all heads would give 10, 5, 10,
    1 and pick token 1 instead of 3).  E = S / M_t with M_t = 2."""
    q = np.array([[[[10.0, 0.0], [0.0, 1.0]]]], np.float32)
    k = np.array([[[1.0, 0.0], [0.0, 5.0], [1.0, 0.0], [0.1, 0.0]]], np.float32)
    w = np.ones((1, 1, 2), np.float32)
    p = make(q, k, w, 3, q_pos0=[3])
    out = oracle_mod.misa(oracle_mod.Inputs(p), 3, block=2, h=1)
    assert out["heads"].tolist() == [[0]]
    assert out["idx"].tolist() == [[0, 2, 3]]
    assert out["score64"][0].tolist() == [10.0, 10.0, float(np.float32(0.1)) * 10.0]
    rep1 = float(np.float32((np.float64(np.float32(0.1)) + 1.0) / 2.0))   # fp32 mean of 1 and 0.1f
    assert out["E"][0].tolist() == [(10.0 * 0.5 + 10.0 * rep1) / 2.0, 2.5 / 2.0]


def test_stacked_hisa_reranks_with_the_routed_heads(oracle_mod):
    """Stacked MISA + HISA, closed form (d = 2, two heads, h = 1): the router
    keeps head 0, so the rerank scores only w_0 ReLU(q_0 . k_s).

    q_0 = (10, 0), q_1 = (0, 1), w = (1, 1); keys (1, 0), (0, 5), (1, 0),
    (0.1, 0); the query sits at position 3.  Router blocks of 2: means
    (0.5, 2.5) and (0.55, 0) give S_0 = 10.5 > S_1 = 2.5.  HISA with blocks of
    one token keeping all four: routed scores 10, 0, 10, 1, so the top 3 are
    tokens 0, 2, 3 with 10, 10, 1 (all heads would give 10, 5, 10, 1 and pick
    token 1 instead of 3)."""
    q = np.array([[[[10.0, 0.0], [0.0, 1.0]]]], np.float32)
    k = np.array([[[1.0, 0.0], [0.0, 5.0], [1.0, 0.0], [0.1, 0.0]]], np.float32)
    w = np.ones((1, 1, 2), np.float32)
    p = make(q, k, w, 3, q_pos0=[3])
    out = oracle_mod.hisa(oracle_mod.Inputs(p), 3, block=1, r=4, route_h=1, route_block=2)
    assert out["heads"].tolist() == [[0]]
    assert out["idx"].tolist() == [[0, 2, 3]]
    assert out["score64"][0].tolist() == [10.0, 10.0, float(np.float32(0.1)) * 10.0]


def test_router_closed_form_constant_keys(oracle_mod):
    """All keys = v => every representative = v, S_j = M |w_j| max(q_j.v, 0)."""
    d, H, nk, blk = 4, 8, 50, 16
    v = np.array([1.0, 0, 0, 0], np.float32)
    k = np.tile(v, (1, nk, 1))
    qc = np.array([3, -1, 2, 2, 0, 5, 1, 2], np.float32)    # q_j . v
    q = np.zeros((1, 1, H, d), np.float32)
    q[0, 0, :, 0] = qc
    w = np.array([[[1, 4, -2, 1, 9, -1, 3, 0.5]]], np.float32)
    p = make(q, k, w, topk=4)
    m = oracle_mod.misa(oracle_mod.Inputs(p), 4, block=blk, h=3)
    M = math.ceil(nk / blk)
    S = M * np.abs(w[0, 0]) * np.maximum(qc, 0)
    assert np.allclose(m["E"][0], S / M, rtol=0, atol=0)
    # S = [3,0,4,2,0,5,3,1]*M -> top-3: head 5 (5), head 2 (4), then tie 3 between heads 0,6 -> 0
    assert list(m["heads"][0]) == [0, 2, 5]


def test_hisa_coarse_closed_form(oracle_mod):
    """Block-constant keys c_b e_0 with one positive head: J_b = w q c_b; kept = top-r c_b."""
    d, blk, nblk = 4, 8, 10
    c = np.array([3, -1, 7, 7, 2, 0, 5, 1, 6, 4], np.float32)
    k = np.zeros((1, blk * nblk, d), np.float32)
    k[0, :, 0] = np.repeat(c, blk)
    q = np.zeros((1, 1, 8, d), np.float32)
    q[0, 0, 0, 0] = 1.0
    w = np.zeros((1, 1, 8), np.float32)
    w[0, 0, 0] = 2.0
    p = make(q, k, w, topk=6)
    h = oracle_mod.hisa(oracle_mod.Inputs(p), 6, block=blk, r=3)
    assert list(h["blocks"][0]) == [2, 3, 8]                 # 7, 7 (lower block first), 6
    assert np.array_equal(h["J"][0], [14.0, 14.0, 12.0])
    # all 24 candidates of blocks 2,3,8 score 2*c; top-6 = the 16 tokens with c=7 -> lowest 6
    assert list(h["idx"][0]) == list(range(16, 22))


def test_block_scores_closed_form(oracle_mod):
    """Same block-constant keys: J_b = w q c_b for every block, in block order."""
    d, blk, nblk = 4, 8, 10
    c = np.array([3, -1, 7, 7, 2, 0, 5, 1, 6, 4], np.float32)
    k = np.zeros((1, blk * nblk, d), np.float32)
    k[0, :, 0] = np.repeat(c, blk)
    q = np.zeros((1, 1, 8, d), np.float32)
    q[0, 0, 0, 0] = 1.0
    w = np.zeros((1, 1, 8), np.float32)
    w[0, 0, 0] = 2.0
    p = make(q, k, w, topk=6)
    J = oracle_mod.block_scores(oracle_mod.Inputs(p), 0, blk)
    assert np.array_equal(J, 2.0 * np.maximum(c, 0))


def test_block_scores_with_unit_blocks_are_token_scores(oracle_mod):
    """b = 1: every block is one token, so J is the DSA score row (any head list)."""
    p = gen.normal_problem(61, 1, 40, 40, 16, 128, 8)
    inp = oracle_mod.Inputs(p)
    for row in (0, 17, 39):
        assert np.array_equal(oracle_mod.block_scores(inp, row, 1), oracle_mod.score_row(inp, row))
        hs = np.array([1, 4, 9], np.int32)
        assert np.array_equal(oracle_mod.block_scores(inp, row, 1, hs),
                              oracle_mod.score_row(inp, row, hs))


def test_segment_problem_pooled_keys_are_exact(oracle_mod):
    """Segment-structured integer keys: every pooled key (full or boundary block,
    block sizes dividing the segment) is c or c + e / blocksize exactly."""
    p = gen.segment_integer_problem(62, 1, 200, 200, 8, 128, 8, seg=64)
    inp = oracle_mod.Inputs(p)
    k = gen.bf16_bits_to_f32(p.k)[0].astype(np.float64)
    for blk in (16, 64):
        for n in (37, 64, 150, 200):
            reps = oracle_mod.pool(inp, 0, n, blk)
            for a in range(reps.shape[0]):
                lo, hi = a * blk, min((a + 1) * blk, n)
                assert np.array_equal(reps[a], k[lo:hi].mean(0))


# ----------------------------------------------------------------- E4M3 codec --

def test_e4m3_ocp_values(oracle_mod):
    g = json.load(open(os.path.join(GOLD, "e4m3_ocp.json")))
    for code, val in g["codes"].items():
        got = oracle_mod.e4m3_decode([int(code, 16)])[0]
        assert got == val and math.copysign(1, got) == math.copysign(1, val)
    for code in g["nan_codes"]:
        assert math.isnan(oracle_mod.e4m3_decode([int(code, 16)])[0])


def test_e4m3_roundtrip_all_codes(oracle_mod):
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    vals = oracle_mod.e4m3_decode(codes).astype(np.float32)
    assert np.array_equal(oracle_mod.e4m3_encode(vals), codes)


def test_e4m3_round_half_even_and_saturation(oracle_mod):
    codes = np.array([c for c in range(0x7E) if c != 0x7F], np.uint8)
    vals = oracle_mod.e4m3_decode(np.arange(0x7F)).astype(np.float64)
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)       # exact in fp32
    got = oracle_mod.e4m3_encode(mids)
    even = np.where(np.arange(0x7E) % 2 == 0, np.arange(0x7E), np.arange(1, 0x7F))
    assert np.array_equal(got, even.astype(np.uint8))
    assert oracle_mod.e4m3_encode([1000.0, -1e6, 449.0])[0] == 0x7E
    assert oracle_mod.e4m3_encode([-1e6])[0] == 0xFE
    del codes


def test_quantize_scale_definition(oracle_mod):
    x = np.array([[0.5, -3.5, 1.0, 0.0], [0, 0, 0, 0]], np.float32)
    codes, sc = oracle_mod.quantize_rows(x, F32)
    assert sc[0] == np.float32(3.5) / np.float32(448.0) and sc[1] == 1.0
    assert codes[0, 1] == 0xFE                                   # -amax maps to -448
    assert np.all(codes[1] == 0)


def test_fp8_margin_bound_keeps_set(oracle_mod):
    """2E < m  =>  the top-k set is unchanged by key quantisation, with
    E = eps * sum_j |w_j| ||q_j||, eps = max_s ||k_s - k^_s||, m = I(k) - I(k+1).
    Each sequence gets k planted keys aligned with its query so that the margin
    clears the (loose) bound on most rows."""
    B, nk, H, d, topk = 6, 300, 8, 32, 10
    p = gen.normal_problem(17, B, 1, nk, H, d, topk=topk)
    qf = gen.bf16_bits_to_f32(p.q)
    kf = gen.bf16_bits_to_f32(p.k).copy()
    rng = np.random.default_rng(17)
    for b in range(B):
        wt = p.w[b, 0]
        u = (np.maximum(wt, 0)[:, None] * qf[b, 0]).sum(0)
        u /= np.linalg.norm(u)
        for s in rng.choice(nk, topk, replace=False):
            kf[b, s] = 6.0 * np.sqrt(d) * u * (1.0 + 0.1 * rng.random())
    p.k = gen.f32_to_bf16_bits(kf)
    kf = gen.bf16_bits_to_f32(p.k)
    codes, ksc = oracle_mod.quantize_rows(p.k, BF16)
    kq = oracle_mod.e4m3_decode(codes.ravel()).reshape(codes.shape) * ksc[..., None]
    inp = oracle_mod.Inputs(p)
    inq = oracle_mod.Inputs(p, k=codes, k_dtype=E4M3, k_scale=ksc)
    ref = oracle_mod.dsa(inp, topk)
    got = oracle_mod.dsa(inq, topk)
    checked = 0
    for row in range(B):
        eps = np.max(np.linalg.norm(kq[row] - kf[row], axis=-1))
        I = np.sort(oracle_mod.score_row(inp, row))[::-1]
        m = I[topk - 1] - I[topk]
        E = eps * np.sum(np.abs(p.w[row, 0]) * np.linalg.norm(qf[row, 0], axis=-1))
        if 2 * E < m:
            checked += 1
            assert set(ref[0][row]) == set(got[0][row])
    assert checked >= 3


# ------------------------------------------------------------- cost counters --

def test_cost_counters_match_page_arithmetic(oracle_mod):
    g = json.load(open(os.path.join(GOLD, "cost_arithmetic.json")))
    ex = g["decode_example"]
    t, H, d = ex["t"], ex["heads"], ex["dim"]
    # one decode query at position t-1 over t keys; cheap integer data
    q = np.ones((1, 1, H, d), np.float32)
    k = np.zeros((1, t, d), np.float32)
    k[0, :, 0] = 1.0
    p = make(q, k, np.ones((1, 1, H), np.float32), topk=ex["topk"])
    inp = oracle_mod.Inputs(p)
    _, _, _, dots = oracle_mod.dsa(inp, ex["topk"])
    assert dots[0] * d == ex["dsa_macs"]
    m = oracle_mod.misa(inp, ex["topk"], block=1024, h=ex["misa_h"])
    assert (m["dots"][0] - H * (t // 1024)) * d == ex["misa_token_macs"]
    h = oracle_mod.hisa(inp, ex["topk"], block=ex["hisa_block"], r=ex["hisa_r"])
    reps = t // ex["hisa_block"]
    assert reps == ex["hisa_representatives"]
    cand = h["dots"][0] // H - reps
    assert cand == ex["hisa_candidates"]
    assert 100.0 * cand / t == ex["hisa_candidate_percent"]
    assert 100.0 * ex["topk"] / t == ex["selected_percent"]
    de = g["dots_example"]
    assert de["N"] * de["heads"] == de["dsa_dots_per_query"]
    by = g["bytes"]
    assert 131072 * 32 == by["fp8_key_bytes_128k_d32"]
    assert 131072 * 128 == by["fp8_key_bytes_128k_d128"]
    assert 2048 * 4 == by["indices_bytes_per_request_k2048"]


# ------------------------------------------------- tolerance scale nu (closed form) --

def test_nu_closed_form(oracle_mod):
    """nu(t, s) = sum_j |w_tj| ||q_tj|| ||k_s|| / sqrt(d).  With q_tj = c_j (1, ..., 1)
    (||q_tj|| = |c_j| sqrt(d)) and k_s = b_s e_0 (||k_s|| = |b_s|) it is
    |b_s| sum_j |w_j| |c_j|, whatever d is; negative weights count by magnitude."""
    d, H = 16, 3
    c = np.array([2.0, -1.0, 0.5], np.float32)
    w = np.array([1.0, -0.5, 3.0], np.float32)
    b = np.array([3.0, -2.0, 0.0, 1.5], np.float32)
    q = np.ones((1, 1, H, d), np.float32) * c[None, None, :, None]
    k = np.zeros((1, len(b), d), np.float32)
    k[0, :, 0] = b
    p = make(q, k, w[None, None], topk=1, q_pos0=[len(b) - 1])
    inp = oracle_mod.Inputs(p)
    s = np.arange(len(b), dtype=np.int64)
    got = oracle_mod.nu_pairs(inp, np.zeros(len(b), np.int64), s)
    want = np.abs(b) * float(np.sum(np.abs(w) * np.abs(c)))   # = |b| * (2 + 0.5 + 1.5)
    assert np.array_equal(got, want.astype(np.float64))
    # restricted to heads (0, 2): |b| (2 + 1.5)
    got2 = oracle_mod.nu_pairs(inp, np.zeros(len(b), np.int64), s,
                               np.tile(np.array([[0, 2]], np.int32), (len(b), 1)))
    assert np.array_equal(got2, np.abs(b) * 3.5)


def test_nu_is_the_typical_score_size(oracle_mod):
    """For independent N(0,1) q and k the dot product of one head has standard
    deviation sqrt(d) = E[||q|| ||k||] / sqrt(d) up to O(1/d): over many pairs the
    single-head nu (|w| = 1) matches the root mean square of q . k within 5 %."""
    rng = np.random.default_rng(8)
    d, n = 128, 4000
    q = rng.standard_normal((1, n, 1, d)).astype(np.float32)
    k = rng.standard_normal((1, n, d)).astype(np.float32)
    p = make(q, k, np.ones((1, n, 1), np.float32), topk=1)
    inp = oracle_mod.Inputs(p)
    rows = np.arange(n, dtype=np.int64)
    s = np.zeros(n, np.int64)                       # key 0 is legal for every row
    nu = oracle_mod.nu_pairs(inp, rows, s)
    dots = np.einsum("nd,d->n", q[0, :, 0].astype(np.float64), k[0, 0].astype(np.float64))
    rms = math.sqrt(float(np.mean(dots ** 2)))
    assert abs(float(np.mean(nu)) / rms - 1.0) < 0.05


# --------------------------------------------------- split query (FP8-key path) --

def test_split_query_worked_values(oracle_mod):
    """amax 448 gives s = 1.  300 -> hi 288 (e4m3 spacing 32 on [256, 512)), residual
    12 (exact) -> 300; 301 -> 288 + 13 = 301; 300.5 -> residual 12.5, an e4m3 tie
    between 12 and 13 (spacing 1 on [8, 16)), rounded to even: 300."""
    x = np.zeros((1, 8), np.float32)
    x[0, :5] = [448.0, 300.0, 301.0, 300.5, -3.0]
    v = oracle_mod.split_query(x, F32)
    assert list(v[0, :5]) == [448.0, 300.0, 301.0, 300.0, -3.0]
    assert np.all(v[0, 5:] == 0.0)
    z = oracle_mod.split_query(np.zeros((2, 8), np.float32), F32)
    assert np.all(z == 0.0)


def test_split_query_error_bound(oracle_mod):
    """Per value: |x - s (hi + lo)| <= 2^-8 |x| + 2^-10 s.  hi has e4m3's four
    significant bits, so the residual is at most half hi's spacing, <= 2^-4 |x|;
    its own code adds at most half its spacing, <= 2^-8 |x|, or at most half the
    subnormal step 2^-9 (times s) below 2^-6.  A bf16 input (eight significant
    bits) is reproduced within the same bound, and exact e4m3 multiples of s are
    reproduced exactly."""
    rng = np.random.default_rng(9)
    x = (rng.standard_normal((64, 128)) * np.exp(rng.uniform(-6, 6, (64, 1)))).astype(np.float32)
    xb = gen.f32_to_bf16_bits(x)
    for arr, dt, vals in ((x, F32, x.astype(np.float64)),
                          (xb, BF16, gen.bf16_bits_to_f32(xb).astype(np.float64))):
        v = oracle_mod.split_query(arr, dt)
        s = np.max(np.abs(vals), axis=1, keepdims=True).astype(np.float32) / np.float32(448.0)
        assert np.all(np.abs(vals - v) <= 2.0 ** -8 * np.abs(vals) + 2.0 ** -10 * s)
    codes = rng.integers(-7, 8, size=(4, 128)).astype(np.float32) * 32.0
    codes[:, 0] = 448.0
    assert np.array_equal(oracle_mod.split_query(codes, F32), codes.astype(np.float64))


# ------------------------------------------------ LISA / LISA-dagger / ResMiSA --

def _golden(name):
    return json.load(open(os.path.join(GOLD, name)))


def test_lisa_decomposition_worked_example(oracle_mod):
    """[PT] 3.1: the fused query 1.5 gives the linear term 4.5 (indexer LISA's score),
    the correction 1.5 restores the score 6; ResMiSA with one residual head picks
    the second head and recovers 6, with none it is LISA."""
    g = _golden("lisa_decomposition.json")
    p = make(np.array(g["q"])[None, None], np.array(g["k"])[None, None],
             np.array(g["w"])[None, None], topk=1)
    inp = oracle_mod.Inputs(p)
    assert oracle_mod.dsa(inp, 1)[2][0, 0] == g["score"]
    assert oracle_mod.lisa(inp, 1)["score64"][0, 0] == g["linear_term"]
    assert g["linear_term"] == g["fused_query"] * g["k"][0]
    assert g["linear_term"] + g["correction"] == g["score"]
    r0 = oracle_mod.resmisa(inp, 1, 1, 0)
    assert r0["score64"][0, 0] == g["linear_term"]
    r1 = oracle_mod.resmisa(inp, 1, 1, 1)
    assert list(r1["heads"][0]) == [g["residual_head"]]
    assert r1["score64"][0, 0] == g["score"]


def test_residual_bound_worked_example(oracle_mod):
    """[PT] 3.2: q = (1, -2) over a block with key ranges [-1, 3] x [0, 4] has U- = 9,
    above both actual negative dot products (1 and 5)."""
    g = _golden("residual_bound_example.json")
    q = np.array(g["q"], np.float32)[None, None, None]          # [1, 1, 1, 2]
    keys = np.array(g["keys"], np.float32)[None]                  # [1, 2, 2]
    p = make(q, keys, np.ones((1, 1, 1), np.float32), topk=1)    # query at position 1
    inp = oracle_mod.Inputs(p)
    U = oracle_mod.residual_bounds(inp, 0, 2)
    assert U.shape == (1, 1) and U[0, 0] == g["bound"]
    neg = -(keys[0] @ np.array(g["q"]))
    assert list(neg) == g["negative_dots"] and np.all(neg <= U[0, 0])


def test_residual_bound_covers_every_legal_key_and_no_future_key(oracle_mod):
    """U-_{b,j} >= -q_j . k_s for every legal key of block b; a future key, however
    extreme, does not move the bound (blocks cover the legal prefix only)."""
    rng = np.random.default_rng(12)
    nq, nk, H, d, blk = 6, 100, 4, 8, 16
    q = rng.standard_normal((1, nq, H, d)).astype(np.float32)
    k = rng.standard_normal((1, nk, d)).astype(np.float32)
    w = rng.standard_normal((1, nq, H)).astype(np.float32)
    p = make(q, k, w, topk=4, q_pos0=[50])
    inp = oracle_mod.Inputs(p)
    k2 = k.copy()
    k2[0, 60:] = 1e3 * np.sign(k2[0, 60:])       # every row sits at position <= 55
    inp2 = oracle_mod.Inputs(make(q, k2, w, topk=4, q_pos0=[50]))
    for row in range(nq):
        U = oracle_mod.residual_bounds(inp, row, blk)
        n = 50 + row + 1
        assert U.shape[0] == (n + blk - 1) // blk
        for a in range(U.shape[0]):
            ks = k[0, a * blk:min((a + 1) * blk, n)].astype(np.float64)
            neg = -(ks @ q[0, row].astype(np.float64).T)           # [keys, H]
            assert np.all(neg <= U[a][None] + 1e-9)
        assert np.array_equal(U, oracle_mod.residual_bounds(inp2, row, blk))


def test_dosa_bound_covers_every_legal_key(oracle_mod):
    """DoSA's block upper bound is >= I_{t,s} and its lower bound <= I_{t,s} for
    every legal key s of the block (brute force over the row), including the
    row's partial last block, and both -inf for blocks past its legal prefix
    ("The new bottleneck of sparse attention", route five: only bounds that
    truly enclose the block keep the top-k exact)."""
    rng = np.random.default_rng(13)
    nq, nk, H, d, shift = 5, 700, 6, 8, 7
    q = rng.standard_normal((1, nq, H, d)).astype(np.float32)
    k = rng.standard_normal((1, nk, d)).astype(np.float32)
    w = rng.standard_normal((1, nq, H)).astype(np.float32)
    inp = oracle_mod.Inputs(make(q, k, w, topk=4, q_pos0=[300]))
    bs = 1 << shift
    for row in range(nq):
        ub, lb, sl = oracle_mod.dosa_bounds(inp, row, shift)
        n = 300 + row + 1
        assert ub.shape == ((nk + bs - 1) // bs,)
        s = np.arange(n)
        I = oracle_mod.score_pairs(inp, np.full(n, row), s)
        for a in range(len(ub)):
            if a * bs >= n:
                assert ub[a] == -np.inf and lb[a] == -np.inf and sl[a] == 0.0
                continue
            blk = I[a * bs:min((a + 1) * bs, n)]
            assert ub[a] >= blk.max() - 1e-12
            assert lb[a] <= blk.min() + 1e-12
            assert sl[a] > 0.0


def test_dosa_bound_is_exact_on_constant_blocks(oracle_mod):
    """Keys constant on each block: the box is a point, hi = lo = q_j . k, and
    the bound equals the score of every key of the block."""
    rng = np.random.default_rng(14)
    nq, nk, H, d, shift = 3, 512, 5, 8, 7
    q = rng.standard_normal((1, nq, H, d)).astype(np.float32)
    c = rng.standard_normal((nk >> shift, d)).astype(np.float32)
    k = np.repeat(c, 1 << shift, axis=0)[None]
    w = rng.standard_normal((1, nq, H)).astype(np.float32)
    inp = oracle_mod.Inputs(make(q, k, w, topk=4))
    for row in range(nq):
        ub, lb, _ = oracle_mod.dosa_bounds(inp, row, shift)
        for a in range(len(ub)):
            I = oracle_mod.score_pairs(inp, [row], [a << shift])[0]
            assert abs(ub[a] - I) <= 1e-12 * max(1.0, abs(I))
            assert abs(lb[a] - I) <= 1e-12 * max(1.0, abs(I))


def test_dosa_seed_is_a_lower_bound_of_the_kth_best(oracle_mod):
    """The seed set guarantees keep legal keys at or above the seed, so the
    row's keep-th best score is >= the seed (brute force over the row); rows
    with fewer than keep legal keys get no seed.  On keys constant per block
    the seed is exactly the score of the block that completes the count."""
    rng = np.random.default_rng(15)
    nq, nk, H, d, shift, keep = 6, 900, 6, 8, 7, 200
    q = rng.standard_normal((1, nq, H, d)).astype(np.float32)
    k = rng.standard_normal((1, nk, d)).astype(np.float32)
    w = rng.standard_normal((1, nq, H)).astype(np.float32)
    inp = oracle_mod.Inputs(make(q, k, w, topk=keep, q_pos0=[300]))
    for row in range(nq):
        n = 300 + row + 1
        seed = oracle_mod.dosa_seed(inp, row, shift, keep)
        if n < keep:
            assert seed == -np.inf
            continue
        I = np.sort(oracle_mod.score_pairs(inp, np.full(n, row), np.arange(n)))[::-1]
        assert seed > -np.inf and I[keep - 1] >= seed
    short = oracle_mod.Inputs(make(q, k, w, topk=keep, q_pos0=[100]))   # rows of 101..106 keys
    assert all(oracle_mod.dosa_seed(short, r, shift, keep) == -np.inf for r in range(nq))
    c = rng.standard_normal((nk >> shift, d)).astype(np.float32)
    kc = np.repeat(c, 1 << shift, axis=0)[None, :nk]
    kc = np.concatenate([kc, np.zeros((1, nk - kc.shape[1], d), np.float32)], axis=1)
    inp = oracle_mod.Inputs(make(q, kc, w, topk=keep))
    for row in range(nq):
        n = nk - nq + row + 1
        blk = oracle_mod.score_pairs(inp, np.full(n, row), np.arange(n))
        per = [blk[a << shift] for a in range((n + (1 << shift) - 1) >> shift)]
        cnt = [min(1 << shift, n - (a << shift)) for a in range(len(per))]
        order = sorted(range(len(per)), key=lambda a: (-per[a], a))
        got, want = 0, None
        for a in order:
            got += cnt[a]
            want = per[a]
            if got >= keep:
                break
        seed = oracle_mod.dosa_seed(inp, row, shift, keep)
        assert abs(seed - want) <= 1e-12 * max(1.0, abs(want))


def test_resmisa_routes_by_weight_magnitude(oracle_mod):
    """S_j = |w_j| max_b ReLU(U-_{b,j}): a head whose weight is negative but large in
    magnitude outranks a positive head with the same bound."""
    d = 4
    q = np.zeros((1, 1, 3, d), np.float32)
    q[0, 0, :, 0] = [-1.0, -1.0, 1.0]             # heads 0, 1 see -q.k = k_0 > 0
    k = np.zeros((1, 8, d), np.float32)
    k[0, :, 0] = np.arange(8)
    w = np.array([[[-3.0, 1.0, 2.0]]], np.float32)
    p = make(q, k, w, topk=3)
    out = oracle_mod.resmisa(oracle_mod.Inputs(p), 3, 4, 1)
    # bounds: heads 0, 1: max k_0 = 7; head 2: -min k_0 = 0
    assert np.allclose(out["S"][0], [21.0, 7.0, 0.0])
    assert list(out["heads"][0]) == [0]


def test_resmisa_with_every_head_is_dsa(oracle_mod):
    """r = H: l + sum_j w_j ReLU(-z_j) = sum_j w_j ReLU(z_j) (integer operands, exact)."""
    p = gen.integer_problem(95, 2, 40, 90, 8, 16, 12, q_pos0=[50, 0], k_len=[90, 60])
    inp = oracle_mod.Inputs(p)
    ri, rs, rs64, _ = oracle_mod.dsa(inp, p.topk)
    out = oracle_mod.resmisa(inp, p.topk, 16, p.heads)
    assert np.array_equal(out["idx"], ri) and np.array_equal(out["score64"], rs64)
    assert np.all(out["heads"] == np.arange(p.heads))


def test_resmisa_without_residual_heads_is_lisa(oracle_mod):
    p = gen.integer_problem(96, 1, 30, 70, 8, 16, 10)
    inp = oracle_mod.Inputs(p)
    a = oracle_mod.resmisa(inp, p.topk, 16, 0)
    b = oracle_mod.lisa(inp, p.topk)
    assert np.array_equal(a["idx"], b["idx"]) and np.array_equal(a["score64"], b["score64"])


def test_lisa_closed_form_line(oracle_mod):
    """q_{t,j} = c_j e_0, k_s = s e_0: l_{t,s} = s sum_j w_j c_j (the ReLU plays no
    part); positive sums rank the latest keys first, negative sums the earliest."""
    rng = np.random.default_rng(14)
    nq, nk, H, topk = 10, 30, 5, 6
    c = rng.integers(-3, 4, size=(nq, H)).astype(np.float32)
    w = rng.integers(-2, 3, size=(nq, H)).astype(np.float32)
    p = _line_problem(nq, nk, c, w, +1.0, topk)
    out = oracle_mod.lisa(oracle_mod.Inputs(p), topk)
    for i in range(nq):
        pos = nk - nq + i
        gsum = float(np.sum(w[i] * c[i]))
        legal = np.arange(pos + 1)
        want = legal[::-1][:topk] if gsum > 0 else legal[:topk]
        assert list(out["idx"][i]) == list(want), (i, gsum)
        assert np.array_equal(out["score64"][i], want * gsum + 0.0)


def test_lisa_dagger_full_pool_is_dsa(oracle_mod):
    p = gen.integer_problem(97, 1, 40, 80, 8, 16, 10)
    inp = oracle_mod.Inputs(p)
    ri, rs, rs64, _ = oracle_mod.dsa(inp, p.topk)
    out = oracle_mod.lisa(inp, p.topk, pool_m=80)
    assert np.array_equal(out["idx"], ri) and np.array_equal(out["score64"], rs64)


def test_lisa_dagger_pool_of_k_keeps_the_lisa_set(oracle_mod):
    """A pool of exactly k keeps LISA's set; only the scores (now the full I) and
    their order change."""
    p = gen.normal_problem(98, 1, 30, 120, 8, 32, 16)
    inp = oracle_mod.Inputs(p)
    a = oracle_mod.lisa(inp, p.topk)
    b = oracle_mod.lisa(inp, p.topk, pool_m=p.topk)
    assert np.array_equal(np.sort(a["idx"], 1), np.sort(b["idx"], 1))
    rows = np.repeat(np.arange(p.n_q), p.topk)
    full = oracle_mod.score_pairs(inp, rows, b["idx"].ravel()).reshape(b["idx"].shape)
    assert np.array_equal(full, b["score64"])


def test_lisa_and_resmisa_cost_counts_match_page_arithmetic(oracle_mod):
    """[PT] 3.2 'one set of numbers': per query at N = 131072, H_I = 64, k = 2048,
    pool M = 8192, r = 7: DSA 8,388,608 key dots, LISA 131,072, ResMiSA 1,048,576
    (1/8), LISA-dagger 655,360 (7.81 %).  Counted on the last row of an
    N-key prefix (d = 4: the counts do not depend on d)."""
    g = _golden("cost_arithmetic.json")["lisa_resmisa_example"]
    N, H = g["N"], g["heads"]
    rng = np.random.default_rng(15)
    q = rng.integers(-2, 3, size=(1, 1, H, 4)).astype(np.float32)
    k = rng.integers(-2, 3, size=(1, N, 4)).astype(np.float32)
    w = rng.integers(-2, 3, size=(1, 1, H)).astype(np.float32)
    inp = oracle_mod.Inputs(make(q, k, w, topk=2048))
    assert oracle_mod.dsa(inp, 2048)[3][0] == g["dsa_dots_per_query"]
    assert oracle_mod.lisa(inp, 2048)["dots"][0] == g["lisa_dots_per_query"]
    assert oracle_mod.resmisa(inp, 2048, 1024, g["residual_heads"])["dots"][0] == \
        g["resmisa_dots_per_query"] == g["dsa_dots_per_query"] * g["resmisa_fraction"]
    ld = oracle_mod.lisa(inp, 2048, pool_m=g["pool"])["dots"][0]
    assert ld == g["lisa_dagger_dots_per_query"]
    assert round(100.0 * ld / g["dsa_dots_per_query"], 2) == g["lisa_dagger_percent"]


def test_pairwise_lisa_and_resmisa_scores_match_the_rankings(oracle_mod):
    """The pairwise scores the tolerance checks use are the ones the row
    functions rank by (same definitions, evaluated at the selected tokens)."""
    p = gen.normal_problem(99, 1, 24, 90, 8, 32, 10, q_pos0=[50])
    inp = oracle_mod.Inputs(p)
    rows = np.repeat(np.arange(p.n_q), p.topk)
    a = oracle_mod.lisa(inp, p.topk)
    assert np.array_equal(oracle_mod.linear_pairs(inp, rows, a["idx"].ravel()),
                          a["score64"].ravel())
    b = oracle_mod.resmisa(inp, p.topk, 16, 3)
    hh = np.repeat(b["heads"], p.topk, 0)
    assert np.array_equal(oracle_mod.resmisa_pairs(inp, rows, b["idx"].ravel(), hh),
                          b["score64"].ravel())


# --------------------------------------------------- Sparse MLA (fixed set) --

def _bf(x):
    return gen.f32_to_bf16_bits(np.asarray(x, np.float32))


def test_sparse_mla_single_key_is_its_value(oracle_mod):
    """One selected position: the softmax weight is 1, the output is that key's
    latent value and lse is its logit."""
    rng = np.random.default_rng(20)
    q = _bf(rng.integers(-2, 3, size=(3, 2, 16)))
    kv = _bf(rng.integers(-2, 3, size=(1, 10, 16)))
    idx = np.full((3, 4), -1, np.int32)
    idx[:, 1] = [7, 0, 9]
    out = oracle_mod.sparse_mla(q, kv, idx, 0.5, 12, 3)
    kvf = gen.bf16_bits_to_f32(kv).astype(np.float64)
    qf = gen.bf16_bits_to_f32(q).astype(np.float64)
    for t, s in enumerate([7, 0, 9]):
        assert np.array_equal(out["o"][t], np.repeat(kvf[0, s, :12][None], 2, 0))
        assert np.array_equal(out["lse"][t], 0.5 * qf[t] @ kvf[0, s])
        assert np.array_equal(out["den"][t], [1.0, 1.0])


def test_sparse_mla_zero_query_is_the_mean_value(oracle_mod):
    """q = 0: every logit is 0, the weights are uniform, o is the mean of the
    selected values and lse = log(n)."""
    rng = np.random.default_rng(21)
    kv = _bf(rng.standard_normal((2, 50, 32)))
    q = np.zeros((4, 3, 32), np.uint16)
    idx = np.array([[3, 9, 12, -1], [0, -1, -1, -1], [5, 6, 7, 8], [49, 1, -1, 2]], np.int32)
    out = oracle_mod.sparse_mla(q, kv, idx, 0.1, 24, 2)     # tokens 0-1: seq 0, 2-3: seq 1
    kvf = gen.bf16_bits_to_f32(kv).astype(np.float64)
    for t in range(4):
        sel = idx[t][idx[t] >= 0]
        want = kvf[t // 2, sel, :24].mean(0)
        np.testing.assert_allclose(out["o"][t], np.repeat(want[None], 3, 0), rtol=1e-14, atol=1e-15)
        np.testing.assert_allclose(out["lse"][t], np.log(len(sel)), rtol=1e-14)


def test_sparse_mla_two_keys_closed_form(oracle_mod):
    """Two positions whose logits differ by log 3 (q . k = 0 and q . k = ln 3 / scale
    chosen exactly): weights 1/4 and 3/4, row max ln 3, denominator 4/3."""
    d = 4
    scale = 0.25
    q = np.zeros((1, 1, d), np.float32)
    q[0, 0, 0] = 1.0
    kv = np.zeros((1, 2, d), np.float32)
    kv[0, 0] = [0.0, 1.0, 0.0, 0.0]
    kv[0, 1] = [4.0, 0.0, 1.0, 0.0]                          # logit 1.0 vs 0.0
    out = oracle_mod.sparse_mla(_bf(q), _bf(kv), np.array([[0, 1]], np.int32), scale, 3, 1)
    e = np.exp(1.0)
    w0, w1 = 1.0 / (1.0 + e), e / (1.0 + e)
    np.testing.assert_allclose(out["o"][0, 0], w0 * kv[0, 0, :3] + w1 * kv[0, 1, :3], rtol=1e-15)
    assert out["max"][0, 0] == 1.0
    np.testing.assert_allclose(out["den"][0, 0], 1.0 + 1.0 / e, rtol=1e-15)
    np.testing.assert_allclose(out["lse"][0, 0], 1.0 + np.log(1.0 + 1.0 / e), rtol=1e-15)


def test_sparse_mla_ignores_order_and_empty_entries(oracle_mod):
    """The candidate set is a set: permuting it, or interleaving empty (-1)
    entries, leaves every output unchanged up to summation order."""
    rng = np.random.default_rng(22)
    q = _bf(rng.standard_normal((5, 4, 64)))
    kv = _bf(rng.standard_normal((1, 300, 64)))
    idx = np.stack([rng.permutation(300)[:40] for _ in range(5)]).astype(np.int32)
    a = oracle_mod.sparse_mla(q, kv, idx, 0.125, 48, 5)
    idx2 = np.full((5, 64), -1, np.int32)
    for t in range(5):
        slots = np.sort(rng.permutation(64)[:40])
        idx2[t, slots] = rng.permutation(idx[t])
    b = oracle_mod.sparse_mla(q, kv, idx2, 0.125, 48, 5)
    for key in ("o", "lse", "max", "den"):
        np.testing.assert_allclose(a[key], b[key], rtol=1e-12, atol=1e-13)
    z = oracle_mod.sparse_mla(q, kv, np.full((5, 3), -1, np.int32), 0.125, 48, 5)
    assert np.all(z["o"] == 0.0) and np.all(np.isneginf(z["lse"])) and np.all(z["den"] == 0.0)


# ---------------------------------------------------------- indexer backward --

def _loss(oracle_mod, p, q, k, w, sel, g):
    """L = sum_{t, s in S_t} g_{t,s} I_{t,s}, evaluated with the oracle's forward
    score (fp32 operands)."""
    pp = gen.Problem(p.batch, p.n_q, p.n_k, p.heads, p.dim, p.topk, F32, F32, q, k, w,
                     p.q_pos0, p.k_len)
    inp = oracle_mod.Inputs(pp)
    rows = np.repeat(np.arange(p.batch * p.n_q), sel.shape[1])
    s = sel.ravel()
    ok = s >= 0
    return float(np.sum(g.ravel()[ok] * oracle_mod.score_pairs(inp, rows[ok], s[ok])))


def test_backward_matches_central_differences(oracle_mod):
    """The three gradients of [PT] 2.3 against central differences of the
    forward score (the definition the chain rule starts from), on inputs whose
    dot products stay far from the ReLU kink."""
    rng = np.random.default_rng(30)
    B_, nq, nk, H, d, kk = 1, 3, 12, 3, 4, 5
    q = rng.standard_normal((B_, nq, H, d))
    k = rng.standard_normal((B_, nk, d))
    w = rng.standard_normal((B_, nq, H))
    z = np.einsum("bthd,bsd->bths", q, k)
    q[np.abs(z).min(axis=(2, 3)) < 0.05] *= 1.1                 # keep |z| away from 0
    q, k, w = (x.astype(np.float32).astype(np.float64) for x in (q, k, w))
    p = gen.Problem(B_, nq, nk, H, d, kk, F32, F32, q.astype(np.float32), k.astype(np.float32),
                    w.astype(np.float32))
    sel = np.array([[0, 3, 7, -1, 9], [1, 2, -1, 4, 10], [11, 0, 5, 6, -1]], np.int32)
    g = rng.standard_normal(sel.shape).astype(np.float32)
    got = oracle_mod.indexer_backward(oracle_mod.Inputs(p), sel, g)
    eps = 1e-3
    for name, arr, grad in (("q", q, got["dq"].reshape(q.shape)), ("k", k, got["dk"].reshape(k.shape)),
                            ("w", w, got["dw"].reshape(w.shape))):
        flat = arr.reshape(-1)
        num = np.empty_like(flat)
        for i in range(flat.size):
            old = flat[i]
            flat[i] = old + eps
            lp = _loss(oracle_mod, p, q.astype(np.float32), k.astype(np.float32),
                       w.astype(np.float32), sel, g)
            flat[i] = old - eps
            lm = _loss(oracle_mod, p, q.astype(np.float32), k.astype(np.float32),
                       w.astype(np.float32), sel, g)
            flat[i] = old
            num[i] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(grad.reshape(-1), num, rtol=1e-3, atol=1e-3, err_msg=name)


def test_backward_relu_kink_has_zero_derivative(oracle_mod):
    """z exactly 0 (integer operands): m = 1[z > 0] = 0, so no gradient flows to
    q or k through that head, and its ReLU(z) = 0 adds nothing to dw."""
    q = np.zeros((1, 1, 2, 4), np.float32)
    q[0, 0, 0] = [1, -1, 0, 0]         # z = 0 against k = (1, 1, 0, 0)
    q[0, 0, 1] = [1, 1, 0, 0]          # z = 2
    k = np.zeros((1, 1, 4), np.float32)
    k[0, 0] = [1, 1, 0, 0]
    w = np.array([[[3.0, 5.0]]], np.float32)
    p = make(q, k, w, topk=1)
    out = oracle_mod.indexer_backward(oracle_mod.Inputs(p), np.array([[0]], np.int32),
                                      np.array([[2.0]], np.float32))
    assert np.all(out["dq"][0, 0] == 0.0)
    assert np.array_equal(out["dq"][0, 1], 2.0 * 5.0 * k[0, 0])
    assert np.array_equal(out["dk"][0, 0], 2.0 * 5.0 * q[0, 0, 1])
    assert np.array_equal(out["dw"][0], [0.0, 2.0 * 2.0])

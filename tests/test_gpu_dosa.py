"""DoSA bound pruning (DSA_FLAG_DOSA): the selected set and every score are
bit-identical to the same call without the flag, on integer inputs (exact, and
also equal to the oracle), on real-valued inputs (and within the tolerance rule
of the oracle), on ragged batches, decode and every supported head count; most
(row, tile) pairs are pruned where the block bounds are tight (keys constant
over blocks), none without the flag.  Where the seeds rule out fewer than 1/32
of the blocks the scan does not check the bounds at all (the counts and
thresholds stay exact either way).

DoSA ("The new bottleneck of sparse attention", route five) keeps the exact
top-k: a (row, key tile) pair is skipped only when an upper bound of every
score in it lies below the row's running threshold, and such candidates are
ones the threshold filter rejects anyway.
"""
import numpy as np
import pytest

import oracle
import parity
from sparse_attention_token_dsa_b200 import inputs as gen

pytestmark = pytest.mark.gpu

TOL_BF16 = 1e-3


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


def both(B, p, extra=0):
    """(idx, score) without and with DSA_FLAG_DOSA, sorted rows, plus the count."""
    import torch
    q, k, w = dev(p.q), dev(p.k), dev(p.w)
    pos0, klen = dev(p.q_pos0), dev(p.k_len)
    out = []
    pruned = []
    for fl in (0, B.DSA_FLAG_DOSA):
        flags = B.DSA_FLAG_SORTED | B.DSA_FLAG_CHECK | extra | fl
        pr = B.problem(q, k, p.topk, pos0, klen, flags)
        ws = torch.empty(B.dsa_workspace_size(pr), dtype=torch.uint8, device="cuda")
        idx, sc = B.dsa_index(q, k, w, p.topk, q_pos0=pos0, k_len=klen, flags=flags,
                              workspace=ws)
        torch.cuda.synchronize()
        pruned.append(B.dsa_read_pruned(ws))
        out.append((idx.cpu().numpy().reshape(-1, p.topk), sc.cpu().numpy().reshape(-1, p.topk)))
    (i0, s0), (i1, s1) = out
    assert pruned[0] == 0
    return i0, s0, i1, s1, pruned[1]


def identical(i0, s0, i1, s1):
    assert np.array_equal(i0, i1), parity._first_diff(i1, i0)
    assert np.array_equal(s0.view(np.uint32), s1.view(np.uint32))


def tile_pairs(p):
    """(row, 128-key tile) pairs of the problem's legal prefixes: the most a call can skip."""
    n = 0
    for b in range(p.batch):
        for t in range(p.n_q):
            n += (min(p.pos0(b) + t + 1, p.klen(b)) + 127) // 128
    return n


def test_integer_segments_bit_exact_and_pruned(B):
    """Keys constant on 1024-token segments (the bound block): the box bound is
    tight, most pairs are skipped, ties are everywhere, and the result is
    bit-exact against both the unpruned scan and the oracle."""
    p = gen.segment_integer_problem(40, 1, 1024, 8192 + 300, 64, 128, 256, seg=1024, tail=False)
    i0, s0, i1, s1, pruned = both(B, p)
    identical(i0, s0, i1, s1)
    ri, rs, _, _ = oracle.dsa(oracle.Inputs(p), p.topk)
    parity.exact(i1, s1, ri, rs)
    total = tile_pairs(p)
    print(f"dosa integer segments: pruned {pruned} of {total} pairs")
    assert total // 2 < pruned <= total          # the seeds rule out most blocks


@pytest.mark.parametrize("heads", [32, 64, 128])
def test_low_noise_clusters_bit_identical(B, heads):
    """Keys with locality (long runs around a centre, small noise): the block
    bound bites on real-valued inputs; result identical, checked against the
    oracle within the tolerance rule on sampled rows."""
    p = gen.normal_problem(41, 1, 1500, 12000, heads, 128, 512, key_structure="clusters",
                           n_centres=64, mean_run=2048.0, noise=0.003)
    i0, s0, i1, s1, pruned = both(B, p)
    identical(i0, s0, i1, s1)
    print(f"dosa clusters H={heads}: pruned {pruned} of {tile_pairs(p)} pairs")
    inp = oracle.Inputs(p)
    rows = np.arange(p.n_q)[::37]
    ri, _, rs64, _ = oracle.dsa(inp, p.topk, rows)
    r = parity.within_tolerance(inp, rows, i1[rows], s1[rows], ri, rs64, TOL_BF16,
                                label=f"dosa H={heads}")
    assert r.iou > 0.99


def test_iid_keys_bit_identical(B):
    """Independent N(0,1) keys: the box of a 1024-token block spans the whole
    key distribution in every dimension, so the bound rarely bites; the call
    must still be identical."""
    p = gen.normal_problem(42, 1, 700, 5000, 64, 128, 512)
    i0, s0, i1, s1, pruned = both(B, p)
    identical(i0, s0, i1, s1)
    print(f"dosa iid: pruned {pruned} of {tile_pairs(p)} pairs")


def test_ragged_batches_bit_identical(B):
    """Several sequences with their own query offsets and key lengths, rows
    with fewer legal keys than k, a ragged last bound block."""
    p = gen.segment_integer_problem(43, 3, 777, 5000, 64, 128, 300, seg=1024,
                                    q_pos0=[4223, 0, 1500], k_len=[5000, 777, 2100], tail=False)
    i0, s0, i1, s1, pruned = both(B, p)
    identical(i0, s0, i1, s1)
    ri, rs, _, _ = oracle.dsa(oracle.Inputs(p), p.topk)
    parity.exact(i1, s1, ri, rs)
    assert pruned > 0


def test_decode_bit_identical(B):
    """One query per sequence over long caches (the decode scan layout)."""
    p = gen.segment_integer_problem(44, 6, 1, 40000, 64, 128, 2048, seg=1024,
                                    q_pos0=[39999, 20000, 35000, 1000, 39000, 30000],
                                    k_len=[40000, 20001, 35001, 1001, 39001, 30001], tail=False)
    i0, s0, i1, s1, pruned = both(B, p)
    identical(i0, s0, i1, s1)
    ri, rs, _, _ = oracle.dsa(oracle.Inputs(p), p.topk)
    parity.exact(i1, s1, ri, rs)
    print(f"dosa decode: pruned {pruned} of {tile_pairs(p)} pairs")
    assert pruned > tile_pairs(p) // 2          # the seeds rule out most blocks


def test_position_order_with_dosa(B):
    """DSA_FLAG_BY_POSITION with pruning: the same set, ordered by index."""
    import torch
    p = gen.segment_integer_problem(45, 1, 512, 6000, 64, 128, 256, seg=1024, tail=False)
    q, k, w = dev(p.q), dev(p.k), dev(p.w)
    a, _ = B.dsa_index(q, k, w, p.topk, flags=B.DSA_FLAG_BY_POSITION)
    b, _ = B.dsa_index(q, k, w, p.topk, flags=B.DSA_FLAG_BY_POSITION | B.DSA_FLAG_DOSA)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_full_size_32k_bit_identical(B):
    """32K-token prefill layer, H = 64, k = 2048, on device-drawn inputs with
    locality (keys: per-2048-token centre + 0.01 noise): identical to the
    unpruned call at full size, with pairs skipped."""
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(46)
    L, H, D, K = 32768, 64, 128, 2048
    q = torch.randn((1, L, H, D), generator=g, device="cuda").to(torch.bfloat16)
    cen = torch.randn((1, L // 2048, 1, D), generator=g, device="cuda")
    k = (cen.expand(1, L // 2048, 2048, D).reshape(1, L, D)
         + 0.01 * torch.randn((1, L, D), generator=g, device="cuda")).to(torch.bfloat16)
    w = torch.randn((1, L, H), generator=g, device="cuda") / 8.0
    res = []
    for fl in (0, B.DSA_FLAG_DOSA):
        pr = B.problem(q, k, K, None, None, fl)
        ws = torch.empty(B.dsa_workspace_size(pr), dtype=torch.uint8, device="cuda")
        idx, sc = B.dsa_index(q, k, w, K, flags=B.DSA_FLAG_SORTED | B.DSA_FLAG_CHECK | fl,
                              workspace=ws)
        torch.cuda.synchronize()
        res.append((idx, sc, B.dsa_read_pruned(ws)))
    assert torch.equal(res[0][0], res[1][0])
    assert torch.equal(res[0][1].view(torch.int32), res[1][1].view(torch.int32))
    print(f"dosa 32k: pruned {res[1][2]} of about {L * (L // 128) // 2} pairs")


@pytest.mark.parametrize("kind", ["integer", "normal"])
def test_block_bounds_match_oracle_and_dominate_every_legal_score(B, kind):
    """The bound kernel (tcgen05 GEMM of [q+ | q-] against the block ranges)
    against the oracle's block bounds with their rounding allowance: exact on
    integer inputs up to the fp32 allowance, within half the allowance on real
    inputs; the upper bound never below and the lower bound never above the
    oracle's score of any legal key of the block (partial last blocks, ragged
    prefixes, blocks past the prefix at -inf)."""
    if kind == "integer":
        p = gen.segment_integer_problem(47, 2, 150, 3000, 64, 128, 32, seg=512,
                                        q_pos0=[2850, 100], k_len=[3000, 2400])
    else:
        p = gen.normal_problem(48, 2, 150, 3000, 64, 128, 32, q_pos0=[2850, 100],
                               k_len=[3000, 2400])
    ubt, lbt = B.dsa_dosa_bounds(dev(p.q), dev(p.k), dev(p.w), q_pos0=dev(p.q_pos0),
                                 k_len=dev(p.k_len))
    ub = ubt.cpu().numpy().astype(np.float64)
    lb = lbt.cpu().numpy().astype(np.float64)
    inp = oracle.Inputs(p)
    nblk = ub.shape[1]
    assert nblk == 3
    worst = 0.0
    for row in range(p.batch * p.n_q):
        ref, lref, sl = oracle.dosa_bounds(inp, row, 10)
        n = p.legal_count(row)
        for a in range(nblk):
            if a * 1024 >= n:
                assert ub[row, a] == -np.inf and lb[row, a] == -np.inf
                continue
            s = np.arange(a * 1024, min((a + 1) * 1024, n))
            I = oracle.score_pairs(inp, np.full(len(s), row), s)
            for got, want in ((ub[row, a], ref[a] + sl[a]), (lb[row, a], lref[a] - sl[a])):
                tol = (1e-6 * (abs(want) + sl[a]) + 1e-6) if kind == "integer" else 0.5 * sl[a]
                assert abs(got - want) <= tol, (row, a, got, want)
                worst = max(worst, abs(got - want) / max(sl[a], 1e-30))
            assert ub[row, a] >= I.max()
            assert lb[row, a] <= I.min()
    print(f"dosa bounds {kind}: largest |gpu - oracle| / allowance {worst:.3e}")

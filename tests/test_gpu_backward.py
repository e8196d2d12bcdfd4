"""GPU parity of dsa_indexer_backward (indexer backward with score recompute,
"PaperTrace 2.2.2 MISA, LISA and ResMiSA", section 2.3) against the oracle.

Integer inputs (q, k in [-3, 3], w and g in [-2, 2]): g w is exact in bf16 and
every sum is an integer below 2^24, so dq, dk and dw are bit-exact whatever the
summation order.  Real inputs: the products g w 1[z > 0] enter the dq / dk
tensor-core products in bf16 (fp32 accumulation), so each element is within
2^-8 of the sum of the absolute values of its terms; dw is reduced in fp32 from
the recomputed z and is checked at 2^-16 of its own absolute-value sum.
"""
import numpy as np
import pytest

import oracle
from sparse_attention_token_dsa_b200 import inputs as gen

pytestmark = pytest.mark.gpu


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


def selection(p, topk, seed, empty=0.1):
    """topk distinct causal positions per row (fewer on short prefixes), -1 padded."""
    r = np.random.default_rng(seed)
    sel = np.full((p.batch * p.n_q, topk), -1, np.int32)
    for row in range(p.batch * p.n_q):
        n = p.legal_count(row)
        pick = r.permutation(n)[:topk]
        pick[r.random(len(pick)) < empty] = -1
        sel[row, :len(pick)] = pick
    return sel


def run(B, p, sel, g):
    import torch
    dq, dk, dw = B.indexer_backward(_t(p.q), _t(p.k), _t(p.w), _t(sel), _t(g),
                                    flags=B.DSA_FLAG_CHECK)
    torch.cuda.synchronize()
    return dq.cpu().numpy().astype(np.float64), dk.cpu().numpy().astype(np.float64), \
        dw.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("topk", [256, 200])
def test_backward_integer_bit_exact(B, topk):
    p = gen.integer_problem(120, 2, 150, 700, 64, 128, topk, dtype=gen.BF16)
    sel = selection(p, topk, 1)
    g = np.random.default_rng(2).integers(-2, 3, size=sel.shape).astype(np.float32)
    dq, dk, dw = run(B, p, sel, g)
    ref = oracle.indexer_backward(oracle.Inputs(p), sel, g)
    assert np.array_equal(dq.reshape(ref["dq"].shape), ref["dq"])
    assert np.array_equal(dw.reshape(ref["dw"].shape), ref["dw"])
    assert np.array_equal(dk.reshape(ref["dk"].shape), ref["dk"])


def test_backward_real_within_bound(B):
    p = gen.normal_problem(121, 1, 300, 900, 64, 128, 384)
    sel = selection(p, 384, 3)
    g = np.random.default_rng(4).standard_normal(sel.shape).astype(np.float32)
    dq, dk, dw = run(B, p, sel, g)
    ref = oracle.indexer_backward(oracle.Inputs(p), sel, g)
    # absolute-value sums of the terms of every element
    q = gen.bf16_bits_to_f32(p.q).astype(np.float64).reshape(-1, 64, 128)
    k = gen.bf16_bits_to_f32(p.k).astype(np.float64).reshape(-1, 128)
    w = p.w.reshape(-1, 64).astype(np.float64)
    aq = np.zeros_like(ref["dq"])
    ak = np.zeros_like(ref["dk"]).reshape(-1, 128)
    aw = np.zeros_like(ref["dw"])
    for row in range(sel.shape[0]):
        ok = sel[row] >= 0
        s = sel[row][ok]
        gg = g[row][ok].astype(np.float64)
        z = q[row] @ k[s].T                                   # [64, n]
        m = (z > 0).astype(np.float64)
        coef = np.abs(gg)[None] * np.abs(w[row])[:, None] * m  # [64, n]
        aq[row] += coef @ np.abs(k[s])
        np.add.at(ak, s, coef.T @ np.abs(q[row]))
        aw[row] += (np.abs(gg)[None] * np.maximum(z, 0)).sum(1)
    ak = ak.reshape(ref["dk"].shape)
    eq = np.abs(dq.reshape(aq.shape) - ref["dq"])
    ek = np.abs(dk.reshape(ak.shape) - ref["dk"])
    ew = np.abs(dw.reshape(aw.shape) - ref["dw"])
    assert np.all(eq <= 2.0 ** -8 * aq + 1e-6), f"dq: {np.max(eq / (aq + 1e-30)):.3e}"
    assert np.all(ek <= 2.0 ** -8 * ak + 1e-6), f"dk: {np.max(ek / (ak + 1e-30)):.3e}"
    assert np.all(ew <= 2.0 ** -16 * aw + 1e-6), f"dw: {np.max(ew / (aw + 1e-30)):.3e}"
    print(f"backward: max |d|/bound dq {np.max(eq / (2.0 ** -8 * aq + 1e-6)):.3f}, "
          f"dk {np.max(ek / (2.0 ** -8 * ak + 1e-6)):.3f}, dw {np.max(ew / (2.0 ** -16 * aw + 1e-6)):.3f}")


def test_backward_accumulates_into_dk(B):
    """dk is added to: two calls on halves of the selection equal one call."""
    import torch
    p = gen.integer_problem(122, 1, 64, 300, 64, 128, 128, dtype=gen.BF16)
    sel = selection(p, 128, 5, empty=0.0)
    g = np.random.default_rng(6).integers(-2, 3, size=sel.shape).astype(np.float32)
    _, dk_all, _ = run(B, p, sel, g)
    a, b = sel.copy(), sel.copy()
    a[:, 64:] = -1
    b[:, :64] = -1
    dk = torch.zeros((1, 300, 128), dtype=torch.float32, device="cuda")
    for part in (a, b):
        B.indexer_backward(_t(p.q), _t(p.k), _t(p.w), _t(part), _t(g), dk=dk)
    torch.cuda.synchronize()
    assert np.array_equal(dk.cpu().numpy().astype(np.float64), dk_all)

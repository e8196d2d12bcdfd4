"""The seeded input generators: bf16 formatting, determinism and the planted
structure the benchmark relies on (needles the exact indexer must find,
clustered key runs for HISA).  CPU only.
"""
import numpy as np
import torch

import oracle
from sparse_attention_token_dsa_b200 import inputs as gen


def test_bf16_words_match_torch_rounding():
    """f32 -> bf16 words round to nearest, ties to even, like torch's cast."""
    rng = np.random.default_rng(0)
    x = rng.standard_normal(4096).astype(np.float32) * np.float32(1e3)
    # exact ties: a bf16 value plus half of its last place, both even and odd
    base = gen.bf16_bits_to_f32(gen.f32_to_bf16_bits(rng.standard_normal(256).astype(np.float32)))
    ties = (base.view(np.uint32) | np.uint32(0x8000)).view(np.float32)
    x = np.concatenate([x, ties, np.array([0.0, -0.0, 1.0, -2.5, 3.4e38], np.float32)])
    ours = gen.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_generators_are_deterministic():
    a = gen.normal_problem(9, 2, 64, 96, 8, 128, 16, n_needles=3, key_structure="clusters")
    b = gen.normal_problem(9, 2, 64, 96, 8, 128, 16, n_needles=3, key_structure="clusters")
    c = gen.normal_problem(10, 2, 64, 96, 8, 128, 16, n_needles=3, key_structure="clusters")
    for f in ("q", "k", "w"):
        assert np.array_equal(getattr(a, f), getattr(b, f))
        assert not np.array_equal(getattr(a, f), getattr(c, f))
    assert a.needles == b.needles
    d1 = gen.decode_problem(3, 2, 300, 8, 128, 16)[0]
    d2 = gen.decode_problem(3, 2, 300, 8, 128, 16)[0]
    assert np.array_equal(d1.k, d2.k) and d1.n_q == 1 and d1.pos0(0) == 299


def test_integer_problem_stays_exact_in_fp32():
    """Integer q, k in [-3, 3], w in [-2, 2]: every partial sum of a score is an
    integer of magnitude at most 3 * 3 * 128 * 64 * 2 < 2^24."""
    p = gen.integer_problem(1, 1, 64, 64, 64, 128, 8)
    assert np.all(np.abs(p.q) <= 3) and np.all(np.abs(p.k) <= 3) and np.all(np.abs(p.w) <= 2)
    assert np.all(p.q == np.round(p.q)) and np.all(p.w == np.round(p.w))
    assert 3 * 3 * 128 * 64 * 2 < 2 ** 24


def test_planted_needles_are_in_the_exact_top_k():
    """Each planted needle key ranks in the exact top-k of its probe row, so a
    needle recall below 1 on the GPU would be the kernel's fault."""
    oracle.build()
    p = gen.normal_problem(2, 1, 1024, 1024, 64, 128, 128, n_needles=6)
    rows = np.array([b * p.n_q + t for b, t in zip(p.needles["b"], p.needles["t"])], np.int64)
    idx, _, _, _ = oracle.dsa(oracle.Inputs(p), p.topk, rows)
    for a, s in enumerate(p.needles["s"]):
        assert s in idx[a], f"needle {s} of row {rows[a]} not in the top-{p.topk}"
        assert s <= p.pos0(0) + p.needles["t"][a]        # a legal (past) key


def test_clustered_keys_form_runs():
    """Neighbouring keys share a centre far more often than independent keys."""
    def neighbour_cos(p):
        k = gen.bf16_bits_to_f32(p.k[0]).astype(np.float64)
        k /= np.linalg.norm(k, axis=1, keepdims=True)
        return float(np.mean(np.sum(k[1:] * k[:-1], axis=1)))
    iid = gen.normal_problem(5, 1, 8, 4096, 8, 128, 16)
    clu = gen.normal_problem(5, 1, 8, 4096, 8, 128, 16, key_structure="clusters")
    assert abs(neighbour_cos(iid)) < 0.05
    assert neighbour_cos(clu) > 0.5


def test_cluster_noise_and_constant_segments():
    """The locality knobs: clustered keys with small noise stay within a narrow
    box along each run, the default noise level reproduces the 0.5 recipe, and
    segment keys without the tail token are exactly constant on each segment."""
    a = gen.normal_problem(11, 1, 32, 4096, 8, 128, 16, key_structure="clusters",
                           n_centres=4, mean_run=4096.0, noise=0.01)
    k = gen.bf16_bits_to_f32(a.k)[0]
    # adjacent keys inside one run differ by the noise only (a centre change is rare)
    d = np.abs(np.diff(k, axis=0)).max(axis=1)
    assert np.median(d) < 0.1
    b = gen.normal_problem(12, 1, 32, 512, 8, 128, 16, key_structure="clusters")
    c = gen.normal_problem(12, 1, 32, 512, 8, 128, 16, key_structure="clusters", noise=0.5)
    assert np.array_equal(b.k, c.k)
    s = gen.segment_integer_problem(13, 1, 16, 3000, 8, 128, 16, seg=1024, tail=False)
    ks = gen.bf16_bits_to_f32(s.k)[0]
    for lo in range(0, 3000, 1024):
        seg = ks[lo:min(lo + 1024, 3000)]
        assert np.all(seg == seg[0])
    t = gen.segment_integer_problem(13, 1, 16, 3000, 8, 128, 16, seg=1024)
    kt = gen.bf16_bits_to_f32(t.k)[0]
    assert not np.all(kt[:1024] == kt[0])           # the tail token differs

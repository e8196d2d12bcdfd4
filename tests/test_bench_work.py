"""The roofline numerators bench.py reports, pinned to closed forms.

`achieved` divides an algorithmic work count by a measured time, so the count
itself is checked here against sums written in closed form for the causal
layouts of the benchmark workloads (CPU only; no problem data is generated).
"""
import numpy as np

import bench
from sparse_attention_token_dsa_b200 import inputs as gen


def _shape(batch, n_q, n_k, heads, dim=128):
    z = np.zeros(1, np.float32)
    return gen.Problem(batch, n_q, n_k, heads, dim, 2048, gen.BF16, gen.BF16, z, z, z)


def _ceil_sum(L, B):
    """sum_{t<L} ceil((t + 1) / B) for L a multiple of B: B * M (M + 1) / 2, M = L / B."""
    M = L // B
    return B * M * (M + 1) // 2


def _min_sum(L, c):
    """sum_{t<L} min(c, t + 1) for c <= L."""
    return c * (c + 1) // 2 + c * (L - c)


def test_dsa_prefill_work():
    for name, L in (("dsa_prefill_32k", 32768), ("dsa_prefill_128k", 131072)):
        p = _shape(1, L, L, 64)
        pairs, dots, flops = bench.algorithmic_work(p, bench.WORKLOADS[name])
        assert pairs == L * (L + 1) // 2
        assert dots == 64 * pairs and flops == 2.0 * dots * 128
    # the 32K layer: 536,887,296 causal pairs, 8.796 TFLOP
    p = _shape(1, 32768, 32768, 64)
    pairs, _, flops = bench.algorithmic_work(p, bench.WORKLOADS["dsa_prefill_32k"])
    assert pairs == 536_887_296 and round(flops / 1e12, 3) == 8.796


def test_decode_bytes():
    p = _shape(32, 1, 131072, 64)
    # 32 x 131072 x (128 B codes + 4 B scale) + 32 x 64 x (256 B bf16 q + 4 B w)
    assert bench.decode_bytes(p) == 32 * 131072 * 132 + 32 * 64 * 260 == 554_180_608
    _, dots, _ = bench.algorithmic_work(p, bench.WORKLOADS["dsa_decode_128k"])
    assert dots == 32 * 64 * 131072


def test_misa_work():
    L = 131072
    for name, H in (("misa_prefill_128k", 64), ("misa_prefill_128k_h32", 32)):
        p = _shape(1, L, L, H)
        _, dots, _ = bench.algorithmic_work(p, bench.WORKLOADS[name])
        router = H * _ceil_sum(L, 1024)          # H M_t block representatives per row
        routed = 8 * L * (L + 1) // 2            # h = 8 heads over every legal key
        assert _ceil_sum(L, 1024) == 8_454_144
        assert dots == router + routed
    p = _shape(1, L, L, 64)
    _, dots, flops = bench.algorithmic_work(p, bench.WORKLOADS["misa_dagger_prefill_128k"])
    rerank = 64 * _min_sum(L, 8192)              # all heads over min(k', legal) candidates
    assert _min_sum(L, 8192) == 1_040_191_488
    assert dots == 64 * 8_454_144 + 8 * L * (L + 1) // 2 + rerank


def test_hisa_work():
    L = 131072
    p = _shape(1, L, L, 64)
    _, dots, flops = bench.algorithmic_work(p, bench.WORKLOADS["hisa_prefill_128k"])
    coarse = 64 * _ceil_sum(L, 64)
    assert _ceil_sum(L, 64) == 134_283_264
    assert dots == coarse + 64 * _min_sum(L, 128 * 64)
    # stacked: router (all heads) + coarse and rerank with h = 8 heads, the
    # scope table's 0.14 + 0.28 + 2.13 TFLOP (2.54 before rounding the parts)
    _, dots, flops = bench.algorithmic_work(p, bench.WORKLOADS["hisa_misa_prefill_128k"])
    parts = (64 * 8_454_144, 8 * 134_283_264, 8 * 1_040_191_488)
    assert dots == sum(parts)
    assert [round(2 * 128 * x / 1e12, 2) for x in parts] == [0.14, 0.28, 2.13]
    assert abs(flops / 1e12 - 2.55) < 0.01


def test_lisa_and_resmisa_work():
    """LISA: one fused-query dot per legal key; LISA-dagger adds H min(M, t + 1);
    ResMiSA: H M_t block bounds + (1 + r) dots per legal key."""
    L = 131072
    p = _shape(1, L, L, 64)
    pairs = L * (L + 1) // 2
    _, dots, _ = bench.algorithmic_work(p, bench.WORKLOADS["lisa_prefill_128k"])
    assert dots == pairs
    _, dots, _ = bench.algorithmic_work(p, bench.WORKLOADS["lisa_dagger_prefill_128k"])
    assert dots == pairs + 64 * _min_sum(L, 8192)
    _, dots, _ = bench.algorithmic_work(p, bench.WORKLOADS["resmisa_prefill_128k"])
    assert dots == 64 * _ceil_sum(L, 1024) + 8 * pairs

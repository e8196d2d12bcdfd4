"""Seeded synthetic inputs for the indexer workloads.

This module only draws numbers and formats them (fp32 -> bf16 words); it holds
none of the indexer arithmetic, so the CPU oracle and the CUDA path can both
consume exactly the same bytes.  Seeds follow ``1000 * workload + tensor_id``
with tensor ids q=1, k=2, w=3, structure (needles / clusters)=4.

Workload shapes come from the pages' own settings: H_I = 64 (DeepSeek-V3.2) or
32 (GLM-5), d = 128, k = 2048, MISA B = 1024 / h = 8 / k' = 8192, HISA b = 64 /
r = 128 ("MISA: Mixture of Indexer Sparse Attention", method steps and results;
"PaperTrace 2.2.2 MISA, LISA and ResMiSA", section 2.3 decode cost example).
"""
from __future__ import annotations

import dataclasses
import numpy as np

F32, BF16, E4M3 = 0, 1, 2


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even) and return the raw uint16 words."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass
class Problem:
    """One synthetic indexer problem (host arrays, C-contiguous)."""
    batch: int
    n_q: int
    n_k: int
    heads: int
    dim: int
    topk: int
    q_dtype: int
    k_dtype: int
    q: np.ndarray                    # [B,n_q,H,d] float32 (F32) or uint16 (BF16)
    k: np.ndarray                    # [B,n_k,d]   float32 (F32) or uint16 (BF16)
    w: np.ndarray                    # [B,n_q,H] float32
    q_pos0: np.ndarray | None = None  # [B] int32
    k_len: np.ndarray | None = None   # [B] int32
    needles: dict | None = None       # planted needle positions / probe rows
    name: str = ""

    def pos0(self, b: int) -> int:
        return int(self.q_pos0[b]) if self.q_pos0 is not None else self.n_k - self.n_q

    def klen(self, b: int) -> int:
        return int(self.k_len[b]) if self.k_len is not None else self.n_k

    def legal_count(self, row: int) -> int:
        b, i = divmod(row, self.n_q)
        return max(0, min(self.pos0(b) + i + 1, self.klen(b)))


def _rng(workload: int, tensor_id: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(1000 * workload + tensor_id))


def _normal(rng: np.random.Generator, shape, scale: float = 1.0) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        x *= np.float32(scale)
    return x


def integer_problem(workload: int, batch: int, n_q: int, n_k: int, heads: int, dim: int,
                    topk: int, qk_max: int = 3, w_max: int = 2, dtype: int = F32,
                    q_pos0=None, k_len=None) -> Problem:
    """q, k uniform integers in [-qk_max, qk_max], w uniform integers in [-w_max, w_max].

    With |q|,|k| <= 3, w <= 2, d = 128 and 64 heads every partial sum is an
    integer below 2^24, so fp32 accumulation is exact in any order.
    """
    q = _rng(workload, 1).integers(-qk_max, qk_max + 1, size=(batch, n_q, heads, dim)).astype(np.float32)
    k = _rng(workload, 2).integers(-qk_max, qk_max + 1, size=(batch, n_k, dim)).astype(np.float32)
    w = _rng(workload, 3).integers(-w_max, w_max + 1, size=(batch, n_q, heads)).astype(np.float32)
    if dtype == BF16:
        q, k = f32_to_bf16_bits(q), f32_to_bf16_bits(k)
    return Problem(batch, n_q, n_k, heads, dim, topk, dtype, dtype, q, k, w,
                   None if q_pos0 is None else np.asarray(q_pos0, np.int32),
                   None if k_len is None else np.asarray(k_len, np.int32), name="integer")


def segment_integer_problem(workload: int, batch: int, n_q: int, n_k: int, heads: int,
                            dim: int, topk: int, seg: int, q_pos0=None, k_len=None,
                            tail: bool = True) -> Problem:
    """Integer problem whose keys are constant on aligned segments of `seg` tokens.

    q uniform integers in [-3, 3], w in [-2, 2]; every key of segment i equals
    an integer vector c_i in [-2, 2]^d except the segment's last token, which
    is c_i + e_i with e_i integers in [-1, 1]^d (bf16 storage, exact).  Any
    mean over a prefix of a power-of-two block aligned inside a segment is
    either c_i or c_i + e_i / (block size): a dyadic number with a small
    numerator, so pooled keys, their dot products with q and the sums over
    heads and blocks stay exactly representable in fp32 at the test sizes.
    tail=False leaves out the e_i (keys exactly constant on each segment).
    """
    q = _rng(workload, 1).integers(-3, 4, size=(batch, n_q, heads, dim)).astype(np.float32)
    r = _rng(workload, 2)
    nseg = (n_k + seg - 1) // seg
    c = r.integers(-2, 3, size=(batch, nseg, dim)).astype(np.float32)
    e = r.integers(-1, 2, size=(batch, nseg, dim)).astype(np.float32)
    k = np.repeat(c, seg, axis=1)[:, :n_k].copy()
    if tail:
        last = np.arange(seg - 1, n_k, seg)
        k[:, last] += e[:, : len(last)]
    w = _rng(workload, 3).integers(-2, 3, size=(batch, n_q, heads)).astype(np.float32)
    return Problem(batch, n_q, n_k, heads, dim, topk, BF16, BF16, f32_to_bf16_bits(q),
                   f32_to_bf16_bits(k), w,
                   None if q_pos0 is None else np.asarray(q_pos0, np.int32),
                   None if k_len is None else np.asarray(k_len, np.int32), name="segments")


def normal_problem(workload: int, batch: int, n_q: int, n_k: int, heads: int, dim: int,
                   topk: int, q_pos0=None, k_len=None, n_needles: int = 0,
                   key_structure: str = "iid", n_centres: int = 256,
                   mean_run: float = 512.0, noise: float = 0.5) -> Problem:
    """q, k ~ N(0,1) rounded to bf16; w ~ N(0, 1/H) fp32.

    key_structure
      "iid"      independent N(0,1) keys;
      "clusters" keys drawn from `n_centres` Gaussian centres assigned to
                 contiguous runs of geometric length (mean `mean_run`), plus
                 `noise` N(0,1), rescaled to unit variance — important tokens
                 gathered in contiguous regions, the structure HISA's block
                 filter relies on ("The new bottleneck of sparse attention",
                 route one: HISA, observation).
    n_needles > 0 plants keys aligned with a probe query: needle position s_i
    uniform in [0, L/2), probe row t_i uniform in [L/2, L);
    u_i = unit(sum_{j: w>0} w_{t_i,j} q_{t_i,j}), k_{s_i} = 0.8 sqrt(d) u_i + 0.6 eps.
    """
    q32 = _normal(_rng(workload, 1), (batch, n_q, heads, dim))
    if key_structure == "iid":
        k32 = _normal(_rng(workload, 2), (batch, n_k, dim))
    elif key_structure == "clusters":
        r = _rng(workload, 4)
        centres = r.standard_normal(size=(batch, n_centres, dim), dtype=np.float32)
        k32 = np.empty((batch, n_k, dim), np.float32)
        eps = _normal(_rng(workload, 2), (batch, n_k, dim), noise)
        for b in range(batch):
            pos = 0
            while pos < n_k:
                run = int(r.geometric(1.0 / mean_run))
                c = int(r.integers(0, n_centres))
                k32[b, pos:pos + run] = centres[b, c]
                pos += run
        k32 += eps
        k32 /= np.float32(np.sqrt(1.0 + noise * noise))
    else:
        raise ValueError(key_structure)
    w = _normal(_rng(workload, 3), (batch, n_q, heads), 1.0 / np.sqrt(heads))
    needles = None
    if n_needles > 0:
        r = _rng(workload, 4)
        needles = {"s": [], "t": [], "b": []}
        pos0 = n_k - n_q if q_pos0 is None else None
        for i in range(n_needles):
            b = int(r.integers(0, batch))
            p0 = pos0 if pos0 is not None else int(q_pos0[b])
            lo_t = max(n_q // 2, 0)
            t = int(r.integers(lo_t, n_q))
            pos_t = p0 + t
            s = int(r.integers(0, max(1, (pos_t + 1) // 2)))
            qt = q32[b, t]
            wt = w[b, t]
            u = (wt[wt > 0][:, None] * qt[wt > 0]).sum(0) if np.any(wt > 0) else qt[0]
            u = u / max(np.linalg.norm(u), 1e-12)
            eps = r.standard_normal(size=dim).astype(np.float32)
            k32[b, s] = (0.8 * np.sqrt(dim) * u + 0.6 * eps).astype(np.float32)
            needles["s"].append(s)
            needles["t"].append(t)
            needles["b"].append(b)
    return Problem(batch, n_q, n_k, heads, dim, topk, BF16, BF16,
                   f32_to_bf16_bits(q32), f32_to_bf16_bits(k32), w,
                   None if q_pos0 is None else np.asarray(q_pos0, np.int32),
                   None if k_len is None else np.asarray(k_len, np.int32),
                   needles, name=key_structure)


def decode_problem(workload: int, batch: int, n_k: int, heads: int, dim: int, topk: int,
                   k_len=None) -> tuple[Problem, np.ndarray]:
    """One new query per sequence at position n_k-1 (its own key already cached).

    Returns the problem with bf16 q and the fp32 keys (to be quantised to e4m3
    by whichever side consumes them); problem.k holds the bf16 rounding of the
    same keys for the unquantised comparison.
    """
    q32 = _normal(_rng(workload, 1), (batch, 1, heads, dim))
    k32 = _normal(_rng(workload, 2), (batch, n_k, dim))
    w = _normal(_rng(workload, 3), (batch, 1, heads), 1.0 / np.sqrt(heads))
    p = Problem(batch, 1, n_k, heads, dim, topk, BF16, BF16, f32_to_bf16_bits(q32),
                f32_to_bf16_bits(k32), w,
                None if k_len is None else np.asarray(k_len, np.int32) - 1,
                None if k_len is None else np.asarray(k_len, np.int32), name="decode")
    return p, k32


def stratified_rows(p: Problem, n: int, seed: int = 7) -> np.ndarray:
    """Rows for sampled checks: first, last, needle probes and n rows stratified over t."""
    total = p.batch * p.n_q
    rows = {0, total - 1}
    if p.needles:
        for b, t in zip(p.needles["b"], p.needles["t"]):
            rows.add(b * p.n_q + t)
    r = np.random.Generator(np.random.PCG64(seed))
    edges = np.linspace(0, total, n + 1).astype(np.int64)
    for a, e in zip(edges[:-1], edges[1:]):
        if e > a:
            rows.add(int(r.integers(a, e)))
    return np.array(sorted(rows), dtype=np.int64)

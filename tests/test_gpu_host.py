"""dsa_index_host: query rows and results in host memory, streamed in chunks
through two device slots with the copies overlapping the scan.  Its results
equal dsa_index's bit for bit (same kernels on the same rows; sorted rows so
the order is fixed), on integer inputs also the oracle's, across ragged
batches, chunk boundaries that cut sequences unevenly, e4m3 operands and a
full 32K layer."""
import numpy as np
import pytest

import oracle
import parity
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


def host(x):
    import torch
    if x is None:
        return None
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
    return torch.from_numpy(np.ascontiguousarray(x)).pin_memory()


def dev(x):
    import torch
    t = host(x)
    return None if t is None else t.cuda()


@pytest.mark.parametrize("chunk", [64, 250, 4096])
def test_integer_ragged_batches_match_dsa_index_and_oracle(B, chunk):
    import torch
    p = gen.integer_problem(130, 3, 700, 1500, 64, 128, 128, q_pos0=[800, 0, 300],
                            k_len=[1500, 700, 1000], dtype=gen.BF16)
    flags = B.DSA_FLAG_SORTED | B.DSA_FLAG_CHECK
    qh, wh = host(p.q), host(p.w)
    k, pos0, klen = dev(p.k), dev(p.q_pos0), dev(p.k_len)
    hi, hs = B.dsa_index_host(qh, k, wh, p.topk, q_pos0=pos0, k_len=klen, flags=flags,
                              chunk_rows=chunk)
    torch.cuda.synchronize()
    di, ds = B.dsa_index(qh.cuda(), k, wh.cuda(), p.topk, q_pos0=pos0, k_len=klen, flags=flags)
    torch.cuda.synchronize()
    assert torch.equal(hi, di.cpu())
    assert torch.equal(hs.view(torch.int32), ds.cpu().view(torch.int32))
    ri, rs, _, _ = oracle.dsa(oracle.Inputs(p), p.topk)
    parity.exact(hi.numpy().reshape(-1, p.topk), hs.numpy().reshape(-1, p.topk), ri, rs)


def test_e4m3_operands_match_dsa_index(B):
    import torch
    p = gen.normal_problem(131, 1, 900, 2000, 64, 128, 256)
    qd, kd = dev(p.q), dev(p.k)
    qc, qs = B.dsa_quantize_e4m3(qd.reshape(p.n_q, -1))
    qc = qc.reshape(qd.shape)
    qs = qs.reshape(1, p.n_q)
    kc, ks = B.dsa_quantize_e4m3(kd)
    w = dev(p.w)
    flags = B.DSA_FLAG_SORTED
    hi, hs = B.dsa_index_host(qc.cpu().pin_memory(), kc, w.cpu().pin_memory(), p.topk,
                              q_scale_host=qs.cpu().pin_memory(), k_scale=ks, flags=flags,
                              chunk_rows=300)
    torch.cuda.synchronize()
    di, ds = B.dsa_index(qc, kc, w, p.topk, q_scale=qs, k_scale=ks, flags=flags)
    torch.cuda.synchronize()
    assert torch.equal(hi, di.cpu())
    assert torch.equal(hs.view(torch.int32), ds.cpu().view(torch.int32))


def test_status_is_kept_in_staging(B):
    import torch
    p = gen.integer_problem(132, 1, 300, 300, 64, 128, 32, dtype=gen.BF16)
    k = dev(p.k)
    prob = B.problem(host(p.q), k, p.topk)
    staging = torch.full((B.dsa_host_staging_size(prob, 100),), 0xFF, dtype=torch.uint8,
                         device="cuda")
    B.dsa_index_host(host(p.q), k, host(p.w), p.topk, chunk_rows=100, staging=staging)
    assert B.dsa_read_status(staging) == 0


def test_full_size_32k_matches_dsa_index(B):
    """A 32K-token layer in 8 chunks of 4096 rows: every row equal to the
    one-call device path."""
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(133)
    L, H, D, K = 32768, 64, 128, 2048
    q = torch.randn((1, L, H, D), generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn((1, L, D), generator=g, device="cuda").to(torch.bfloat16)
    w = torch.randn((1, L, H), generator=g, device="cuda") / 8.0
    flags = B.DSA_FLAG_SORTED
    hi, hs = B.dsa_index_host(q.cpu().pin_memory(), k, w.cpu().pin_memory(), K, flags=flags,
                              chunk_rows=4096)
    torch.cuda.synchronize()
    di, ds = B.dsa_index(q, k, w, K, flags=flags)
    torch.cuda.synchronize()
    assert torch.equal(hi, di.cpu())
    assert torch.equal(hs.view(torch.int32), ds.cpu().view(torch.int32))

"""Host-side checks of the C ABI: the library builds, loads without a GPU,
exports every symbol its header declares, and rejects bad arguments before any
CUDA call.  CPU only."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsaidx.h")


@pytest.fixture(scope="module")
def lib():
    from sparse_attention_token_dsa_b200 import build
    path = build.build()
    return C.CDLL(path)


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for f in ("dsa_index", "misa_index", "misa_dagger_index", "hisa_index", "dsa_workspace_size",
              "dsa_status_string", "dsa_quantize_e4m3", "dsa_read_status"):
        assert f in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


@pytest.fixture(scope="module")
def bind(lib):
    from sparse_attention_token_dsa_b200 import binding
    return binding


def _prob(bind, **kw):
    base = dict(batch=1, n_q=16, n_k=64, heads=64, dim=128, topk=8, q_dtype=1, k_dtype=1)
    base.update(kw)
    return bind.DsaProblem(base["batch"], base["n_q"], base["n_k"], base["heads"], base["dim"],
                           base["topk"], base["q_dtype"], base["k_dtype"], None, None, 0)


def test_status_strings(bind):
    for s in (0, -1, -2, -3, -4, -5, -6, -7):
        assert bind.status_string(s) and bind.status_string(s) != "unknown status"
    assert bind.status_string(-99) == "unknown status"


@pytest.mark.parametrize("kw,status", [
    (dict(batch=0), -1), (dict(n_q=0), -1), (dict(topk=0), -1), (dict(dim=64), -2),
    (dict(heads=48), -2), (dict(heads=4), -2), (dict(topk=9000), -2), (dict(q_dtype=7), -1),
    (dict(q_dtype=2, k_dtype=1), -2), (dict(n_k=1 << 25), -2)])
def test_workspace_size_rejects(bind, kw, status):
    n = C.c_size_t(0)
    rc = bind.lib.dsa_workspace_size(C.byref(_prob(bind, **kw)), 0, None, C.byref(n))
    assert rc == status


def test_workspace_size_grows_with_problem(bind):
    a = bind.dsa_workspace_size(_prob(bind, n_q=64, n_k=64))
    b = bind.dsa_workspace_size(_prob(bind, n_q=4096, n_k=4096))
    assert 0 < a < b


def test_dsa_index_rejects_before_launch(bind):
    p = _prob(bind)
    fake = C.c_void_p(0x1000)   # never dereferenced: validation fails first
    f = bind.lib.dsa_index
    assert f(None, fake, None, fake, None, fake, fake, fake, fake, 1 << 30, None) == -1
    assert f(C.byref(p), None, None, fake, None, fake, fake, fake, fake, 1 << 30, None) == -1
    assert f(C.byref(p), C.c_void_p(0x1001), None, fake, None, fake, fake, fake, fake, 1 << 30,
             None) == -1                                           # misaligned q
    assert f(C.byref(p), fake, None, fake, None, fake, fake, fake, None, 0, None) == -3
    assert f(C.byref(p), fake, None, fake, None, fake, fake, fake, fake, 16, None) == -3
    assert f(C.byref(p), fake, None, fake, None, fake, fake, fake, C.c_void_p(0x1008), 1 << 30,
             None) == -1                                           # misaligned workspace
    e4 = _prob(bind, q_dtype=2, k_dtype=2)
    assert f(C.byref(e4), fake, None, fake, None, fake, fake, fake, fake, 1 << 30, None) == -1


def test_quantize_rejects(bind):
    f = bind.lib.dsa_quantize_e4m3
    fake = C.c_void_p(0x1000)
    assert f(None, 1, 4, 128, fake, fake, None) == -1
    assert f(fake, 2, 4, 128, fake, fake, None) == -2
    assert f(fake, 1, 4, 0, fake, fake, None) == -1


def _ws(bind, p, algo, rp):
    n = C.c_size_t(0)
    rc = bind.lib.dsa_workspace_size(C.byref(p), algo, None if rp is None else C.byref(rp),
                                     C.byref(n))
    return rc, n.value


@pytest.mark.parametrize("algo,rp,status", [
    (1, None, -1),                                                  # route params required
    (1, dict(misa_block=128, misa_h=8), 0),
    (1, dict(misa_block=100, misa_h=8), -2),                         # block not a power of two
    (1, dict(misa_block=128, misa_h=12), -2),                        # h not a power of two
    (1, dict(misa_block=128, misa_h=128), -1),                       # h > heads
    (1, dict(misa_block=8, misa_h=8), -2),                           # block below 16
    (2, dict(misa_block=128, misa_h=8, k_prime=4), -1),              # k' < topk
    (2, dict(misa_block=128, misa_h=8, k_prime=9000), -2),           # k' above 8192
    (2, dict(misa_block=128, misa_h=8, k_prime=64), 0),
    (3, dict(hisa_block=64, hisa_r=0), -1),                          # r < 1
    (3, dict(hisa_block=64, hisa_r=16), 0),
    (3, dict(hisa_block=64, hisa_r=16, misa_block=128, misa_h=8), 0),  # stacked
    (3, dict(hisa_block=48, hisa_r=16), -2),
    (7, dict(hisa_block=64, hisa_r=16), -1),                         # unknown algorithm
])
def test_route_workspace_validation(bind, algo, rp, status):
    p = _prob(bind, n_q=256, n_k=1024)
    rc, n = _ws(bind, p, algo, None if rp is None else bind.route_params(**rp))
    assert rc == status
    if status == 0:
        assert n > 0


def test_route_rejects_unsupported_operands(bind):
    rp = bind.route_params(misa_block=128, misa_h=8)
    assert _ws(bind, _prob(bind, q_dtype=0, k_dtype=0), 1, rp)[0] == -2      # fp32: bf16 only
    assert _ws(bind, _prob(bind, q_dtype=1, k_dtype=2), 1, rp)[0] == -2      # e4m3 keys
    # more than 224 full router blocks per sequence
    assert _ws(bind, _prob(bind, n_k=225 * 16), 1, bind.route_params(misa_block=16, misa_h=8))[0] == -2
    assert _ws(bind, _prob(bind, n_k=224 * 16), 1, bind.route_params(misa_block=16, misa_h=8))[0] == 0


def test_route_workspace_is_bounded_by_row_chunks(bind):
    """The candidate logs of 128K prefill rows are chunked: the workspace stays far
    below rows x per-row log size."""
    p = _prob(bind, n_q=131072, n_k=131072, topk=2048)
    rc, n = _ws(bind, p, 2, bind.route_params(misa_block=1024, misa_h=8, k_prime=8192))
    assert rc == 0
    per_row_pass1 = 4 * (2 * 8192 + 768) * 8
    assert n < 131072 * per_row_pass1 / 4
    rc, n2 = _ws(bind, p, 3, bind.route_params(hisa_block=64, hisa_r=128))
    assert rc == 0 and n2 > 0


def test_route_entry_points_reject_before_launch(bind):
    p = _prob(bind, n_q=256, n_k=1024)
    rp = bind.route_params(misa_block=128, misa_h=8, k_prime=64, hisa_block=64, hisa_r=16)
    fake = C.c_void_p(0x1000)
    L = bind.lib
    assert L.misa_index(C.byref(p), None, fake, fake, fake, fake, fake, None, None, fake,
                        1 << 40, None) == -1
    assert L.misa_index(C.byref(p), C.byref(rp), None, fake, fake, fake, fake, None, None, fake,
                        1 << 40, None) == -1
    assert L.misa_index(C.byref(p), C.byref(rp), fake, fake, fake, fake, fake, None, None, fake,
                        16, None) == -3
    assert L.misa_dagger_index(C.byref(p), C.byref(rp), fake, fake, fake, None, fake, None, None,
                               fake, 1 << 40, None) == -1
    assert L.hisa_index(C.byref(p), C.byref(rp), fake, fake, fake, fake, fake, None, None, None,
                        0, None) == -3
    assert L.hisa_index(C.byref(p), C.byref(rp), fake, fake, fake, fake, fake, None, None,
                        C.c_void_p(0x1008), 1 << 40, None) == -1   # misaligned workspace


def test_binding_checks_tensors_before_any_call(bind):
    """The Python binding refuses host, strided or mistyped tensors itself: the
    library takes raw device pointers and could not tell."""
    import torch
    q = torch.zeros((1, 4, 8, 128), dtype=torch.bfloat16)
    k = torch.zeros((1, 16, 128), dtype=torch.bfloat16)
    w = torch.zeros((1, 4, 8), dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA device"):
        bind.dsa_index(q, k, w, 4)
    with pytest.raises(TypeError, match="w: dtype"):
        bind.dsa_index(q, k, w.double(), 4)
    with pytest.raises(ValueError, match="q: must be contiguous"):
        bind.dsa_index(q.transpose(2, 3), k, w, 4)
    with pytest.raises(TypeError, match="k_len: dtype"):
        bind.dsa_index(q, k, w, 4, k_len=torch.zeros(1, dtype=torch.int64))
    with pytest.raises(TypeError, match="q: dtype"):
        bind.dsa_index(q.half(), k, w, 4)
    with pytest.raises(TypeError, match="out_score: dtype"):
        bind.dsa_index(q, k, w, 4, out=(torch.zeros((1, 4, 4), dtype=torch.int32),
                                        torch.zeros((1, 4, 4), dtype=torch.float64)))
    with pytest.raises(ValueError, match="CUDA device"):
        bind.misa_index(q, k, w, 4, 16, 8)
    with pytest.raises(TypeError, match="out_pool: dtype"):
        bind.misa_dagger_index(q, k, w, 4, 16, 8, 8, out_pool=torch.zeros(1, dtype=torch.int64))
    with pytest.raises(ValueError, match="CUDA device"):
        bind.hisa_index(q, k, w, 4, 16, 2)
    with pytest.raises(ValueError, match="CUDA device"):
        bind.dsa_quantize_e4m3(k)
    with pytest.raises(TypeError, match="workspace: dtype"):
        bind.dsa_read_status(torch.zeros(4, dtype=torch.int32))


def _flagged(bind, flags, **kw):
    p = _prob(bind, **kw)
    p.flags = flags
    return p


def test_dosa_flag_validation_and_workspace(bind):
    D = bind.DSA_FLAG_DOSA
    # bf16 q and k with >= 32 heads only
    for kw in (dict(heads=16), dict(q_dtype=2, k_dtype=2), dict(q_dtype=0, k_dtype=0)):
        rc, _ = _ws(bind, _flagged(bind, D, **kw), 0, None)
        assert rc == -2, kw
    # routed algorithms take no DoSA bounds
    rc, _ = _ws(bind, _flagged(bind, D, n_q=256, n_k=1024), 1,
                bind.route_params(misa_block=128, misa_h=8))
    assert rc == -2
    # extra workspace: two range rows and a magnitude per block, bounds per (row, block)
    for nq, nk in ((16, 64), (300, 5000), (4096, 4096)):
        rc0, plain = _ws(bind, _prob(bind, n_q=nq, n_k=nk), 0, None)
        rc1, dosa = _ws(bind, _flagged(bind, D, n_q=nq, n_k=nk), 0, None)
        assert rc0 == 0 and rc1 == 0
        nblk = (nk + 1023) // 1024
        need = nblk * 2 * 512 + nblk * 4 + 2 * nq * nblk * 4 + nq * 4
        assert need <= dosa - plain <= need + 5 * 256, (nq, nk, dosa - plain)


def test_read_pruned_rejects_null(bind):
    n = C.c_ulonglong(0)
    assert bind.lib.dsa_read_pruned(None, None, C.byref(n)) == -1
    assert bind.lib.dsa_read_pruned(C.c_void_p(0x1000), None, None) == -1


def test_host_path_validation(bind):
    f = bind.lib.dsa_index_host
    fake = C.c_void_p(0x1000)
    p = _prob(bind)
    n = C.c_size_t(0)
    assert bind.lib.dsa_host_staging_size(C.byref(p), 0, C.byref(n)) == -1     # chunk rows < 1
    assert bind.lib.dsa_host_staging_size(C.byref(_prob(bind, dim=64)), 16, C.byref(n)) == -2
    sizes = []
    for rows in (1, 8, 16, 1000):
        assert bind.lib.dsa_host_staging_size(C.byref(p), rows, C.byref(n)) == 0
        sizes.append(n.value)
    assert sizes[0] < sizes[1] < sizes[2] == sizes[3]      # chunks never exceed n_q = 16 rows
    big = 1 << 34
    assert f(None, fake, None, fake, None, fake, fake, fake, 8, fake, big, None) == -1
    assert f(C.byref(p), None, None, fake, None, fake, fake, fake, 8, fake, big, None) == -1
    assert f(C.byref(p), fake, None, fake, None, fake, None, fake, 8, fake, big, None) == -1
    assert f(C.byref(p), fake, None, fake, None, fake, fake, fake, 0, fake, big, None) == -1
    assert f(C.byref(p), fake, None, fake, None, fake, fake, fake, 8, fake, 16, None) == -3
    assert f(C.byref(p), fake, None, fake, None, fake, fake, fake, 8, C.c_void_p(0x1008), big,
             None) == -1                                              # misaligned staging
    e4 = _prob(bind, q_dtype=2, k_dtype=2)
    assert f(C.byref(e4), fake, None, fake, fake, fake, fake, fake, 8, fake, big, None) == -1


def test_host_path_binding_checks_devices(bind):
    import torch
    q = torch.zeros((1, 4, 64, 128), dtype=torch.bfloat16)
    w = torch.zeros((1, 4, 64), dtype=torch.float32)
    with pytest.raises(ValueError):
        bind.dsa_index_host(q, q[0, :, 0], w, 2)       # keys must be on the GPU
    with pytest.raises(TypeError):
        bind.dsa_index_host(q.float().int(), q[0, :, 0], w, 2)

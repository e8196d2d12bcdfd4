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
    for s in (0, -1, -2, -3, -4, -5, -6):
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
    e4 = _prob(bind, q_dtype=2, k_dtype=2)
    assert f(C.byref(e4), fake, None, fake, None, fake, fake, fake, fake, 1 << 30, None) == -1


def test_quantize_rejects(bind):
    f = bind.lib.dsa_quantize_e4m3
    fake = C.c_void_p(0x1000)
    assert f(None, 1, 4, 128, fake, fake, None) == -1
    assert f(fake, 2, 4, 128, fake, fake, None) == -2
    assert f(fake, 1, 4, 0, fake, fake, None) == -1

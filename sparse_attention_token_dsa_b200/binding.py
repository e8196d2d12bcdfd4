"""Thin ctypes binding of libdsaidx.so (C ABI declared in include/dsaidx.h).

Argument marshalling only: PyTorch provides device memory and the current
stream; every step of the computation runs in the library's CUDA kernels.
There is no CPU fallback — importing this module without the built library
raises.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdsaidx.so")

DSA_OK, DSA_ERR_INVALID, DSA_ERR_UNSUPPORTED, DSA_ERR_WORKSPACE = 0, -1, -2, -3
DSA_ERR_CUDA, DSA_ERR_NONFINITE, DSA_ERR_TIMEOUT, DSA_ERR_INTERNAL = -4, -5, -6, -7
DSA_F32, DSA_BF16, DSA_E4M3 = 0, 1, 2
DSA_ALGO_DSA, DSA_ALGO_MISA, DSA_ALGO_MISA_DAGGER, DSA_ALGO_HISA = 0, 1, 2, 3
DSA_ALGO_LISA, DSA_ALGO_RESMISA = 4, 5
DSA_FLAG_CHECK = 1
DSA_FLAG_SORTED = 2
DSA_FLAG_BY_POSITION = 4
DSA_FLAG_DOSA = 8                    # exact bound pruning of the dense scan
DSA_FLAG_TEST_STALL = 0x80000000   # tests of the timeout path only (see include/dsaidx.h)


class DsaProblem(C.Structure):
    _fields_ = [("batch", C.c_int32), ("n_q", C.c_int32), ("n_k", C.c_int32),
                ("heads", C.c_int32), ("dim", C.c_int32), ("topk", C.c_int32),
                ("q_dtype", C.c_int32), ("k_dtype", C.c_int32), ("q_pos0", C.c_void_p),
                ("k_len", C.c_void_p), ("flags", C.c_uint32)]


class DsaRouteParams(C.Structure):
    _fields_ = [("misa_block", C.c_int32), ("misa_h", C.c_int32), ("k_prime", C.c_int32),
                ("hisa_block", C.c_int32), ("hisa_r", C.c_int32), ("lisa_pool", C.c_int32),
                ("res_block", C.c_int32), ("res_r", C.c_int32)]


class DsaMlaProblem(C.Structure):
    _fields_ = [("batch", C.c_int32), ("tokens_per_seq", C.c_int32), ("n_k", C.c_int32),
                ("heads", C.c_int32), ("dim_qk", C.c_int32), ("dim_v", C.c_int32),
                ("topk", C.c_int32), ("scale", C.c_float), ("flags", C.c_uint32)]


class DsaError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} ({status})")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m sparse_attention_token_dsa_b200.build`")
    lib = C.CDLL(LIB_PATH)
    vp, i32, i64, sz = C.c_void_p, C.c_int32, C.c_int64, C.c_size_t
    P = C.POINTER(DsaProblem)
    R = C.POINTER(DsaRouteParams)
    lib.dsa_status_string.restype = C.c_char_p
    lib.dsa_status_string.argtypes = [i32]
    lib.dsa_read_status.argtypes = [vp, vp]
    lib.dsa_read_pruned.argtypes = [vp, vp, C.POINTER(C.c_ulonglong)]
    lib.dsa_host_staging_size.argtypes = [P, i32, C.POINTER(sz)]
    lib.dsa_dosa_bounds.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.dsa_index_host.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, i32, vp, sz, vp]
    lib.dsa_workspace_size.argtypes = [P, i32, R, C.POINTER(sz)]
    lib.dsa_index.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.dsa_route_chunk_rows.argtypes = [P, i32, R, C.POINTER(i32)]
    lib.dsa_index_noalloc.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.dsa_index_scan.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.dsa_index_select.argtypes = [P, vp, vp, vp, sz, vp]
    lib.misa_index.argtypes = [P, R, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.misa_dagger_index.argtypes = [P, R, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.hisa_index.argtypes = [P, R, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.lisa_index.argtypes = [P, R, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.resmisa_index.argtypes = [P, R, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.dsa_quantize_e4m3.argtypes = [vp, i32, i64, i32, vp, vp, vp]
    lib.dsa_sparse_mla.argtypes = [C.POINTER(DsaMlaProblem), vp, vp, vp, vp, vp, vp, sz, vp]
    lib.dsa_indexer_backward.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    for f in ("dsa_read_status", "dsa_read_pruned", "dsa_host_staging_size", "dsa_index_host",
              "dsa_dosa_bounds",
              "dsa_workspace_size", "dsa_route_chunk_rows", "dsa_index",
              "dsa_index_noalloc",
              "dsa_index_scan",
              "dsa_index_select", "misa_index",
              "misa_dagger_index", "hisa_index", "lisa_index", "resmisa_index",
              "dsa_quantize_e4m3", "dsa_sparse_mla", "dsa_indexer_backward"):
        getattr(lib, f).restype = C.c_int
    return lib


lib = _load()


def status_string(s: int) -> str:
    return lib.dsa_status_string(s).decode()


def _check(rc: int, what: str):
    if rc != DSA_OK:
        raise DsaError(rc, what)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return DSA_F32
    if t.dtype == torch.bfloat16:
        return DSA_BF16
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return DSA_E4M3
    raise TypeError(f"unsupported operand dtype {t.dtype}")


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


_OPERAND = (torch.float32, torch.bfloat16, torch.uint8, torch.float8_e4m3fn)
_F32 = (torch.float32,)
_I32 = (torch.int32,)
_U8 = (torch.uint8,)


def _args(**named):
    """Check tensor arguments before any library call: dtype, C-contiguous
    layout and a CUDA device (the kernels take raw device pointers, so a host or
    strided tensor would be misread).  Each value is (tensor or None, dtypes)."""
    given = [(name, t, dtypes) for name, (t, dtypes) in named.items() if t is not None]
    for name, t, dtypes in given:
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
        if t.dtype not in dtypes:
            raise TypeError(f"{name}: dtype {t.dtype}, expected one of {dtypes}")
        if not t.is_contiguous():
            raise ValueError(f"{name}: must be contiguous")
    for name, t, _ in given:
        if t.device.type != "cuda":
            raise ValueError(f"{name}: must be on a CUDA device, not {t.device}")


def _common_args(q, k, w, q_scale=None, k_scale=None, q_pos0=None, k_len=None, out=None,
                 workspace=None, **extra):
    idx, sc = (None, None) if out is None else out
    _args(q=(q, _OPERAND), k=(k, _OPERAND), w=(w, _F32), q_scale=(q_scale, _F32),
          k_scale=(k_scale, _F32), q_pos0=(q_pos0, _I32), k_len=(k_len, _I32),
          out_idx=(idx, _I32), out_score=(sc, _F32), workspace=(workspace, _U8), **extra)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


def problem(q: torch.Tensor, k: torch.Tensor, topk: int, q_pos0=None, k_len=None,
            flags: int = 0) -> DsaProblem:
    """q [batch, n_q, heads, dim], k [batch, n_k, dim]."""
    B, nq, H, d = q.shape
    nk = k.shape[1]
    return DsaProblem(B, nq, nk, H, d, topk, _dtype_code(q), _dtype_code(k), _ptr(q_pos0),
                      _ptr(k_len), flags)


def route_params(misa_block=0, misa_h=0, k_prime=0, hisa_block=0, hisa_r=0, lisa_pool=0,
                 res_block=0, res_r=0) -> DsaRouteParams:
    return DsaRouteParams(misa_block, misa_h, k_prime, hisa_block, hisa_r, lisa_pool, res_block,
                          res_r)


def dsa_workspace_size(p: DsaProblem, algo: int = DSA_ALGO_DSA, rp: DsaRouteParams | None = None) -> int:
    n = C.c_size_t(0)
    _check(lib.dsa_workspace_size(C.byref(p), algo, None if rp is None else C.byref(rp),
                                  C.byref(n)), "dsa_workspace_size")
    return n.value


def dsa_route_chunk_rows(p: DsaProblem, algo: int, rp: DsaRouteParams) -> int:
    """Query rows per sequence of one row chunk of a routed entry point."""
    n = C.c_int32(0)
    _check(lib.dsa_route_chunk_rows(C.byref(p), algo, C.byref(rp), C.byref(n)),
           "dsa_route_chunk_rows")
    return n.value


def _workspace(nbytes: int, device, workspace):
    if workspace is not None and workspace.numel() >= nbytes:
        return workspace
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def _outputs(B, nq, topk, device, out):
    if out is not None:
        return out
    return (torch.empty((B, nq, topk), dtype=torch.int32, device=device),
            torch.empty((B, nq, topk), dtype=torch.float32, device=device))


def dsa_index(q, k, w, topk, q_scale=None, k_scale=None, q_pos0=None, k_len=None, flags=0,
              out=None, workspace=None, stream=None):
    """DSA indexer top-k.  Returns (idx int32 [B,n_q,k], score fp32 [B,n_q,k])."""
    _common_args(q, k, w, q_scale, k_scale, q_pos0, k_len, out, workspace)
    p = problem(q, k, topk, q_pos0, k_len, flags)
    ws = _workspace(dsa_workspace_size(p), q.device, workspace)
    idx, sc = _outputs(q.shape[0], q.shape[1], topk, q.device, out)
    _check(lib.dsa_index(C.byref(p), _ptr(q), _ptr(q_scale), _ptr(k), _ptr(k_scale), _ptr(w),
                         _ptr(idx), _ptr(sc), _ptr(ws), ws.numel(), _stream(stream)), "dsa_index")
    return idx, sc


def dsa_index_noalloc(q, k, w, topk, q_scale=None, k_scale=None, q_pos0=None, k_len=None,
                      flags=0, out=None, stream=None):
    """dsa_index on the library's fixed internal scratch (no workspace argument).

    For callers that cannot allocate device memory at call time; problems that
    need more than the library's 64 MiB scratch raise DsaError(DSA_ERR_WORKSPACE),
    and calls that overlap on the GPU race on the shared scratch."""
    _common_args(q, k, w, q_scale, k_scale, q_pos0, k_len, out)
    p = problem(q, k, topk, q_pos0, k_len, flags)
    idx, sc = _outputs(q.shape[0], q.shape[1], topk, q.device, out)
    _check(lib.dsa_index_noalloc(C.byref(p), _ptr(q), _ptr(q_scale), _ptr(k), _ptr(k_scale),
                                 _ptr(w), _ptr(idx), _ptr(sc), _stream(stream)),
           "dsa_index_noalloc")
    return idx, sc


def _host_args(**named):
    """Host-side tensors of dsa_index_host: dtype, C-contiguous, on the CPU."""
    for name, (t, dtypes) in named.items():
        if t is None:
            continue
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
        if t.dtype not in dtypes:
            raise TypeError(f"{name}: dtype {t.dtype}, expected one of {dtypes}")
        if not t.is_contiguous():
            raise ValueError(f"{name}: must be contiguous")
        if t.device.type != "cpu":
            raise ValueError(f"{name}: must be in host memory, not {t.device}")


def dsa_host_staging_size(p: DsaProblem, chunk_rows: int) -> int:
    n = C.c_size_t(0)
    _check(lib.dsa_host_staging_size(C.byref(p), chunk_rows, C.byref(n)), "dsa_host_staging_size")
    return n.value


def dsa_index_host(q_host, k, w_host, topk, q_scale_host=None, k_scale=None, q_pos0=None,
                   k_len=None, flags=0, chunk_rows=16384, out=None, staging=None, stream=None):
    """dsa_index with q, w (and q_scale) in (page-locked) host memory and the
    results written to host tensors; the rows stream in chunks so the copies
    overlap the scan.  k, k_scale, q_pos0, k_len on the GPU.  Returns host
    (idx int32 [B, n_q, k], score fp32 [B, n_q, k]); with `out` given, writes there."""
    _host_args(q_host=(q_host, _OPERAND), w_host=(w_host, _F32), q_scale_host=(q_scale_host, _F32))
    _args(k=(k, _OPERAND), k_scale=(k_scale, _F32), q_pos0=(q_pos0, _I32), k_len=(k_len, _I32),
          staging=(staging, _U8))
    p = problem(q_host, k, topk, q_pos0, k_len, flags)
    B, nq = q_host.shape[0], q_host.shape[1]
    if out is None:
        out = (torch.empty((B, nq, topk), dtype=torch.int32).pin_memory(),
               torch.empty((B, nq, topk), dtype=torch.float32).pin_memory())
    idx, sc = out
    _host_args(out_idx=(idx, _I32), out_score=(sc, _F32))
    nbytes = dsa_host_staging_size(p, chunk_rows)
    if staging is None or staging.numel() < nbytes:
        staging = torch.empty(nbytes, dtype=torch.uint8, device=k.device)
    _check(lib.dsa_index_host(C.byref(p), _ptr(q_host), _ptr(q_scale_host), _ptr(k), _ptr(k_scale),
                              _ptr(w_host), _ptr(idx), _ptr(sc), chunk_rows, _ptr(staging),
                              staging.numel(), _stream(stream)), "dsa_index_host")
    return idx, sc


def dsa_index_scan(p: DsaProblem, q, k, w, workspace, q_scale=None, k_scale=None, stream=None):
    """First stage of dsa_index (scores + candidate logs in `workspace`)."""
    _common_args(q, k, w, q_scale, k_scale, workspace=workspace)
    _check(lib.dsa_index_scan(C.byref(p), _ptr(q), _ptr(q_scale), _ptr(k), _ptr(k_scale), _ptr(w),
                              _ptr(workspace), workspace.numel(), _stream(stream)), "dsa_index_scan")


def dsa_index_select(p: DsaProblem, idx, score, workspace, stream=None):
    """Second stage of dsa_index (exact top-k per row from the logs)."""
    _args(idx=(idx, _I32), score=(score, _F32), workspace=(workspace, _U8))
    _check(lib.dsa_index_select(C.byref(p), _ptr(idx), _ptr(score), _ptr(workspace),
                                workspace.numel(), _stream(stream)), "dsa_index_select")


def misa_index(q, k, w, topk, block, h, q_pos0=None, k_len=None, flags=0, out=None,
               out_heads=None, out_E=None, workspace=None, stream=None):
    _common_args(q, k, w, None, None, q_pos0, k_len, out, workspace,
                 out_heads=(out_heads, _I32), out_E=(out_E, _F32))
    p = problem(q, k, topk, q_pos0, k_len, flags)
    rp = route_params(misa_block=block, misa_h=h)
    ws = _workspace(dsa_workspace_size(p, DSA_ALGO_MISA, rp), q.device, workspace)
    idx, sc = _outputs(q.shape[0], q.shape[1], topk, q.device, out)
    _check(lib.misa_index(C.byref(p), C.byref(rp), _ptr(q), _ptr(k), _ptr(w), _ptr(idx), _ptr(sc),
                          _ptr(out_heads), _ptr(out_E), _ptr(ws), ws.numel(), _stream(stream)),
           "misa_index")
    return idx, sc


def misa_dagger_index(q, k, w, topk, block, h, k_prime, q_pos0=None, k_len=None, flags=0,
                      out=None, out_heads=None, out_pool=None, workspace=None, stream=None):
    _common_args(q, k, w, None, None, q_pos0, k_len, out, workspace,
                 out_heads=(out_heads, _I32), out_pool=(out_pool, _I32))
    p = problem(q, k, topk, q_pos0, k_len, flags)
    rp = route_params(misa_block=block, misa_h=h, k_prime=k_prime)
    ws = _workspace(dsa_workspace_size(p, DSA_ALGO_MISA_DAGGER, rp), q.device, workspace)
    idx, sc = _outputs(q.shape[0], q.shape[1], topk, q.device, out)
    _check(lib.misa_dagger_index(C.byref(p), C.byref(rp), _ptr(q), _ptr(k), _ptr(w), _ptr(idx),
                                 _ptr(sc), _ptr(out_heads), _ptr(out_pool), _ptr(ws), ws.numel(),
                                 _stream(stream)), "misa_dagger_index")
    return idx, sc


def hisa_index(q, k, w, topk, block, r, route_h=0, route_block=1024, q_pos0=None, k_len=None,
               flags=0, out=None, out_blocks=None, out_heads=None, workspace=None, stream=None):
    _common_args(q, k, w, None, None, q_pos0, k_len, out, workspace,
                 out_blocks=(out_blocks, _I32), out_heads=(out_heads, _I32))
    p = problem(q, k, topk, q_pos0, k_len, flags)
    rp = route_params(misa_block=route_block if route_h else 0, misa_h=route_h, hisa_block=block,
                      hisa_r=r)
    ws = _workspace(dsa_workspace_size(p, DSA_ALGO_HISA, rp), q.device, workspace)
    idx, sc = _outputs(q.shape[0], q.shape[1], topk, q.device, out)
    _check(lib.hisa_index(C.byref(p), C.byref(rp), _ptr(q), _ptr(k), _ptr(w), _ptr(idx), _ptr(sc),
                          _ptr(out_blocks), _ptr(out_heads), _ptr(ws), ws.numel(), _stream(stream)),
           "hisa_index")
    return idx, sc


def lisa_index(q, k, w, topk, pool=0, q_pos0=None, k_len=None, flags=0, out=None,
               out_pool=None, workspace=None, stream=None):
    """Indexer LISA (pool == 0: top-k by the linear term g . k) or LISA-dagger
    (pool = M: the top-M by g . k reranked by the full score over every head)."""
    _common_args(q, k, w, None, None, q_pos0, k_len, out, workspace, out_pool=(out_pool, _I32))
    p = problem(q, k, topk, q_pos0, k_len, flags)
    rp = route_params(lisa_pool=pool)
    ws = _workspace(dsa_workspace_size(p, DSA_ALGO_LISA, rp), q.device, workspace)
    idx, sc = _outputs(q.shape[0], q.shape[1], topk, q.device, out)
    _check(lib.lisa_index(C.byref(p), C.byref(rp), _ptr(q), _ptr(k), _ptr(w), _ptr(idx), _ptr(sc),
                          _ptr(out_pool), _ptr(ws), ws.numel(), _stream(stream)), "lisa_index")
    return idx, sc


def resmisa_index(q, k, w, topk, block, r, q_pos0=None, k_len=None, flags=0, out=None,
                  out_heads=None, out_S=None, workspace=None, stream=None):
    """ResMiSA: the linear term of every head plus r routed residual heads."""
    _common_args(q, k, w, None, None, q_pos0, k_len, out, workspace,
                 out_heads=(out_heads, _I32), out_S=(out_S, _F32))
    p = problem(q, k, topk, q_pos0, k_len, flags)
    rp = route_params(res_block=block, res_r=r)
    ws = _workspace(dsa_workspace_size(p, DSA_ALGO_RESMISA, rp), q.device, workspace)
    idx, sc = _outputs(q.shape[0], q.shape[1], topk, q.device, out)
    _check(lib.resmisa_index(C.byref(p), C.byref(rp), _ptr(q), _ptr(k), _ptr(w), _ptr(idx),
                             _ptr(sc), _ptr(out_heads), _ptr(out_S), _ptr(ws), ws.numel(),
                             _stream(stream)), "resmisa_index")
    return idx, sc


def sparse_mla(q, kv, idx, scale, tokens_per_seq=None, flags=0, out=None, out_lse=None,
               workspace=None, stream=None):
    """Sparse MLA over fixed selected positions.  q [T, heads, 576] bf16,
    kv [batch, n_k, 576] bf16, idx [T, k] int32 (-1 empty).  Returns (out
    [T, heads, 512] bf16, lse [T, heads] fp32)."""
    _args(q=(q, (torch.bfloat16,)), kv=(kv, (torch.bfloat16,)), idx=(idx, _I32),
          out=(out, (torch.bfloat16,)), out_lse=(out_lse, _F32), workspace=(workspace, _U8))
    T, H, dqk = q.shape
    B, n_k, _ = kv.shape
    tps = T // B if tokens_per_seq is None else tokens_per_seq
    p = DsaMlaProblem(B, tps, n_k, H, dqk, 512, idx.shape[1], float(scale), flags)
    if out is None:
        out = torch.empty((T, H, 512), dtype=torch.bfloat16, device=q.device)
    if out_lse is None:
        out_lse = torch.empty((T, H), dtype=torch.float32, device=q.device)
    ws = _workspace(256, q.device, workspace)
    _check(lib.dsa_sparse_mla(C.byref(p), _ptr(q), _ptr(kv), _ptr(idx), _ptr(out), _ptr(out_lse),
                              _ptr(ws), ws.numel(), _stream(stream)), "dsa_sparse_mla")
    return out, out_lse


def indexer_backward(q, k, w, sel, grad, dk=None, flags=0, workspace=None, stream=None):
    """Gradients of sum g I over the selected positions: returns (dq [B, n_q, H, d],
    dk [B, n_k, d], dw [B, n_q, H]) in fp32; dk is added to when given."""
    _args(q=(q, (torch.bfloat16,)), k=(k, (torch.bfloat16,)), w=(w, _F32), sel=(sel, _I32),
          grad=(grad, _F32), dk=(dk, _F32), workspace=(workspace, _U8))
    p = problem(q, k, sel.shape[-1], flags=flags)
    dq = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    dw = torch.empty(w.shape, dtype=torch.float32, device=q.device)
    if dk is None:
        dk = torch.zeros(k.shape, dtype=torch.float32, device=q.device)
    ws = _workspace(256, q.device, workspace)
    _check(lib.dsa_indexer_backward(C.byref(p), _ptr(q), _ptr(k), _ptr(w), _ptr(sel), _ptr(grad),
                                    _ptr(dq), _ptr(dk), _ptr(dw), _ptr(ws), ws.numel(),
                                    _stream(stream)), "dsa_indexer_backward")
    return dq, dk, dw


def dsa_quantize_e4m3(x: torch.Tensor, stream=None):
    """Per-row e4m3 codes (uint8, same shape) and fp32 scales (shape[:-1])."""
    _args(x=(x, (torch.float32, torch.bfloat16)))
    cols = x.shape[-1]
    rows = x.numel() // cols
    out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    sc = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    _check(lib.dsa_quantize_e4m3(_ptr(x), _dtype_code(x), rows, cols, _ptr(out), _ptr(sc),
                                 _stream(stream)), "dsa_quantize_e4m3")
    return out, sc


def dsa_read_status(workspace: torch.Tensor, stream=None) -> int:
    _args(workspace=(workspace, _U8))
    return lib.dsa_read_status(_ptr(workspace), _stream(stream))


def dsa_read_pruned(workspace: torch.Tensor, stream=None) -> int:
    """(query row, key tile) pairs the last DSA_FLAG_DOSA call on `workspace` skipped."""
    _args(workspace=(workspace, _U8))
    n = C.c_ulonglong(0)
    _check(lib.dsa_read_pruned(_ptr(workspace), _stream(stream), C.byref(n)), "dsa_read_pruned")
    return int(n.value)


def dsa_dosa_bounds(q, k, w, q_pos0=None, k_len=None, flags=0, workspace=None, stream=None):
    """DoSA block upper and lower bounds, each [B * n_q, ceil(n_k / 1024)] fp32
    (see include/dsaidx.h)."""
    _common_args(q, k, w, q_pos0=q_pos0, k_len=k_len, workspace=workspace)
    p = problem(q, k, 1, q_pos0, k_len, flags | DSA_FLAG_DOSA)
    ws = _workspace(dsa_workspace_size(p), q.device, workspace)
    nblk = (k.shape[1] + 1023) // 1024
    ub = torch.empty((q.shape[0] * q.shape[1], nblk), dtype=torch.float32, device=q.device)
    lb = torch.empty_like(ub)
    _check(lib.dsa_dosa_bounds(C.byref(p), _ptr(q), _ptr(k), _ptr(w), _ptr(ub), _ptr(lb),
                               _ptr(ws), ws.numel(), _stream(stream)), "dsa_dosa_bounds")
    return ub, lb

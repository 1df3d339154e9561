"""fp64 CPU oracle for block top-k sparse decode attention over a paged KV cache.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the CPU-baseline
leg of ``bench.py`` may import this package; the library under
``paged_block_sparse_vt_b200`` never does, and shares no code with it.

The arithmetic lives in ``vt_oracle.c`` (plain C, fp64, OpenMP over
(request, KV head)); this module compiles it with gcc on first use and wraps it
with ctypes.  Arguments are host torch tensors; bf16 tensors are handed to C as
their 16-bit patterns.  Every function cites the passage it follows in the C
source's header.

``kind="f32"`` selects a second build of the same C source with fp32 arithmetic
(``-DVTO_REAL=float -O3 -march=native``).  It is a timing-only copy for the
benchmark's CPU baseline, never a correctness reference.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "vt_oracle.c")
_LIB = os.path.join(_HERE, "libvt_oracle.so")
_LIB_F32 = os.path.join(_HERE, "libvt_oracle_f32.so")
_lock = threading.Lock()
_libs = {}

OK, ERR_ARG, ERR_LEN, ERR_PAGE = 0, 1, 2, 3


class OracleError(RuntimeError):
    pass


def build(force: bool = False, kind: str = "f64") -> str:
    """Compile vt_oracle.c next to it: libvt_oracle.so (the fp64 oracle: gcc -O2, no FMA
    contraction, OpenMP), or with kind="f32" the timing-only fp32 copy libvt_oracle_f32.so."""
    lib = _LIB if kind == "f64" else _LIB_F32
    if force or not os.path.exists(lib) or os.path.getmtime(lib) < os.path.getmtime(_SRC):
        tmp = lib + f".tmp{os.getpid()}"
        if kind == "f64":
            flags = ["-O2", "-ffp-contract=off"]
        elif kind == "f32":
            flags = ["-O3", "-march=native", "-DVTO_REAL=float"]
        else:
            raise ValueError(kind)
        cmd = ["gcc", "-std=c11", *flags, "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, lib)
    return lib


def _load(kind: str = "f64"):
    with _lock:
        if kind not in _libs:
            lib = ctypes.CDLL(build(kind=kind))
            i32, i64, f64, p = ctypes.c_int32, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
            lib.vto_set_threads.argtypes = [ctypes.c_int]
            lib.vto_get_threads.restype = ctypes.c_int
            lib.vto_build_centroids.argtypes = [p, i64, i32, i32, i32, i64, i64, i64, p, i32, p]
            lib.vto_build_centroids.restype = ctypes.c_int
            lib.vto_select_pages.argtypes = [p, i32, i32, i32, i32, p, i64, p, p, i64, i32, i32,
                                             i32, i32, p, p, p]
            lib.vto_select_pages.restype = ctypes.c_int
            lib.vto_select_pages_approx.argtypes = [p, i32, i32, i32, i32, p, i64, p, p, i64,
                                                    i32, i32, i32, i32, ctypes.c_uint64, p, p]
            lib.vto_select_pages_approx.restype = ctypes.c_int
            lib.vto_sparse_attention.argtypes = [p, i32, i32, i32, i32, i32, p, i64, i64, i64, p,
                                                 i64, i64, i64, i64, i32, p, i64, p, p, p, i32,
                                                 f64, p, p]
            lib.vto_sparse_attention.restype = ctypes.c_int
            lib.vto_decode_step.argtypes = [p, i32, i32, i32, i32, i32, p, i64, i64, i64, p, i64,
                                            i64, i64, i64, i32, p, i64, p, p, i32, i32, i32, f64,
                                            p, p, p, p]
            lib.vto_decode_step.restype = ctypes.c_int
            _libs[kind] = lib
    return _libs[kind]


def set_threads(n: int, kind: str = "f64") -> None:
    """Threads of the OpenMP loops (0: the OpenMP default, every core of the affinity mask)."""
    _load(kind).vto_set_threads(int(n))


def get_threads(kind: str = "f64") -> int:
    return int(_load(kind).vto_get_threads())


def _ptr(t) -> int:
    return t.data_ptr() if isinstance(t, torch.Tensor) else t.ctypes.data


def _bits(t: torch.Tensor) -> torch.Tensor:
    assert t.dtype == torch.bfloat16 and t.device.type == "cpu"
    return t.view(torch.int16)


def _i32(t: torch.Tensor) -> torch.Tensor:
    assert t.dtype == torch.int32 and t.device.type == "cpu" and t.is_contiguous()
    return t


def _check(rc: int, what: str) -> None:
    if rc != OK:
        raise OracleError(f"{what}: oracle error code {rc}")


def _pool_strides(pool: torch.Tensor):
    assert pool.dim() == 4, "pool is [P, page_size, Hkv, D]"
    assert pool.stride(3) == 1
    return pool.stride(0), pool.stride(1), pool.stride(2)


def build_centroids(k_pool: torch.Tensor, pages: torch.Tensor, centroids: torch.Tensor,
                    kind: str = "f64") -> None:
    """centroids[p] = mean over the page's tokens of K[p] (fp64 sum, fp32 store), in place."""
    P, page_size, hkv, d = k_pool.shape
    assert centroids.dtype == torch.float32 and centroids.is_contiguous()
    assert tuple(centroids.shape) == (P, hkv, d)
    sk = _pool_strides(k_pool)
    pages = _i32(pages)
    rc = _load(kind).vto_build_centroids(_ptr(_bits(k_pool)), P, page_size, hkv, d, *sk,
                                     _ptr(pages), pages.numel(), _ptr(centroids))
    _check(rc, "build_centroids")


def select_pages(q, page_table, seq_lens, centroids, topk, bos, eos, page_size=16,
                 want_scores=False):
    """Group mean -> score vs centroids -> top-k + reserved.  Returns (sel, n_sel[, scores])."""
    B, hq, d = q.shape
    P, hkv, dc = centroids.shape
    assert dc == d and q.is_contiguous() and centroids.is_contiguous()
    page_table, seq_lens = _i32(page_table), _i32(seq_lens)
    kmax = topk + bos + eos
    sel = torch.empty((B, hkv, kmax), dtype=torch.int32)
    n_sel = torch.empty((B, hkv), dtype=torch.int32)
    scores = torch.empty((B, hkv, page_table.shape[1]), dtype=torch.float64) if want_scores else None
    rc = _load().vto_select_pages(_ptr(_bits(q)), B, hq, hkv, d, _ptr(page_table),
                                  page_table.shape[1], _ptr(seq_lens), _ptr(centroids), P,
                                  page_size, topk, bos, eos, _ptr(sel), _ptr(n_sel),
                                  _ptr(scores) if want_scores else None)
    _check(rc, "select_pages")
    return (sel, n_sel, scores) if want_scores else (sel, n_sel)


def select_pages_approx(q, page_table, seq_lens, centroids, topk, bos, eos, seed,
                        page_size=16):
    """The lossy indexer mode: one radix pass over the fp32 scores (1024 bins linear between
    the smallest and largest), every bin above the topk-th score's bin kept, that bin's
    candidates taken in cyclic order from a SplitMix64-drawn start.  Returns (sel, n_sel)."""
    B, hq, d = q.shape
    P, hkv, dc = centroids.shape
    assert dc == d and q.is_contiguous() and centroids.is_contiguous()
    page_table, seq_lens = _i32(page_table), _i32(seq_lens)
    kmax = topk + bos + eos
    sel = torch.empty((B, hkv, kmax), dtype=torch.int32)
    n_sel = torch.empty((B, hkv), dtype=torch.int32)
    rc = _load().vto_select_pages_approx(_ptr(_bits(q)), B, hq, hkv, d, _ptr(page_table),
                                         page_table.shape[1], _ptr(seq_lens), _ptr(centroids),
                                         P, page_size, topk, bos, eos,
                                         ctypes.c_uint64(seed & (2**64 - 1)), _ptr(sel),
                                         _ptr(n_sel))
    _check(rc, "select_pages_approx")
    return sel, n_sel


def sparse_attention(q, k_pool, v_pool, page_table, seq_lens, sel, n_sel, sm_scale,
                     head_dim_v=None):
    """Exact fp64 softmax attention over the selected pages.  Returns (out [B,Hq,Dv], lse [B,Hq])."""
    B, hq, d = q.shape
    P, page_size, hkv, _ = k_pool.shape
    dv = head_dim_v if head_dim_v is not None else v_pool.shape[3]
    sk, sv = _pool_strides(k_pool), _pool_strides(v_pool)
    page_table, seq_lens = _i32(page_table), _i32(seq_lens)
    sel, n_sel = _i32(sel), _i32(n_sel)
    out = torch.empty((B, hq, dv), dtype=torch.float64)
    lse = torch.empty((B, hq), dtype=torch.float64)
    rc = _load().vto_sparse_attention(_ptr(_bits(q)), B, hq, hkv, d, dv, _ptr(_bits(k_pool)), *sk,
                                      _ptr(_bits(v_pool)), *sv, P, page_size, _ptr(page_table),
                                      page_table.shape[1], _ptr(seq_lens), _ptr(sel), _ptr(n_sel),
                                      sel.shape[2], float(sm_scale), _ptr(out), _ptr(lse))
    _check(rc, "sparse_attention")
    return out, lse


def decode_step(q, k_pool, v_pool, page_table, seq_lens, centroids, topk, bos, eos, sm_scale,
                head_dim_v=None, kind: str = "f64"):
    """select_pages followed by sparse_attention.  Returns (sel, n_sel, out, lse)."""
    B, hq, d = q.shape
    P, page_size, hkv, _ = k_pool.shape
    dv = head_dim_v if head_dim_v is not None else v_pool.shape[3]
    sk, sv = _pool_strides(k_pool), _pool_strides(v_pool)
    page_table, seq_lens = _i32(page_table), _i32(seq_lens)
    kmax = topk + bos + eos
    sel = torch.empty((B, hkv, kmax), dtype=torch.int32)
    n_sel = torch.empty((B, hkv), dtype=torch.int32)
    out = torch.empty((B, hq, dv), dtype=torch.float64)
    lse = torch.empty((B, hq), dtype=torch.float64)
    rc = _load(kind).vto_decode_step(_ptr(_bits(q)), B, hq, hkv, d, dv, _ptr(_bits(k_pool)), *sk,
                                 _ptr(_bits(v_pool)), *sv, P, page_size, _ptr(page_table),
                                 page_table.shape[1], _ptr(seq_lens), _ptr(centroids), topk, bos,
                                 eos, float(sm_scale), _ptr(sel), _ptr(n_sel), _ptr(out), _ptr(lse))
    _check(rc, "decode_step")
    return sel, n_sel, out, lse

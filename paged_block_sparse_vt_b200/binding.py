"""ctypes binding of libvt (include/vt.h).  Argument marshalling only.

Every function takes CUDA torch tensors, passes their device pointers, sizes and strides to
the C entry point of the same name, and enqueues on the current torch CUDA stream.  All
computation happens in libvt's kernels; there is no fallback of any kind: if libvt.so is
missing or a call fails, a ``VtError`` is raised.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libvt.so")

VT_OK, VT_ERR_INVALID_ARG, VT_ERR_UNSUPPORTED, VT_ERR_CUDA = 0, 1, 2, 3
VT_DEV_BAD_PAGE, VT_DEV_BAD_LEN, VT_DEV_BAD_SEL, VT_DEV_BAD_ORDER, VT_DEV_TIMEOUT = 1, 2, 4, 8, 16
PAGE_SIZE = 16


class VtError(RuntimeError):
    def __init__(self, code: int, where: str, detail: str):
        super().__init__(f"{where}: {_status_name(code)}: {detail}")
        self.code = code


class PagedKV(ctypes.Structure):
    _fields_ = [
        ("k_pool", ctypes.c_void_p), ("v_pool", ctypes.c_void_p),
        ("num_pages", ctypes.c_int64), ("page_size", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("head_dim_v", ctypes.c_int32),
        ("sk_p", ctypes.c_int64), ("sk_t", ctypes.c_int64), ("sk_h", ctypes.c_int64),
        ("sv_p", ctypes.c_int64), ("sv_t", ctypes.c_int64), ("sv_h", ctypes.c_int64),
    ]


class DecodeArgs(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
        ("q", ctypes.c_void_p), ("page_table", ctypes.c_void_p), ("pt_stride", ctypes.c_int64),
        ("seq_lens", ctypes.c_void_p), ("centroids", ctypes.c_void_p),
        ("topk", ctypes.c_int32), ("bos", ctypes.c_int32), ("eos", ctypes.c_int32),
        ("sm_scale", ctypes.c_float),
        ("order", ctypes.c_void_p), ("status", ctypes.c_void_p),
    ]


EXPORTS = ("vt_build_centroids", "vt_select_pages", "vt_select_pages_approx",
           "vt_select_pages_ws", "vt_sparse_decode_ws",
           "vt_sparse_decode", "vt_sparse_decode_fused", "vt_sparse_decode_step",
           "vt_fused_workspace_size", "vt_sparse_decode_fused_static", "vt_plan_requests",
           "vt_status_string",
           "vt_last_error_detail", "vt_abi_version")

_lock = threading.Lock()
_lib = None


def load_library(path: str = LIB_PATH):
    """Load libvt.so (once).  Raises VtError if it is missing: there is no fallback."""
    global _lib
    lib = _lib
    if lib is not None:
        return lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise VtError(-1, "load", f"{path} not found; build it with "
                                          "`python -m paged_block_sparse_vt_b200.build`")
            lib = ctypes.CDLL(path)
            P, I32, I64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
            kv, args = ctypes.POINTER(PagedKV), ctypes.POINTER(DecodeArgs)
            sigs = {
                "vt_build_centroids": [kv, P, I32, P, P, P],
                "vt_select_pages": [kv, args, P, P, P],
                "vt_select_pages_approx": [kv, args, ctypes.c_uint64, P, P, P],
                "vt_select_pages_ws": [kv, args, P, P, P, ctypes.c_size_t, P],
                "vt_sparse_decode_ws": [kv, args, P, P, P, P, P, ctypes.c_size_t, P],
                "vt_sparse_decode": [kv, args, P, P, P, P, P],
                "vt_sparse_decode_fused": [kv, args, P, P, P, P, P, ctypes.c_size_t, P],
                "vt_sparse_decode_step": [kv, args, P, I32, P, P, P, P, P, P, ctypes.c_size_t, P],
                "vt_sparse_decode_fused_static": [kv, args, P, P, P, P, P],
                "vt_plan_requests": [P, I32, P, P],
            }
            for name, argtypes in sigs.items():
                fn = getattr(lib, name)
                fn.argtypes = argtypes
                fn.restype = ctypes.c_int
            lib.vt_fused_workspace_size.argtypes = [kv, args]
            lib.vt_fused_workspace_size.restype = ctypes.c_size_t
            lib.vt_status_string.argtypes = [ctypes.c_int]
            lib.vt_status_string.restype = ctypes.c_char_p
            lib.vt_last_error_detail.argtypes = []
            lib.vt_last_error_detail.restype = ctypes.c_char_p
            lib.vt_abi_version.argtypes = []
            lib.vt_abi_version.restype = ctypes.c_int32
            _lib = lib
    return _lib


def _status_name(code: int) -> str:
    return {0: "VT_OK", 1: "VT_ERR_INVALID_ARG", 2: "VT_ERR_UNSUPPORTED", 3: "VT_ERR_CUDA"}.get(
        code, f"status {code}")


def _check(rc: int, where: str) -> None:
    if rc != VT_OK:
        detail = load_library().vt_last_error_detail().decode()
        raise VtError(rc, where, detail)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


# The current stream's handle without building a torch.cuda.Stream object per call.
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(t: torch.Tensor) -> int:
    if _raw_stream is not None:
        return _raw_stream(t.get_device())
    return torch.cuda.current_stream(t.device).cuda_stream


def _need(t: torch.Tensor, name: str, dtype=None, contiguous: bool = False) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise VtError(VT_ERR_INVALID_ARG, name, "must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise VtError(VT_ERR_INVALID_ARG, name, f"must be {dtype}, got {t.dtype}")
    if contiguous and not t.is_contiguous():
        raise VtError(VT_ERR_INVALID_ARG, name, "must be contiguous")


def paged_kv(k_pool: torch.Tensor, v_pool: torch.Tensor, head_dim_v: Optional[int] = None) -> PagedKV:
    """Descriptor of the pools [P, 16, Hkv, D] (bf16, any strides with the last one 1)."""
    _need(k_pool, "k_pool", torch.bfloat16)
    _need(v_pool, "v_pool", torch.bfloat16)
    if k_pool.dim() != 4 or v_pool.dim() != 4:
        raise VtError(VT_ERR_INVALID_ARG, "pools", "must be [P, page_size, Hkv, D]")
    P, ps, hkv, d = k_pool.shape
    dv = head_dim_v if head_dim_v is not None else v_pool.shape[3]
    if k_pool.stride(3) != 1 or v_pool.stride(3) != 1:
        raise VtError(VT_ERR_UNSUPPORTED, "pools", "innermost stride must be 1")
    return PagedKV(k_pool.data_ptr(), v_pool.data_ptr(), P, ps, hkv, d, dv,
                   k_pool.stride(0), k_pool.stride(1), k_pool.stride(2),
                   v_pool.stride(0), v_pool.stride(1), v_pool.stride(2))


def decode_args(q, page_table, seq_lens, centroids=None, topk=0, bos=0, eos=0, sm_scale=1.0,
                order=None, status=None) -> DecodeArgs:
    _need(q, "q", torch.bfloat16, contiguous=True)
    _need(page_table, "page_table", torch.int32)
    _need(seq_lens, "seq_lens", torch.int32, contiguous=True)
    if page_table.dim() != 2 or page_table.stride(1) != 1:
        raise VtError(VT_ERR_INVALID_ARG, "page_table", "must be [B, max_pages] with unit inner stride")
    if centroids is not None:
        _need(centroids, "centroids", torch.float32, contiguous=True)
    if order is not None:
        _need(order, "order", torch.int32, contiguous=True)
    if status is not None:
        _need(status, "status", torch.int32)
    B, hq, _ = q.shape
    return DecodeArgs(B, hq, q.data_ptr(), page_table.data_ptr(), page_table.stride(0),
                      seq_lens.data_ptr(), _ptr(centroids), int(topk), int(bos), int(eos),
                      float(sm_scale), _ptr(order), _ptr(status))


def vt_build_centroids(k_pool: torch.Tensor, pages: torch.Tensor, centroids: torch.Tensor,
                       status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """centroids[p] = mean over the 16 tokens of K[p] for every physical page p in ``pages``."""
    lib = load_library()
    _need(pages, "pages", torch.int32, contiguous=True)
    _need(centroids, "centroids", torch.float32, contiguous=True)
    kv = paged_kv(k_pool, k_pool)
    rc = lib.vt_build_centroids(ctypes.byref(kv), pages.data_ptr(), pages.numel(),
                                centroids.data_ptr(), _ptr(status), _stream(k_pool))
    _check(rc, "vt_build_centroids")
    return centroids


def vt_select_pages(q, k_pool, v_pool, page_table, seq_lens, centroids, topk, bos, eos,
                    sel=None, n_sel=None, order=None, status=None, head_dim_v=None,
                    workspace=None):
    """Top-k page selection per (request, KV head).  Returns (sel [B,Hkv,kmax], n_sel [B,Hkv]).

    With ``workspace`` (from fused_workspace() for the same arguments) it calls
    vt_select_pages_ws (the persistent kernel, B <= 2048)."""
    lib = load_library()
    kv = paged_kv(k_pool, v_pool, head_dim_v)
    a = decode_args(q, page_table, seq_lens, centroids, topk, bos, eos, 1.0, order, status)
    kmax = topk + bos + eos
    B, hkv = q.shape[0], k_pool.shape[2]
    if sel is None:
        sel = torch.empty((B, hkv, kmax), dtype=torch.int32, device=q.device)
    if n_sel is None:
        n_sel = torch.empty((B, hkv), dtype=torch.int32, device=q.device)
    if workspace is not None:
        _need(workspace, "workspace", torch.uint8, contiguous=True)
        rc = lib.vt_select_pages_ws(ctypes.byref(kv), ctypes.byref(a), sel.data_ptr(),
                                    n_sel.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                    _stream(q))
        _check(rc, "vt_select_pages_ws")
        return sel, n_sel
    rc = lib.vt_select_pages(ctypes.byref(kv), ctypes.byref(a), sel.data_ptr(), n_sel.data_ptr(),
                             _stream(q))
    _check(rc, "vt_select_pages")
    return sel, n_sel


def vt_select_pages_approx(q, k_pool, v_pool, page_table, seq_lens, centroids, topk, bos, eos,
                           seed, sel=None, n_sel=None, order=None, status=None, head_dim_v=None):
    """The indexer's lossy mode (one radix pass, seeded start in the last bin).  Returns
    (sel [B,Hkv,kmax], n_sel [B,Hkv])."""
    lib = load_library()
    kv = paged_kv(k_pool, v_pool, head_dim_v)
    a = decode_args(q, page_table, seq_lens, centroids, topk, bos, eos, 1.0, order, status)
    kmax = topk + bos + eos
    B, hkv = q.shape[0], k_pool.shape[2]
    if sel is None:
        sel = torch.empty((B, hkv, kmax), dtype=torch.int32, device=q.device)
    if n_sel is None:
        n_sel = torch.empty((B, hkv), dtype=torch.int32, device=q.device)
    rc = lib.vt_select_pages_approx(ctypes.byref(kv), ctypes.byref(a),
                                    ctypes.c_uint64(int(seed) & (2 ** 64 - 1)), sel.data_ptr(),
                                    n_sel.data_ptr(), _stream(q))
    _check(rc, "vt_select_pages_approx")
    return sel, n_sel


def vt_sparse_decode(q, k_pool, v_pool, page_table, seq_lens, sel, n_sel, sm_scale, out=None,
                     lse=None, status=None, head_dim_v=None, want_lse=True, workspace=None):
    """Attention over a given page selection.  Returns (out [B,Hq,Dv] bf16, lse [B,Hq] or None).

    With ``workspace`` (decode_workspace() for these arguments) it calls vt_sparse_decode_ws
    (the persistent kernel, B <= 2048)."""
    lib = load_library()
    kv = paged_kv(k_pool, v_pool, head_dim_v)
    kmax = sel.shape[2]
    a = decode_args(q, page_table, seq_lens, None, kmax, 0, 0, sm_scale, None, status)
    B, hq = q.shape[0], q.shape[1]
    if out is None:
        out = torch.empty((B, hq, kv.head_dim_v), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, hq), dtype=torch.float32, device=q.device)
    if workspace is not None:
        _need(workspace, "workspace", torch.uint8, contiguous=True)
        rc = lib.vt_sparse_decode_ws(ctypes.byref(kv), ctypes.byref(a), sel.data_ptr(),
                                     n_sel.data_ptr(), out.data_ptr(), _ptr(lse),
                                     workspace.data_ptr(), workspace.numel(), _stream(q))
        _check(rc, "vt_sparse_decode_ws")
        return out, lse
    rc = lib.vt_sparse_decode(ctypes.byref(kv), ctypes.byref(a), sel.data_ptr(), n_sel.data_ptr(),
                              out.data_ptr(), _ptr(lse), _stream(q))
    _check(rc, "vt_sparse_decode")
    return out, lse


def decode_workspace(q, k_pool, v_pool, page_table, seq_lens, sel, head_dim_v=None):
    """A zeroed workspace for vt_sparse_decode(..., workspace=) with these arguments (the
    decode call's arguments: kmax = sel.shape[2] selected pages, no centroids), or None."""
    lib = load_library()
    kv = paged_kv(k_pool, v_pool, head_dim_v)
    kmax = sel.shape[2]
    a = decode_args(q, page_table, seq_lens, None, kmax, 0, 0, 1.0, None, None)
    n = int(lib.vt_fused_workspace_size(ctypes.byref(kv), ctypes.byref(a)))
    return torch.zeros(n, dtype=torch.uint8, device=q.device) if n else None


def vt_fused_workspace_size(q, k_pool, v_pool, page_table, seq_lens, centroids, topk, bos, eos,
                            head_dim_v=None) -> int:
    """Bytes of workspace vt_sparse_decode_fused needs for these shapes (0 if none)."""
    lib = load_library()
    kv = paged_kv(k_pool, v_pool, head_dim_v)
    a = decode_args(q, page_table, seq_lens, centroids, topk, bos, eos, 1.0)
    return int(lib.vt_fused_workspace_size(ctypes.byref(kv), ctypes.byref(a)))


def fused_workspace(q, k_pool, v_pool, page_table, seq_lens, centroids, topk, bos, eos,
                    head_dim_v=None) -> Optional[torch.Tensor]:
    """A zero-filled workspace for vt_sparse_decode_fused (None when none is needed).

    Zero it once; every call leaves it ready for the next call with the same B * Hkv (zero it
    again before one with another B * Hkv).  Calls sharing one workspace must not overlap on
    the GPU.
    """
    n = vt_fused_workspace_size(q, k_pool, v_pool, page_table, seq_lens, centroids, topk, bos,
                                eos, head_dim_v)
    return torch.zeros(n, dtype=torch.uint8, device=q.device) if n else None


def vt_sparse_decode_fused(q, k_pool, v_pool, page_table, seq_lens, centroids, topk, bos, eos,
                           sm_scale, out=None, lse=None, sel=None, n_sel=None, order=None,
                           status=None, head_dim_v=None, want_lse=True, workspace=None):
    """Selection + attention in one call.  Returns (out, lse, sel, n_sel).

    ``workspace``: from fused_workspace(); allocated (zeroed) here when not given.
    """
    lib = load_library()
    kv = paged_kv(k_pool, v_pool, head_dim_v)
    a = decode_args(q, page_table, seq_lens, centroids, topk, bos, eos, sm_scale, order, status)
    B, hq = q.shape[0], q.shape[1]
    if out is None:
        out = torch.empty((B, hq, kv.head_dim_v), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, hq), dtype=torch.float32, device=q.device)
    if workspace is None:
        n = int(lib.vt_fused_workspace_size(ctypes.byref(kv), ctypes.byref(a)))
        workspace = torch.zeros(n, dtype=torch.uint8, device=q.device) if n else None
    if workspace is not None:
        _need(workspace, "workspace", torch.uint8, contiguous=True)
    rc = lib.vt_sparse_decode_fused(ctypes.byref(kv), ctypes.byref(a), out.data_ptr(), _ptr(lse),
                                    _ptr(sel), _ptr(n_sel), _ptr(workspace),
                                    0 if workspace is None else workspace.numel(), _stream(q))
    _check(rc, "vt_sparse_decode_fused")
    return out, lse, sel, n_sel


def vt_sparse_decode_step(q, k_pool, v_pool, page_table, seq_lens, centroids, topk, bos, eos,
                          sm_scale, fill_pages, out=None, lse=None, sel=None, n_sel=None,
                          order=None, status=None, head_dim_v=None, want_lse=True,
                          workspace=None):
    """One step in one launch: the centroid build of fill_pages (int32, the pages filled at this
    step; written into ``centroids``) and the fused selection + attention.  Returns
    (out, lse, sel, n_sel)."""
    lib = load_library()
    kv = paged_kv(k_pool, v_pool, head_dim_v)
    a = decode_args(q, page_table, seq_lens, centroids, topk, bos, eos, sm_scale, order, status)
    _need(fill_pages, "fill_pages", torch.int32, contiguous=True)
    B, hq = q.shape[0], q.shape[1]
    if out is None:
        out = torch.empty((B, hq, kv.head_dim_v), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, hq), dtype=torch.float32, device=q.device)
    if workspace is None:
        n = int(lib.vt_fused_workspace_size(ctypes.byref(kv), ctypes.byref(a)))
        workspace = torch.zeros(n, dtype=torch.uint8, device=q.device) if n else None
    if workspace is not None:
        _need(workspace, "workspace", torch.uint8, contiguous=True)
    rc = lib.vt_sparse_decode_step(ctypes.byref(kv), ctypes.byref(a), fill_pages.data_ptr(),
                                   fill_pages.numel(), centroids.data_ptr(), out.data_ptr(),
                                   _ptr(lse), _ptr(sel), _ptr(n_sel), _ptr(workspace),
                                   0 if workspace is None else workspace.numel(), _stream(q))
    _check(rc, "vt_sparse_decode_step")
    return out, lse, sel, n_sel


def vt_sparse_decode_fused_static(q, k_pool, v_pool, page_table, seq_lens, centroids, topk, bos,
                                  eos, sm_scale, out=None, lse=None, sel=None, n_sel=None,
                                  order=None, status=None, head_dim_v=None, want_lse=True):
    """vt_sparse_decode_fused on the library's own static scratch (no workspace argument).

    Calls on one device share that scratch: they must not overlap on the GPU.
    """
    lib = load_library()
    kv = paged_kv(k_pool, v_pool, head_dim_v)
    a = decode_args(q, page_table, seq_lens, centroids, topk, bos, eos, sm_scale, order, status)
    B, hq = q.shape[0], q.shape[1]
    if out is None:
        out = torch.empty((B, hq, kv.head_dim_v), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, hq), dtype=torch.float32, device=q.device)
    rc = lib.vt_sparse_decode_fused_static(ctypes.byref(kv), ctypes.byref(a), out.data_ptr(),
                                           _ptr(lse), _ptr(sel), _ptr(n_sel), _stream(q))
    _check(rc, "vt_sparse_decode_fused_static")
    return out, lse, sel, n_sel


def vt_plan_requests(seq_lens: torch.Tensor, order: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Request order, longest (most pages) first; equal lengths keep index order."""
    lib = load_library()
    _need(seq_lens, "seq_lens", torch.int32, contiguous=True)
    if order is None:
        order = torch.empty_like(seq_lens)
    rc = lib.vt_plan_requests(seq_lens.data_ptr(), seq_lens.numel(), order.data_ptr(),
                              _stream(seq_lens))
    _check(rc, "vt_plan_requests")
    return order


class PreparedCall:
    """One C entry point bound to fixed tensors: the arguments are checked and marshalled
    once, and each ``run()`` only launches (on the current stream).

    For a serving loop that calls the same operation on the same buffers every step (inputs
    refreshed in place, as with CUDA graphs).  The bound tensors must keep their storage,
    shapes and strides for the object's lifetime; it holds references to them.
    """

    def __init__(self, fn, args, device_index: int, where: str, keep, result):
        self._fn = fn
        self._args = args
        self._dev = device_index
        self._where = where
        self._keep = keep
        self.result = result

    def run(self):
        stream = _raw_stream(self._dev) if _raw_stream is not None else \
            torch.cuda.current_stream(self._dev).cuda_stream
        rc = self._fn(*self._args, stream)
        if rc != VT_OK:
            _check(rc, self._where)
        return self.result


def prepare_build_centroids(k_pool: torch.Tensor, pages: torch.Tensor, centroids: torch.Tensor,
                            status: Optional[torch.Tensor] = None) -> PreparedCall:
    """vt_build_centroids bound to these tensors; ``run()`` returns ``centroids``."""
    lib = load_library()
    _need(pages, "pages", torch.int32, contiguous=True)
    _need(centroids, "centroids", torch.float32, contiguous=True)
    if status is not None:
        _need(status, "status", torch.int32)
    kv = paged_kv(k_pool, k_pool)
    P = ctypes.c_void_p
    args = (ctypes.byref(kv), P(pages.data_ptr()), ctypes.c_int32(pages.numel()),
            P(centroids.data_ptr()), P(_ptr(status)))
    return PreparedCall(lib.vt_build_centroids, args, k_pool.get_device(), "vt_build_centroids",
                        (kv, k_pool, pages, centroids, status), centroids)


def prepare_sparse_decode_fused(q, k_pool, v_pool, page_table, seq_lens, centroids, topk, bos,
                                eos, sm_scale, out, lse=None, sel=None, n_sel=None, order=None,
                                status=None, head_dim_v=None, workspace=None) -> PreparedCall:
    """vt_sparse_decode_fused bound to these tensors; ``run()`` returns (out, lse, sel, n_sel).

    ``out`` (and ``lse`` if wanted) must be given; ``workspace`` as for the unprepared call
    (from fused_workspace(); required when the shapes need one).
    """
    lib = load_library()
    kv = paged_kv(k_pool, v_pool, head_dim_v)
    a = decode_args(q, page_table, seq_lens, centroids, topk, bos, eos, sm_scale, order, status)
    _need(out, "out", torch.bfloat16, contiguous=True)
    if lse is not None:
        _need(lse, "lse", torch.float32, contiguous=True)
    for t, name in ((sel, "sel"), (n_sel, "n_sel")):
        if t is not None:
            _need(t, name, torch.int32, contiguous=True)
    need = int(lib.vt_fused_workspace_size(ctypes.byref(kv), ctypes.byref(a)))
    if need:
        if workspace is None:
            raise VtError(VT_ERR_INVALID_ARG, "workspace", f"{need} bytes needed (fused_workspace())")
        _need(workspace, "workspace", torch.uint8, contiguous=True)
    P = ctypes.c_void_p
    args = (ctypes.byref(kv), ctypes.byref(a), P(out.data_ptr()), P(_ptr(lse)), P(_ptr(sel)),
            P(_ptr(n_sel)), P(_ptr(workspace)),
            ctypes.c_size_t(0 if workspace is None else workspace.numel()))
    keep = (kv, a, q, k_pool, v_pool, page_table, seq_lens, centroids, out, lse, sel, n_sel,
            order, status, workspace)
    return PreparedCall(lib.vt_sparse_decode_fused, args, q.get_device(), "vt_sparse_decode_fused",
                        keep, (out, lse, sel, n_sel))


def prepare_sparse_decode_step(q, k_pool, v_pool, page_table, seq_lens, centroids, topk, bos,
                               eos, sm_scale, fill_pages, out, lse=None, sel=None, n_sel=None,
                               order=None, status=None, head_dim_v=None,
                               workspace=None) -> PreparedCall:
    """vt_sparse_decode_step bound to these tensors (``fill_pages`` included: its contents may
    change between runs, its length may not); ``run()`` returns (out, lse, sel, n_sel)."""
    lib = load_library()
    fused = prepare_sparse_decode_fused(q, k_pool, v_pool, page_table, seq_lens, centroids, topk,
                                        bos, eos, sm_scale, out, lse, sel, n_sel, order, status,
                                        head_dim_v, workspace)
    _need(fill_pages, "fill_pages", torch.int32, contiguous=True)
    kv_ref, a_ref = fused._args[0], fused._args[1]
    P = ctypes.c_void_p
    args = (kv_ref, a_ref, P(fill_pages.data_ptr()), ctypes.c_int32(fill_pages.numel()),
            P(centroids.data_ptr())) + fused._args[2:]
    return PreparedCall(lib.vt_sparse_decode_step, args, q.get_device(), "vt_sparse_decode_step",
                        fused._keep + (fill_pages,), fused.result)


def vt_abi_version() -> int:
    return int(load_library().vt_abi_version())

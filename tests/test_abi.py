"""The C ABI without a GPU: the library loads, exports what include/vt.h declares, and its
host-side argument checks reject bad calls before anything is launched.

Pointers below are fake, 16-byte-aligned addresses: every call here must fail (or return
VT_OK for an empty batch) during host validation, so no device memory is ever touched.
"""
import ctypes
import os
import re

import pytest

import paged_block_sparse_vt_b200 as vt
from paged_block_sparse_vt_b200 import binding
from paged_block_sparse_vt_b200.build import build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "vt.h")
OK, INV, UNS = 0, 1, 2
FAKE = 0x7F0000000000  # aligned, never dereferenced


@pytest.fixture(scope="module")
def lib():
    build()
    return vt.load_library()


def test_exports_every_declared_symbol(lib):
    text = open(HEADER).read()
    declared = set(re.findall(r"^\s*(?:vt_status|const char\*|int32_t|size_t)\s+(vt_\w+)\s*\(", text, re.M))
    assert declared == set(binding.EXPORTS)
    for name in declared:
        assert hasattr(lib, name), name
    assert lib.vt_abi_version() == 1


def test_status_strings(lib):
    assert lib.vt_status_string(0) == b"VT_OK"
    assert lib.vt_status_string(1) == b"VT_ERR_INVALID_ARG"
    assert lib.vt_status_string(2) == b"VT_ERR_UNSUPPORTED"
    assert lib.vt_status_string(3) == b"VT_ERR_CUDA"


def _kv(**over):
    f = dict(k_pool=FAKE, v_pool=FAKE + 0x100000, num_pages=1000, page_size=16, num_kv_heads=8,
             head_dim=128, head_dim_v=128, sk_p=16 * 8 * 128, sk_t=8 * 128, sk_h=128,
             sv_p=16 * 8 * 128, sv_t=8 * 128, sv_h=128)
    f.update(over)
    return binding.PagedKV(**f)


def _args(**over):
    f = dict(batch=4, num_q_heads=32, q=FAKE + 0x200000, page_table=FAKE + 0x300000,
             pt_stride=64, seq_lens=FAKE + 0x400000, centroids=FAKE + 0x500000, topk=30, bos=1,
             eos=1, sm_scale=0.088, order=None, status=None)
    f.update(over)
    return binding.DecodeArgs(**f)


def _fused(lib, kv, a, out=FAKE + 0x600000, lse=None, sel=None, n_sel=None, ws=FAKE + 0x8000000,
           ws_bytes=1 << 40):
    return lib.vt_sparse_decode_fused(ctypes.byref(kv), ctypes.byref(a), out, lse, sel, n_sel, ws,
                                      ws_bytes, None)


@pytest.mark.parametrize("kv_over,args_over,code", [
    (dict(page_size=8), {}, UNS),
    (dict(k_pool=None), {}, INV),
    (dict(num_pages=0), {}, INV),
    (dict(num_kv_heads=0), {}, INV),
    (dict(head_dim=96, head_dim_v=96), {}, UNS),
    (dict(head_dim=128, head_dim_v=64), {}, UNS),
    (dict(k_pool=FAKE + 8), {}, UNS),
    (dict(sk_t=8 * 128 + 4), {}, UNS),
    (dict(sv_h=-128), {}, UNS),
    ({}, dict(num_q_heads=30), INV),
    ({}, dict(num_q_heads=72), UNS),            # G = 9
    ({}, dict(topk=-1), INV),
    ({}, dict(topk=0, bos=0, eos=0), INV),
    ({}, dict(topk=5000), UNS),
    ({}, dict(pt_stride=0), UNS),
    ({}, dict(pt_stride=40000), UNS),
    ({}, dict(sm_scale=float("nan")), INV),
    ({}, dict(q=None), INV),
    ({}, dict(centroids=None), INV),
    ({}, dict(q=FAKE + 0x200004), UNS),
    ({}, dict(batch=-1), INV),
    ({}, dict(batch=0), OK),                    # empty batch: nothing to launch
    (dict(num_kv_heads=2, head_dim=576, head_dim_v=512), dict(num_q_heads=64), UNS),
    (dict(num_kv_heads=1, head_dim=576, head_dim_v=512, sk_h=576, sv_h=576), dict(num_q_heads=32), UNS),
    (dict(num_kv_heads=1, head_dim=576, head_dim_v=512, v_pool=FAKE, sk_h=576, sv_h=576,
          sk_p=16 * 576, sv_p=16 * 576, sk_t=576, sv_t=576), dict(num_q_heads=48), UNS),
])
def test_fused_host_validation(lib, kv_over, args_over, code):
    rc = _fused(lib, _kv(**kv_over), _args(**args_over))
    assert rc == code
    if code != OK:
        assert lib.vt_last_error_detail()


def test_call_level_checks(lib):
    kv, a = _kv(), _args()
    assert lib.vt_sparse_decode_fused(ctypes.byref(kv), ctypes.byref(a), None, None, None, None,
                                      FAKE, 1 << 40, None) == INV        # out missing
    assert _fused(lib, kv, a, sel=FAKE + 0x700000) == INV                # sel without n_sel
    assert lib.vt_select_pages(ctypes.byref(kv), ctypes.byref(a), None, FAKE, None) == INV
    assert lib.vt_sparse_decode(ctypes.byref(kv), ctypes.byref(a), FAKE, None, FAKE, None,
                                None) == INV
    assert lib.vt_select_pages(None, ctypes.byref(a), FAKE, FAKE, None) == INV
    assert lib.vt_build_centroids(ctypes.byref(kv), FAKE, -1, FAKE, None, None) == INV
    assert lib.vt_build_centroids(ctypes.byref(kv), FAKE, 0, FAKE, None, None) == OK
    assert lib.vt_build_centroids(ctypes.byref(kv), None, 5, FAKE, None, None) == INV
    assert lib.vt_build_centroids(ctypes.byref(kv), FAKE, 5, FAKE + 4, None, None) == UNS
    assert lib.vt_build_centroids(ctypes.byref(_kv(page_size=32)), FAKE, 5, FAKE, None, None) == UNS
    assert lib.vt_plan_requests(FAKE, 70000, FAKE, None) == UNS
    assert lib.vt_plan_requests(FAKE, -2, FAKE, None) == INV
    assert lib.vt_plan_requests(FAKE, 0, FAKE, None) == OK
    assert lib.vt_plan_requests(None, 3, FAKE, None) == INV


def test_fused_workspace_contract(lib):
    kv, a = _kv(), _args()
    need = lib.vt_fused_workspace_size(ctypes.byref(kv), ctypes.byref(a))
    assert need > 0 and need % 256 == 0
    assert _fused(lib, kv, a, ws=None, ws_bytes=0) == INV                   # missing
    assert _fused(lib, kv, a, ws=FAKE, ws_bytes=need - 1) == INV            # too small
    assert _fused(lib, kv, a, ws=FAKE + 16, ws_bytes=need) == INV           # misaligned
    # MLA takes its own persistent path (with a workspace); very large batches need none
    mla = _kv(num_kv_heads=1, head_dim=576, head_dim_v=512, v_pool=FAKE, sk_h=576, sv_h=576,
              sk_p=16 * 576, sv_p=16 * 576, sk_t=576, sv_t=576)
    assert lib.vt_fused_workspace_size(ctypes.byref(mla), ctypes.byref(_args(num_q_heads=32))) > 0
    assert lib.vt_fused_workspace_size(ctypes.byref(mla),
                                       ctypes.byref(_args(num_q_heads=32, batch=5000))) == 0
    assert lib.vt_fused_workspace_size(ctypes.byref(kv), ctypes.byref(_args(batch=5000))) == 0
    assert lib.vt_fused_workspace_size(ctypes.byref(kv), ctypes.byref(_args(topk=-1))) == 0
    # grows with the batch and with the chunks of the page-table row
    assert lib.vt_fused_workspace_size(ctypes.byref(kv), ctypes.byref(_args(batch=8))) > need
    assert lib.vt_fused_workspace_size(ctypes.byref(kv), ctypes.byref(_args(pt_stride=1024))) > need


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(vt.VtError):
        vt.vt_sparse_decode_fused(q, q.view(1, 1, 2, 64), q.view(1, 1, 2, 64),
                                  torch.zeros(1, 1, dtype=torch.int32), torch.ones(1, dtype=torch.int32),
                                  torch.zeros(1, 2, 64), 1, 0, 0, 0.125)

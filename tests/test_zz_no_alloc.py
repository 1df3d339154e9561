"""vt_sparse_decode_fused_static: the fused call on the library's own static scratch.

It must give exactly what vt_sparse_decode_fused gives with a caller-owned workspace, call
after call (each call has to leave the shared scratch ready for the next), whether it runs
alone or after every other test in the process.  Collected last on purpose (file name).
"""
import ctypes

import pytest
import torch

import paged_block_sparse_vt_b200 as vt
from paged_block_sparse_vt_b200 import binding
from paged_block_sparse_vt_b200.build import build
from paged_block_sparse_vt_b200.workloads import config, make_workload
from parity import all_full_pages, to_device

FAKE = 0x7F0000000000  # aligned, never dereferenced (host checks fail first)
STATIC_BYTES = 32 << 20  # VT_STATIC_SCRATCH_BYTES


def _kv(**over):
    f = dict(k_pool=FAKE, v_pool=FAKE + 0x100000, num_pages=1000, page_size=16, num_kv_heads=8,
             head_dim=128, head_dim_v=128, sk_p=16 * 8 * 128, sk_t=8 * 128, sk_h=128,
             sv_p=16 * 8 * 128, sv_t=8 * 128, sv_h=128)
    f.update(over)
    return binding.PagedKV(**f)


def _args(**over):
    f = dict(batch=4, num_q_heads=16, q=FAKE + 0x200000, page_table=FAKE + 0x300000,
             pt_stride=64, seq_lens=FAKE + 0x400000, centroids=FAKE + 0x500000, topk=30, bos=1,
             eos=1, sm_scale=0.088, order=None, status=None)
    f.update(over)
    return binding.DecodeArgs(**f)


def test_static_host_checks():
    """Too much scratch is refused before launch; bad arguments fail as in the fused call."""
    build()
    lib = vt.load_library()
    big = _args(batch=2048, pt_stride=32768, topk=256)
    need = lib.vt_fused_workspace_size(ctypes.byref(_kv()), ctypes.byref(big))
    assert need > STATIC_BYTES
    rc = lib.vt_sparse_decode_fused_static(ctypes.byref(_kv()), ctypes.byref(big), FAKE + 0x600000,
                                           None, None, None, None)
    assert rc == 2 and b"static scratch" in lib.vt_last_error_detail()
    many = _kv(num_kv_heads=64, sk_p=16 * 64 * 128, sk_t=64 * 128, sv_p=16 * 64 * 128,
               sv_t=64 * 128)  # B * Hkv = 131072 units: more counters than the scratch lays out
    rc = lib.vt_sparse_decode_fused_static(ctypes.byref(many),
                                           ctypes.byref(_args(batch=2048, num_q_heads=64)),
                                           FAKE + 0x600000, None, None, None, None)
    assert rc == 2 and b"static scratch" in lib.vt_last_error_detail()
    for kv, a, code in ((_kv(page_size=8), _args(), 2), (_kv(), _args(num_q_heads=30), 1),
                        (_kv(), _args(q=None), 1), (_kv(), _args(batch=-1), 1)):
        assert lib.vt_sparse_decode_fused_static(ctypes.byref(kv), ctypes.byref(a), FAKE + 0x600000,
                                                 None, None, None, None) == code
    assert lib.vt_sparse_decode_fused_static(ctypes.byref(_kv()), ctypes.byref(_args()), None,
                                             None, None, None, None) == 1  # out missing


CASES = {
    "gqa_d128_g2": dict(cfg=2, B=6, len_lo=600, len_hi=5000, pool_pages=2500),
    "gqa_d128_g8": dict(cfg=2, B=3, Hq=16, Hkv=2, len_lo=700, len_hi=3000, pool_pages=800),
    "gqa_d64_g5": dict(cfg=1, B=3, Hq=10, Hkv=2, len_lo=300, len_hi=2000, pool_pages=500,
                       lengths="uniform"),
    "mixed_lengths": dict(cfg=5, B=40, len_lo=100, len_hi=12000, filled=3),
    "mla_no_scratch": dict(cfg=4, B=2, Hq=16, len_lo=2500, len_hi=2500, pool_pages=400),
}


@pytest.mark.gpu
@pytest.mark.parametrize("name", list(CASES))
def test_static_matches_workspace_call(name):
    kw = dict(CASES[name])
    c = config(kw.pop("cfg"), **kw)
    w = make_workload(c, poison=True)
    d = to_device(w)
    cent = torch.full((w["P"], c.Hkv, c.D), float("nan"), device="cuda")
    vt.vt_build_centroids(d["k_pool"], all_full_pages(d), cent)
    args = (d["q"], d["k_pool"], d["v_pool"], d["page_table"], d["seq_lens"], cent, c.topk, c.bos,
            c.eos, c.sm_scale)

    def outputs(fn, **extra):
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        sel = torch.full((c.B, c.Hkv, c.kmax), -7, dtype=torch.int32, device="cuda")
        n_sel = torch.full((c.B, c.Hkv), -7, dtype=torch.int32, device="cuda")
        out, lse, _, _ = fn(*args, sel=sel, n_sel=n_sel, status=st, head_dim_v=c.Dv, **extra)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        return out, lse, sel, n_sel

    ws = vt.fused_workspace(*args[:9], head_dim_v=c.Dv)
    want = outputs(vt.vt_sparse_decode_fused, workspace=ws)
    for _ in range(2):  # two calls in a row on the same static scratch
        got = outputs(vt.vt_sparse_decode_fused_static)
        for g, r in zip(got, want):
            assert torch.equal(g, r)
    # and the workspace path is unaffected by the static calls in between
    again = outputs(vt.vt_sparse_decode_fused, workspace=ws)
    for g, r in zip(again, want):
        assert torch.equal(g, r)

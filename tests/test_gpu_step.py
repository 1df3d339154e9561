"""vt_sparse_decode_step: the centroid build of the pages filled at this step folded into the
fused launch.  Against the oracle (every built centroid row, the selection within the tie
rule, every output) and bit for bit against the two-call step (vt_build_centroids, then
vt_sparse_decode_fused) on the same inputs; through the persistent kernels (GQA and MLA) and
through the cluster path (more than 2048 requests), where the build is its own launch."""
import ctypes

import pytest
import torch

import paged_block_sparse_vt_b200 as vt
from paged_block_sparse_vt_b200 import binding
from paged_block_sparse_vt_b200.workloads import config, make_workload
from parity import check_centroids, check_step, oracle_centroids, oracle_step, to_device

pytestmark = pytest.mark.gpu

CASES = {
    "c2s": dict(cfg=2, B=6, len_lo=600, len_hi=5000, pool_pages=2500, filled=3),
    "c5s": dict(cfg=5, B=40, len_lo=100, len_hi=12000, filled=5),
    "c4s": dict(cfg=4, B=3, len_lo=3000, len_hi=3000, pool_pages=700, filled=2),
    "c2_full": dict(cfg=2),
    "big_batch": dict(cfg=1, B=2100, len_lo=200, len_hi=900, lengths="uniform",
                      pool_pages=80000, filled=40),
}


@pytest.mark.parametrize("name", list(CASES))
def test_one_launch_step_equals_two_calls_and_the_oracle(name, oracle):
    kw = dict(CASES[name])
    c = config(kw.pop("cfg"), **kw)
    w = make_workload(c, poison=True)
    assert c.eos >= 1 and w["fill_pages"].numel() > 0
    d = to_device(w)
    args = lambda cent: (d["q"], d["k_pool"], d["v_pool"], d["page_table"], d["seq_lens"], cent,
                         c.topk, c.bos, c.eos)
    res = []
    for one_launch in (True, False):
        cent = torch.full((w["P"], c.Hkv, c.D), float("nan"), device="cuda")
        vt.vt_build_centroids(d["k_pool"], d["prebuilt_pages"], cent)
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        sel = torch.empty((c.B, c.Hkv, c.kmax), dtype=torch.int32, device="cuda")
        n_sel = torch.empty((c.B, c.Hkv), dtype=torch.int32, device="cuda")
        ws = vt.fused_workspace(*args(cent), head_dim_v=c.Dv)
        if one_launch:
            out, lse, _, _ = vt.vt_sparse_decode_step(*args(cent), c.sm_scale, d["fill_pages"],
                                                      sel=sel, n_sel=n_sel, status=st,
                                                      head_dim_v=c.Dv, workspace=ws)
        else:
            vt.vt_build_centroids(d["k_pool"], d["fill_pages"], cent, status=st)
            out, lse, _, _ = vt.vt_sparse_decode_fused(*args(cent), c.sm_scale, sel=sel,
                                                       n_sel=n_sel, status=st, head_dim_v=c.Dv,
                                                       workspace=ws)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        res.append((cent, sel, n_sel, out, lse))
    (c1, s1, n1, o1, l1), (c2, s2, n2, o2, l2) = res
    assert torch.equal(c1.nan_to_num(7.0), c2.nan_to_num(7.0))
    assert torch.equal(s1, s2) and torch.equal(n1, n2)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)
    cent_ref = oracle_centroids(oracle, w)
    pages = torch.cat([w["prebuilt_pages"], w["fill_pages"]]).to(torch.int32)
    check_centroids(c1, cent_ref, pages)
    ref = oracle_step(oracle, w, cent_ref)
    check_step(oracle, w, ref, cent_ref, s1, n1, o1, l1, label=f"one-launch step {name}")


def test_step_host_checks():
    """eos = 0 with pages to build, and a build target other than the scored cache, are
    refused before anything is launched."""
    lib = vt.load_library()
    fake = 0x7F0000000000
    kv = binding.PagedKV(k_pool=fake, v_pool=fake + 0x100000, num_pages=1000, page_size=16,
                         num_kv_heads=8, head_dim=128, head_dim_v=128, sk_p=16 * 8 * 128,
                         sk_t=8 * 128, sk_h=128, sv_p=16 * 8 * 128, sv_t=8 * 128, sv_h=128)
    cent = fake + 0x500000

    def a(eos):
        return binding.DecodeArgs(batch=4, num_q_heads=16, q=fake + 0x200000,
                                  page_table=fake + 0x300000, pt_stride=64,
                                  seq_lens=fake + 0x400000, centroids=cent, topk=30, bos=1,
                                  eos=eos, sm_scale=0.088, order=None, status=None)
    call = lib.vt_sparse_decode_step
    assert call(ctypes.byref(kv), ctypes.byref(a(0)), fake + 0x600000, 2, cent, fake + 0x700000,
                None, None, None, None, 0, None) == 2
    assert call(ctypes.byref(kv), ctypes.byref(a(1)), fake + 0x600000, 2, cent + 4096,
                fake + 0x700000, None, None, None, None, 0, None) == 1
    assert call(ctypes.byref(kv), ctypes.byref(a(1)), None, 2, cent, fake + 0x700000, None, None,
                None, None, 0, None) == 1
    assert call(ctypes.byref(kv), ctypes.byref(a(1)), fake + 0x600000, -1, cent,
                fake + 0x700000, None, None, None, None, 0, None) == 1

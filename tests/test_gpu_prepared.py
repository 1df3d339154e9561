"""Prepared calls (prepare_build_centroids / prepare_sparse_decode_fused): arguments checked
and marshalled once, then run() launches.  Each run must give bitwise what the plain call
gives on the same inputs, including after the inputs are refreshed in place, which is how a
serving loop uses them.
"""
import pytest
import torch

import paged_block_sparse_vt_b200 as vt
from paged_block_sparse_vt_b200.workloads import config, make_workload
from parity import all_full_pages, to_device


def test_prepare_rejects_host_tensors():
    """The checks run at prepare time: host tensors fail before anything launches."""
    k = torch.zeros((4, 16, 1, 64), dtype=torch.bfloat16)
    pages = torch.zeros(2, dtype=torch.int32)
    cent = torch.zeros((4, 1, 64))
    with pytest.raises(vt.VtError):
        vt.prepare_build_centroids(k, pages, cent)


CASES = {
    "gqa": dict(cfg=2, B=6, len_lo=2000, len_hi=9000, pool_pages=3000),
    "gqa_d64": dict(cfg=1, B=5, Hq=10, Hkv=2, lengths="uniform", len_lo=800, len_hi=6000,
                    pool_pages=2500),
    "mla": dict(cfg=4, B=3, Hq=16, len_lo=5000, len_hi=5000, pool_pages=1200),
}


@pytest.mark.gpu
@pytest.mark.parametrize("name", list(CASES))
def test_prepared_equals_plain(name):
    kw = dict(CASES[name])
    c = config(kw.pop("cfg"), **kw)
    w = make_workload(c)
    d = to_device(w)
    pages = all_full_pages(d)
    # a finite fill: pages outside the list stay as they are and must compare equal
    cent_a = torch.full((w["P"], c.Hkv, c.D), -7.0, device="cuda")
    cent_b = cent_a.clone()
    vt.vt_build_centroids(d["k_pool"], pages, cent_a)
    build = vt.prepare_build_centroids(d["k_pool"], pages, cent_b)
    assert build.run() is cent_b
    torch.cuda.synchronize()
    assert torch.equal(cent_a, cent_b)

    args = (d["q"], d["k_pool"], d["v_pool"], d["page_table"], d["seq_lens"], cent_a, c.topk,
            c.bos, c.eos)
    ws_a = vt.fused_workspace(*args, head_dim_v=c.Dv)
    ws_b = vt.fused_workspace(*args, head_dim_v=c.Dv)
    out_b = torch.empty((c.B, c.Hq, c.Dv), dtype=torch.bfloat16, device="cuda")
    lse_b = torch.empty((c.B, c.Hq), dtype=torch.float32, device="cuda")
    sel_b = torch.empty((c.B, c.Hkv, c.kmax), dtype=torch.int32, device="cuda")
    nsel_b = torch.empty((c.B, c.Hkv), dtype=torch.int32, device="cuda")
    fused = vt.prepare_sparse_decode_fused(*args, c.sm_scale, out=out_b, lse=lse_b, sel=sel_b,
                                           n_sel=nsel_b, head_dim_v=c.Dv, workspace=ws_b)
    for step in range(3):
        if step:  # refresh the inputs in place, as a serving loop does between steps
            g = torch.Generator(device="cuda").manual_seed(step)
            d["q"].copy_(torch.randn(d["q"].shape, generator=g, device="cuda").to(torch.bfloat16))
        out_a, lse_a, sel_a, nsel_a = vt.vt_sparse_decode_fused(
            *args, c.sm_scale, sel=torch.empty_like(sel_b), n_sel=torch.empty_like(nsel_b),
            head_dim_v=c.Dv, workspace=ws_a)
        res = fused.run()
        assert res[0] is out_b and res[1] is lse_b
        torch.cuda.synchronize()
        assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16))
        assert torch.equal(lse_a, lse_b)
        assert torch.equal(sel_a, sel_b) and torch.equal(nsel_a, nsel_b)


@pytest.mark.gpu
def test_prepared_needs_a_workspace():
    c = config(2, B=4, len_lo=3000, len_hi=6000, pool_pages=2000)
    w = make_workload(c)
    d = to_device(w)
    cent = torch.zeros((w["P"], c.Hkv, c.D), device="cuda")
    out = torch.empty((c.B, c.Hq, c.Dv), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(vt.VtError):
        vt.prepare_sparse_decode_fused(d["q"], d["k_pool"], d["v_pool"], d["page_table"],
                                       d["seq_lens"], cent, c.topk, c.bos, c.eos, c.sm_scale,
                                       out=out)

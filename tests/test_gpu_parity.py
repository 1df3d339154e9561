"""GPU parity: libvt (through its C ABI) against the fp64 CPU oracle on the same seeded inputs.

Sizes are chosen so the oracle finishes in seconds while every case still spans several
CTAs per unit, several score tiles and ragged last pages.  Pool pages that belong to no
request, and token slots past the end of each request, hold NaN: a wrong gather cannot pass.
"""
import functools

import pytest
import torch

import paged_block_sparse_vt_b200 as vt
from paged_block_sparse_vt_b200.workloads import config, make_workload
from parity import (all_full_pages, check_centroids, check_step, compare_outputs,
                    compare_selection, oracle_centroids, oracle_step, to_device)

pytestmark = pytest.mark.gpu

CASES = {
    "c1": dict(cfg=1),
    "c2s": dict(cfg=2, B=6, len_lo=600, len_hi=5000, pool_pages=2500),
    "c3s": dict(cfg=3, B=3, len_lo=4096, len_hi=4096, pool_pages=1000),
    "c4s": dict(cfg=4, B=3, len_lo=3000, len_hi=3000, pool_pages=700),
    "c5s": dict(cfg=5, B=40, len_lo=100, len_hi=12000, filled=3),
    "g1_d128": dict(cfg=2, B=3, Hq=8, Hkv=8, len_lo=700, len_hi=3000, pool_pages=800),
    "g2_d64": dict(cfg=1, B=4, Hq=4, Hkv=2, len_lo=300, len_hi=2000, pool_pages=500, lengths="uniform"),
    "g3_d128": dict(cfg=2, B=3, Hq=6, Hkv=2, len_lo=700, len_hi=3000, pool_pages=800),
    "g5_d64": dict(cfg=1, B=3, Hq=10, Hkv=2, len_lo=300, len_hi=2000, pool_pages=500, lengths="uniform"),
    "g6_d128": dict(cfg=2, B=3, Hq=12, Hkv=2, len_lo=700, len_hi=3000, pool_pages=800),
    "g7_d64": dict(cfg=1, B=3, Hq=7, Hkv=1, len_lo=300, len_hi=2000, pool_pages=500, lengths="uniform"),
    "g8_d128": dict(cfg=2, B=3, Hq=16, Hkv=2, len_lo=700, len_hi=3000, pool_pages=800),
    "mla16": dict(cfg=4, B=2, Hq=16, len_lo=2500, len_hi=2500, pool_pages=400),
    # top-k large enough that the chunks keep more candidates than the fused merge's fast path
    # takes (GQA: more than 256; MLA: more than 512, and 13 attention pieces per request)
    "bigk_gqa": dict(cfg=2, B=3, Hq=4, Hkv=2, topk=300, len_lo=18000, len_hi=22000,
                     pool_pages=5000),
    "bigk_mla": dict(cfg=4, B=2, Hq=16, topk=100, len_lo=16000, len_hi=16000, pool_pages=2100),
    # more requests than the persistent path takes: the fused call runs the cluster kernel
    "big_batch": dict(cfg=1, B=2100, len_lo=200, len_hi=900, lengths="uniform",
                      pool_pages=80000),
}


@functools.lru_cache(maxsize=None)
def _case(name):
    kw = dict(CASES[name])
    cfg = kw.pop("cfg")
    w = make_workload(config(cfg, **kw), poison=True)
    return w


@functools.lru_cache(maxsize=None)
def _reference(name):
    import oracle
    w = _case(name)
    cent = oracle_centroids(oracle, w)
    return cent, oracle_step(oracle, w, cent)


def _gpu_centroids(d, w):
    c = w["config"]
    cent = torch.full((w["P"], c.Hkv, c.D), float("nan"), device="cuda")
    vt.vt_build_centroids(d["k_pool"], all_full_pages(d), cent)
    return cent


def _status():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


@pytest.mark.parametrize("name", list(CASES))
def test_centroid_build(name, oracle):
    w = _case(name)
    d = to_device(w)
    cent_ref, _ = _reference(name)
    st = _status()
    cent = torch.full((w["P"], w["config"].Hkv, w["config"].D), float("nan"), device="cuda")
    vt.vt_build_centroids(d["k_pool"], all_full_pages(d), cent, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    check_centroids(cent, cent_ref, all_full_pages(w))
    # rows of pages not listed stay untouched
    untouched = torch.ones(w["P"], dtype=torch.bool)
    untouched[all_full_pages(w).long()] = False
    assert torch.isnan(cent.cpu()[untouched]).all()


@pytest.mark.parametrize("name", list(CASES))
def test_select_pages(name, oracle):
    """Selection from the oracle's centroids (an input here) vs the oracle's selection."""
    w = _case(name)
    c = w["config"]
    d = to_device(w)
    cent_ref, ref = _reference(name)
    st = _status()
    sel, n_sel = vt.vt_select_pages(d["q"], d["k_pool"], d["v_pool"], d["page_table"],
                                    d["seq_lens"], cent_ref.cuda(), c.topk, c.bos, c.eos,
                                    status=st, head_dim_v=c.Dv)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    compare_selection(w, ref, cent_ref, sel, n_sel, label=f"select {name}")


@pytest.mark.parametrize("name", list(CASES))
def test_sparse_decode(name, oracle):
    """Attention over the oracle's selection (an input here) vs the oracle's output."""
    w = _case(name)
    c = w["config"]
    d = to_device(w)
    _, ref = _reference(name)
    st = _status()
    out, lse = vt.vt_sparse_decode(d["q"], d["k_pool"], d["v_pool"], d["page_table"],
                                   d["seq_lens"], ref["sel"].cuda(), ref["n_sel"].cuda(),
                                   c.sm_scale, status=st, head_dim_v=c.Dv)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    compare_outputs(out, lse, ref["out"], ref["lse"])


@pytest.mark.parametrize("name", list(CASES))
def test_fused_pipeline(name, oracle):
    """GPU centroids -> fused select+attend vs the oracle pipeline; unfused path identical."""
    w = _case(name)
    c = w["config"]
    d = to_device(w)
    cent_ref, ref = _reference(name)
    st = _status()
    cent = _gpu_centroids(d, w)
    B, hkv = c.B, c.Hkv
    sel = torch.full((B, hkv, c.kmax), -7, dtype=torch.int32, device="cuda")
    n_sel = torch.full((B, hkv), -7, dtype=torch.int32, device="cuda")
    out, lse, _, _ = vt.vt_sparse_decode_fused(d["q"], d["k_pool"], d["v_pool"], d["page_table"],
                                               d["seq_lens"], cent, c.topk, c.bos, c.eos,
                                               c.sm_scale, sel=sel, n_sel=n_sel, status=st,
                                               head_dim_v=c.Dv)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    check_step(oracle, w, ref, cent_ref, sel, n_sel, out, lse, label=f"fused {name}")
    # the two-launch path (select, then decode) meets the same bar
    sel2, n_sel2 = vt.vt_select_pages(d["q"], d["k_pool"], d["v_pool"], d["page_table"],
                                      d["seq_lens"], cent, c.topk, c.bos, c.eos, head_dim_v=c.Dv)
    out2, lse2 = vt.vt_sparse_decode(d["q"], d["k_pool"], d["v_pool"], d["page_table"],
                                     d["seq_lens"], sel2, n_sel2, c.sm_scale, head_dim_v=c.Dv)
    check_step(oracle, w, ref, cent_ref, sel2, n_sel2, out2, lse2, label=f"select+decode {name}")


@pytest.mark.parametrize("name", ["c2s", "c5s", "g3_d128", "g7_d64"])
def test_fused_workspace_reuse(name, oracle):
    """One workspace, zeroed once, serves repeated calls: identical results every time."""
    w = _case(name)
    c = w["config"]
    d = to_device(w)
    cent = _gpu_centroids(d, w)
    args = (d["q"], d["k_pool"], d["v_pool"], d["page_table"], d["seq_lens"], cent, c.topk,
            c.bos, c.eos)
    ws = vt.fused_workspace(*args)
    assert ws is not None and int(ws.count_nonzero()) == 0
    st = _status()
    outs = [vt.vt_sparse_decode_fused(*args, c.sm_scale, status=st, workspace=ws)[0].clone()
            for _ in range(3)]
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
    # after a complete call the claim count equals the next launch's starting count, and the
    # per-unit counters (after the first 256 bytes, B * Hkv int32 each, 256-byte aligned) are 0
    head = ws[:8].view(torch.int32)
    assert int(head[0]) == int(head[1]) > 0
    units = c.B * c.Hkv
    span = 2 * ((units * 4 + 255) // 256 * 256)
    assert int(ws[256:256 + span].count_nonzero()) == 0


def test_planner_order_and_invariance(oracle):
    w = _case("c5s")
    c = w["config"]
    d = to_device(w)
    order = vt.vt_plan_requests(d["seq_lens"])
    n = (w["seq_lens"].long() + 15) // 16
    want = sorted(range(c.B), key=lambda b: (-int(n[b]), b))
    assert order.cpu().tolist() == want
    cent = _gpu_centroids(d, w)
    args = (d["q"], d["k_pool"], d["v_pool"], d["page_table"], d["seq_lens"], cent, c.topk,
            c.bos, c.eos, c.sm_scale)
    out_a, lse_a, _, _ = vt.vt_sparse_decode_fused(*args)
    out_b, lse_b, _, _ = vt.vt_sparse_decode_fused(*args, order=order)
    assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16))
    assert torch.equal(lse_a, lse_b)


EDGE_LENS = (1, 15, 16, 17, 95, 96, 97, 100, 255, 256, 257, 16 * 38 + 3, 4000)


@pytest.mark.parametrize("topk,bos,eos", [(6, 1, 1), (0, 1, 1), (5, 0, 0), (4, 2, 0), (3, 0, 3),
                                          (300, 1, 1)])
def test_edge_lengths_and_knobs(topk, bos, eos, oracle):
    """Single-token requests, exact page boundaries, the dense threshold, k=0, no reserved
    pages, and a top-k that covers everything."""
    c = config(2, B=len(EDGE_LENS), lengths="explicit", explicit=EDGE_LENS, pool_pages=600,
               topk=topk, bos=bos, eos=eos)
    w = make_workload(c, poison=True)
    # with eos = 0 the partial last page is a candidate: give it a finite centroid
    cent_ref = torch.full((w["P"], c.Hkv, c.D), float("nan"))
    n = (w["seq_lens"].long() + 15) // 16
    pages = torch.cat([w["page_table"][b, : int(n[b])] for b in range(c.B)]).to(torch.int32)
    oracle.build_centroids(w["k_pool"].nan_to_num(0.0), pages, cent_ref)
    ref = oracle_step(oracle, w, cent_ref)
    d = to_device(w)
    st = _status()
    sel = torch.empty((c.B, c.Hkv, c.kmax), dtype=torch.int32, device="cuda")
    n_sel = torch.empty((c.B, c.Hkv), dtype=torch.int32, device="cuda")
    out, lse, _, _ = vt.vt_sparse_decode_fused(d["q"], d["k_pool"], d["v_pool"], d["page_table"],
                                               d["seq_lens"], cent_ref.cuda(), topk, bos, eos,
                                               c.sm_scale, sel=sel, n_sel=n_sel, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    check_step(oracle, w, ref, cent_ref, sel, n_sel, out, lse,
               label=f"edge k={topk} bos={bos} eos={eos}")


def test_strided_pools_match_contiguous(oracle):
    """K and V as views into one [P, 16, 2, Hkv, D] tensor (non-contiguous strides)."""
    w = _case("c2s")
    c = w["config"]
    d = to_device(w)
    kv = torch.stack([d["k_pool"], d["v_pool"]], dim=2)  # [P, 16, 2, Hkv, D]
    k_view, v_view = kv[:, :, 0], kv[:, :, 1]
    assert not k_view.is_contiguous()
    cent = _gpu_centroids(d, w)
    a = vt.vt_sparse_decode_fused(d["q"], d["k_pool"], d["v_pool"], d["page_table"],
                                  d["seq_lens"], cent, c.topk, c.bos, c.eos, c.sm_scale)
    cent2 = torch.full_like(cent, float("nan"))
    vt.vt_build_centroids(k_view, all_full_pages(d), cent2)
    b = vt.vt_sparse_decode_fused(d["q"], k_view, v_view, d["page_table"], d["seq_lens"], cent2,
                                  c.topk, c.bos, c.eos, c.sm_scale)
    assert torch.equal(cent.nan_to_num(7.0), cent2.nan_to_num(7.0))
    assert torch.equal(a[0].view(torch.int16), b[0].view(torch.int16))


def test_bad_inputs_set_status_and_spare_other_units(oracle):
    """An out-of-range page id and a zero length are reported, not faulted on."""
    w = _case("c2s")
    c = w["config"]
    cent_ref, ref = _reference("c2s")
    d = to_device(w)
    pt = d["page_table"].clone()
    pt[0, 5] = w["P"] + 1000  # a middle page of request 0 -> unit skipped, bit set
    seq = d["seq_lens"].clone()
    seq[1] = 0                 # request 1 -> skipped, bit set
    st = _status()
    out, lse, sel, n_sel = vt.vt_sparse_decode_fused(
        d["q"], d["k_pool"], d["v_pool"], pt, seq, cent_ref.cuda(), c.topk, c.bos, c.eos,
        c.sm_scale, sel=torch.empty((c.B, c.Hkv, c.kmax), dtype=torch.int32, device="cuda"),
        n_sel=torch.empty((c.B, c.Hkv), dtype=torch.int32, device="cuda"), status=st)
    torch.cuda.synchronize()
    bits = int(st.item())
    assert bits & vt.VT_DEV_BAD_PAGE and bits & vt.VT_DEV_BAD_LEN
    assert torch.all(out[1].float() == 0) and torch.all(n_sel[1] == 0)
    keep = torch.ones((c.B, c.Hkv), dtype=torch.bool)
    keep[0] = keep[1] = False
    rows = keep.repeat_interleave(c.G, dim=1)
    err = (out.cpu().double()[rows] - ref["out"][rows]).abs().max().item()
    assert err <= 1e-2
    # build: a bad page id is skipped and reported
    st.zero_()
    cent = torch.zeros((w["P"], c.Hkv, c.D), device="cuda")
    vt.vt_build_centroids(d["k_pool"], torch.tensor([3, -1, w["P"]], dtype=torch.int32,
                                                    device="cuda"), cent, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == vt.VT_DEV_BAD_PAGE
    # decode: a selection entry past the request's pages is reported
    st.zero_()
    bad_sel = ref["sel"].clone().cuda()
    bad_sel[2, 0, 0] = 10 ** 6
    vt.vt_sparse_decode(d["q"], d["k_pool"], d["v_pool"], d["page_table"], d["seq_lens"], bad_sel,
                        ref["n_sel"].cuda(), c.sm_scale, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == vt.VT_DEV_BAD_SEL
    # the same through the decode-only persistent launch: reported, the unit's output zeroed
    st.zero_()
    ws = vt.decode_workspace(d["q"], d["k_pool"], d["v_pool"], d["page_table"], d["seq_lens"],
                             bad_sel)
    out, _ = vt.vt_sparse_decode(d["q"], d["k_pool"], d["v_pool"], d["page_table"], d["seq_lens"],
                                 bad_sel, ref["n_sel"].cuda(), c.sm_scale, status=st, workspace=ws)
    torch.cuda.synchronize()
    assert int(st.item()) == vt.VT_DEV_BAD_SEL
    assert torch.all(out[2, :c.G].float() == 0)


def test_mla_decode_workspace_rejects_bad_selection(oracle):
    """The MLA decode-only persistent launch: a selection entry past its request's pages is
    reported and zeroes that request's outputs; the other requests still match the oracle."""
    w = _case("c4s")
    c = w["config"]
    _, ref = _reference("c4s")
    d = to_device(w)
    bad_sel = ref["sel"].clone().cuda()
    bad_sel[1, 0, 3] = 10 ** 6
    ws = vt.decode_workspace(d["q"], d["k_pool"], d["v_pool"], d["page_table"], d["seq_lens"],
                             bad_sel, head_dim_v=c.Dv)
    assert ws is not None
    st = _status()
    out, lse = vt.vt_sparse_decode(d["q"], d["k_pool"], d["v_pool"], d["page_table"],
                                   d["seq_lens"], bad_sel, ref["n_sel"].cuda(), c.sm_scale,
                                   status=st, head_dim_v=c.Dv, workspace=ws)
    torch.cuda.synchronize()
    assert int(st.item()) == vt.VT_DEV_BAD_SEL
    assert torch.all(out[1].float() == 0)
    keep = [0, 2]
    compare_outputs(out[keep], lse[keep], ref["out"][keep], ref["lse"][keep])


@pytest.mark.parametrize("name", ["c2s", "c4s", "c5s"])
def test_last_page_centroid_is_never_read(name):
    """With eos >= 1 a request's last page is reserved, so no score reads its centroid: the
    fused call gives the same bits with those centroid rows set to NaN.  (This is what lets a
    serving loop build the centroid of a page that fills at this step beside this step's
    call, as bench.py does.)"""
    kw = dict(CASES[name])
    c = config(kw.pop("cfg"), **kw)
    assert c.eos >= 1
    w = make_workload(c)
    d = to_device(w)
    cent = torch.zeros((w["P"], c.Hkv, c.D), device="cuda")
    vt.vt_build_centroids(d["k_pool"], all_full_pages(d), cent)
    n = (d["seq_lens"].long() + 15) // 16
    last = d["page_table"][torch.arange(c.B, device="cuda"), n - 1].long()
    poisoned = cent.clone()
    poisoned[last] = float("nan")
    args = (d["q"], d["k_pool"], d["v_pool"], d["page_table"], d["seq_lens"])
    res = []
    for cc in (cent, poisoned):
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        sel = torch.empty((c.B, c.Hkv, c.kmax), dtype=torch.int32, device="cuda")
        n_sel = torch.empty((c.B, c.Hkv), dtype=torch.int32, device="cuda")
        out, lse, _, _ = vt.vt_sparse_decode_fused(*args, cc, c.topk, c.bos, c.eos, c.sm_scale,
                                                   sel=sel, n_sel=n_sel, status=st,
                                                   head_dim_v=c.Dv)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        res.append((out.view(torch.int16), lse, sel, n_sel))
    for a, b in zip(*res):
        assert torch.equal(a, b)


@pytest.mark.parametrize("name", list(CASES))
def test_select_and_decode_with_workspace(name, oracle):
    """vt_select_pages_ws and vt_sparse_decode_ws (the persistent kernels' select-only and
    decode-only launches, GQA and MLA, B <= 2048; larger batches keep the cluster kernels)
    against the oracle, twice in a row on the same workspaces."""
    w = _case(name)
    c = w["config"]
    d = to_device(w)
    cent_ref, ref = _reference(name)
    cent = cent_ref.cuda()
    args = (d["q"], d["k_pool"], d["v_pool"], d["page_table"], d["seq_lens"], cent, c.topk, c.bos,
            c.eos)
    ws_sel = vt.fused_workspace(*args, head_dim_v=c.Dv)
    ref_sel, ref_n = ref["sel"].cuda(), ref["n_sel"].cuda()
    ws_dec = vt.decode_workspace(d["q"], d["k_pool"], d["v_pool"], d["page_table"], d["seq_lens"],
                                 ref_sel, head_dim_v=c.Dv)
    for _ in range(2):
        st = _status()
        sel, n_sel = vt.vt_select_pages(*args, status=st, head_dim_v=c.Dv, workspace=ws_sel)
        out, lse = vt.vt_sparse_decode(d["q"], d["k_pool"], d["v_pool"], d["page_table"],
                                       d["seq_lens"], ref_sel, ref_n, c.sm_scale, status=st,
                                       head_dim_v=c.Dv, workspace=ws_dec)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        compare_selection(w, ref, cent_ref, sel, n_sel, label=f"select with workspace {name}")
        compare_outputs(out, lse, ref["out"], ref["lse"])

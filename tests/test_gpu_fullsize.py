"""Full-size parity: the benchmark workloads at their real sizes, through the calls bench.py
times (centroid build of the prebuilt and of the newly filled pages, then the fused call on a
workspace), against the oracle on EVERY request (the fp64 oracle runs these sizes in seconds
on the host cores): every centroid row, every selection within the tie rule, every output
row and lse.  Every request is also checked through properties that hold at any size.

Pool pages that belong to no request and token slots past the end of each request hold NaN,
so a gather from the wrong place cannot pass.
"""
import pytest
import torch

import paged_block_sparse_vt_b200 as vt
from paged_block_sparse_vt_b200.workloads import config, make_workload
from parity import PS, all_full_pages, check_centroids, check_step, oracle_step, to_device

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _check_invariants(c, seq_lens, sel, n_sel, out) -> None:
    """What holds for every request whatever the scores: counts, order, range, reserved pages."""
    kmax = c.topk + c.bos + c.eos
    n = (seq_lens.long() + PS - 1) // PS
    want = torch.minimum(n, torch.full_like(n, kmax))
    assert torch.equal(n_sel.long(), want[:, None].expand_as(n_sel))
    pos = torch.arange(kmax, device=sel.device)
    live = pos[None, None, :] < n_sel[:, :, None]
    assert bool((sel[~live] == -1).all())
    s = torch.where(live, sel, torch.full_like(sel, 1 << 30)).long()
    assert bool((s[:, :, 1:] > s[:, :, :-1])[live[:, :, 1:]].all()), "not strictly ascending"
    assert bool((s[live] >= 0).all())
    assert bool((s < n[:, None, None])[live].all()), "page past the end of its request"
    sparse = n > kmax
    for r in range(c.bos):  # reserved first pages, then the last eos pages, of sparse requests
        assert bool((sel[sparse, :, r] == r).all())
    for r in range(c.eos):
        last = (n[sparse] - c.eos + r)[:, None]
        assert bool((sel[sparse][:, :, c.bos + c.topk + r] == last).all())
    assert bool(torch.isfinite(out.float()).all())


@pytest.mark.parametrize("cfg", [2, 3, 4, 5])
def test_full_size_fused_against_oracle(cfg, oracle):
    c = config(cfg)
    w = make_workload(c, poison=True)
    d = to_device(w)
    cent = torch.full((w["P"], c.Hkv, c.D), float("nan"), device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    vt.vt_build_centroids(d["k_pool"], d["prebuilt_pages"], cent, status=st)
    vt.vt_build_centroids(d["k_pool"], d["fill_pages"], cent, status=st)
    sel = torch.full((c.B, c.Hkv, c.kmax), -7, dtype=torch.int32, device="cuda")
    n_sel = torch.full((c.B, c.Hkv), -7, dtype=torch.int32, device="cuda")
    args = (d["q"], d["k_pool"], d["v_pool"], d["page_table"], d["seq_lens"], cent, c.topk, c.bos,
            c.eos)
    ws = vt.fused_workspace(*args, head_dim_v=c.Dv)
    out, lse, _, _ = vt.vt_sparse_decode_fused(*args, c.sm_scale, sel=sel, n_sel=n_sel, status=st,
                                               head_dim_v=c.Dv, workspace=ws)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    _check_invariants(c, d["seq_lens"], sel, n_sel, out)
    del d

    cent_ref = torch.full((w["P"], c.Hkv, c.D), float("nan"))
    pages = all_full_pages(w)
    oracle.build_centroids(w["k_pool"], pages, cent_ref)
    check_centroids(cent, cent_ref, pages)
    del cent
    ref = oracle_step(oracle, w, cent_ref)
    check_step(oracle, w, ref, cent_ref, sel, n_sel, out, lse, label=f"full-size config {cfg}")

"""Bounded waits of the persistent kernels: a counter that never reaches its target makes the
waiting CTAs give up after their time limit, report VT_DEV_TIMEOUT in the status word and
finish the launch; the context stays usable and a re-zeroed workspace gives exact results.

The failure is made on the host, in the workspace: unit 0's scan counter (the first int32
after the 256-byte queue block) is set far below any count its scan items can reach, so its
attention items wait for a signal that never comes.  No kernel faults, traps or hangs.
"""
import pytest
import torch

import paged_block_sparse_vt_b200 as vt
from paged_block_sparse_vt_b200.workloads import config, make_workload
from parity import all_full_pages, to_device

pytestmark = pytest.mark.gpu

CASES = {
    "gqa": dict(cfg=2, B=4, len_lo=3000, len_hi=6000, pool_pages=2000),
    "mla": dict(cfg=4, B=2, Hq=16, len_lo=4000, len_hi=4000, pool_pages=600),
}


@pytest.mark.parametrize("name", list(CASES))
def test_wait_that_never_ends_reports_timeout(name):
    kw = dict(CASES[name])
    c = config(kw.pop("cfg"), **kw)
    w = make_workload(c)
    d = to_device(w)
    cent = torch.full((w["P"], c.Hkv, c.D), float("nan"), device="cuda")
    vt.vt_build_centroids(d["k_pool"], all_full_pages(d), cent)
    args = (d["q"], d["k_pool"], d["v_pool"], d["page_table"], d["seq_lens"], cent, c.topk, c.bos,
            c.eos)
    ws = vt.fused_workspace(*args, head_dim_v=c.Dv)
    assert ws is not None

    def run():
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        out, lse, _, _ = vt.vt_sparse_decode_fused(*args, c.sm_scale, status=st, workspace=ws,
                                                   head_dim_v=c.Dv)
        torch.cuda.synchronize()
        return int(st.item()), out.clone(), lse.clone()

    status, want_out, want_lse = run()
    assert status == 0
    # unit 0's scan counter can no longer reach its target
    ws.zero_()
    ws[256:260].view(torch.int32)[0] = -(1 << 30)
    status, _, _ = run()
    assert status & vt.VT_DEV_TIMEOUT, status
    # the context is usable: a re-zeroed workspace serves the next call exactly
    ws.zero_()
    status, out, lse = run()
    assert status == 0
    assert torch.equal(out.view(torch.int16), want_out.view(torch.int16))
    assert torch.equal(lse, want_lse)

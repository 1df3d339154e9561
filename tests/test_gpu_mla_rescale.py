"""MLA attention whose scores climb steeply from round to round, so that every round of the
fused kernel moves its heads' reference maxima and rescales the output accumulator (held in
tensor memory): random keys almost never exercise that step.

The climb lives in the 64 rope dims, so that V (the latent 512 dims of the same rows) keeps
its O(1) values: request b's query heads share a rope direction u_b (plus noise), and the rope
part of its logical page j's keys is beta_j * u_b (plus noise), beta_j climbing over the last
pages.  The top-k then selects those pages, and their maxima (base 2, sm_scale * log2 e) grow
by more than the kernel's reference threshold (8) between consecutive rounds of four pages.
Selection, output and lse are checked against the oracle as in every parity test.
"""
import math

import pytest
import torch

import paged_block_sparse_vt_b200 as vt
from paged_block_sparse_vt_b200.workloads import config, make_workload
from parity import all_full_pages, check_step, oracle_centroids, oracle_step, to_device

pytestmark = pytest.mark.gpu

CLIMB_PAGES = 40   # pages whose keys climb (covers the top-32 + the reserved last page)
STEP = 9.0         # beta per page
ROPE = 512         # first rope dim of the 576-dim rows


def _climbing_workload(Hq: int, seed: int):
    c = config(4, B=2, Hq=Hq, len_lo=3000, len_hi=3000, pool_pages=600)
    w = make_workload(c, poison=True, seed=seed)
    g = torch.Generator().manual_seed(seed + 1)
    k = w["k_pool"]
    for b in range(c.B):
        cvec = torch.randn(c.D - ROPE, generator=g)
        w["q"][b, :, ROPE:] = (cvec + 0.3 * torch.randn((c.Hq, c.D - ROPE), generator=g)).to(torch.bfloat16)
        u = cvec / cvec.norm()
        L = int(w["seq_lens"][b])
        n = (L + 15) // 16
        for j in range(n):
            beta = STEP * max(0, j - (n - CLIMB_PAGES))
            valid = min(16, L - 16 * j)
            phys = int(w["page_table"][b, j])
            rows = beta * u + 0.3 * torch.randn((valid, c.D - ROPE), generator=g)
            k[phys, :valid, 0, ROPE:] = rows.to(torch.bfloat16)  # NaN stays past the last token
    return w


def _round_growth(w, sel, n_sel):
    """Per request and head, the rise of the running base-2 maximum at each round of four
    selected pages (host fp32, from the keys as stored)."""
    c = w["config"]
    qs = c.sm_scale * math.log2(math.e)
    rises = []
    for b in range(c.B):
        L = int(w["seq_lens"][b])
        pages = [int(p) for p in sel[b, 0, : int(n_sel[b, 0])]]
        q = w["q"][b].float()  # [Hq, D]
        run = torch.full((c.Hq,), -math.inf)
        for r0 in range(0, len(pages), 4):
            m = torch.full((c.Hq,), -math.inf)
            for lp in pages[r0: r0 + 4]:
                valid = min(16, L - 16 * lp)
                kk = w["k_pool"][int(w["page_table"][b, lp]), :valid, 0, :].float()
                m = torch.maximum(m, (q @ kk.T).max(1).values * qs)
            if r0 > 0:
                rises.append((m - run).min().item())
            run = torch.maximum(run, m)
    return rises


@pytest.mark.parametrize("Hq", [32, 16])
def test_mla_rescale_every_round(Hq, oracle):
    w = _climbing_workload(Hq, seed=4100 + Hq)
    c = w["config"]
    d = to_device(w)
    cent_ref = oracle_centroids(oracle, w)
    ref = oracle_step(oracle, w, cent_ref)
    # the premise: most rounds raise every head's maximum by more than 8 (base 2)
    rises = _round_growth(w, ref["sel"], ref["n_sel"])
    assert sum(r > 8.0 for r in rises) >= len(rises) // 2, rises
    cent = torch.full((w["P"], c.Hkv, c.D), float("nan"), device="cuda")
    vt.vt_build_centroids(d["k_pool"], all_full_pages(d), cent)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    sel = torch.full((c.B, c.Hkv, c.kmax), -7, dtype=torch.int32, device="cuda")
    n_sel = torch.full((c.B, c.Hkv), -7, dtype=torch.int32, device="cuda")
    out, lse, _, _ = vt.vt_sparse_decode_fused(d["q"], d["k_pool"], d["v_pool"], d["page_table"],
                                               d["seq_lens"], cent, c.topk, c.bos, c.eos,
                                               c.sm_scale, sel=sel, n_sel=n_sel, status=st,
                                               head_dim_v=c.Dv)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    check_step(oracle, w, ref, cent_ref, sel, n_sel, out, lse,
               label=f"MLA climbing scores, G = {Hq}")

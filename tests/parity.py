"""Helpers for the GPU-vs-oracle parity tests: run both sides on the same seeded inputs.

Tolerances (from the target the method is built to):
  * centroids: |c_gpu - c_ref| <= 1e-5 |c_ref| + 1e-6 (fp32 storage of an fp64 mean);
  * selected pages: identical sets per (request, KV head), except a swap at the top-k
    boundary between pages whose oracle scores are within 1e-4 relative of the k-th score
    (relative to max(|s_i|, |s_k|, sum_d |qm_d c_id|): the fp32 GPU score error scales with
    the magnitude of the terms, not of the possibly cancelling sum);
  * attention output: max-abs error <= 1e-2 (bf16 output of an fp32 accumulation);
  * lse: abs error <= 1e-3.
"""
from __future__ import annotations

import torch

CENTROID_RTOL, CENTROID_ATOL = 1e-5, 1e-6
SCORE_RTOL = 1e-4
OUT_ATOL = 1e-2
LSE_ATOL = 1e-3
PS = 16


def to_device(w: dict, device="cuda") -> dict:
    d = dict(w)
    for key in ("q", "k_pool", "page_table", "seq_lens", "prebuilt_pages", "fill_pages"):
        d[key] = w[key].to(device)
    d["v_pool"] = d["k_pool"] if w["v_pool"] is w["k_pool"] else w["v_pool"].to(device)
    return d


def all_full_pages(w: dict) -> torch.Tensor:
    return torch.cat([w["prebuilt_pages"], w["fill_pages"]]).to(torch.int32)


def oracle_centroids(oracle, w: dict) -> torch.Tensor:
    c = w["config"]
    cent = torch.full((w["P"], c.Hkv, c.D), float("nan"))
    oracle.build_centroids(w["k_pool"], all_full_pages(w), cent)
    return cent


def oracle_step(oracle, w: dict, cent: torch.Tensor, topk=None, bos=None, eos=None):
    """Oracle selection (with fp64 scores) and attention.  Returns a dict of host tensors."""
    c = w["config"]
    topk = c.topk if topk is None else topk
    bos = c.bos if bos is None else bos
    eos = c.eos if eos is None else eos
    sel, n_sel, scores = oracle.select_pages(w["q"], w["page_table"], w["seq_lens"], cent, topk, bos,
                                             eos, want_scores=True)
    out, lse = oracle.sparse_attention(w["q"], w["k_pool"], w["v_pool"], w["page_table"],
                                       w["seq_lens"], sel, n_sel, c.sm_scale, head_dim_v=c.Dv)
    return dict(sel=sel, n_sel=n_sel, scores=scores, out=out, lse=lse, topk=topk, bos=bos, eos=eos)


def check_centroids(gpu: torch.Tensor, ref: torch.Tensor, pages: torch.Tensor) -> None:
    g = gpu.cpu()[pages.long()].double()
    r = ref[pages.long()].double()
    assert torch.isfinite(r).all()
    err = (g - r).abs()
    bound = CENTROID_RTOL * r.abs() + CENTROID_ATOL
    bad = err > bound
    assert not bad.any(), f"{int(bad.sum())} centroid elements off, max err {err.max().item():.3g}"


def _sigma(w: dict, cent: torch.Tensor, b: int, h: int, i: int) -> float:
    """sum_d |qm_d c_{page(i),h,d}|: the magnitude scale of the fp32 score of page i."""
    c = w["config"]
    qm = w["q"][b, h * c.G:(h + 1) * c.G].double().mean(dim=0)
    p = int(w["page_table"][b, i])
    return float((qm * cent[p, h].double()).abs().sum())


def compare_selection(w: dict, ref: dict, cent: torch.Tensor, sel: torch.Tensor,
                      n_sel: torch.Tensor) -> torch.Tensor:
    """Assert GPU selection == oracle selection up to tolerated boundary swaps.

    Returns a bool [B, Hkv] mask of units whose selected set is identical.
    """
    c = w["config"]
    sel, n_sel = sel.cpu(), n_sel.cpu()
    same = torch.ones((c.B, c.Hkv), dtype=torch.bool)
    kmax = ref["topk"] + ref["bos"] + ref["eos"]
    for b in range(c.B):
        n = (int(w["seq_lens"][b]) + PS - 1) // PS
        for h in range(c.Hkv):
            assert int(n_sel[b, h]) == int(ref["n_sel"][b, h]), (b, h)
            got = sel[b, h, : n_sel[b, h]].tolist()
            want = ref["sel"][b, h, : ref["n_sel"][b, h]].tolist()
            assert got == sorted(set(got)), f"unit {(b, h)}: not ascending/unique: {got}"
            assert all(x == -1 for x in sel[b, h, int(n_sel[b, h]):kmax].tolist())
            if got == want:
                continue
            same[b, h] = False
            s = ref["scores"][b, h]
            chosen = [s[i].item() for i in want if ref["bos"] <= i < n - ref["eos"]]
            kth = min(chosen)
            for i in set(got) ^ set(want):
                assert ref["bos"] <= i < n - ref["eos"], f"unit {(b, h)}: reserved page {i} differs"
                si = s[i].item()
                tol = SCORE_RTOL * max(abs(si), abs(kth), _sigma(w, cent, b, h, i))
                assert abs(si - kth) <= tol, (
                    f"unit {(b, h)}: page {i} score {si!r} vs k-th {kth!r} (tol {tol:.3g})")
    return same


def compare_outputs(out: torch.Tensor, lse, ref: dict, mask=None, G: int = 1) -> float:
    """Max-abs check of out [B,Hq,Dv] (and lse) against the oracle, over units in mask."""
    o = out.cpu().double()
    r = ref["out"]
    if mask is not None:
        rows = mask.repeat_interleave(G, dim=1)  # [B, Hq]
        o, r = o[rows], r[rows]
    assert torch.isfinite(o).all()
    err = (o - r).abs().max().item() if o.numel() else 0.0
    assert err <= OUT_ATOL, f"max abs error {err:.4g} > {OUT_ATOL}"
    if lse is not None:
        lg, lr = lse.cpu().double(), ref["lse"]
        if mask is not None:
            lg, lr = lg[rows], lr[rows]
        lerr = (lg - lr).abs().max().item() if lg.numel() else 0.0
        assert lerr <= LSE_ATOL, f"lse max abs error {lerr:.4g}"
    return err

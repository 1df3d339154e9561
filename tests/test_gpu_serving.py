"""A serving-shaped decode pass: L layers, each one vt_sparse_decode_step launch (the centroid
build of the pages that filled at this step, then select + attend), the first layer dense
(every page attended: the README's vortex_layers_skip of layer 0, read as a top-k that covers
every candidate), captured as ONE CUDA graph and replayed twice, as a serving engine replays its
captured decode step.  Every layer's output, lse and selection are checked against the oracle
for that layer's inputs (its own query, its own K/V pool and centroid cache)."""
import pytest
import torch

import paged_block_sparse_vt_b200 as vt
from paged_block_sparse_vt_b200.workloads import config, make_workload
from parity import check_centroids, check_step, oracle_centroids, oracle_step, to_device

pytestmark = pytest.mark.gpu

LAYERS = 4


def test_layered_pass_in_one_graph_matches_the_oracle_per_layer(oracle):
    base = config(2, B=5, len_lo=900, len_hi=6000, pool_pages=3000, filled=2)
    dense_topk = 400  # >= every request's candidates: every page is attended
    layers = []
    for l in range(LAYERS):
        w = make_workload(base, seed=4242 + l, poison=True)  # own q, pool, page placement
        c = w["config"]
        d = to_device(w)
        topk = dense_topk if l == 0 else c.topk
        d["topk"] = topk
        d["cent"] = torch.full((w["P"], c.Hkv, c.D), float("nan"), device="cuda")
        vt.vt_build_centroids(d["k_pool"], d["prebuilt_pages"], d["cent"])
        kmax = topk + c.bos + c.eos
        d["out"] = torch.empty((c.B, c.Hq, c.Dv), dtype=torch.bfloat16, device="cuda")
        d["lse"] = torch.empty((c.B, c.Hq), dtype=torch.float32, device="cuda")
        d["sel"] = torch.empty((c.B, c.Hkv, kmax), dtype=torch.int32, device="cuda")
        d["n_sel"] = torch.empty((c.B, c.Hkv), dtype=torch.int32, device="cuda")
        d["status"] = torch.zeros(1, dtype=torch.int32, device="cuda")
        d["ws"] = vt.fused_workspace(d["q"], d["k_pool"], d["v_pool"], d["page_table"],
                                     d["seq_lens"], d["cent"], topk, c.bos, c.eos)
        layers.append((w, d))
    torch.cuda.synchronize()

    def pass_():
        for w, d in layers:
            c = w["config"]
            vt.vt_sparse_decode_step(d["q"], d["k_pool"], d["v_pool"], d["page_table"],
                                     d["seq_lens"], d["cent"], d["topk"], c.bos, c.eos,
                                     c.sm_scale, d["fill_pages"], out=d["out"], lse=d["lse"],
                                     sel=d["sel"], n_sel=d["n_sel"], status=d["status"],
                                     workspace=d["ws"])

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        pass_()
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    for l, (w, d) in enumerate(layers):
        c = w["config"]
        assert int(d["status"].item()) == 0, l
        cent_ref = oracle_centroids(oracle, w)
        check_centroids(d["cent"], cent_ref,
                        torch.cat([w["prebuilt_pages"], w["fill_pages"]]).to(torch.int32))
        ref = oracle_step(oracle, w, cent_ref, topk=d["topk"])
        n = (w["seq_lens"].long() + 15) // 16
        if l == 0:
            assert torch.equal(d["n_sel"].cpu().long(), n[:, None].expand(c.B, c.Hkv))
        check_step(oracle, w, ref, cent_ref, d["sel"], d["n_sel"], d["out"], d["lse"],
                   label=f"layer {l} of a {LAYERS}-layer pass in one graph")

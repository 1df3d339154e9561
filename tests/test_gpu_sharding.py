"""Tensor parallelism by KV head on one GPU: the N shard calls of the Qwen3-0.6B-like decode
layer, run one after another (each with its own K/V head views, its own centroid cache built
from them and its own query heads, as N ranks would hold them), put back together, against
the unsharded call and the oracle.

Centroids and selections are bit-identical to the unsharded call (their arithmetic per
(page, head) and per unit does not depend on the launch).  The attention output is compared
with the oracle at the usual bound and with the unsharded call within bf16 rounding (out) and
the lse bound: how a unit's selected pages are split into attention pieces depends on how
many units the launch holds, and each piece rounds its probabilities to bf16 against its own
running maximum, so the partials differ in their last bits.
"""
import pytest
import torch

import paged_block_sparse_vt_b200 as vt
from paged_block_sparse_vt_b200.sharding import (gather_heads, kv_head_shard, shard_pool,
                                                 shard_queries)
from paged_block_sparse_vt_b200.workloads import config, make_workload
from parity import all_full_pages, check_step, oracle_centroids, oracle_step, to_device

pytestmark = pytest.mark.gpu


def _call(q, k, v, d, c, pages):
    cent = torch.full((d["P"], k.shape[2], c.D), float("nan"), device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    vt.vt_build_centroids(k, pages, cent, status=st)
    hkv = k.shape[2]
    sel = torch.empty((c.B, hkv, c.kmax), dtype=torch.int32, device="cuda")
    n_sel = torch.empty((c.B, hkv), dtype=torch.int32, device="cuda")
    args = (q, k, v, d["page_table"], d["seq_lens"], cent, c.topk, c.bos, c.eos)
    ws = vt.fused_workspace(*args)
    out, lse, _, _ = vt.vt_sparse_decode_fused(*args, c.sm_scale, sel=sel, n_sel=n_sel, status=st,
                                               workspace=ws)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return cent, sel, n_sel, out, lse


@pytest.mark.parametrize("world", [2, 4, 8])
def test_kv_head_shards_equal_the_unsharded_call(world, oracle):
    c = config(2)
    w = make_workload(c, poison=True)
    d = to_device(w)
    pages = all_full_pages(d)
    full = _call(d["q"], d["k_pool"], d["v_pool"], d, c, pages)
    parts = []
    for r in range(world):
        s = kv_head_shard(c.Hq, c.Hkv, world, r)
        parts.append(_call(shard_queries(d["q"], s), shard_pool(d["k_pool"], s),
                           shard_pool(d["v_pool"], s), d, c, pages))
    cent, sel, n_sel, out, lse = (gather_heads([p[i] for p in parts]) for i in range(5))
    rows = pages.long()
    assert torch.equal(cent[rows], full[0][rows])
    assert torch.equal(sel, full[1]) and torch.equal(n_sel, full[2])
    diff = (out.float() - full[3].float()).abs().max().item()
    assert diff <= 2 ** -7 * max(1.0, full[3].float().abs().max().item()), diff
    assert (lse - full[4]).abs().max().item() <= 1e-3
    cent_ref = oracle_centroids(oracle, w)
    ref = oracle_step(oracle, w, cent_ref)
    check_step(oracle, w, ref, cent_ref, sel, n_sel, out, lse, label=f"TP by KV head, {world} shards")

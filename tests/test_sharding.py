"""Tensor parallelism by KV head, on the CPU: the head partition, and two gloo ranks that each
run the oracle on their shard (their own K/V heads, their own centroid cache built from
them, their own query heads) and gather the results, which must equal the unsharded oracle
step bit for bit -- the method has no exchange between KV heads."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from paged_block_sparse_vt_b200.sharding import (gather_heads, kv_head_shard, shard_centroids,
                                                 shard_pool, shard_queries)
from paged_block_sparse_vt_b200.workloads import config, make_workload

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("hq,hkv,world", [(16, 8, 1), (16, 8, 2), (16, 8, 4), (16, 8, 8),
                                          (48, 8, 4), (4, 2, 2)])
def test_partition_covers_every_head_once(hq, hkv, world):
    shards = [kv_head_shard(hq, hkv, world, r) for r in range(world)]
    kv = [h for s in shards for h in range(s.kv0, s.kv1)]
    qh = [h for s in shards for h in range(s.q0, s.q1)]
    assert kv == list(range(hkv)) and qh == list(range(hq))
    G = hq // hkv
    for s in shards:  # each shard's query heads are exactly the groups of its KV heads
        assert s.q0 == s.kv0 * G and s.q1 == s.kv1 * G
        assert s.num_q_heads == G * s.num_kv_heads


def test_partition_rejects_uneven_splits():
    with pytest.raises(ValueError):
        kv_head_shard(16, 8, 3, 0)
    with pytest.raises(ValueError):
        kv_head_shard(32, 1, 2, 0)  # the MLA latent form: one KV head, shard by request
    with pytest.raises(ValueError):
        kv_head_shard(16, 8, 2, 2)


def _shard_step(oracle, w, s):
    """The oracle step of one shard, from the shard's own tensors only."""
    c = w["config"]
    k, v = shard_pool(w["k_pool"], s), shard_pool(w["v_pool"], s)
    q = shard_queries(w["q"], s)
    cent = torch.full((w["P"], s.num_kv_heads, c.D), float("nan"))
    oracle.build_centroids(k, torch.cat([w["prebuilt_pages"], w["fill_pages"]]).to(torch.int32),
                           cent)
    sel, n_sel, out, lse = oracle.decode_step(q, k, v, w["page_table"], w["seq_lens"], cent,
                                              c.topk, c.bos, c.eos, c.sm_scale)
    return cent, sel, n_sel, out, lse


def _full_step(oracle, w):
    c = w["config"]
    s = kv_head_shard(c.Hq, c.Hkv, 1, 0)
    return _shard_step(oracle, w, s)


WORKLOAD = dict(cfg=2, B=3, len_lo=700, len_hi=3000, pool_pages=800)


def _workload():
    kw = dict(WORKLOAD)
    return make_workload(config(kw.pop("cfg"), **kw))


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        w = _workload()
        c = w["config"]
        s = kv_head_shard(c.Hq, c.Hkv, world, rank)
        parts = _shard_step(oracle, w, s)
        gathered = []
        for t in parts:
            buf = [torch.empty_like(t) for _ in range(world)]
            dist.all_gather(buf, t.contiguous())
            gathered.append(buf)
        if rank == 0:
            q.put([gather_heads(g) for g in gathered])
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_equal_the_unsharded_step(oracle):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want = _full_step(oracle, _workload())
    for got, ref in zip(res, want):
        assert torch.equal(got.nan_to_num(7.0), ref.nan_to_num(7.0))


def test_four_shards_in_one_process_equal_the_unsharded_step(oracle):
    w = _workload()
    c = w["config"]
    parts = [_shard_step(oracle, w, kv_head_shard(c.Hq, c.Hkv, 4, r)) for r in range(4)]
    want = _full_step(oracle, w)
    for i, ref in enumerate(want):
        got = gather_heads([p[i] for p in parts])
        assert torch.equal(got.nan_to_num(7.0), ref.nan_to_num(7.0))

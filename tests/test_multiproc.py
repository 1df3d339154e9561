"""The N > 1 host path of bench.py on CPU: two gloo ranks, no GPU.

Every rank runs its own batch (no collective on the data path); the only cross-rank steps are
the barriers around the timed region and the max-over-ranks of the elapsed time.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        bench.barrier(world)
        elapsed = [0.25, 0.40][rank]            # rank 1 is the slow one
        t = bench.max_over_ranks(elapsed, world, "cpu")
        value = bench.aggregate_value(world, 32 * 16, 10, t)
        bench.barrier(world)
        q.put((rank, t, value))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, t, value in res:
        assert t == pytest.approx(0.40)
        assert value == pytest.approx(2 * 32 * 16 * 10 / 0.40)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(1.5, 1, "cpu") == 1.5
    assert bench.aggregate_value(1, 512, 4, 2.0) == 1024.0


def test_algorithmic_bytes_formula_by_hand():
    """Two requests, hand-counted bytes (B=2, Hq=4, Hkv=2, D=Dv=8, top-2+1+1)."""
    sys.path.insert(0, ROOT)
    import bench
    from paged_block_sparse_vt_b200.workloads import config
    c = config(2, B=2, Hq=4, Hkv=2, D=8, Dv=8, topk=2, bos=1, eos=1)
    L = torch.tensor([100, 48], dtype=torch.int32)  # n = 7 (sparse, last page 4 tokens), 3 (dense)
    nb = bench.algorithmic_bytes(c, L)
    q_out_lse = 2 * (2 * 4 * 8 + 2 * 4 * 8 + 4 * 4)
    pt = 4 * (7 + 3)
    cent = 2 * 4 * 8 * (7 - 2)                     # 5 candidates, both KV heads
    kv_tokens = (16 * 3 + 4) + (16 * 2 + 16)       # 4 selected pages (last partial); 3 pages
    kv = 2 * 2 * (8 + 8) * kv_tokens
    assert nb["fused"] == q_out_lse + pt + cent + kv
    assert nb["build"] == 1 * (16 * 2 * 8 * 2 + 2 * 8 * 4 + 4)   # request 1 ends on a boundary


def test_split_call_bytes_by_hand():
    """select-only and decode-only algorithmic bytes, hand-counted (B=2, Hq=4, Hkv=2, D=Dv=8,
    top-2+1+1: request 0 has 7 pages, the last with 4 tokens, request 1 has 3 full pages)."""
    sys.path.insert(0, ROOT)
    import bench
    from paged_block_sparse_vt_b200.workloads import config
    c = config(2, B=2, Hq=4, Hkv=2, D=8, Dv=8, topk=2, bos=1, eos=1)
    L = torch.tensor([100, 48], dtype=torch.int32)
    vb = bench.variant_bytes(c, L)
    q = 2 * 4 * 8 * 2                     # bf16 q of both requests
    sel = 4 * 2 * 2 * (4 + 1)             # sel rows (kmax = 4) and n_sel, int32
    select = q + 4 * (7 + 3) + 2 * 4 * 8 * 5 + sel   # page tables; 5 candidates x 2 heads, fp32
    assert vb["select"] == select
    # decode: q, bf16 out, fp32 lse, sel; per head one page-table entry per selected page and
    # the K and V rows of 4 pages (52 tokens) and of 3 pages (48 tokens)
    decode = q + 2 * 4 * 8 * 2 + 4 * 4 * 2 + sel + 2 * (4 * (4 + 3) + 2 * (8 + 8) * (52 + 48))
    assert vb["decode"] == decode


def test_mla_decode_bytes_read_v_once():
    """MLA: V is the first Dv dims of the K row, so a selected token costs its 576-dim row
    once (B=1, Hq=16, one KV head, top-1+1+1, 40 tokens over 3 pages)."""
    sys.path.insert(0, ROOT)
    import bench
    from paged_block_sparse_vt_b200.workloads import config
    c = config(4, B=1, Hq=16, topk=1, bos=1, eos=1)
    L = torch.tensor([40], dtype=torch.int32)      # 3 pages, the last with 8 tokens: dense
    vb = bench.variant_bytes(c, L)
    q = 2 * 16 * 576
    sel = 4 * 1 * 1 * (3 + 1)
    decode = q + 2 * 16 * 512 + 4 * 16 + sel + (4 * 3 + 2 * 576 * (16 + 16 + 8))
    assert vb["decode"] == decode

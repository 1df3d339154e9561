"""The seeded input generator: determinism, shapes and the per-config recipes."""
import torch

from paged_block_sparse_vt_b200.workloads import PAGE_SIZE, config, make_workload


def _bits(t):
    return t.view(torch.int16)


def test_deterministic_and_seed_sensitive():
    a = make_workload(1)
    b = make_workload(1)
    c = make_workload(1, seed=77)
    for key in ("q", "k_pool", "v_pool", "page_table", "seq_lens"):
        x, y = a[key], b[key]
        if x.dtype == torch.bfloat16:
            x, y = _bits(x), _bits(y)
        assert torch.equal(x, y)
    assert not torch.equal(_bits(a["k_pool"]), _bits(c["k_pool"]))


def test_config1_shapes():
    w = make_workload(1)
    c = w["config"]
    assert w["q"].shape == (1, 2, 64) and w["k_pool"].shape == (128, PAGE_SIZE, 1, 64)
    assert w["seq_lens"].tolist() == [1024] and w["page_table"].shape == (1, 64)
    assert len(set(w["page_table"][0].tolist())) == 64
    assert c.kmax == 6


def test_page_tables_are_injective_and_in_range():
    c = config(5, B=40, len_lo=16, len_hi=4000, filled=3)
    w = make_workload(c)
    L = w["seq_lens"]
    n = (L + PAGE_SIZE - 1) // PAGE_SIZE
    used = torch.cat([w["page_table"][b, : int(n[b])] for b in range(c.B)])
    assert used.unique().numel() == used.numel()
    assert int(used.min()) >= 0 and int(used.max()) < w["P"]
    assert w["P"] == int(torch.ceil(torch.tensor(1.25 * int(n.sum()))))


def test_config5_fill_recipe():
    c = config(5, B=64, filled=4)
    w = make_workload(c)
    L = w["seq_lens"]
    assert int((L % PAGE_SIZE == 0).sum()) == 4
    assert w["fill_pages"].numel() == 4
    assert int(L.min()) >= 511 and int(L.max()) <= 65536
    n = (L + PAGE_SIZE - 1) // PAGE_SIZE
    last = {int(w["page_table"][b, int(n[b]) - 1]) for b in range(c.B) if int(L[b]) % PAGE_SIZE == 0}
    assert set(w["fill_pages"].tolist()) == last
    assert not (set(w["prebuilt_pages"].tolist()) & last)


def test_poison_marks_unused_pages_and_tails():
    c = config(2, B=3, len_lo=100, len_hi=300, pool_pages=80)
    w = make_workload(c, poison=True)
    L = w["seq_lens"]
    n = (L + PAGE_SIZE - 1) // PAGE_SIZE
    used = set()
    for b in range(c.B):
        used |= set(w["page_table"][b, : int(n[b])].tolist())
        last = int(w["page_table"][b, int(n[b]) - 1])
        valid = int(L[b]) - PAGE_SIZE * (int(n[b]) - 1)
        assert torch.isfinite(w["k_pool"][last, :valid].float()).all()
        assert torch.isnan(w["k_pool"][last, valid:].float()).all()
    unused = [p for p in range(w["P"]) if p not in used]
    assert unused and torch.isnan(w["k_pool"][unused].float()).all()
    assert torch.isnan(w["v_pool"][unused].float()).all()


def test_mla_shares_one_pool():
    w = make_workload(config(4, B=2, len_lo=64, len_hi=64, pool_pages=10))
    assert w["v_pool"] is w["k_pool"] and w["k_pool"].shape[-1] == 576


def test_page_offsets_shift_page_means():
    """Config 2 adds an N(0, 0.5^2) vector per (page, head): page means spread ~0.5."""
    w = make_workload(config(2, B=2, len_lo=2000, len_hi=2000, pool_pages=400))
    means = w["k_pool"].float().mean(dim=1)          # [P, H, D]
    std = means.std().item()
    assert 0.45 < std < 0.62  # sqrt(0.25 + 1/16) ~= 0.56

"""Pins for the CPU oracle against facts fixed by the method's definition and by mathematics.

Nothing here compares the oracle with itself: each test checks it against a
hand-worked example, a closed form, a brute-force enumeration, an independent
library routine (torch fp64 softmax over the gathered sequence), or an invariant
that the method guarantees.  Each is chosen so that a plausible slip in the
oracle (a dropped term, a wrong index, a transposed operand, a wrong tie rule)
fails at least one of them.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from dense_ref import dense_attention, gather_sequence

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
PS = 16


def _bf16(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16)


def _pool_from_rows(rows_by_page, page_table, P, poison_tail_of=None, valid_last=None):
    """Pool [P,16,1,D] whose logical page i holds rows_by_page[i] in every token slot."""
    D = len(rows_by_page[0])
    pool = torch.full((P, PS, 1, D), float("nan"), dtype=torch.bfloat16)
    for i, row in enumerate(rows_by_page):
        pool[page_table[i], :, 0, :] = _bf16(row)
    if poison_tail_of is not None:
        pool[page_table[poison_tail_of], valid_last:, 0, :] = float("nan")
    return pool


# --------------------------------------------------------------------------------------
# the hand-worked example (tests/golden/worked_example_tiny.json)
# --------------------------------------------------------------------------------------

def test_golden_fixture_closed_forms_are_consistent():
    fx = json.load(open(os.path.join(GOLDEN, "worked_example_tiny.json")))
    e = math.e
    want = [[18 / (18 + 16 * e), (16 * e + 2) / (18 + 16 * e)],
            [18 / (18 + 16 * e ** 2), (16 * e ** 2 + 2) / (18 + 16 * e ** 2)]]
    assert np.allclose(fx["expected_out"], want, rtol=0, atol=1e-15)
    assert np.allclose(fx["expected_lse"], [math.log(18 + 16 * e), math.log(18 + 16 * e * e)])


def test_golden_worked_example(oracle):
    fx = json.load(open(os.path.join(GOLDEN, "worked_example_tiny.json")))
    pt = fx["page_table"]
    L = fx["seq_len"]
    n = (L + PS - 1) // PS
    valid_last = L - PS * (n - 1)
    k_pool = _pool_from_rows(fx["k_rows_by_logical_page"], pt, fx["num_pages"], n - 1, valid_last)
    v_pool = _pool_from_rows(fx["v_rows_by_logical_page"], pt, fx["num_pages"], n - 1, valid_last)
    q = _bf16(fx["q"]).view(1, 2, 2).contiguous()
    page_table = torch.tensor([pt], dtype=torch.int32)
    seq_lens = torch.tensor([L], dtype=torch.int32)

    cent = torch.full((fx["num_pages"], 1, 2), float("nan"), dtype=torch.float32)
    oracle.build_centroids(k_pool, torch.tensor(pt[: n - 1], dtype=torch.int32), cent)
    for i, row in enumerate(fx["expected_centroids_by_logical_page"]):
        assert cent[pt[i], 0].tolist() == row

    sel, n_sel, scores = oracle.select_pages(q, page_table, seq_lens, cent, fx["topk"], fx["bos"],
                                             fx["eos"], want_scores=True)
    for i, s in fx["expected_scores"].items():
        assert scores[0, 0, int(i)].item() == s
    assert n_sel[0, 0].item() == len(fx["expected_selection"])
    assert sel[0, 0, : n_sel[0, 0]].tolist() == fx["expected_selection"]

    out, lse = oracle.sparse_attention(q, k_pool, v_pool, page_table, seq_lens, sel, n_sel,
                                       fx["sm_scale"])
    assert np.allclose(out[0].numpy(), fx["expected_out"], rtol=0, atol=1e-14)
    assert np.allclose(lse[0].numpy(), fx["expected_lse"], rtol=0, atol=1e-13)


# --------------------------------------------------------------------------------------
# centroids (CMean over the tokens of a finished page)
# --------------------------------------------------------------------------------------

def test_centroid_of_constant_page_is_its_row(oracle):
    g = torch.Generator().manual_seed(1)
    P, H, D = 6, 3, 32
    rows = torch.randn(P, H, D, generator=g).to(torch.bfloat16)
    pool = rows.unsqueeze(1).expand(P, PS, H, D).contiguous()
    cent = torch.full((P, H, D), float("nan"))
    oracle.build_centroids(pool, torch.arange(P, dtype=torch.int32), cent)
    assert torch.equal(cent, rows.float())


def test_centroid_is_exact_mean_rounded_once(oracle):
    """16 bf16 values sum exactly in rationals; the centroid is that mean rounded once to fp32."""
    g = torch.Generator().manual_seed(2)
    P, H, D = 4, 2, 16
    pool = (3.0 * torch.randn(P, PS, H, D, generator=g)).to(torch.bfloat16)
    cent = torch.zeros(P, H, D)
    oracle.build_centroids(pool, torch.arange(P, dtype=torch.int32), cent)
    vals = pool.float()  # torch's own bf16 -> fp32 widening (exact)
    for p in range(P):
        for h in range(H):
            for d in range(D):
                exact = sum(Fraction(float(vals[p, t, h, d])) for t in range(PS)) / PS
                f = float(exact)
                assert Fraction(f) == exact  # the mean is a dyadic rational with < 53 bits here
                assert cent[p, h, d].item() == float(np.float32(f))


def test_centroid_total_equals_pool_total(oracle):
    """sum over pages of 16*c equals the sum of every K element (linearity of the mean)."""
    g = torch.Generator().manual_seed(3)
    P, H, D = 40, 4, 64
    pool = torch.randn(P, PS, H, D, generator=g).to(torch.bfloat16)
    cent = torch.zeros(P, H, D)
    oracle.build_centroids(pool, torch.arange(P, dtype=torch.int32), cent)
    lhs = (PS * cent.double()).sum(dim=0)
    rhs = pool.double().sum(dim=(0, 1))
    # each centroid carries one fp32 rounding: |err| <= 16 * 2^-24 * |c| per element
    bound = (PS * cent.double().abs() * 2.0 ** -24).sum(dim=0) + 1e-12
    assert torch.all((lhs - rhs).abs() <= bound)


def test_centroid_pages_and_heads_not_transposed(oracle):
    """Page p, head h gets a value only its own slab can produce."""
    P, H, D = 5, 3, 8
    pool = torch.zeros(P, PS, H, D)
    for p in range(P):
        for h in range(H):
            pool[p, :, h, :] = 10 * p + h
        pool[p, 0, :, :] += 16.0  # token 0 differs: mean shifts by exactly 1
    pool = pool.to(torch.bfloat16)
    cent = torch.full((P, H, D), float("nan"))
    oracle.build_centroids(pool, torch.tensor([4, 1], dtype=torch.int32), cent)
    for p in (1, 4):
        for h in range(H):
            assert torch.all(cent[p, h] == 10 * p + h + 1)
    assert torch.isnan(cent[[0, 2, 3]]).all()  # unlisted pages untouched


def test_centroid_strided_pool(oracle):
    g = torch.Generator().manual_seed(4)
    P, H, D = 7, 2, 32
    big = torch.randn(P, PS + 3, H + 1, D + 8, generator=g).to(torch.bfloat16)
    view = big[:, :PS, :H, :D]
    cent_a = torch.zeros(P, H, D)
    cent_b = torch.zeros(P, H, D)
    oracle.build_centroids(view, torch.arange(P, dtype=torch.int32), cent_a)
    oracle.build_centroids(view.contiguous(), torch.arange(P, dtype=torch.int32), cent_b)
    assert torch.equal(cent_a, cent_b)
    assert torch.allclose(cent_a.double(), view.double().mean(dim=1), rtol=1e-6, atol=1e-7)


def test_centroid_rejects_bad_page(oracle):
    pool = torch.zeros(3, PS, 1, 8, dtype=torch.bfloat16)
    cent = torch.zeros(3, 1, 8)
    with pytest.raises(oracle.OracleError):
        oracle.build_centroids(pool, torch.tensor([3], dtype=torch.int32), cent)


# --------------------------------------------------------------------------------------
# indexer: group mean -> GeMV -> topK + reserved pages
# --------------------------------------------------------------------------------------

def _identity_batch(n_pages, D=4, H=1):
    pt = torch.arange(n_pages, dtype=torch.int32).view(1, -1)
    return pt, torch.tensor([n_pages * PS], dtype=torch.int32)


def test_scores_read_off_the_centroid_table(oracle):
    """q heads (e0, e0) -> mean e0 -> s_i = c_i[0]; (e0, 2e1 - e0) -> mean e1 -> s_i = c_i[1]."""
    n = 10
    g = torch.Generator().manual_seed(5)
    cent = torch.randn(n, 1, 4, generator=g)
    pt, L = _identity_batch(n)
    for qrows, col in (([[1, 0, 0, 0], [1, 0, 0, 0]], 0), ([[1, 0, 0, 0], [-1, 2, 0, 0]], 1)):
        q = _bf16(qrows).view(1, 2, 4).contiguous()
        _, _, s = oracle.select_pages(q, pt, L, cent, 3, 1, 1, want_scores=True)
        for i in range(1, n - 1):
            assert s[0, 0, i].item() == float(cent[i, 0, col])
        assert math.isnan(s[0, 0, 0]) and math.isnan(s[0, 0, n - 1])  # reserved: not scored


def test_query_mean_is_per_kv_head_group(oracle):
    """Hkv=2, G=2: each KV head ranks pages by the mean of its own two query heads."""
    n = 12
    cent = torch.zeros(n, 2, 2)
    cent[:, 0, 0] = torch.arange(n, dtype=torch.float32)        # head 0 prefers late pages
    cent[:, 1, 1] = -torch.arange(n, dtype=torch.float32)       # head 1 prefers early pages
    pt, L = _identity_batch(n)
    q = _bf16([[1, 0], [1, 0], [0, 1], [0, 1]]).view(1, 4, 2).contiguous()
    sel, n_sel = oracle.select_pages(q, pt, L, cent, 3, 1, 1)
    assert sel[0, 0].tolist() == [0, 8, 9, 10, 11]
    assert sel[0, 1].tolist() == [0, 1, 2, 3, 11]


def test_topk_equals_best_subset_by_enumeration(oracle):
    """With distinct scores the top-k set is the unique k-subset of candidates with maximal sum."""
    g = torch.Generator().manual_seed(6)
    for trial in range(20):
        n = int(torch.randint(6, 13, (1,), generator=g))
        k = int(torch.randint(1, 4, (1,), generator=g))
        bos, eos = int(torch.randint(0, 3, (1,), generator=g)), int(torch.randint(0, 3, (1,), generator=g))
        if n <= k + bos + eos:
            continue
        D, G = 8, 2
        cent = torch.randn(n, 1, D, generator=g)
        q = torch.randn(1, G, D, generator=g).to(torch.bfloat16)
        L = torch.tensor([n * PS - int(torch.randint(0, PS, (1,), generator=g))], dtype=torch.int32)
        pt = torch.randperm(n, generator=g).to(torch.int32).view(1, -1)
        sel, n_sel = oracle.select_pages(q, pt, L, cent, k, bos, eos)
        # independent score: numpy fp64 (qm . c) for each middle page
        qm = q[0].double().numpy().mean(axis=0)
        s = {i: float(np.dot(qm, cent[int(pt[0, i]), 0].double().numpy())) for i in range(bos, n - eos)}
        best = max(itertools.combinations(sorted(s), k), key=lambda sub: sum(s[i] for i in sub))
        want = sorted(set(range(bos)) | set(range(n - eos, n)) | set(best))
        assert sel[0, 0, : n_sel[0, 0]].tolist() == want


def test_equal_scores_break_toward_lower_index(oracle):
    n = 20
    cent = torch.ones(n, 1, 4)
    cent[[5, 9, 13], 0, :] = 2.0            # three clear winners
    pt, L = _identity_batch(n)
    q = _bf16([[1, 1, 1, 1]]).view(1, 1, 4).contiguous()
    sel, n_sel = oracle.select_pages(q, pt, L, cent, 6, 2, 1)
    # winners 5, 9, 13, then the three lowest-index ties among the middle pages [2, 19)
    assert sel[0, 0].tolist() == [0, 1, 2, 3, 4, 5, 9, 13, 19]


def test_dense_rule_and_k_zero(oracle):
    cent = torch.randn(8, 1, 4, generator=torch.Generator().manual_seed(7))
    q = _bf16([[1, 2, 3, 4]]).view(1, 1, 4).contiguous()
    pt = torch.arange(8, dtype=torch.int32).view(1, -1)
    # n = 5 <= k+bos+eos = 5: every page, then -1 padding
    sel, n_sel = oracle.select_pages(q, pt, torch.tensor([70], dtype=torch.int32), cent, 3, 1, 1)
    assert n_sel.item() == 5 and sel[0, 0].tolist() == [0, 1, 2, 3, 4]
    # n = 8 > 4 and k = 0: only the reserved pages
    sel, n_sel = oracle.select_pages(q, pt, torch.tensor([128], dtype=torch.int32), cent, 0, 2, 2)
    assert n_sel.item() == 4 and sel[0, 0].tolist() == [0, 1, 6, 7]
    # a single token: one page, attended densely
    sel, n_sel = oracle.select_pages(q, pt, torch.tensor([1], dtype=torch.int32), cent, 2, 1, 1)
    assert n_sel.item() == 1 and sel[0, 0].tolist() == [0, -1, -1, -1]


def test_selection_invariants_random(oracle):
    from paged_block_sparse_vt_b200.workloads import make_workload, config
    c = config(5, B=24, len_lo=40, len_hi=3000, filled=2)
    w = make_workload(c)
    cent = torch.full((w["P"], c.Hkv, c.D), float("nan"))
    oracle.build_centroids(w["k_pool"], torch.cat([w["prebuilt_pages"], w["fill_pages"]]), cent)
    sel, n_sel, s = oracle.select_pages(w["q"], w["page_table"], w["seq_lens"], cent, c.topk, c.bos,
                                        c.eos, want_scores=True)
    for b in range(c.B):
        n = (int(w["seq_lens"][b]) + PS - 1) // PS
        for h in range(c.Hkv):
            got = sel[b, h, : n_sel[b, h]].tolist()
            assert got == sorted(set(got)) and all(0 <= i < n for i in got)
            assert all(x == -1 for x in sel[b, h, n_sel[b, h]:].tolist())
            assert n_sel[b, h] == min(n, c.kmax)
            if n > c.kmax:
                assert set(range(c.bos)) | set(range(n - c.eos, n)) <= set(got)
                cand = range(c.bos, n - c.eos)
                chosen = [s[b, h, i].item() for i in cand if i in got]
                rest = [s[b, h, i].item() for i in cand if i not in got]
                assert len(chosen) == c.topk and min(chosen) >= max(rest)


def test_mla_score_is_latent_plus_rope(oracle):
    """Rope-aware scoring q_lat.c_lat + q_rope.c_rope equals the score on the 576-d row."""
    g = torch.Generator().manual_seed(8)
    n, Hq = 40, 8
    pool = torch.randn(n, PS, 1, 576, generator=g).to(torch.bfloat16)
    q = torch.randn(1, Hq, 576, generator=g).to(torch.bfloat16)
    cent = torch.zeros(n, 1, 576)
    oracle.build_centroids(pool, torch.arange(n, dtype=torch.int32), cent)
    pt, L = _identity_batch(n)
    _, _, s = oracle.select_pages(q, pt, L, cent, 8, 1, 1, want_scores=True)
    qm = q[0].double().mean(dim=0)
    c_lat = pool[:, :, 0, :512].double().mean(dim=1)   # page means of each part, separately
    c_rope = pool[:, :, 0, 512:].double().mean(dim=1)
    want = c_lat @ qm[:512] + c_rope @ qm[512:]
    for i in range(1, n - 1):
        assert abs(s[0, 0, i].item() - want[i].item()) <= 1e-6 * (1 + abs(want[i].item()))


def test_select_errors(oracle):
    cent = torch.zeros(4, 1, 4)
    q = torch.zeros(1, 1, 4, dtype=torch.bfloat16)
    pt = torch.arange(4, dtype=torch.int32).view(1, -1)
    with pytest.raises(oracle.OracleError):
        oracle.select_pages(q, pt, torch.tensor([0], dtype=torch.int32), cent, 1, 1, 1)
    with pytest.raises(oracle.OracleError):
        oracle.select_pages(q, pt, torch.tensor([65], dtype=torch.int32), cent, 1, 1, 1)
    with pytest.raises(oracle.OracleError):
        oracle.select_pages(q, torch.tensor([[0, 1, 9, 2]], dtype=torch.int32),
                            torch.tensor([64], dtype=torch.int32), cent, 1, 1, 1)


# --------------------------------------------------------------------------------------
# attention over the selected pages
# --------------------------------------------------------------------------------------

def test_attention_constant_keys_one_hot_values(oracle):
    """K = a_i e0 on page i, V = e_i: out[i] = w_i e^{s q0 a_i} / sum_j w_j e^{s q0 a_j}."""
    n, D, L = 6, 8, 6 * PS - 11
    a = [0.5, -1.0, 2.0, 0.25, 1.5, -0.75]
    last_valid = L - PS * (n - 1)
    pt = [3, 0, 5, 1, 4, 2]
    k_pool = _pool_from_rows([[ai] + [0] * (D - 1) for ai in a], pt, 7, n - 1, last_valid)
    v_pool = _pool_from_rows([[1.0 if d == i else 0.0 for d in range(D)] for i in range(n)], pt, 7,
                             n - 1, last_valid)
    q = _bf16([[1.5] + [0.0] * (D - 1)]).view(1, 1, D).contiguous()
    scale = 0.3
    page_table = torch.tensor([pt], dtype=torch.int32)
    seq = torch.tensor([L], dtype=torch.int32)
    sel = torch.tensor([[[0, 2, 3, 5]]], dtype=torch.int32)
    n_sel = torch.tensor([[4]], dtype=torch.int32)
    out, lse = oracle.sparse_attention(q, k_pool, v_pool, page_table, seq, sel, n_sel, scale)
    w = {i: (last_valid if i == n - 1 else PS) * math.exp(scale * 1.5 * a[i]) for i in (0, 2, 3, 5)}
    Z = sum(w.values())
    want = [w.get(i, 0.0) / Z for i in range(D)]
    assert np.allclose(out[0, 0].numpy(), want, rtol=0, atol=1e-15)
    assert abs(lse[0, 0].item() - math.log(Z)) < 1e-13


def test_attention_equal_keys_average_values(oracle):
    g = torch.Generator().manual_seed(9)
    n, D, L = 9, 16, 9 * PS - 5
    k_pool = torch.ones(n, PS, 1, D, dtype=torch.bfloat16)
    v_pool = torch.randn(n, PS, 1, D, generator=g).to(torch.bfloat16)
    q = torch.randn(1, 2, D, generator=g).to(torch.bfloat16)
    pt = torch.randperm(n, generator=g).to(torch.int32).view(1, -1)
    chosen = [0, 4, 8]
    sel = torch.tensor([[chosen]], dtype=torch.int32)
    out, _ = oracle.sparse_attention(q, k_pool, v_pool, pt, torch.tensor([L], dtype=torch.int32), sel,
                                     torch.tensor([[3]], dtype=torch.int32), 0.7)
    V = gather_sequence(v_pool, pt, 0, L).double()[:, 0]
    rows = [t for i in chosen for t in range(PS * i, min(L, PS * (i + 1)))]
    want = V[rows].mean(dim=0)
    assert torch.allclose(out[0, 0], want, rtol=0, atol=1e-14)
    assert torch.allclose(out[0, 1], want, rtol=0, atol=1e-14)


def test_all_pages_selected_equals_dense_attention(oracle):
    """k >= number of middle pages: the method is plain attention; compare with torch fp64."""
    from paged_block_sparse_vt_b200.workloads import make_workload, config
    c = config(2, B=5, len_lo=17, len_hi=700, pool_pages=300, topk=64)
    w = make_workload(c, poison=True)
    cent = torch.full((w["P"], c.Hkv, c.D), float("nan"))
    oracle.build_centroids(w["k_pool"], torch.cat([w["prebuilt_pages"], w["fill_pages"]]), cent)
    sel, n_sel, out, lse = oracle.decode_step(w["q"], w["k_pool"], w["v_pool"], w["page_table"],
                                              w["seq_lens"], cent, c.topk, c.bos, c.eos, c.sm_scale)
    ref_out, ref_lse = dense_attention(w["q"], w["k_pool"], w["v_pool"], w["page_table"],
                                       w["seq_lens"], c.sm_scale)
    assert torch.isfinite(out).all()
    assert torch.allclose(out, ref_out, rtol=0, atol=1e-12)
    assert torch.allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_sparse_output_equals_dense_over_selected_tokens(oracle):
    """A sparse selection gives plain attention restricted to the selected pages' tokens."""
    from paged_block_sparse_vt_b200.workloads import make_workload, config
    c = config(2, B=3, len_lo=900, len_hi=1500, pool_pages=400, topk=6)
    w = make_workload(c, poison=True)
    cent = torch.full((w["P"], c.Hkv, c.D), float("nan"))
    oracle.build_centroids(w["k_pool"], torch.cat([w["prebuilt_pages"], w["fill_pages"]]), cent)
    sel, n_sel, out, lse = oracle.decode_step(w["q"], w["k_pool"], w["v_pool"], w["page_table"],
                                              w["seq_lens"], cent, c.topk, c.bos, c.eos, c.sm_scale)
    for h in range(c.Hkv):
        pages = [sel[b, h, : n_sel[b, h]].tolist() for b in range(c.B)]
        ref, ref_lse = dense_attention(w["q"], w["k_pool"], w["v_pool"], w["page_table"],
                                       w["seq_lens"], c.sm_scale, pages=pages)
        hs = slice(h * c.G, (h + 1) * c.G)
        assert torch.allclose(out[:, hs], ref[:, hs], rtol=0, atol=1e-12)
        assert torch.allclose(lse[:, hs], ref_lse[:, hs], rtol=0, atol=1e-12)


def test_physical_placement_does_not_matter(oracle):
    """Same logical data under two pool permutations: identical selection, bit-identical output."""
    from paged_block_sparse_vt_b200.workloads import make_workload, config
    c = config(2, B=3, len_lo=600, len_hi=1400, pool_pages=320, topk=5)
    w = make_workload(c)
    P = w["P"]
    perm = torch.randperm(P, generator=torch.Generator().manual_seed(10))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(P)
    k2, v2 = torch.empty_like(w["k_pool"]), torch.empty_like(w["v_pool"])
    k2[perm], v2[perm] = w["k_pool"], w["v_pool"]          # page p moves to perm[p]
    pt2 = perm[w["page_table"].long()].to(torch.int32)
    res = []
    for kp, vp, pt in ((w["k_pool"], w["v_pool"], w["page_table"]), (k2, v2, pt2)):
        cent = torch.full((P, c.Hkv, c.D), float("nan"))
        n = (w["seq_lens"] + PS - 1) // PS
        full = torch.cat([pt[b, : int(n[b]) - 1] for b in range(c.B)])
        oracle.build_centroids(kp, full, cent)
        res.append(oracle.decode_step(w["q"], kp, vp, pt, w["seq_lens"], cent, c.topk, c.bos, c.eos,
                                      c.sm_scale))
    assert torch.equal(res[0][0], res[1][0]) and torch.equal(res[0][1], res[1][1])
    assert torch.equal(res[0][2], res[1][2]) and torch.equal(res[0][3], res[1][3])


def test_unused_slots_are_never_read(oracle):
    """NaN in every unused pool page and past each request's end leaves the output finite."""
    from paged_block_sparse_vt_b200.workloads import make_workload, config
    c = config(5, B=10, len_lo=20, len_hi=2500, filled=2)
    w = make_workload(c, poison=True)
    cent = torch.full((w["P"], c.Hkv, c.D), float("nan"))
    oracle.build_centroids(w["k_pool"], torch.cat([w["prebuilt_pages"], w["fill_pages"]]), cent)
    sel, n_sel, out, lse = oracle.decode_step(w["q"], w["k_pool"], w["v_pool"], w["page_table"],
                                              w["seq_lens"], cent, c.topk, c.bos, c.eos, c.sm_scale)
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()


def test_last_page_centroid_is_not_a_candidate(oracle):
    """With eos >= 1 each request's last page is reserved, never scored (reading S4): the
    oracle's selection and output do not change when every last page's centroid is NaN."""
    from paged_block_sparse_vt_b200.workloads import make_workload, config
    c = config(5, B=12, len_lo=200, len_hi=3000, filled=4)
    assert c.eos >= 1
    w = make_workload(c)
    cent = torch.zeros((w["P"], c.Hkv, c.D))
    oracle.build_centroids(w["k_pool"], torch.cat([w["prebuilt_pages"], w["fill_pages"]]), cent)
    n = (w["seq_lens"].long() + PS - 1) // PS
    last = w["page_table"][torch.arange(c.B), n - 1].long()
    poisoned = cent.clone()
    poisoned[last] = float("nan")
    res = [oracle.decode_step(w["q"], w["k_pool"], w["v_pool"], w["page_table"], w["seq_lens"],
                              cc, c.topk, c.bos, c.eos, c.sm_scale) for cc in (cent, poisoned)]
    for a, b in zip(*res):
        assert torch.equal(a, b)


def test_mla_value_is_prefix_of_key_row(oracle):
    """MLA: V = K[:, :512] read from the same pool; equals dense attention with that V."""
    from paged_block_sparse_vt_b200.workloads import make_workload, config
    c = config(4, B=2, len_lo=300, len_hi=300, pool_pages=40, topk=64)
    w = make_workload(c)
    assert w["v_pool"] is w["k_pool"]
    cent = torch.full((w["P"], 1, c.D), float("nan"))
    oracle.build_centroids(w["k_pool"], torch.cat([w["prebuilt_pages"], w["fill_pages"]]), cent)
    sel, n_sel, out, lse = oracle.decode_step(w["q"], w["k_pool"], w["v_pool"], w["page_table"],
                                              w["seq_lens"], cent, c.topk, c.bos, c.eos, c.sm_scale,
                                              head_dim_v=c.Dv)
    vcopy = w["k_pool"][..., : c.Dv].contiguous()
    ref, ref_lse = dense_attention(w["q"], w["k_pool"], vcopy, w["page_table"], w["seq_lens"],
                                   c.sm_scale)
    assert out.shape == (2, 32, 512)
    assert torch.allclose(out, ref, rtol=0, atol=1e-12)
    assert torch.allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_fp32_timing_copy_tracks_the_oracle(oracle):
    """The fp32 build of the same source (the benchmark's CPU-baseline copy, never a
    reference) computes the same step: same selections here, outputs within fp32 rounding."""
    from paged_block_sparse_vt_b200.workloads import config, make_workload
    w = make_workload(config(2, B=4, len_lo=600, len_hi=3000, pool_pages=1000))
    c = w["config"]
    full = torch.cat([w["prebuilt_pages"], w["fill_pages"]]).to(torch.int32)
    res = []
    for kind in ("f64", "f32"):
        cent = torch.zeros((w["P"], c.Hkv, c.D))
        oracle.build_centroids(w["k_pool"], full, cent, kind=kind)
        res.append((cent,) + oracle.decode_step(w["q"], w["k_pool"], w["v_pool"], w["page_table"],
                                                w["seq_lens"], cent, c.topk, c.bos, c.eos,
                                                c.sm_scale, kind=kind))
    (c64, s64, n64, o64, l64), (c32, s32, n32, o32, l32) = res
    assert torch.allclose(c32, c64, rtol=1e-6, atol=1e-7)
    assert torch.equal(n32, n64) and torch.equal(s32, s64)
    assert (o32 - o64).abs().max().item() < 1e-4 and (l32 - l64).abs().max().item() < 1e-4


# --------------------------------------------------------------------------------------
# the lossy indexer mode (one radix pass, early termination, random start in the last bin)
# --------------------------------------------------------------------------------------

# SplitMix64's published output sequence from state 0 (Steele, Lea and Flood 2014; the
# reference generator's first three outputs): the start of the cyclic fill for unit 0 with
# seed = 0, gamma and 2 gamma.
GAMMA = 0x9E3779B97F4A7C15
SPLITMIX64_FROM_ZERO = (0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F)


def _one_head_case(values, topk, bos=1, eos=1):
    """One request, Hkv = G = 1, D = 4, q = e0, centroid of page i = (values[i], 0, 0, 0):
    the score of page i is values[i]."""
    n = len(values)
    pt, seq = _identity_batch(n)
    q = torch.zeros(1, 1, 4)
    q[0, 0, 0] = 1.0
    cent = torch.zeros(n, 1, 4)
    cent[:, 0, 0] = torch.tensor(values, dtype=torch.float32)
    return q.to(torch.bfloat16), pt, seq, cent


def test_approx_equals_exact_when_every_score_has_its_own_bin(oracle):
    """m <= 1024 candidates with evenly spaced scores: one per bin, so the single pass is exact."""
    g = torch.Generator().manual_seed(21)
    m = 300
    vals = (torch.randperm(m + 2, generator=g).float() * 0.5).tolist()
    q, pt, seq, cent = _one_head_case(vals, 30)
    exact = oracle.select_pages(q, pt, seq, cent, 30, 1, 1)
    for seed in (0, 5, 2 ** 63 + 11):
        approx = oracle.select_pages_approx(q, pt, seq, cent, 30, 1, 1, seed)
        assert torch.equal(approx[0], exact[0]) and torch.equal(approx[1], exact[1])


@pytest.mark.parametrize("which", [0, 1, 2])
def test_approx_fill_of_the_last_bin_starts_at_the_published_draw(oracle, which):
    """Every score equal: all candidates share bin 0, so the pass keeps topk of them in cyclic
    order from r = splitmix64(seed + unit) mod m; for unit 0 and seed = which * gamma that is
    the generator's published output number which + 1."""
    n, topk = 50, 7
    m = n - 2
    q, pt, seq, cent = _one_head_case([1.5] * n, topk)
    seed = (which * GAMMA) % 2 ** 64
    sel, n_sel = oracle.select_pages_approx(q, pt, seq, cent, topk, 1, 1, seed)
    r = SPLITMIX64_FROM_ZERO[which] % m
    want = sorted([0, n - 1] + [1 + (r + t) % m for t in range(topk)])
    assert int(n_sel[0, 0]) == topk + 2
    assert sel[0, 0, : topk + 2].tolist() == want


def test_approx_keeps_every_page_clear_of_the_boundary_and_is_valid(oracle):
    """Random batches: the lossy set has the exact size, holds the reserved pages, and keeps
    every candidate scoring more than two bin widths above the exact k-th score; its recall of
    the exact top-k stays high."""
    from paged_block_sparse_vt_b200.workloads import config, make_workload
    w = make_workload(config(2, B=6, len_lo=2000, len_hi=12000, pool_pages=6000))
    c = w["config"]
    full = torch.cat([w["prebuilt_pages"], w["fill_pages"]]).to(torch.int32)
    cent = torch.zeros((w["P"], c.Hkv, c.D))
    oracle.build_centroids(w["k_pool"], full, cent)
    sel, n_sel, scores = oracle.select_pages(w["q"], w["page_table"], w["seq_lens"], cent, c.topk,
                                             c.bos, c.eos, want_scores=True)
    asel, an = oracle.select_pages_approx(w["q"], w["page_table"], w["seq_lens"], cent, c.topk,
                                          c.bos, c.eos, 99)
    assert torch.equal(an, n_sel)
    recalls = []
    for b in range(c.B):
        n = (int(w["seq_lens"][b]) + 15) // 16
        for h in range(c.Hkv):
            got = set(asel[b, h, : an[b, h]].tolist())
            want = set(sel[b, h, : n_sel[b, h]].tolist())
            assert {0, n - 1} <= got and len(got) == c.kmax
            s = scores[b, h, 1:n - 1]
            kth = min(scores[b, h, i].item() for i in want if 0 < i < n - 1)
            width = (s.max() - s.min()).item() / 1024
            for i in range(1, n - 1):
                if scores[b, h, i].item() > kth + 2 * width:
                    assert i in got
            recalls.append(len(got & want) / len(want))
    assert min(recalls) >= 0.9 and sum(recalls) / len(recalls) >= 0.97

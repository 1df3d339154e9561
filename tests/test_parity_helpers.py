"""The parity checker itself, on the CPU: a selection that swaps a tied page is accepted,
counted and its output held against the oracle's attention over that selection; a swap of
pages that do not tie, or an output off by more than the bound on a swapped unit, fails.
The "GPU" results here are the oracle's own, with the mistakes planted in them."""
import pytest
import torch

from paged_block_sparse_vt_b200.workloads import config, make_workload
from parity import (compare_outputs, compare_selection, oracle_centroids, oracle_step,
                    reference_outputs)


def _tied_case(oracle):
    """Config-1 workload whose k-th selected page and best unselected candidate have equal
    centroids (so equal scores); returns the workload, centroids, oracle result, the two pages."""
    w = make_workload(config(1))
    c = w["config"]
    cent = oracle_centroids(oracle, w)
    ref = oracle_step(oracle, w, cent)
    s = ref["scores"][0, 0]
    n = (int(w["seq_lens"][0]) + 15) // 16
    chosen = [i for i in ref["sel"][0, 0, : ref["n_sel"][0, 0]].tolist() if c.bos <= i < n - c.eos]
    kth = min(chosen, key=lambda i: (s[i].item(), -i))
    rest = [i for i in range(c.bos, n - c.eos) if i not in chosen]
    best = max(rest, key=lambda i: (s[i].item(), -i))
    pt = w["page_table"][0]
    cent[int(pt[best])] = cent[int(pt[kth])]
    ref = oracle_step(oracle, w, cent)
    return w, cent, ref, kth, best


def test_tied_swap_is_accepted_counted_and_its_output_checked(oracle):
    w, cent, ref, kth, best = _tied_case(oracle)
    want = ref["sel"][0, 0, : ref["n_sel"][0, 0]].tolist()
    a, b = min(kth, best), max(kth, best)
    assert a in want and b not in want  # ties go to the lower index
    alt = sorted((set(want) - {a}) | {b})
    sel = ref["sel"].clone()
    sel[0, 0, : len(alt)] = torch.tensor(alt, dtype=torch.int32)
    rep = compare_selection(w, ref, cent, sel, ref["n_sel"], label="planted tie")
    assert rep.swapped == [(0, 0)] and rep.swapped_pages == 2 and rep.strict_fail == 0
    ro, rl = reference_outputs(oracle, w, ref, sel, ref["n_sel"], rep)
    assert not torch.allclose(ro, ref["out"])  # another page set: another output
    alt_out, alt_lse = oracle.sparse_attention(w["q"], w["k_pool"], w["v_pool"], w["page_table"],
                                               w["seq_lens"], sel, ref["n_sel"],
                                               w["config"].sm_scale)
    compare_outputs(alt_out.to(torch.bfloat16), alt_lse.float(), ro, rl)
    with pytest.raises(AssertionError):  # the swapped unit's output is compared too
        compare_outputs((alt_out + 0.02).to(torch.bfloat16), alt_lse.float(), ro, rl)
    with pytest.raises(AssertionError):  # and not against the oracle's own selection
        compare_outputs(alt_out.to(torch.bfloat16), alt_lse.float(), ref["out"], ref["lse"])


def test_swap_without_a_tie_fails(oracle):
    w = make_workload(config(1))
    c = w["config"]
    cent = oracle_centroids(oracle, w)
    ref = oracle_step(oracle, w, cent)
    n = (int(w["seq_lens"][0]) + 15) // 16
    want = ref["sel"][0, 0, : ref["n_sel"][0, 0]].tolist()
    s = ref["scores"][0, 0]
    chosen = [i for i in want if c.bos <= i < n - c.eos]
    rest = [i for i in range(c.bos, n - c.eos) if i not in chosen]
    worst = min(rest, key=lambda i: s[i].item())
    alt = sorted((set(want) - {chosen[0]}) | {worst})
    sel = ref["sel"].clone()
    sel[0, 0, : len(alt)] = torch.tensor(alt, dtype=torch.int32)
    with pytest.raises(AssertionError):
        compare_selection(w, ref, cent, sel, ref["n_sel"])


def test_reserved_page_must_match(oracle):
    w = make_workload(config(1))
    cent = oracle_centroids(oracle, w)
    ref = oracle_step(oracle, w, cent)
    want = ref["sel"][0, 0, : ref["n_sel"][0, 0]].tolist()
    n = (int(w["seq_lens"][0]) + 15) // 16
    x = next(i for i in range(1, n - 1) if i not in want)
    alt = sorted((set(want) - {0}) | {x})  # reserved page 0 replaced by a candidate
    sel = ref["sel"].clone()
    sel[0, 0, : len(alt)] = torch.tensor(alt, dtype=torch.int32)
    with pytest.raises(AssertionError, match="reserved page"):
        compare_selection(w, ref, cent, sel, ref["n_sel"])

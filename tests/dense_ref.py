"""An independent dense-attention routine (torch fp64 on the CPU) used only by tests.

It gathers each request's pages into one contiguous sequence and calls the
library softmax; it shares nothing with the oracle's C code, so the two can
check each other where the method reduces to plain attention (every page
selected).
"""
import torch


def gather_sequence(pool, page_table, b, seq_len, page_size=16):
    n = (seq_len + page_size - 1) // page_size
    idx = page_table[b, :n].long()
    rows = pool[idx]                              # [n, page, H, D]
    return rows.reshape(n * page_size, *rows.shape[2:])[:seq_len]


def dense_attention(q, k_pool, v_pool, page_table, seq_lens, sm_scale, head_dim_v=None,
                    pages=None):
    """softmax(scale * q K^T) V over the listed logical pages (all pages if None), fp64.

    Returns (out [B, Hq, Dv], lse [B, Hq]).
    """
    B, Hq, D = q.shape
    Hkv = k_pool.shape[2]
    G = Hq // Hkv
    Dv = head_dim_v if head_dim_v is not None else v_pool.shape[3]
    out = torch.zeros((B, Hq, Dv), dtype=torch.float64)
    lse = torch.zeros((B, Hq), dtype=torch.float64)
    for b in range(B):
        L = int(seq_lens[b])
        K = gather_sequence(k_pool, page_table, b, L).double()
        V = gather_sequence(v_pool, page_table, b, L)[..., :Dv].double()
        if pages is not None:
            keep = torch.zeros(L, dtype=torch.bool)
            for i in pages[b]:
                keep[16 * i: min(L, 16 * (i + 1))] = True
            K, V = K[keep], V[keep]
        for hq in range(Hq):
            h = hq // G
            z = (K[:, h, :] @ q[b, hq].double()) * sm_scale
            out[b, hq] = torch.softmax(z, dim=0) @ V[:, h, :]
            lse[b, hq] = torch.logsumexp(z, dim=0)
    return out, lse

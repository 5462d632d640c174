"""Test-side helpers: dense views of a paged problem and problem transforms.

These move data only (page-table gathers, page renumbering, head repeats); none
of them computes attention.
"""
from __future__ import annotations

import copy

import numpy as np

import workloads as W


def kv_values(pr, which: str) -> np.ndarray:
    """Pool values as float64 [num_pages][Hkv][P][d] (FP8: code value x page scale)."""
    pool = pr.k_pages if which == "k" else pr.v_pages
    if pr.kv_dtype == "bf16":
        return W.bf16_bits_to_f32(pool).astype(np.float64)
    import torch
    vals = torch.from_numpy(np.ascontiguousarray(pool)).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    sc = pr.kv_scales[0 if which == "k" else 1].astype(np.float64)
    return vals * sc[:, :, None, None]


def dense_kv(pr, b: int, which: str) -> np.ndarray:
    """Logical K or V of request b as float64 [Hkv][Lb][d], gathered through the page table (only
    the request's pages are converted)."""
    Lb, P = int(pr.seq_lens[b]), pr.page_size
    npg = (Lb + P - 1) // P
    pages = pr.page_table[b, :npg]
    pool = pr.k_pages if which == "k" else pr.v_pages
    raw = pool[pages]                    # [npg][Hkv][P][d]
    if pr.kv_dtype == "bf16":
        x = W.bf16_bits_to_f32(raw).astype(np.float64)
    else:
        import torch
        x = torch.from_numpy(np.ascontiguousarray(raw)).view(torch.float8_e4m3fn).to(torch.float64).numpy()
        sc = pr.kv_scales[0 if which == "k" else 1].astype(np.float64)[pages]   # [npg][Hkv]
        x = x * sc[:, :, None, None]
    x = x.transpose(1, 0, 2, 3).reshape(pr.n_kv_heads, npg * P, pr.head_dim)
    return x[:, :Lb]


def q_values(pr) -> np.ndarray:
    return W.bf16_bits_to_f32(pr.q).astype(np.float64)


def repage(pr, seed: int):
    """Same logical KV under another physical page numbering (and a larger pool)."""
    rng = np.random.default_rng(seed)
    n_old = pr.num_pages
    n_new = n_old + 7
    new_of_old = rng.permutation(n_new)[:n_old]
    k = np.zeros((n_new,) + pr.k_pages.shape[1:], dtype=pr.k_pages.dtype)
    v = np.zeros_like(k)
    k[new_of_old] = pr.k_pages
    v[new_of_old] = pr.v_pages
    out = copy.copy(pr)
    out.k_pages, out.v_pages = k, v
    tab = pr.page_table.copy()
    m = tab >= 0
    tab[m] = new_of_old[tab[m]]
    out.page_table = tab
    if pr.kv_scales is not None:
        s = np.ones((2, n_new, pr.n_kv_heads), dtype=np.float32)
        s[:, new_of_old] = pr.kv_scales
        out.kv_scales = s
    return out


def as_mha(pr):
    """Repeat every KV head G times so that each query head has its own KV head."""
    G = pr.group
    out = copy.copy(pr)
    out.k_pages = np.repeat(pr.k_pages, G, axis=1)
    out.v_pages = np.repeat(pr.v_pages, G, axis=1)
    out.n_kv_heads = pr.n_q_heads
    if pr.kv_scales is not None:
        out.kv_scales = np.repeat(pr.kv_scales, G, axis=2)
    return out


def with_lens(pr, seq_lens, q_tokens=None, q=None):
    """Same pools and page table, other lengths / query tokens."""
    out = copy.copy(pr)
    out.seq_lens = np.asarray(seq_lens, dtype=np.int32)
    if q_tokens is not None:
        out.q_tokens = q_tokens
    if q is not None:
        out.q = np.ascontiguousarray(q)
    return out

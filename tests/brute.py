"""Brute-force dense attention in numpy fp64, written independently of the
oracle: gather each request's keys and values into contiguous arrays by
walking its page table, build the full [q_b, kv_b] score matrix per head,
apply an explicit boolean mask matrix, and take a softmax of each row.

Used only to pin the oracle on small inputs.
"""
from __future__ import annotations

import numpy as np


def bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def dense_attention(q_bits, k_bits, v_bits, page_table, seq_lens, cu_q_lens, scale,
                    causal=True):
    return dense_attention_values(bits_to_f64(q_bits), bits_to_f64(k_bits), bits_to_f64(v_bits),
                                  page_table, seq_lens, cu_q_lens, scale, causal)


def dense_attention_values(q, kp, vp, page_table, seq_lens, cu_q_lens, scale, causal=True):
    """The same on float64 values: q [T, Hq, D], pools [P, ps, Hkv, D]."""
    T, Hq, D = q.shape
    P, ps, Hkv, _ = kp.shape
    B = len(seq_lens)
    G = Hq // Hkv
    if cu_q_lens is None:
        cu_q_lens = np.arange(B + 1)
    out = np.zeros((T, Hq, D))
    lse = np.zeros((T, Hq))
    for b in range(B):
        kv = int(seq_lens[b])
        t0, t1 = int(cu_q_lens[b]), int(cu_q_lens[b + 1])
        qb = t1 - t0
        if qb == 0:
            continue
        n_pages = -(-kv // ps)
        pages = [int(p) for p in page_table[b, :n_pages]]
        # contiguous [kv, Hkv, D]
        K = np.concatenate([kp[p] for p in pages], axis=0)[:kv] if kv else np.zeros((0, Hkv, D))
        V = np.concatenate([vp[p] for p in pages], axis=0)[:kv] if kv else np.zeros((0, Hkv, D))
        # explicit mask matrix: row i (query), column j (key)
        rows = np.arange(qb)[:, None]
        cols = np.arange(kv)[None, :]
        visible = (cols <= rows + (kv - qb)) if causal else np.ones((qb, kv), dtype=bool)
        for h in range(Hq):
            g = h // G
            S = scale * (q[t0:t1, h, :] @ K[:, g, :].T)          # [qb, kv]
            S = np.where(visible, S, -np.inf)
            for i in range(qb):
                row = S[i]
                if not np.any(visible[i]):
                    out[t0 + i, h] = 0.0
                    lse[t0 + i, h] = -np.inf
                    continue
                m = row.max()
                e = np.exp(row - m)
                out[t0 + i, h] = (e / e.sum()) @ V[:, g, :]
                lse[t0 + i, h] = m + np.log(e.sum())
    return out, lse

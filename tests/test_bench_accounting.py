"""The algorithmic work counts behind bench.py's roofline figures, checked on
the CPU against brute force: every visible (query, key) pair enumerated with
the end-aligned causal rule (query i of a request with q queries and kv keys
sees keys j < kv - q + i + 1), and every byte of K, V, Q, O, LSE and the live
page-table entries counted from the shapes."""
import numpy as np
import pytest

import bench


def brute_counts(q_lens, kv_lens, Hq, Hkv, D, ps):
    pairs = 0
    for q, kv in zip(q_lens, kv_lens):
        for i in range(q):
            for j in range(kv):
                if j < kv - q + i + 1:
                    pairs += 1
    T = sum(q_lens)
    kv_bytes = 0
    for kv in kv_lens:
        kv_bytes += kv * Hkv * D * 2      # K, bf16
        kv_bytes += kv * Hkv * D * 2      # V, bf16
    table = sum((kv + ps - 1) // ps for kv in kv_lens) * 4
    lens = len(kv_lens) * 4 + (len(kv_lens) + 1) * 4
    total = kv_bytes + 2 * T * Hq * D * 2 + T * Hq * 4 + table + lens
    return dict(kv_bytes=kv_bytes, bytes=total, flops=4 * D * Hq * pairs, T=T)


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_work_counts_match_brute_force(seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 6))
    kv = [int(x) for x in rng.integers(1, 90, size=B)]
    q = [int(rng.integers(1, k + 1)) for k in kv]
    if seed == 3:
        q = [1] * B                       # decode: one query token per request
    Hkv = int(rng.choice([1, 2, 8]))
    G = int(rng.choice([1, 4, 32]))
    D = int(rng.choice([64, 128, 256]))
    ps = int(rng.choice([16, 64, 128]))
    w = dict(q_lens=q, kv_lens=kv, Hq=Hkv * G, Hkv=Hkv, D=D, ps=ps)
    assert bench.work_counts(w) == brute_counts(q, kv, Hkv * G, Hkv, D, ps)


def test_work_counts_headline_shape():
    """Workload-2 style batch: K+V bytes are 4 * D * Hkv per key and there is
    exactly one visible key per (query, key) of a decode row."""
    kv = [1024, 2048, 1500]
    w = dict(q_lens=[1, 1, 1], kv_lens=kv, Hq=32, Hkv=8, D=128, ps=16)
    c = bench.work_counts(w)
    assert c["kv_bytes"] == sum(kv) * 8 * 128 * 4
    assert c["flops"] == 4 * 128 * 32 * sum(kv)
    assert c["T"] == 3

"""Pins of the oracle's non-causal mode (``causal=False``): every query row
sees all keys of its request ("Unified Triton kernel that doesn't distinguish
between prefill + decode", vLLM PR #16828, review thread on the masking).

Checked against the brute-force dense attention with an all-true mask, a
closed form (q = 0: O is the mean of all of the request's V rows and LSE =
ln kv_b), and decode, where causal and non-causal coincide.  A planted
mistake in a copy of the oracle source is caught."""
import math
import os
import subprocess

import numpy as np
import pytest

from oracle import oracle as O
from paged_kv_gqa_fmha_b200 import workloads as W
from tests.brute import bits_to_f64, dense_attention


def _w(seed, prefill=True, **kw):
    rng = np.random.default_rng(seed)
    spec = W.random_small(rng, prefill=prefill, max_kv=200, **kw)
    return W.generate(spec, seed, device="cpu")


def _args(w):
    return (W.bf16_bits(w["q"]), W.bf16_bits(w["k_pool"]), W.bf16_bits(w["v_pool"]),
            w["page_table_cpu"].numpy(), w["seq_lens_cpu"].numpy(), w["cu_q_lens_cpu"].numpy(),
            w["scale"])


@pytest.mark.parametrize("seed", [1, 2, 3, 4, 5, 6])
def test_noncausal_matches_brute_force(seed):
    w = _w(seed)
    o, l = O.paged_attention(*_args(w), causal=False)
    ob, lb = dense_attention(*_args(w), causal=False)
    assert np.max(np.abs(o - ob)) < 1e-12
    fin = np.isfinite(lb)
    assert np.array_equal(fin, np.isfinite(l))
    assert np.max(np.abs(l[fin] - lb[fin])) < 1e-12


def test_noncausal_zero_query_closed_form():
    w = _w(11, D=64, G=2, Hkv=2)
    q, k, v, table, seq, cu, scale = _args(w)
    q = np.zeros_like(q)
    o, l = O.paged_attention(q, k, v, table, seq, cu, scale, causal=False)
    vp = bits_to_f64(v)
    ps = vp.shape[1]
    G = q.shape[1] // vp.shape[2]
    for b in range(len(seq)):
        kv = int(seq[b])
        if kv == 0:
            continue
        rows = np.concatenate([vp[table[b, p]] for p in range(-(-kv // ps))], axis=0)[:kv]
        mean = rows.mean(axis=0)                      # [Hkv, D]
        for t in range(int(cu[b]), int(cu[b + 1])):
            for h in range(q.shape[1]):
                assert np.max(np.abs(o[t, h] - mean[h // G])) < 1e-12
                assert abs(l[t, h] - math.log(kv)) < 1e-12


def test_decode_is_the_same_in_both_modes():
    w = _w(21, prefill=False)
    o1, l1 = O.paged_attention(*_args(w), causal=True)
    o2, l2 = O.paged_attention(*_args(w), causal=False)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_noncausal_differs_from_causal_on_prefill():
    w = _w(31)
    o1, _ = O.paged_attention(*_args(w), causal=True)
    o2, _ = O.paged_attention(*_args(w), causal=False)
    assert np.max(np.abs(o1 - o2)) > 1e-3


def test_pin_catches_a_planted_mistake(tmp_path):
    src = open(os.path.join(os.path.dirname(O.__file__), "oracle.c")).read()
    old = "if (J->non_causal) n = kv_b;"
    assert src.count(old) == 1
    c = tmp_path / "nc.c"
    so = tmp_path / "nc.so"
    c.write_text(src.replace(old, "if (J->non_causal) n = kv_b - 1;", 1))
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread", "-o",
                           str(so), str(c), "-lm"])
    lib = O.load_library(str(so))
    w = _w(41)
    o, _ = O.paged_attention(*_args(w), causal=False, lib=lib)
    ob, _ = dense_attention(*_args(w), causal=False)
    assert np.max(np.abs(o - ob)) > 1e-6

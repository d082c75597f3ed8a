"""Pins of the oracle's row-selective entry point (``oracle_paged_attention_rows``).

The full-size GPU parity tests check every element of the smaller workloads
with ``oracle_paged_attention`` and, where the host cannot hold a whole
output, rows chosen by index through this entry point.  It computes the same
attention as the all-rows entry point (softmax(scale * Q K^T + causal mask) V
over paged KV, with the page table of "integrate PrimTS FMHA kernels",
TensorRT-LLM PR #17399, "Unified page-table metadata", and the varlen packed
queries of "Unified Triton kernel that doesn't distinguish between prefill +
decode", vLLM PR #16828), but picks its rows from two index lists and writes
row u of the result at position u.  These tests pin that selection and
placement against the independent brute-force dense attention of
``tests/brute.py``, and plant mistakes in the row path of copies of the C
source (swapped token / head lists, a wrong output offset, a wrong LSE
offset) to show the pins catch them.
"""
import os
import subprocess

import numpy as np
import pytest

from oracle import oracle as O
from paged_kv_gqa_fmha_b200 import workloads as W
from tests.brute import dense_attention


def _brute(w):
    return dense_attention(W.bf16_bits(w["q"]), W.bf16_bits(w["k_pool"]),
                           W.bf16_bits(w["v_pool"]), w["page_table_cpu"].numpy(),
                           w["seq_lens_cpu"].numpy(), w["cu_q_lens_cpu"].numpy(), w["scale"])


def _rows(w, rows_t, rows_h, lib=None):
    return O.paged_attention_rows(W.bf16_bits(w["q"]), W.bf16_bits(w["k_pool"]),
                                  W.bf16_bits(w["v_pool"]), w["page_table_cpu"].numpy(),
                                  w["seq_lens_cpu"].numpy(), w["cu_q_lens_cpu"].numpy(),
                                  w["scale"], rows_t, rows_h, lib=lib)


def _workloads(seed, n=3, **kw):
    rng = np.random.default_rng(seed)
    return [W.generate(W.random_small(rng, name="rows%d" % i, **kw), seed=20_000 + seed * 10 + i)
            for i in range(n)]


def _shuffled_rows(w, rng, n):
    """n (token, head) pairs drawn with repeats, in random order."""
    return (rng.integers(0, w["T"], size=n).astype(np.int32),
            rng.integers(0, w["Hq"], size=n).astype(np.int32))


@pytest.mark.parametrize("seed", range(4))
def test_rows_match_brute_force_in_any_order(seed):
    rng = np.random.default_rng(700 + seed)
    for w in _workloads(seed, max_kv=220, prefill=bool(seed % 2)):
        ob, lb = _brute(w)
        rt, rh = _shuffled_rows(w, rng, 3 * w["T"] * w["Hq"] // 2 + 5)
        o, l = _rows(w, rt, rh)
        assert o.shape == (rt.size, w["D"]) and l.shape == (rt.size,)
        assert np.max(np.abs(o - ob[rt, rh])) < 1e-12
        fin = np.isfinite(lb[rt, rh])
        assert np.array_equal(fin, np.isfinite(l))
        assert np.max(np.abs(l[fin] - lb[rt, rh][fin])) < 1e-12


def test_rows_cover_every_row_and_agree_with_all_rows_entry():
    """Every (token, head) once, in reverse order, equals the all-rows result
    read backwards; both equal brute force."""
    for w in _workloads(9, n=2, max_kv=300, prefill=True):
        T, Hq = w["T"], w["Hq"]
        tt, hh = np.meshgrid(np.arange(T), np.arange(Hq), indexing="ij")
        rt = tt.reshape(-1)[::-1].astype(np.int32).copy()
        rh = hh.reshape(-1)[::-1].astype(np.int32).copy()
        o, l = _rows(w, rt, rh)
        oa, la = O.paged_attention(W.bf16_bits(w["q"]), W.bf16_bits(w["k_pool"]),
                                   W.bf16_bits(w["v_pool"]), w["page_table_cpu"].numpy(),
                                   w["seq_lens_cpu"].numpy(), w["cu_q_lens_cpu"].numpy(),
                                   w["scale"])
        ob, lb = _brute(w)
        assert np.max(np.abs(o - oa[rt, rh])) == 0.0
        assert np.max(np.abs(o - ob[rt, rh])) < 1e-12


def test_empty_row_list():
    w = _workloads(11, n=1, max_kv=50)[0]
    o, l = _rows(w, np.zeros(0, np.int32), np.zeros(0, np.int32))
    assert o.shape == (0, w["D"]) and l.shape == (0,)


# ---------------------------------------------------------------- planted mistakes
ROW_MUTANTS = {
    "row_lists_swapped": ("t = J->row_t[u];\n            h = J->row_h[u];",
                          "t = J->row_h[u];\n            h = J->row_t[u];"),
    "row_output_offset": ("o = J->out + u * J->D;\n            l = J->lse + u;\n        } else",
                          "o = J->out + (J->n_rows - 1 - u) * J->D;\n            l = J->lse + u;\n"
                          "        } else"),
    "row_lse_offset": ("l = J->lse + u;\n        } else",
                       "l = J->lse + (J->n_rows - 1 - u);\n        } else"),
}


def _row_pins_pass(lib) -> bool:
    """The pin above on rows whose token and head indices are both below
    min(T, Hq), so that a mutant that swaps the lists still reads inside the
    arrays (and therefore fails by value, not by a crash)."""
    rng = np.random.default_rng(5)
    for w in _workloads(13, n=2, max_kv=150, prefill=True, G=8, Hkv=2):
        lim = min(w["T"], w["Hq"])
        ob, lb = _brute(w)
        rt = rng.integers(0, lim, size=40).astype(np.int32)
        rh = rng.integers(0, lim, size=40).astype(np.int32)
        try:
            o, l = _rows(w, rt, rh, lib=lib)
        except ValueError:
            return False
        fin = np.isfinite(lb[rt, rh])
        if not (np.max(np.abs(o - ob[rt, rh])) < 1e-12 and
                np.array_equal(fin, np.isfinite(l)) and
                np.max(np.abs(l[fin] - lb[rt, rh][fin])) < 1e-12):
            return False
    return True


def test_unmutated_rows_entry_passes():
    assert _row_pins_pass(None)


@pytest.mark.parametrize("name", sorted(ROW_MUTANTS))
def test_row_pins_catch_planted_mistake(name, tmp_path):
    src = open(os.path.join(os.path.dirname(O.__file__), "oracle.c")).read()
    old, new = ROW_MUTANTS[name]
    assert src.count(old) == 1, "mutation anchor not found once: %s" % name
    c = tmp_path / ("r_%s.c" % name)
    so = tmp_path / ("r_%s.so" % name)
    c.write_text(src.replace(old, new, 1))
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread", "-o",
                           str(so), str(c), "-lm"])
    assert not _row_pins_pass(O.load_library(str(so))), "row pins did not catch %s" % name

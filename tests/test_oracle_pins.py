"""Pins of the fp64 CPU oracle against things other than itself.

Each test checks the oracle against a brute-force dense implementation
written separately (``tests/brute.py``), a closed form, an invariant of the
method, or a special case.  The last test plants mistakes in copies of the
oracle's C source and shows that these pins catch each one.

The attention being pinned is softmax(scale * Q K^T + causal mask) V over
paged KV, as stated in "integrate PrimTS FMHA kernels" (TensorRT-LLM PR
#17399, "Unified page-table metadata") for the page table and in "Unified
Triton kernel that doesn't distinguish between prefill + decode" (vLLM PR
#16828) for varlen queries, GQA packing and the mask by select.
"""
import math
import os
import re
import subprocess

import numpy as np
import pytest
import torch

from oracle import oracle as O
from paged_kv_gqa_fmha_b200 import workloads as W
from tests.brute import dense_attention

pytestmark = pytest.mark.filterwarnings("ignore")


def _np(w, key):
    return w[key + "_cpu"].numpy() if key + "_cpu" in w else w[key].numpy()


def run_oracle(w, lib=None, q=None, k=None, v=None, table=None, seq=None, cu="default"):
    qb = W.bf16_bits(w["q"]) if q is None else q
    kb = W.bf16_bits(w["k_pool"]) if k is None else k
    vb = W.bf16_bits(w["v_pool"]) if v is None else v
    tb = _np(w, "page_table") if table is None else table
    sl = _np(w, "seq_lens") if seq is None else seq
    cq = _np(w, "cu_q_lens") if cu == "default" else cu
    return O.paged_attention(qb, kb, vb, tb, sl, cq, w["scale"], num_pages=kb.shape[0], lib=lib)


def run_brute(w, q=None, k=None, v=None):
    qb = W.bf16_bits(w["q"]) if q is None else q
    kb = W.bf16_bits(w["k_pool"]) if k is None else k
    vb = W.bf16_bits(w["v_pool"]) if v is None else v
    return dense_attention(qb, kb, vb, _np(w, "page_table"), _np(w, "seq_lens"),
                           _np(w, "cu_q_lens"), w["scale"])


def to_bits(x: torch.Tensor) -> np.ndarray:
    return W.bf16_bits(x.to(torch.bfloat16))


def bits_f64(b):
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def visible_counts(w):
    """n_vis[t] = number of keys token t may see (end-aligned causal)."""
    cu = _np(w, "cu_q_lens")
    seq = _np(w, "seq_lens")
    out = np.zeros(w["T"], dtype=np.int64)
    for b in range(w["B"]):
        qb = cu[b + 1] - cu[b]
        for i in range(qb):
            out[cu[b] + i] = min(seq[b], max(0, seq[b] - qb + i + 1))
    return out


def gather_rows(pool_f64, w, b, n):
    """Rows 0..n-1 of request b, [n, Hkv, D], by walking its page table."""
    ps = w["ps"]
    table = _np(w, "page_table")
    return np.stack([pool_f64[table[b, j // ps], j % ps] for j in range(n)], 0)


def random_workloads(n, seed=0, **kw):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        spec = W.random_small(rng, name="pin%d" % i, **kw)
        out.append(W.generate(spec, seed=10_000 + seed * 100 + i))
    return out


# ---------------------------------------------------------------- P-a brute force
@pytest.mark.parametrize("seed", range(6))
def test_brute_force_random(seed):
    for w in random_workloads(3, seed=seed, max_kv=200):
        o, l = run_oracle(w)
        ob, lb = run_brute(w)
        assert np.max(np.abs(o - ob)) < 1e-12
        assert np.max(np.abs(l - lb)) < 1e-12


@pytest.mark.parametrize("G,D,ps", [(32, 256, 128), (32, 64, 16), (1, 128, 32), (8, 128, 64)])
def test_brute_force_geometries(G, D, ps):
    rng = np.random.default_rng(G * 1000 + D + ps)
    for prefill in (False, True):
        spec = W.random_small(rng, G=G, D=D, ps=ps, Hkv=1, max_kv=160, prefill=prefill)
        w = W.generate(spec, seed=77 + G + D + ps)
        o, l = run_oracle(w)
        ob, lb = run_brute(w)
        assert np.max(np.abs(o - ob)) < 1e-12
        assert np.max(np.abs(l - lb)) < 1e-12


def test_brute_force_tiny_decode_config():
    w = W.generate(W.CONFIGS["tiny_decode"], W.default_seed("tiny_decode"))
    assert w["P"] == 12 and w["C"] == 4
    assert (_np(w, "page_table")[0, 3] == -1)
    o, l = run_oracle(w)
    ob, lb = run_brute(w)
    assert np.max(np.abs(o - ob)) < 1e-12 and np.max(np.abs(l - lb)) < 1e-12


# ---------------------------------------------------------------- P-b q = 0
def test_zero_query_closed_form():
    """With q = 0 every visible score is 0: O is the plain mean of the visible
    V rows and LSE = ln(number of visible keys).  Pins the mask alignment and
    the natural-log base of LSE."""
    for w in random_workloads(4, seed=11, prefill=True, max_kv=150):
        q0 = np.zeros_like(W.bf16_bits(w["q"]))
        o, l = run_oracle(w, q=q0)
        nvis = visible_counts(w)
        vp = bits_f64(W.bf16_bits(w["v_pool"]))
        cu = _np(w, "cu_q_lens")
        G = w["Hq"] // w["Hkv"]
        for b in range(w["B"]):
            for t in range(cu[b], cu[b + 1]):
                n = nvis[t]
                V = gather_rows(vp, w, b, n)            # [n, Hkv, D]
                for h in range(w["Hq"]):
                    assert abs(l[t, h] - math.log(n)) < 1e-13
                    assert np.max(np.abs(o[t, h] - V[:, h // G].mean(0))) < 1e-13


# ---------------------------------------------------------------- P-c single key
def test_single_key():
    """kv = 1: O = V_0 and LSE = the single scaled score."""
    spec = W.custom_spec("one", 8, 2, 128, 16, [1, 1, 1], [1, 1, 1])
    w = W.generate(spec, seed=5)
    o, l = run_oracle(w)
    qf = bits_f64(W.bf16_bits(w["q"]))
    kp = bits_f64(W.bf16_bits(w["k_pool"]))
    vp = bits_f64(W.bf16_bits(w["v_pool"]))
    table = _np(w, "page_table")
    for b in range(3):
        p = table[b, 0]
        for h in range(8):
            g = h // 4
            assert np.array_equal(o[b, h], vp[p, 0, g])
            s = w["scale"] * float(np.dot(qf[b, h], kp[p, 0, g]))
            assert abs(l[b, h] - s) < 1e-12


# ---------------------------------------------------------------- P-d equal logits
def test_equal_logits():
    """If all keys of a head are equal, every visible score is the same:
    O = mean of the visible V rows, LSE = s + ln(n)."""
    spec = W.custom_spec("eq", 8, 2, 64, 16, [5, 1, 40], [37, 20, 40])
    w = W.generate(spec, seed=9)
    k = W.bf16_bits(w["k_pool"]).copy()
    k[:] = k[0, 0][None, None]                  # one key vector per head, everywhere
    o, l = run_oracle(w, k=k)
    qf = bits_f64(W.bf16_bits(w["q"]))
    kf = bits_f64(k)
    vp = bits_f64(W.bf16_bits(w["v_pool"]))
    nvis = visible_counts(w)
    cu = _np(w, "cu_q_lens")
    for b in range(w["B"]):
        for t in range(cu[b], cu[b + 1]):
            V = gather_rows(vp, w, b, nvis[t])
            for h in range(8):
                g = h // 4
                s = w["scale"] * float(np.dot(qf[t, h], kf[0, 0, g]))
                assert abs(l[t, h] - (s + math.log(nvis[t]))) < 1e-12
                assert np.max(np.abs(o[t, h] - V[:, g].mean(0))) < 1e-12


# ---------------------------------------------------------------- P-e GQA = MHA
def test_gqa_equals_mha_with_repeated_kv_heads():
    spec = W.custom_spec("gqa", 16, 2, 64, 32, [3, 1, 17], [50, 33, 17])
    w = W.generate(spec, seed=21)
    G = 8
    k = W.bf16_bits(w["k_pool"])
    v = W.bf16_bits(w["v_pool"])
    k_mha = np.repeat(k, G, axis=2)             # KV head g -> query heads g*G..g*G+G-1
    v_mha = np.repeat(v, G, axis=2)
    o1, l1 = run_oracle(w)
    o2, l2 = run_oracle(w, k=np.ascontiguousarray(k_mha), v=np.ascontiguousarray(v_mha))
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


# ---------------------------------------------------------------- P-f permutation
def test_page_permutation_invariance():
    for w in random_workloads(3, seed=31, max_kv=250):
        k = W.bf16_bits(w["k_pool"])
        v = W.bf16_bits(w["v_pool"])
        table = _np(w, "page_table")
        P = k.shape[0]
        perm = np.random.default_rng(3).permutation(P)
        k2 = np.empty_like(k)
        v2 = np.empty_like(v)
        k2[perm] = k
        v2[perm] = v
        t2 = np.where(table >= 0, perm[np.maximum(table, 0)], -1).astype(np.int32)
        o1, l1 = run_oracle(w)
        o2, l2 = run_oracle(w, k=k2, v=v2, table=t2)
        assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


# ---------------------------------------------------------------- P-g poisoning
@pytest.mark.parametrize("fill", [-1, 2**31 - 1, "nan_page"])
def test_poisoned_columns_and_tails_are_never_read(fill):
    for w in random_workloads(3, seed=41, max_kv=200):
        k = W.bf16_bits(w["k_pool"]).copy()
        v = W.bf16_bits(w["v_pool"]).copy()
        table = _np(w, "page_table").copy()
        seq = _np(w, "seq_lens")
        ps = w["ps"]
        o1, l1 = run_oracle(w)
        nan = np.uint16(0x7FC0)
        live = set()
        for b in range(w["B"]):
            n = -(-seq[b] // ps)
            live.update(int(p) for p in table[b, :n])
            last = table[b, n - 1]
            tail = seq[b] - (n - 1) * ps
            k[last, tail:] = nan                 # tail slots of the last live page
            v[last, tail:] = nan
        dead = [p for p in range(k.shape[0]) if p not in live]
        for p in dead:
            k[p] = nan
            v[p] = nan
        for b in range(w["B"]):
            n = -(-seq[b] // ps)
            if fill == "nan_page":
                if dead:
                    table[b, n:] = dead[0]
            else:
                table[b, n:] = fill
        o2, l2 = O.paged_attention(W.bf16_bits(w["q"]), k, v, table, seq, _np(w, "cu_q_lens"),
                                   w["scale"], num_pages=0)
        assert np.all(np.isfinite(o2)) and np.all(np.isfinite(l2))
        assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


# ---------------------------------------------------------------- P-i chunked prefill
def test_chunked_prefill_equivalence():
    """Rows a..n-1 of a full prefill (q = kv = n) equal a prefill of only the
    last n-a tokens with kv = n: the mask is aligned to the end of KV."""
    n, a = 150, 97
    full = W.generate(W.custom_spec("full", 8, 2, 64, 16, [n], [n]), seed=51)
    o1, l1 = run_oracle(full)
    q_tail = W.bf16_bits(full["q"])[a:]
    o2, l2 = O.paged_attention(q_tail, W.bf16_bits(full["k_pool"]), W.bf16_bits(full["v_pool"]),
                               _np(full, "page_table"), _np(full, "seq_lens"),
                               np.array([0, n - a], dtype=np.int32), full["scale"])
    assert np.array_equal(o1[a:], o2) and np.array_equal(l1[a:], l2)


# ---------------------------------------------------------------- P-j large logits
def test_large_logits_stay_finite_and_match_brute_force():
    for w in random_workloads(2, seed=61, max_kv=180, prefill=True):
        q30 = to_bits(w["q"].float() * 30.0)
        o, l = run_oracle(w, q=q30)
        ob, lb = run_brute(w, q=q30)
        assert np.all(np.isfinite(o)) and np.all(np.isfinite(l))
        assert np.max(np.abs(o - ob)) < 1e-10
        assert np.max(np.abs(l - lb) / np.maximum(1.0, np.abs(lb))) < 1e-12


# ---------------------------------------------------------------- degenerate rows
def test_rows_without_visible_keys_and_empty_requests():
    """q_b > kv_b (invalid input) leaves the first q_b - kv_b rows without a
    key: O = 0, LSE = -inf.  A request with q_b = 0 contributes no rows."""
    spec = W.custom_spec("deg", 4, 1, 64, 16, [6, 0, 1], [4, 9, 9])
    w = W.generate(spec, seed=71)
    o, l = run_oracle(w)
    assert w["T"] == 7
    assert np.all(o[0:2] == 0) and np.all(np.isneginf(l[0:2]))
    assert np.all(np.isfinite(l[2:]))
    ob, lb = run_brute(w)
    assert np.max(np.abs(o - ob)) < 1e-12
    assert np.array_equal(np.isneginf(l), np.isneginf(lb))


# ---------------------------------------------------------------- split-KV merge identity
def test_merge_of_disjoint_key_ranges_equals_full_attention():
    """Split-KV decode: attention over keys [0, k) and [k, n), merged by
    log-sum-exp, equals attention over [0, n)."""
    ps, n = 16, 200
    for k_split in (16, 96, 192):
        w = W.generate(W.custom_spec("m", 8, 2, 128, ps, [1], [n]), seed=81 + k_split)
        o_full, l_full = run_oracle(w)
        table = _np(w, "page_table")
        t_a = table.copy()
        t_b = np.full_like(table, -1)
        nb = -(-(n - k_split) // ps)
        t_b[0, :nb] = table[0, k_split // ps: k_split // ps + nb]
        o_a, l_a = run_oracle(w, table=t_a, seq=np.array([k_split], np.int32))
        o_b, l_b = run_oracle(w, table=t_b, seq=np.array([n - k_split], np.int32))
        for h in range(8):
            o_m, l_m = O.merge_states(np.stack([o_a[0, h], o_b[0, h]]),
                                      np.array([l_a[0, h], l_b[0, h]]))
            assert abs(l_m - l_full[0, h]) < 1e-12
            assert np.max(np.abs(o_m - o_full[0, h])) < 1e-12


def test_merge_ignores_empty_states():
    o_s = np.array([[1.0, 2.0], [np.nan, np.nan] ])
    o, l = O.merge_states(np.nan_to_num(o_s), np.array([0.5, -np.inf]))
    assert np.allclose(o, [1.0, 2.0]) and abs(l - 0.5) < 1e-15
    o, l = O.merge_states(np.zeros((2, 2)), np.array([-np.inf, -np.inf]))
    assert np.all(o == 0) and np.isneginf(l)


# ---------------------------------------------------------------- planted mistakes
MUTANTS = {
    "mask_off_by_one": ("long n = kv_b - q_b + i + 1;", "long n = kv_b - q_b + i;"),
    "mask_start_aligned": ("long n = kv_b - q_b + i + 1;", "long n = i + 1;"),
    "kv_head_map": ("const int g = h / G;", "const int g = h % J->Hkv;"),
    "dropped_scale": ("s[j] = J->scale * acc;", "s[j] = acc;"),
    "lse_dropped_max": ("*lse_out = m + log(l);", "*lse_out = log(l);"),
    "softmax_sign": ("s[j] = exp(s[j] - m);", "s[j] = exp(m - s[j]);"),
    "pool_transposed": ("long idx = ((page * J->ps + slot) * J->Hkv + g) * J->D + d;",
                        "long idx = ((page * J->Hkv + g) * J->ps + slot) * J->D + d;"),
    "page_column": ("long page = J->page_table[(long)b * J->C + j / J->ps];\n        if",
                    "long page = J->page_table[(long)b * J->C + j % J->C];\n        if"),
    "slot_index": ("long slot = j % J->ps;\n        double acc",
                   "long slot = (j + 1) % J->ps;\n        double acc"),
    "v_not_normalised": ("double w = s[j] / l;", "double w = s[j];"),
}


def _pins_pass(lib) -> bool:
    """A compact run of the pins above against another oracle build."""
    try:
        for w in random_workloads(3, seed=2, max_kv=120, prefill=True) + \
                random_workloads(2, seed=3, max_kv=120, prefill=False, Hkv=2, G=4):
            o, l = run_oracle(w, lib=lib)
            ob, lb = run_brute(w)
            if not (np.max(np.abs(o - ob)) < 1e-12 and np.max(np.abs(l - lb)) < 1e-12):
                return False
        return True
    except ValueError:
        return False


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    src = open(os.path.join(os.path.dirname(O.__file__), "oracle.c")).read()
    old, new = MUTANTS[name]
    assert src.count(old) >= 1, "mutation anchor not found: %s" % name
    mutated = src.replace(old, new, 1)
    c = tmp_path / ("m_%s.c" % name)
    so = tmp_path / ("m_%s.so" % name)
    c.write_text(mutated)
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread", "-o",
                           str(so), str(c), "-lm"])
    assert not _pins_pass(O.load_library(str(so))), "pins did not catch %s" % name


def test_unmutated_oracle_passes_compact_pins():
    assert _pins_pass(None)


# ---------------------------------------------------------------- golden fixture
def load_golden(name):
    """Values written by tests/golden/make_golden.py (oracle only)."""
    path = os.path.join(os.path.dirname(__file__), "golden", name + ".txt")
    vals = [float(x) for x in open(path) if not x.startswith("#")]
    return np.array(vals)


def test_tiny_decode_golden_fixture_is_reproduced():
    """Regression fixture: the generator and the oracle still give the stored
    tiny-decode outputs (brute force pins those values above)."""
    name = "tiny_decode"
    w = W.generate(W.CONFIGS[name], W.default_seed(name))
    o, l = run_oracle(w, cu=None)
    g = load_golden(name)
    assert g.size == 8 + 8 * 64
    assert np.max(np.abs(g[:8] - l.reshape(-1))) < 1e-14
    assert np.max(np.abs(g[8:] - o.reshape(-1))) < 1e-14
    ob, lb = run_brute(w)
    assert np.max(np.abs(g[8:] - ob.reshape(-1))) < 1e-12

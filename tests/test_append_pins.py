"""Pins of the oracle's paged KV append (``oracle_append_kv``).

The pins do not restate the slot formula.  Each request's keys and values
are drawn as contiguous [kv_b, Hkv, D] arrays; the pool is filled from them
by the definition of paging (page p of the request's table row holds rows
p*ps .. p*ps+ps-1, as tests/brute.py reads it back), with the rows of this
step's new tokens left out (poisoned with NaN).  After the append, reading
the request back page by page must give the contiguous arrays bit for bit,
attention over the pool must equal attention over the contiguous arrays,
and nothing outside the live rows may change.  Planted mistakes in copies of
the oracle's source are caught by the same checks.

Source: "integrate PrimTS FMHA kernels" (TensorRT-LLM PR #17399), sections
"Unified page-table metadata" and "Planning, preprocessing, and workspace
ownership" (the KV-cache append that precedes attention).
"""
import os
import subprocess

import numpy as np
import pytest

from oracle import oracle as O
from tests.brute import dense_attention

NAN_BITS = 0x7FC0


def _case(seed, B=4, Hkv=2, G=2, D=32, ps=16, decode=False, extra_pages=3):
    """Contiguous K/V per request, a shuffled pool, the pool before the
    append (new rows poisoned) and the packed new rows."""
    rng = np.random.default_rng(seed)
    kv = [int(x) for x in rng.integers(1, 5 * ps, size=B)]
    q = [1 if decode else int(rng.integers(0, k + 1)) for k in kv]
    C = max(-(-k // ps) for k in kv)
    n_live = sum(-(-k // ps) for k in kv)
    P = n_live + extra_pages
    perm = rng.permutation(P)
    table = np.full((B, C), -1, dtype=np.int32)
    used = 0
    for b in range(B):
        n = -(-kv[b] // ps)
        table[b, :n] = perm[used:used + n]
        used += n

    def bf16(shape):
        return (rng.standard_normal(shape).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)

    Kc = [bf16((kv[b], Hkv, D)) for b in range(B)]
    Vc = [bf16((kv[b], Hkv, D)) for b in range(B)]
    k_pool = bf16((P, ps, Hkv, D))       # unrelated content everywhere else
    v_pool = bf16((P, ps, Hkv, D))
    for b in range(B):
        old = kv[b] - q[b]                # rows already in the cache
        for p in range(-(-kv[b] // ps)):
            lo, hi = p * ps, min(kv[b], (p + 1) * ps)
            page = table[b, p]
            for r in range(lo, hi):
                if r < old:
                    k_pool[page, r - lo] = Kc[b][r]
                    v_pool[page, r - lo] = Vc[b][r]
                else:
                    k_pool[page, r - lo] = NAN_BITS
                    v_pool[page, r - lo] = NAN_BITS
    cu = np.concatenate([[0], np.cumsum(q)]).astype(np.int32)
    k_new = np.concatenate([Kc[b][kv[b] - q[b]:] for b in range(B)], axis=0)
    v_new = np.concatenate([Vc[b][kv[b] - q[b]:] for b in range(B)], axis=0)
    return dict(kv=np.array(kv, dtype=np.int32), q=q, cu=cu, table=table, Kc=Kc, Vc=Vc,
                k_pool=k_pool, v_pool=v_pool, k_new=k_new, v_new=v_new, ps=ps, P=P,
                Hkv=Hkv, G=G, D=D)


def _read_back(pool, table, kv, ps, b):
    """Rows 0..kv-1 of request b, page by page (the definition of paging)."""
    n = -(-kv // ps)
    return np.concatenate([pool[table[b, p]] for p in range(n)], axis=0)[:kv]


def _check(c, k_out, v_out, flags):
    """All three pins; returns an error string or None."""
    if flags != 0:
        return "flags %d" % flags
    live = np.zeros(k_out.shape[:2], dtype=bool)
    for b in range(len(c["kv"])):
        kvb = int(c["kv"][b])
        if not np.array_equal(_read_back(k_out, c["table"], kvb, c["ps"], b), c["Kc"][b]):
            return "K of request %d differs" % b
        if not np.array_equal(_read_back(v_out, c["table"], kvb, c["ps"], b), c["Vc"][b]):
            return "V of request %d differs" % b
        for p in range(-(-kvb // c["ps"])):
            live[c["table"][b, p], : min(c["ps"], kvb - p * c["ps"])] = True
    if not (np.array_equal(k_out[~live], c["k_pool"][~live]) and
            np.array_equal(v_out[~live], c["v_pool"][~live])):
        return "rows outside the live ranges changed"
    return None


def _attention_check(c, k_out, v_out, seed):
    """Attention over the appended pool equals attention over the contiguous
    arrays (a pool whose pages are the requests' rows in order)."""
    rng = np.random.default_rng(seed + 100)
    B, Hkv, G, D, ps = len(c["kv"]), c["Hkv"], c["G"], c["D"], c["ps"]
    T = int(c["cu"][-1])
    q = (rng.standard_normal((T, Hkv * G, D)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    scale = 1.0 / np.sqrt(D)
    o1, l1 = dense_attention(q, k_out, v_out, c["table"], c["kv"], c["cu"], scale)
    # contiguous reference: request b's rows in pages of its own, in order
    pages = []
    table2 = np.full_like(c["table"], -1)
    for b in range(B):
        n = -(-int(c["kv"][b]) // ps)
        padk = np.zeros((n * ps, Hkv, D), dtype=np.uint16)
        padv = np.zeros((n * ps, Hkv, D), dtype=np.uint16)
        padk[: c["kv"][b]] = c["Kc"][b]
        padv[: c["kv"][b]] = c["Vc"][b]
        for p in range(n):
            table2[b, p] = len(pages)
            pages.append((padk[p * ps:(p + 1) * ps], padv[p * ps:(p + 1) * ps]))
    k2 = np.stack([x[0] for x in pages])
    v2 = np.stack([x[1] for x in pages])
    o2, l2 = dense_attention(q, k2, v2, table2, c["kv"], c["cu"], scale)
    return np.array_equal(o1, o2) and np.array_equal(l1, l2)


@pytest.mark.parametrize("seed,decode", [(1, False), (2, False), (3, True), (4, False)])
def test_append_rebuilds_contiguous_kv(seed, decode):
    c = _case(seed, decode=decode)
    k_out, v_out, flags = O.append_kv(c["k_new"], c["v_new"], c["k_pool"], c["v_pool"],
                                      c["table"], c["kv"], None if decode else c["cu"])
    assert _check(c, k_out, v_out, flags) is None
    assert _attention_check(c, k_out, v_out, seed)


def test_append_geometries():
    for seed, (Hkv, D, ps) in enumerate([(1, 64, 16), (8, 128, 32), (2, 256, 128), (4, 64, 64)]):
        c = _case(10 + seed, Hkv=Hkv, D=D, ps=ps)
        k_out, v_out, flags = O.append_kv(c["k_new"], c["v_new"], c["k_pool"], c["v_pool"],
                                          c["table"], c["kv"], c["cu"])
        assert _check(c, k_out, v_out, flags) is None


def test_append_rejects_bad_requests_and_leaves_them_untouched():
    c = _case(20, B=3)
    rb = next(b for b in range(3) if c["q"][b] > 0)
    # request rb: a page id past the pool on the page of its last new row
    table = c["table"].copy()
    last_page = (int(c["kv"][rb]) - 1) // c["ps"]
    table[rb, last_page] = c["P"] + 5
    k_out, v_out, flags = O.append_kv(c["k_new"], c["v_new"], c["k_pool"], c["v_pool"],
                                      table, c["kv"], c["cu"], num_pages=c["P"])
    assert flags & 1
    # only the tokens on the bad page are skipped: the request's other pages
    # hold its rows, the bad page's rows in the pool are untouched
    for p in range(last_page):
        lo = p * c["ps"]
        assert np.array_equal(k_out[table[rb, p]][: min(c["ps"], int(c["kv"][rb]) - lo)],
                              c["Kc"][rb][lo: lo + c["ps"]])
    assert np.array_equal(k_out[c["table"][rb, last_page]], c["k_pool"][c["table"][rb, last_page]])
    # q > kv
    kv = c["kv"].copy()
    kv[rb] = c["q"][rb] - 1
    _, _, f2 = O.append_kv(c["k_new"], c["v_new"], c["k_pool"], c["v_pool"], c["table"], kv,
                           c["cu"])
    assert f2 & 2
    # malformed cu_q_lens
    bad_cu = c["cu"].copy()
    bad_cu[1] = bad_cu[2] + 1
    _, _, f3 = O.append_kv(c["k_new"], c["v_new"], c["k_pool"], c["v_pool"], c["table"],
                           c["kv"], bad_cu)
    assert f3 == 8


APPEND_MUTANTS = {
    "position_shift": ("const int j = kv - qb + i;\n            const long page",
                       "const int j = kv - qb + i - 1 + (i == 0);\n            const long page"),
    "slot_index": ("const long dst = (page * ps + j % ps) * row;",
                   "const long dst = (page * ps + (j + 1) % ps) * row;"),
    "page_column": ("const long page = page_table[(long)b * C + j / ps];",
                    "const long page = page_table[(long)b * C + j % C];"),
    "one_head_only": ("for (long e = 0; e < row; ++e) {", "for (long e = 0; e < D; ++e) {"),
    "source_row": ("const long src = (t0 + i) * row;", "const long src = (t0 + qb - 1 - i) * row;"),
}


def _append_pins_pass(lib) -> bool:
    for seed in (5, 6, 7):
        c = _case(seed, Hkv=2, D=32, ps=16)
        k_out = c["k_pool"].copy()
        v_out = c["v_pool"].copy()
        flags = lib.oracle_append_kv(
            len(c["kv"]), c["Hkv"], c["D"], c["ps"], c["table"].shape[1], 0,
            O._ptr(c["k_new"]), O._ptr(c["v_new"]), O._ptr(k_out), O._ptr(v_out),
            O._ptr(np.ascontiguousarray(c["table"])), O._ptr(c["kv"]), O._ptr(c["cu"]))
        if _check(c, k_out, v_out, int(flags)) is not None:
            return False
    return True


@pytest.mark.parametrize("name", sorted(APPEND_MUTANTS))
def test_append_pins_catch_planted_mistake(name, tmp_path):
    src = open(os.path.join(os.path.dirname(O.__file__), "oracle.c")).read()
    old, new = APPEND_MUTANTS[name]
    assert src.count(old) == 1, "mutation anchor not found: %s" % name
    c = tmp_path / ("a_%s.c" % name)
    so = tmp_path / ("a_%s.so" % name)
    c.write_text(src.replace(old, new, 1))
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread", "-o",
                           str(so), str(c), "-lm"])
    assert not _append_pins_pass(O.load_library(str(so))), "pins did not catch %s" % name


def test_unmutated_append_passes():
    assert _append_pins_pass(O._load())

"""Helpers shared by the GPU tests: run the CUDA path through the C-ABI
binding and compare it with the CPU oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

from oracle import oracle as O
from paged_kv_gqa_fmha_b200 import Plan
from paged_kv_gqa_fmha_b200 import workloads as W

# Tolerances: bf16 outputs within 1e-2 absolute, fp32 LSE within 1e-3 absolute
# (N(0,1) inputs); both against the fp64 oracle.
TOL_O = 1e-2
TOL_LSE = 1e-3


def make_plan(w, num_splits=0, num_pages=None):
    return Plan(w["B"], w["Hq"], w["Hkv"], w["D"], w["ps"], w["C"], scale=w["scale"],
                num_pages=w["P"] if num_pages is None else num_pages, num_splits=num_splits)


def gpu_run(w, plan=None, use_cu=True, **over):
    plan = plan or make_plan(w)
    args = dict(q=w["q"], k_pool=w["k_pool"], v_pool=w["v_pool"], page_table=w["page_table"],
                seq_lens=w["seq_lens"], cu_q_lens=w["cu_q_lens"] if use_cu else None)
    args.update(over)
    out, lse = plan.run(**args)
    torch.cuda.synchronize()
    return out, lse, plan


def oracle_all(w, q=None, k=None, v=None, table=None, seq=None):
    return O.paged_attention(
        W.bf16_bits(w["q"]) if q is None else q,
        W.bf16_bits(w["k_pool"]) if k is None else k,
        W.bf16_bits(w["v_pool"]) if v is None else v,
        w["page_table_cpu"].numpy() if table is None else table,
        w["seq_lens_cpu"].numpy() if seq is None else seq,
        w["cu_q_lens_cpu"].numpy(), w["scale"], num_pages=0)


def compare(out, lse, o_ref, l_ref, tol_o=TOL_O, tol_l=TOL_LSE):
    """Max abs errors over finite reference entries; -inf LSE rows must match exactly."""
    o = out.float().cpu().numpy().astype(np.float64)
    l = lse.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(o)), "non-finite output"
    err_o = float(np.max(np.abs(o - o_ref))) if o.size else 0.0
    inf_ref = np.isneginf(l_ref)
    assert np.array_equal(inf_ref, np.isneginf(l)), "LSE -inf pattern differs"
    fin = ~inf_ref
    err_l = float(np.max(np.abs(l[fin] - l_ref[fin]))) if fin.any() else 0.0
    assert err_o <= tol_o, "max |O - oracle| = %g > %g" % (err_o, tol_o)
    assert err_l <= tol_l, "max |LSE - oracle| = %g > %g" % (err_l, tol_l)
    return err_o, err_l


def sample_rows(w, n, seed=0):
    """n (token, head) rows spread over the batch, including first/last tokens."""
    rng = np.random.default_rng(seed)
    T, Hq = w["T"], w["Hq"]
    cu = w["cu_q_lens_cpu"].numpy()
    ts = set()
    for b in rng.choice(w["B"], size=min(w["B"], max(1, n // 4)), replace=False):
        ts.add(int(cu[b]))
        ts.add(int(cu[b + 1] - 1))
    while len(ts) < min(n // 2, T):
        ts.add(int(rng.integers(0, T)))
    ts = sorted(t for t in ts if 0 <= t < T)
    rows_t, rows_h = [], []
    for t in ts:
        for h in rng.choice(Hq, size=min(Hq, 2), replace=False):
            rows_t.append(t)
            rows_h.append(int(h))
    return np.array(rows_t, np.int32), np.array(rows_h, np.int32)


def oracle_rows(w, rows_t, rows_h):
    """Oracle on selected rows; copies to the host only the pages those rows'
    requests use (the pools of the full-size workloads are gigabytes)."""
    cu = w["cu_q_lens_cpu"].numpy()
    seq = w["seq_lens_cpu"].numpy()
    table = w["page_table_cpu"].numpy()
    ps = w["ps"]
    reqs = sorted(set(int(np.searchsorted(cu, t, side="right") - 1) for t in rows_t))
    pages = sorted(set(int(p) for b in reqs for p in table[b, : -(-int(seq[b]) // ps)]))
    remap = {p: i for i, p in enumerate(pages)}
    idx = torch.tensor(pages, dtype=torch.long, device=w["k_pool"].device)
    k = W.bf16_bits(w["k_pool"].index_select(0, idx))
    v = W.bf16_bits(w["v_pool"].index_select(0, idx))
    t2 = np.full_like(table, -1)
    for b in reqs:
        n = -(-int(seq[b]) // ps)
        t2[b, :n] = [remap[int(p)] for p in table[b, :n]]
    # rows of other requests are never read, so their table rows stay -1
    q = W.bf16_bits(w["q"])
    return O.paged_attention_rows(q, k, v, t2, seq, cu, w["scale"], rows_t, rows_h)

"""Helpers shared by the GPU tests: run the CUDA path through the C-ABI
binding and compare it with the CPU oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

from oracle import oracle as O
from paged_kv_gqa_fmha_b200 import Plan
from paged_kv_gqa_fmha_b200 import workloads as W

# Tolerances against the fp64 oracle: fp32 LSE within 1e-3 absolute; bf16
# outputs within 1e-2 absolute (N(0,1) inputs), except where the bf16 format
# itself cannot get that close: an output of magnitude |x| is rounded to a
# grid of spacing up to 2^-7 |x|, so even the exact result, correctly rounded,
# may be 2^-8 |x| away -- more than 1e-2 once |x| > 2.56 (two keys with
# values 4 and 4.03125 and equal weights give exactly 4.015625, 0.0156 from
# both neighbouring bf16 values; tests/test_tolerance_reading.py).  There the
# bound is bf16's unit roundoff 2^-8 |x|, with 1/128 of it as slack for the
# fp32 arithmetic before the rounding.  Below |x| = 2.54 the bound is 1e-2.
TOL_O = 1e-2
TOL_LSE = 1e-3


def o_tolerance(o_ref):
    """Per-element bound on |O_gpu - O_oracle| for bf16 outputs."""
    return np.maximum(TOL_O, 2.0 ** -8 * np.abs(o_ref) * (1.0 + 2.0 ** -7))


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


def compare(out, lse, o_ref, l_ref, tol_o=None, tol_l=TOL_LSE):
    """Max abs errors over finite reference entries; -inf LSE rows must match
    exactly.  ``tol_o`` defaults to the per-element bar ``o_tolerance``; a
    scalar replaces it.  ``tol_l`` is a scalar or an array of per-row bounds
    shaped like ``l_ref``.  Returns (max |O - ref|, max |LSE - ref|)."""
    o = out.float().cpu().numpy().astype(np.float64)
    l = lse.float().cpu().numpy().astype(np.float64)
    n_bad = int(np.count_nonzero(~np.isfinite(o)))
    assert n_bad == 0, "%d non-finite output elements" % n_bad
    d_o = np.abs(o - o_ref)
    err_o = float(np.max(d_o)) if o.size else 0.0
    inf_ref = np.isneginf(l_ref)
    assert np.array_equal(inf_ref, np.isneginf(l)), "LSE -inf pattern differs"
    fin = ~inf_ref
    d_l = np.abs(l[fin] - l_ref[fin])
    err_l = float(np.max(d_l)) if fin.any() else 0.0
    if tol_o is None:
        bound = o_tolerance(o_ref)
        if o.size and not np.all(d_o <= bound):
            i = np.unravel_index(int(np.argmax(d_o - bound)), d_o.shape)
            raise AssertionError("|O - oracle| = %g > bound %g at %s (oracle %g, gpu %g)"
                                 % (d_o[i], bound[i], i, o_ref[i], o[i]))
    else:
        assert err_o <= tol_o, "max |O - oracle| = %g > %g" % (err_o, tol_o)
    if np.ndim(tol_l) == 0:
        assert err_l <= tol_l, "max |LSE - oracle| = %g > %g" % (err_l, tol_l)
    else:
        bound = np.broadcast_to(np.asarray(tol_l, dtype=np.float64), l_ref.shape)[fin]
        worst = int(np.argmax(d_l - bound)) if d_l.size else 0
        assert d_l.size == 0 or np.all(d_l <= bound), \
            "|LSE - oracle| = %g > per-row bound %g" % (d_l[worst], bound[worst])
    return err_o, err_l

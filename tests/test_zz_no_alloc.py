"""pa_run_noalloc: the attention pass for callers that cannot allocate device
memory where they run attention -- an engine whose device memory is fully
budgeted by its own allocator (a raw cudaMalloc would bypass its accounting
and may fail late), or a serving loop that must not stall on a synchronous
allocation.  It uses the library's static scratch array instead of a plan
workspace, and reports bad request data through pa_noalloc_get_status.

The GPU tests call it through the C ABI and compare it with the plan-based
pa_run (the existing entry point) and with the fp64 oracle, on two calls in a
row with different request lengths (so the second call must not see the
first call's scratch contents), within the tolerances of the other GPU tests.
This file is collected last so that a run stopping at the first failure has
already run every other test; it passes alone in a fresh process and after
the rest of the suite.
"""
import pytest
import torch

from oracle import oracle as O
from paged_kv_gqa_fmha_b200 import binding
from paged_kv_gqa_fmha_b200 import workloads as W
from tests.gpu_common import compare, o_tolerance

TOL_O = 1e-2
TOL_LSE = 1e-3


def test_noalloc_rejects_geometry_beyond_its_scratch():
    """Checked on the host before any device work: a worst-case work list
    larger than the static scratch is refused with a clear message."""
    lib = binding.load_library()
    rc = lib.pa_run_noalloc(8, 64, 2, 256, 128, 1024, 0, 0.0, None, None, None, None, None,
                            None, None, None, None)
    assert rc == binding.PA_ERR_UNSUPPORTED
    msg = lib.pa_last_error().decode()
    assert "scratch" in msg and "pa_create_plan" in msg


def _oracle(w, use_cu=True):
    return O.paged_attention(W.bf16_bits(w["q"]), W.bf16_bits(w["k_pool"]),
                             W.bf16_bits(w["v_pool"]), w["page_table_cpu"].numpy(),
                             w["seq_lens_cpu"].numpy(),
                             w["cu_q_lens_cpu"].numpy() if use_cu else None, w["scale"])


def _noalloc(w, out, lse, use_cu=True, table=None):
    binding.run_noalloc(w["q"], w["k_pool"], w["v_pool"],
                        w["page_table"] if table is None else table, w["seq_lens"],
                        w["cu_q_lens"] if use_cu else None, out, lse, heads_kv=w["Hkv"],
                        page_size=w["ps"], capacity=w["C"], num_pages=w["P"], scale=w["scale"])


@pytest.mark.gpu
def test_noalloc_matches_plan_entry_point_on_two_calls():
    spec1 = W.custom_spec("na1", 32, 8, 128, 16, [1, 40, 1, 300], [1500, 40, 77, 700], C=128)
    spec2 = W.custom_spec("na2", 32, 8, 128, 16, [1, 1, 200, 1], [33, 2000, 900, 5], C=128)
    for spec, seed in ((spec1, 31), (spec2, 32)):
        w = W.generate(spec, seed, device="cuda")
        args = (w["q"], w["k_pool"], w["v_pool"], w["page_table"], w["seq_lens"],
                w["cu_q_lens"])
        # existing entry point (plan with its own workspace)
        plan = binding.Plan(w["B"], w["Hq"], w["Hkv"], w["D"], w["ps"], w["C"],
                            scale=w["scale"], num_pages=w["P"])
        ref_o, ref_l = plan.run(*args)
        # the no-allocation entry point, writing into caller-provided outputs
        out = torch.full_like(ref_o, float("nan"))
        lse = torch.full_like(ref_l, float("nan"))
        _noalloc(w, out, lse)
        assert binding.noalloc_status() == 0
        assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
        assert torch.max(torch.abs(out.float() - ref_o.float())).item() <= TOL_O
        assert torch.max(torch.abs(lse - ref_l)).item() <= TOL_LSE
        compare(out, lse, *_oracle(w))
        plan.close()


@pytest.mark.gpu
def test_noalloc_decode_without_cu_q_lens_or_lse():
    """One query token per request (cu_q_lens = NULL) and no LSE output, on
    two calls in a row, against the plan entry point and the oracle."""
    for kv, seed in (([1, 129, 2048, 700, 64], 33), ([300, 1, 17], 34)):
        spec = W.custom_spec("na_dec", 16, 4, 128, 32, [1] * len(kv), kv, decode_only=True)
        w = W.generate(spec, seed, device="cuda")
        plan = binding.Plan(w["B"], w["Hq"], w["Hkv"], w["D"], w["ps"], w["C"],
                            scale=w["scale"], num_pages=w["P"])
        ref_o, _ = plan.run(w["q"], w["k_pool"], w["v_pool"], w["page_table"], w["seq_lens"],
                            None)
        out = torch.full_like(ref_o, float("nan"))
        _noalloc(w, out, None, use_cu=False)
        assert binding.noalloc_status() == 0
        assert torch.max(torch.abs(out.float() - ref_o.float())).item() <= TOL_O
        o_ref, l_ref = _oracle(w, use_cu=False)
        err = (out.float().cpu().double().numpy() - o_ref)
        assert (abs(err) <= o_tolerance(o_ref)).all()
        plan.close()


@pytest.mark.gpu
def test_noalloc_status_reports_bad_page_and_next_call_clears_it():
    """A live page id past num_pages is skipped on the device and flagged:
    the accessor returns PA_STATUS_BAD_PAGE; the next clean call starts from a
    zero status word."""
    spec = W.custom_spec("na_bad", 8, 2, 64, 16, [1, 1], [40, 90], decode_only=True)
    w = W.generate(spec, 35, device="cuda")
    bad = w["page_table"].clone()
    bad[1, 2] = w["P"] + 7            # inside request 1's live pages
    out = torch.empty_like(w["q"])
    lse = torch.empty(w["T"], w["Hq"], dtype=torch.float32, device="cuda")
    _noalloc(w, out, lse, use_cu=False, table=bad)
    assert binding.noalloc_status(clear=False) & binding.STATUS_BAD_PAGE
    _noalloc(w, out, lse, use_cu=False)
    assert binding.noalloc_status() == 0
    compare(out, lse, *_oracle(w, use_cu=False))

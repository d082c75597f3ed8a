"""pa_run_noalloc: the attention pass for callers that cannot allocate device
memory (inside a region captured in global mode, or under an engine whose
device memory is fully budgeted by its own allocator).  It uses the library's
static scratch array instead of a plan workspace.

The GPU test compares it, through the C ABI, with the plan-based pa_run on two
calls in a row (different request lengths, so the second call must not see the
first call's scratch contents), within the tolerances of the other GPU tests.
This file is collected last so that a run stopping at the first failure has
already run every other test; it passes alone in a fresh process and after the
rest of the suite.
"""
import pytest
import torch

from paged_kv_gqa_fmha_b200 import binding
from paged_kv_gqa_fmha_b200 import workloads as W

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
        binding.run_noalloc(*args, out, lse, heads_kv=w["Hkv"], page_size=w["ps"],
                            capacity=w["C"], num_pages=w["P"], scale=w["scale"])
        torch.cuda.synchronize()
        assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
        assert torch.max(torch.abs(out.float() - ref_o.float())).item() <= TOL_O
        assert torch.max(torch.abs(lse - ref_l)).item() <= TOL_LSE
        plan.close()

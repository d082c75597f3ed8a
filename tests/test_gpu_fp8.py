"""GPU parity of the E4M3 (FP8) KV paths (pa_set_kv_fp8 + pa_run, through
the C ABI) with the oracle's attention over fp8 pools: decode-only runs on the
keys-as-M decode kernel, prefill, chunked prefill and mixed batches on the
one-stage kernel (codes widened to fp16 in shared memory).

The pools hold E4M3 codes of N(0,1) * 4 values (torch's round-to-nearest
quantisation); the descales are arbitrary non-powers of two so that a missing
or misplaced descale cannot pass.  Rows of each request's last page past its
KV length hold NaN codes: the kernel must never let them reach O."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from paged_kv_gqa_fmha_b200 import binding, workloads as W
from tests.gpu_common import compare

pytestmark = pytest.mark.gpu

K_SCALE, V_SCALE = 0.22, 0.31
NAN_CODE = 0x7F


def _codes(shape, gen, dev):
    x = torch.randn(shape, generator=gen, device=dev, dtype=torch.float32) * 4
    return x.to(torch.float8_e4m3fn).view(torch.uint8)


def _poison_tails(k8, v8, w):
    """NaN codes in the rows past kv_len of every request's last page."""
    table = w["page_table_cpu"].numpy()
    ps = w["ps"]
    for b, kv in enumerate(w["seq_lens_cpu"].tolist()):
        if kv % ps:
            page = int(table[b, (kv - 1) // ps])
            k8[page, kv % ps:] = NAN_CODE
            v8[page, kv % ps:] = NAN_CODE


def _fp8_workload(spec, seed, dev="cuda"):
    w = W.generate(spec, seed, device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(seed + 7)
    k8 = _codes(tuple(w["k_pool"].shape), g, dev)
    v8 = _codes(tuple(w["v_pool"].shape), g, dev)
    _poison_tails(k8, v8, w)
    return w, k8, v8


def _plan(w, num_splits=0):
    plan = binding.Plan(w["B"], w["Hq"], w["Hkv"], w["D"], w["ps"], w["C"], scale=w["scale"],
                        num_pages=w["P"], num_splits=num_splits)
    plan.set_kv_fp8(True, K_SCALE, V_SCALE)
    return plan


def _oracle(w, k8, v8):
    return O.paged_attention_fp8(W.bf16_bits(w["q"]), k8.cpu().numpy(), v8.cpu().numpy(),
                                 K_SCALE, V_SCALE, w["page_table_cpu"].numpy(),
                                 w["seq_lens_cpu"].numpy(), w["cu_q_lens_cpu"].numpy(),
                                 w["scale"])


def _run(plan, w, k8, v8, use_cu=False):
    out, lse = plan.run(w["q"], k8, v8, w["page_table"], w["seq_lens"],
                        w["cu_q_lens"] if use_cu else None)
    torch.cuda.synchronize()
    assert plan.status() == 0
    return out, lse


GEOMS = [  # seed, D, G, ps, Hkv, B, max_kv
    (1, 128, 4, 16, 2, 5, 700),
    (2, 128, 8, 32, 1, 3, 1000),
    (3, 128, 16, 64, 2, 4, 600),
    (4, 128, 32, 16, 1, 3, 500),
    (5, 128, 1, 128, 2, 4, 900),
    (6, 256, 4, 16, 2, 3, 500),
    (7, 256, 32, 64, 1, 2, 400),
    (8, 128, 5, 32, 2, 3, 400),
]


@pytest.mark.parametrize("other_kernel", [False, True])
@pytest.mark.parametrize("seed,D,G,ps,Hkv,B,max_kv", GEOMS)
def test_fp8_decode_matches_oracle(seed, D, G, ps, Hkv, B, max_kv, other_kernel):
    """Decode-only runs over E4M3 pools on the default kernel (the decode
    kernel at head_dim 128, the one-stage kernel at 256) and on the other one
    (pa_set_decode_kernel)."""
    rng = np.random.default_rng(seed)
    spec = W.random_small(rng, D=D, ps=ps, G=G, Hkv=Hkv, B=B, max_kv=max_kv, prefill=False)
    w, k8, v8 = _fp8_workload(spec, 500 + seed)
    plan = _plan(w)
    if other_kernel:
        plan.set_decode_kernel(D == 256)
    out, lse = _run(plan, w, k8, v8)
    o_ref, l_ref = _oracle(w, k8, v8)
    compare(out, lse, o_ref, l_ref)


@pytest.mark.parametrize("fused", [False, True])
def test_fp8_splits_and_tile_edges(fused):
    """KV lengths on and next to the 128-key tile edges, forced splits, with
    the separate merge kernel and with the fused merge."""
    kv = [1, 127, 128, 129, 255, 256, 257, 1000]
    spec = W.custom_spec("fp8_edges", 16, 2, 128, 32, [1] * len(kv), kv)
    w, k8, v8 = _fp8_workload(spec, 77)
    o_ref, l_ref = _oracle(w, k8, v8)
    for splits in (1, 3):
        plan = _plan(w, num_splits=splits)
        plan.set_fused_merge(fused)
        out, lse = _run(plan, w, k8, v8)
        compare(out, lse, o_ref, l_ref)


def test_fp8_descales_are_applied():
    """The same codes with other descales: still the oracle's answer (a
    kernel that ignored either descale could not match both)."""
    rng = np.random.default_rng(91)
    spec = W.random_small(rng, D=128, ps=16, G=4, Hkv=2, B=3, max_kv=300, prefill=False)
    w, k8, v8 = _fp8_workload(spec, 91)
    plan = _plan(w)
    for ks, vs in ((K_SCALE, V_SCALE), (0.05, 0.9)):
        plan.set_kv_fp8(True, ks, vs)
        out, lse = _run(plan, w, k8, v8)
        o_ref, l_ref = O.paged_attention_fp8(
            W.bf16_bits(w["q"]), k8.cpu().numpy(), v8.cpu().numpy(), ks, vs,
            w["page_table_cpu"].numpy(), w["seq_lens_cpu"].numpy(),
            w["cu_q_lens_cpu"].numpy(), w["scale"])
        compare(out, lse, o_ref, l_ref)


def test_fp8_rejections():
    rng = np.random.default_rng(3)
    spec = W.random_small(rng, D=128, ps=16, G=4, Hkv=2, B=2, max_kv=100, prefill=True)
    w, k8, v8 = _fp8_workload(spec, 3)
    plan = _plan(w)
    with pytest.raises(binding.PAError) as e:
        plan.set_kv_fp8(True, 0.0, 1.0)
    assert e.value.code == binding.PA_ERR_INVALID
    p64 = binding.Plan(2, 8, 2, 64, 16, 8)
    with pytest.raises(binding.PAError) as e:
        p64.set_kv_fp8(True, 1.0, 1.0)
    assert e.value.code == binding.PA_ERR_UNSUPPORTED


PREFILL_GEOMS = [  # seed, D, G, ps, Hkv, q_lens, kv_lens
    (11, 128, 4, 16, 2, [300, 1, 77, 129, 1], [300, 900, 500, 129, 64]),
    (12, 128, 8, 64, 1, [64, 200, 1], [64, 1000, 40]),
    (13, 128, 1, 128, 2, [100, 31], [700, 31]),
    (14, 128, 32, 32, 1, [9, 4, 1], [9, 300, 800]),
    (15, 256, 4, 32, 2, [90, 1, 40], [90, 500, 300]),
    (16, 256, 2, 128, 1, [130, 3], [400, 3]),
    (17, 128, 3, 16, 2, [50, 1, 2], [50, 60, 500]),
]


@pytest.mark.parametrize("seed,D,G,ps,Hkv,q_lens,kv_lens", PREFILL_GEOMS)
def test_fp8_prefill_and_mixed_match_oracle(seed, D, G, ps, Hkv, q_lens, kv_lens):
    """Causal prefill, chunked prefill (kv > q) and decode rows in one batch
    over E4M3 pools, on the one-stage kernel, against the oracle; NaN codes
    in every request's tail slots must not reach O."""
    spec = W.custom_spec("fp8_pf", G * Hkv, Hkv, D, ps, q_lens, kv_lens)
    w, k8, v8 = _fp8_workload(spec, 700 + seed)
    out, lse = _run(_plan(w), w, k8, v8, use_cu=True)
    compare(out, lse, *_oracle(w, k8, v8))


@pytest.mark.parametrize("splits,fused,two_stage", [(0, False, False), (3, False, False),
                                                    (3, True, False), (0, False, True)])
def test_fp8_mixed_batch_options(splits, fused, two_stage):
    """A mixed batch over E4M3 pools with KV splits for its single-token
    requests (separate or fused merge), and with the two-stage prefill option
    on (E4M3 runs stay on the one-stage kernel)."""
    spec = W.custom_spec("fp8_mix", 32, 8, 128, 16, [200, 1, 1, 64, 1], [200, 1500, 90, 700, 3000])
    w, k8, v8 = _fp8_workload(spec, 41)
    plan = _plan(w, num_splits=splits)
    plan.set_fused_merge(fused)
    if two_stage:
        plan.set_two_stage_prefill(True)
    out, lse = _run(plan, w, k8, v8, use_cu=True)
    compare(out, lse, *_oracle(w, k8, v8))


def test_fp8_prefill_non_causal_and_descales():
    """Non-causal mode and a second pair of descales on the same codes."""
    spec = W.custom_spec("fp8_nc", 16, 4, 128, 32, [100, 1, 37], [300, 200, 37])
    w, k8, v8 = _fp8_workload(spec, 43)
    plan = _plan(w)
    plan.set_causal(False)
    for ks, vs in ((K_SCALE, V_SCALE), (0.05, 0.9)):
        plan.set_kv_fp8(True, ks, vs)
        out, lse = _run(plan, w, k8, v8, use_cu=True)
        compare(out, lse, *_oracle_nc(w, k8, v8, ks, vs))


def _oracle_nc(w, k8, v8, ks, vs):
    """Non-causal reference over E4M3 pools: every query token becomes a
    one-token request with its own request's page-table row and KV length, so
    the oracle's (end-aligned causal) fp8 entry lets it see all of its keys."""
    cu = w["cu_q_lens_cpu"].numpy()
    seq = w["seq_lens_cpu"].numpy()
    table = w["page_table_cpu"].numpy()
    q = W.bf16_bits(w["q"])
    T = w["T"]
    rows_req = np.concatenate([np.full(cu[b + 1] - cu[b], b, dtype=np.int64) for b in range(w["B"])])
    o, l = O.paged_attention_fp8(q, k8.cpu().numpy(), v8.cpu().numpy(), ks, vs,
                                 table[rows_req], seq[rows_req], np.arange(T + 1, dtype=np.int32),
                                 w["scale"])
    return o, l


@pytest.mark.slow
def test_fp8_full_size_llama_decode_every_element():
    """The Llama-3.1-8B decode shape at full size (the timed launch), fp8 pools
    quantised on the device: every element of O and LSE against the oracle
    over the whole fp8 pools."""
    w = W.generate(W.CONFIGS["llama8b_decode"], W.default_seed("llama8b_decode"), device="cuda")
    k8 = (w["k_pool"].float() * 4).to(torch.float8_e4m3fn).view(torch.uint8)
    v8 = (w["v_pool"].float() * 4).to(torch.float8_e4m3fn).view(torch.uint8)
    del w["k_pool"], w["v_pool"]
    plan = _plan(w)
    out, lse = _run(plan, w, k8, v8)
    o_ref, l_ref = _oracle(w, k8, v8)
    err_o, err_l = compare(out, lse, o_ref, l_ref)
    print("llama8b_decode/fp8: %d elements, max|O-oracle| %.3e, max|LSE-oracle| %.3e"
          % (out.numel(), err_o, err_l))


@pytest.mark.slow
@pytest.mark.parametrize("name", ["llama8b_causal_prefill", "unified_mixed"])
def test_fp8_full_size_prefill_and_mixed_every_element(name):
    """The causal-prefill and mixed-batch workloads at full size over E4M3 pools
    (quantised on the device): every element of O and LSE against the oracle."""
    w = W.generate(W.CONFIGS[name], W.default_seed(name), device="cuda")
    k8 = (w["k_pool"].float() * 4).to(torch.float8_e4m3fn).view(torch.uint8)
    v8 = (w["v_pool"].float() * 4).to(torch.float8_e4m3fn).view(torch.uint8)
    del w["k_pool"], w["v_pool"]
    plan = _plan(w)
    out, lse = _run(plan, w, k8, v8, use_cu=True)
    o_ref, l_ref = _oracle(w, k8, v8)
    err_o, err_l = compare(out, lse, o_ref, l_ref)
    print("%s/fp8: %d elements, max|O-oracle| %.3e, max|LSE-oracle| %.3e"
          % (name, out.numel(), err_o, err_l))


# q_lens / kv_lens of a batch with three multi-block requests (G = 4: 32 tokens
# per block) and two decode rows; page size 16, so the multi-block requests
# own 19, 32 and 10 pages
WIDE_Q = [300, 1, 200, 150, 1]
WIDE_KV = [300, 900, 500, 150, 2000]


# launches: the scheduler, [the widening pass and the bf16 kernel,] the E4M3
# one-stage kernel and the decode kernel (the batch's two decode rows)
@pytest.mark.parametrize("max_pages,launches", [(-1, 5), (0, 3), (19, 5), (20, 5), (61, 5)])
def test_fp8_widened_requests_match_oracle(max_pages, launches):
    """Requests of two or more query blocks over E4M3 pools are widened once
    into the bf16 scratch pool (in request order while their pages fit) and
    run on the bf16 kernel; the rest stay on the E4M3 one-stage kernel.  Every
    capacity -- all widened (-1, 61), none (0), only the first request (19:
    its pages exactly; 20: one spare page, the next request does not fit) --
    matches the oracle, and the run enqueues the widening pass and the bf16
    launch only when the capacity is not 0."""
    spec = W.custom_spec("fp8_wide", 16, 4, 128, 16, WIDE_Q, WIDE_KV)
    w, k8, v8 = _fp8_workload(spec, 47)
    o_ref, l_ref = _oracle(w, k8, v8)
    plan = _plan(w, num_splits=1)
    plan.set_kv_fp8_widen(max_pages)
    for _ in range(2):      # the second run reuses the scratch pool
        plan.profile_start(1)
        out, lse = _run(plan, w, k8, v8, use_cu=True)
        _, n, per_run = plan.profile_read()
        assert n == 1 and per_run == launches
        compare(out, lse, o_ref, l_ref)


def test_fp8_widen_paths_agree_and_d256():
    """head_dim 256 over E4M3 pools with and without widening: both match the
    oracle (the two paths round q and P differently, so they agree only
    within the tolerances)."""
    spec = W.custom_spec("fp8_wide256", 8, 2, 256, 32, [70, 1, 9], [300, 400, 9])
    w, k8, v8 = _fp8_workload(spec, 53)
    o_ref, l_ref = _oracle(w, k8, v8)
    for max_pages in (-1, 0):
        plan = _plan(w)
        plan.set_kv_fp8_widen(max_pages)
        out, lse = _run(plan, w, k8, v8, use_cu=True)
        compare(out, lse, o_ref, l_ref)


def test_fp8_widened_bad_page_is_reported():
    """A page id outside [0, num_pages) inside a widened request's pages is
    reported as PA_STATUS_BAD_PAGE (the page reads as zeros), and the plan
    keeps working: the next run with a valid table matches the oracle."""
    spec = W.custom_spec("fp8_wide_bad", 16, 4, 128, 16, WIDE_Q, WIDE_KV)
    w, k8, v8 = _fp8_workload(spec, 59)
    plan = _plan(w)
    bad = w["page_table"].clone()
    bad[0, 3] = w["P"] + 5
    plan.run(w["q"], k8, v8, bad, w["seq_lens"], w["cu_q_lens"])
    torch.cuda.synchronize()
    assert plan.status() & binding.STATUS_BAD_PAGE
    out, lse = _run(plan, w, k8, v8, use_cu=True)
    compare(out, lse, *_oracle(w, k8, v8))


def test_fp8_widen_rejects_bad_capacity():
    spec = W.custom_spec("fp8_wide_rej", 8, 2, 128, 16, [40], [40])
    w, _, _ = _fp8_workload(spec, 61)
    plan = _plan(w)
    with pytest.raises(binding.PAError) as e:
        plan.set_kv_fp8_widen(-2)
    assert e.value.code == binding.PA_ERR_INVALID


def test_fp8_batch_larger_than_scheduler_cache():
    """3 200 requests over E4M3 pools (more than the scheduler's 3 072 cached
    unit offsets): widened multi-block requests, one-token rows on the decode
    kernel's segment (some of them split) and the rest, against the oracle."""
    rng = np.random.default_rng(3201)
    B = 3200
    q_lens = [1] * B
    kv_lens = [int(x) for x in rng.integers(1, 120, size=B)]
    for b in range(0, B, 97):
        q_lens[b] = kv_lens[b] = int(rng.integers(40, 160))
    for b in range(3, B, 211):         # one-block chunks (q_len 2..8) stay on the E4M3 kernel
        q_lens[b] = int(rng.integers(2, 9))
        kv_lens[b] = max(kv_lens[b], q_lens[b])
    for b in range(5, B, 401):
        kv_lens[b] = 3000
    spec = W.custom_spec("fp8_big_batch", 8, 2, 128, 16, q_lens, kv_lens)
    w, k8, v8 = _fp8_workload(spec, 3201)
    out, lse = _run(_plan(w), w, k8, v8, use_cu=True)
    compare(out, lse, *_oracle(w, k8, v8))


@pytest.mark.parametrize("decode_kernel", [True, False])
def test_fp8_mixed_decode_rows_on_either_kernel(decode_kernel):
    """Decode rows of a mixed batch over E4M3 pools run on the decode kernel
    (default at head_dim 128: a second segment of the work list) or, with
    pa_set_decode_kernel(0), on the one-stage kernel; both match the oracle,
    with KV splits and the launch count of each path."""
    spec = W.custom_spec("fp8_segs", 32, 8, 128, 16, [300, 1, 1, 5, 1, 64],
                         [300, 2500, 90, 700, 1, 64])
    w, k8, v8 = _fp8_workload(spec, 67)
    plan = _plan(w, num_splits=3)
    plan.set_decode_kernel(decode_kernel)
    plan.profile_start(1)
    out, lse = _run(plan, w, k8, v8, use_cu=True)
    _, n, per_run = plan.profile_read()
    # scheduler, widening, bf16 kernel (widened), E4M3 one-stage, [decode kernel], merge
    assert per_run == (6 if decode_kernel else 5)
    compare(out, lse, *_oracle(w, k8, v8))


def test_fp8_run_allocates_nothing():
    """pa_set_kv_fp8 allocates the widening scratch pool; pa_run over E4M3
    pools with cu_q_lens (widening pass included) then allocates no device
    memory: free memory is unchanged across runs with preallocated outputs."""
    spec = W.custom_spec("fp8_noalloc", 16, 4, 128, 16, WIDE_Q, WIDE_KV)
    w, k8, v8 = _fp8_workload(spec, 71)
    plan = _plan(w)
    out = torch.empty_like(w["q"])
    lse = torch.empty(w["T"], w["Hq"], device="cuda")
    args = (w["q"], k8, v8, w["page_table"], w["seq_lens"], w["cu_q_lens"])
    plan.run(*args, out=out, lse=lse)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        plan.run(*args, out=out, lse=lse)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert plan.status() == 0
    compare(out, lse, *_oracle(w, k8, v8))

"""GPU parity: the CUDA path, called through the C ABI, against the fp64 CPU
oracle on the same seeded inputs.  Bar: max |O - oracle| <= 1e-2 on bf16
outputs and max |LSE - oracle| <= 1e-3 on the fp32 LSE (N(0,1) inputs)."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from paged_kv_gqa_fmha_b200 import workloads as W
from tests.gpu_common import compare, gpu_run, make_plan, oracle_all

pytestmark = pytest.mark.gpu


def gen(spec, seed):
    return W.generate(spec, seed, device="cuda")


# ------------------------------------------------------------------ tiny decode (config 1)
def test_tiny_decode_matches_oracle_and_golden():
    w = gen(W.CONFIGS["tiny_decode"], W.default_seed("tiny_decode"))
    # the golden fixture was drawn on the CPU generator: regenerate values there
    wc = W.generate(W.CONFIGS["tiny_decode"], W.default_seed("tiny_decode"))
    for key in ("q", "k_pool", "v_pool"):
        w[key] = wc[key].cuda()
    out, lse, _ = gpu_run(w, use_cu=False)
    o_ref, l_ref = oracle_all(w)
    compare(out, lse, o_ref, l_ref)
    import os
    g = np.array([float(x) for x in open(os.path.join(os.path.dirname(__file__), "golden",
                                                      "tiny_decode.txt"))
                  if not x.startswith("#")])
    assert np.max(np.abs(lse.cpu().numpy().reshape(-1) - g[:8])) <= 1e-3
    assert np.max(np.abs(out.float().cpu().numpy().reshape(-1) - g[8:])) <= 1e-2


# ------------------------------------------------------------------ small geometries, all rows
GEOMS = [  # (D, ps, G, Hkv, prefill)
    (128, 16, 4, 2, False), (128, 16, 4, 2, True), (64, 16, 2, 2, True), (64, 64, 8, 1, False),
    (256, 128, 32, 1, False), (256, 32, 2, 2, True), (128, 64, 1, 3, True), (128, 128, 16, 2, True),
    (64, 32, 32, 1, True), (256, 16, 8, 1, True), (128, 32, 3, 2, True), (128, 16, 6, 1, False),
]


@pytest.mark.parametrize("D,ps,G,Hkv,prefill", GEOMS)
def test_small_geometry_all_rows(D, ps, G, Hkv, prefill):
    rng = np.random.default_rng(D * 7 + ps * 3 + G + Hkv + int(prefill))
    spec = W.random_small(rng, D=D, ps=ps, G=G, Hkv=Hkv, B=int(rng.integers(1, 6)),
                          max_kv=700, prefill=prefill)
    w = gen(spec, 500 + D + ps + G)
    out, lse, _ = gpu_run(w)
    compare(out, lse, *oracle_all(w))


def test_prefill_many_tiles_ragged():
    """Several 128-row query blocks and KV tiles, with a ragged tail and chunked
    prefill (kv > q)."""
    spec = W.custom_spec("ragged", 32, 8, 128, 16, [300, 1, 77, 129], [300, 901, 500, 129])
    w = gen(spec, 11)
    out, lse, _ = gpu_run(w)
    compare(out, lse, *oracle_all(w))


def test_decode_without_cu_q_lens():
    spec = W.custom_spec("dec", 32, 8, 128, 16, [1] * 9, [1, 15, 16, 17, 127, 128, 129, 600, 2048])
    w = gen(spec, 12)
    out, lse, _ = gpu_run(w, use_cu=False)
    compare(out, lse, *oracle_all(w))


@pytest.mark.parametrize("D,ps,G,splits", [(128, 16, 4, 0), (128, 64, 1, 1), (128, 128, 8, 3),
                                            (128, 32, 16, 0), (128, 16, 32, 2), (256, 128, 32, 0),
                                            (256, 16, 2, 5), (256, 64, 12, 1)])
def test_decode_kernel(D, ps, G, splits):
    """Decode-only runs (no cu_q_lens) on the keys-as-M decode kernel: against
    the oracle, and against the one-stage kernel on the same inputs.  Lengths
    cover a single key, tails on both sides of the 128-key tile and of a page,
    and requests long enough to be split."""
    kv = [1, 15, 127, 128, 129, 300, 2048, 4097]
    spec = W.custom_spec("deck", G * 2, 2, D, ps, [1] * len(kv), kv, decode_only=True)
    w = gen(spec, 60 + D + ps + G + splits)
    plan = make_plan(w, num_splits=splits)
    plan.set_decode_kernel(True)
    out, lse, _ = gpu_run(w, plan, use_cu=False)
    assert plan.status() == 0
    compare(out, lse, *oracle_all(w))
    ref = make_plan(w, num_splits=splits)
    ref.set_decode_kernel(False)
    out1, lse1, _ = gpu_run(w, ref, use_cu=False)
    assert torch.max(torch.abs(out.float() - out1.float())).item() <= 1e-2
    assert torch.max(torch.abs(lse - lse1)).item() <= 1e-3


@pytest.mark.parametrize("D,ps,G", [(128, 16, 4), (128, 64, 1), (64, 32, 8), (128, 128, 3)])
def test_two_stage_prefill_kernel(D, ps, G):
    """The optional two-stage kernel (query-block pairs) against the oracle,
    with odd block counts, partial pairs, chunked prefill and decode rows in
    the same batch (those stay on the one-stage kernel)."""
    spec = W.custom_spec("pairs", 2 * G, 2, D, ps, [300, 1, 129, 77, 5], [300, 700, 400, 77, 900])
    w = gen(spec, 30 + D + ps + G)
    plan = make_plan(w)
    plan.set_two_stage_prefill(True)
    out, lse, _ = gpu_run(w, plan)
    assert plan.status() == 0
    compare(out, lse, *oracle_all(w))


@pytest.mark.parametrize("scale_q", [1.0, 30.0])
def test_two_stage_long_requests(scale_q):
    """The two-stage kernel over many 128-key tiles per item (the slot ring
    wraps many times), a chunked-prefill request whose keys start far before
    its queries, and (q x 30) a peaked softmax that rescales O in TMEM (bound
    of the large-logit test below)."""
    spec = W.custom_spec("pairs_long", 16, 4, 128, 64, [1024, 200, 33], [1024, 1500, 2100])
    w = gen(spec, 41)
    if scale_q != 1.0:
        w["q"] = (w["q"].float() * scale_q).to(torch.bfloat16)
    plan = make_plan(w)
    plan.set_two_stage_prefill(True)
    out, lse, _ = gpu_run(w, plan)
    assert plan.status() == 0
    o_ref, l_ref = oracle_all(w)
    if scale_q == 1.0:
        compare(out, lse, o_ref, l_ref)
    else:
        vmax = float(w["v_pool"].float().abs().max())
        compare(out, lse, o_ref, l_ref, tol_o=2.0 ** -7 * vmax,
                tol_l=1e-3 * np.maximum(1.0, np.abs(l_ref)))


# ------------------------------------------------------------------ split-KV (a8)
@pytest.mark.parametrize("splits,fused", [(1, True), (2, True), (7, True), (0, True), (2, False),
                                          (7, False), (0, False)])
def test_split_invariance(splits, fused):
    """Split counts give the same result, merged by the last split warp
    (fused) or by the separate merge kernel."""
    spec = W.custom_spec("split", 16, 2, 128, 32, [1, 1, 3, 1], [3000, 1200, 2500, 64])
    w = gen(spec, 13)
    plan = make_plan(w, num_splits=splits)
    plan.set_fused_merge(fused)
    out, lse, _ = gpu_run(w, plan)
    compare(out, lse, *oracle_all(w))
    ref_plan = make_plan(w, num_splits=1)
    out1, lse1, _ = gpu_run(w, ref_plan)
    assert torch.max(torch.abs(out.float() - out1.float())).item() <= 1e-2
    assert torch.max(torch.abs(lse - lse1)).item() <= 1e-3


def test_split_long_gqa32_head_dim_256():
    spec = W.custom_spec("split256", 64, 2, 256, 128, [1, 1], [20000, 7000])
    w = gen(spec, 14)
    for splits in (0, 5):
        for fused in (True, False):
            plan = make_plan(w, num_splits=splits)
            plan.set_fused_merge(fused)
            out, lse, _ = gpu_run(w, plan)
            assert plan.status() == 0
            compare(out, lse, *oracle_all(w))


@pytest.mark.parametrize("D,decode_kernel", [(128, True), (128, False), (256, False)])
def test_up_to_64_splits(D, decode_kernel):
    """One long request on one KV head: the automatic split count reaches its
    cap of 64 (the merge's second LSE lane, splits 33..64, is in use); the
    result must match the oracle and the unsplit run."""
    spec = W.custom_spec("split64", 8, 1, D, 64, [1], [60000])
    w = gen(spec, 15)
    plan = make_plan(w)
    plan.set_decode_kernel(decode_kernel)
    assert plan.max_splits == 64
    out, lse, _ = gpu_run(w, plan, use_cu=False)
    assert plan.status() == 0
    compare(out, lse, *oracle_all(w))
    one = make_plan(w, num_splits=1)
    out1, lse1, _ = gpu_run(w, one, use_cu=False)
    assert torch.max(torch.abs(out.float() - out1.float())).item() <= 1e-2
    assert torch.max(torch.abs(lse - lse1)).item() <= 1e-3


@pytest.mark.parametrize("G,splits,fused", [(4, 0, False), (8, 3, False), (4, 3, True),
                                            (32, 0, False)])
def test_mixed_batch_splits_and_edges(G, splits, fused):
    """Mixed batch: single-token requests long enough to be split (merge
    kernel or fused merge), a single key, a tile edge, prefill requests of one
    and of several query blocks, two tokens over two keys."""
    q = [1, 200, 1, 1, 37, 1, 130, 1, 2]
    kv = [3000, 600, 129, 1, 500, 2048, 130, 77, 2]
    spec = W.custom_spec("mixed_edges", 2 * G, 2, 128, 32, q, kv)
    w = gen(spec, 17 + G + splits)
    plan = make_plan(w, num_splits=splits)
    plan.set_fused_merge(fused)
    out, lse, _ = gpu_run(w, plan)
    assert plan.status() == 0
    compare(out, lse, *oracle_all(w))


# ------------------------------------------------------------------ invariants on the GPU path
def test_page_permutation_invariance_gpu():
    spec = W.custom_spec("perm", 16, 4, 64, 16, [1, 40, 1], [500, 300, 77])
    w = gen(spec, 15)
    out1, lse1, _ = gpu_run(w)
    perm = torch.randperm(w["P"], generator=torch.Generator().manual_seed(3)).cuda()
    k2 = torch.empty_like(w["k_pool"])
    v2 = torch.empty_like(w["v_pool"])
    k2[perm] = w["k_pool"]
    v2[perm] = w["v_pool"]
    t = w["page_table"].long()
    t2 = torch.where(t >= 0, perm[t.clamp(min=0)], t).to(torch.int32)
    out2, lse2, _ = gpu_run(w, k_pool=k2, v_pool=v2, page_table=t2)
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2)


@pytest.mark.parametrize("fill", [-1, 2**31 - 1])
def test_poisoned_tails_and_columns_gpu(fill):
    """NaN in tail slots of the last live page and in every unused page; table
    columns past the live pages set to -1 or INT32_MAX: output unchanged and
    finite (pages never read, V tail sanitised)."""
    spec = W.custom_spec("poison", 16, 2, 128, 16, [1, 20, 1, 5], [37, 100, 64, 5])
    w = gen(spec, 16)
    out1, lse1, _ = gpu_run(w)
    k, v = w["k_pool"].clone(), w["v_pool"].clone()
    table = w["page_table"].clone()
    seq = w["seq_lens_cpu"].tolist()
    live = set()
    for b, kv in enumerate(seq):
        n = -(-kv // 16)
        pages = w["page_table_cpu"][b, :n].tolist()
        live.update(pages)
        tail = kv - (n - 1) * 16
        k[pages[-1], tail:] = float("nan")
        v[pages[-1], tail:] = float("nan")
        table[b, n:] = fill
    for p in range(w["P"]):
        if p not in live:
            k[p] = float("nan")
            v[p] = float("nan")
    plan = make_plan(w, num_pages=0)
    out2, lse2, _ = gpu_run(w, plan, k_pool=k, v_pool=v, page_table=table)
    assert torch.isfinite(out2.float()).all() and torch.isfinite(lse2).all()
    assert torch.max(torch.abs(out1.float() - out2.float())).item() == 0.0
    assert torch.max(torch.abs(lse1 - lse2)).item() == 0.0


def test_metadata_mutation_between_runs_same_plan():
    """One plan, new request metadata bound on every run."""
    spec = W.custom_spec("mut", 16, 2, 128, 32, [1, 7, 1], [900, 400, 33])
    w = gen(spec, 17)
    plan = make_plan(w)
    out, lse, _ = gpu_run(w, plan)
    compare(out, lse, *oracle_all(w))
    seq2 = torch.tensor([513, 7, 1], dtype=torch.int32)
    w2 = dict(w)
    w2["seq_lens"] = seq2.cuda()
    w2["seq_lens_cpu"] = seq2
    out2, lse2, _ = gpu_run(w2, plan)
    compare(out2, lse2, *oracle_all(w2))


def test_cuda_graph_replay_with_new_seq_lens():
    spec = W.custom_spec("graph", 32, 8, 128, 16, [1] * 6, [100, 2000, 37, 64, 1500, 999])
    w = gen(spec, 18)
    plan = make_plan(w)
    seq = w["seq_lens"].clone()
    out = torch.empty_like(w["q"])
    lse = torch.empty(w["T"], w["Hq"], device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        plan.run(w["q"], w["k_pool"], w["v_pool"], w["page_table"], seq, None, out=out, lse=lse)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        plan.run(w["q"], w["k_pool"], w["v_pool"], w["page_table"], seq, None, out=out, lse=lse)
    for new in ([100, 2000, 37, 64, 1500, 999], [1, 1999, 38, 17, 1024, 1000]):
        seq.copy_(torch.tensor(new, dtype=torch.int32))
        g.replay()
        torch.cuda.synchronize()
        w2 = dict(w)
        w2["seq_lens_cpu"] = torch.tensor(new, dtype=torch.int32)
        w2["cu_q_lens_cpu"] = torch.arange(7, dtype=torch.int32)
        compare(out, lse, *oracle_all(w2))


def test_status_bits_for_bad_requests():
    spec = W.custom_spec("bad", 8, 2, 64, 16, [1, 1], [40, 30])
    w = gen(spec, 19)
    plan = make_plan(w)
    assert plan.status() == 0
    gpu_run(w, plan)
    assert plan.status() == 0
    table = w["page_table"].clone()
    table[0, 1] = w["P"] + 5                       # live column out of the pool
    gpu_run(w, plan, page_table=table)
    assert plan.status() & 1
    seq = torch.tensor([40, 10**6], dtype=torch.int32, device="cuda")
    gpu_run(w, plan, seq_lens=seq)
    assert plan.status() & 4


def test_rows_without_visible_keys_get_zero_and_minus_inf():
    """q_b > kv_b (invalid): the first q_b - kv_b rows see no key."""
    spec = W.custom_spec("qgt", 8, 2, 64, 16, [6, 3], [4, 40])
    w = gen(spec, 20)
    plan = make_plan(w)
    out, lse, _ = gpu_run(w, plan)
    assert plan.status() & 2
    compare(out, lse, *oracle_all(w))


def test_empty_requests():
    spec = W.custom_spec("empty", 8, 2, 128, 16, [0, 5, 0, 1], [0, 5, 17, 1])
    w = gen(spec, 21)
    out, lse, _ = gpu_run(w)
    compare(out, lse, *oracle_all(w))


def test_zero_query_closed_form_gpu():
    """q = 0: O is the mean of the visible V rows, LSE = ln(#visible keys)."""
    spec = W.custom_spec("q0", 16, 4, 128, 16, [50, 1], [300, 200])
    w = gen(spec, 22)
    w["q"] = torch.zeros_like(w["q"])
    out, lse, _ = gpu_run(w)
    compare(out, lse, *oracle_all(w))
    cu = w["cu_q_lens_cpu"]
    n = np.array([300 - 50 + i + 1 for i in range(50)] + [200], dtype=np.float64)
    assert np.max(np.abs(lse.cpu().numpy()[:, 0] - np.log(n))) < 1e-4


def test_large_logits_gpu():
    """q x 30: a very peaked softmax must neither overflow nor lose accuracy
    beyond what bf16 allows.  bf16 carries an 8-bit significand, so rounding
    to nearest has relative error <= 2^-8: with P rounded to bf16 for P V
    (the row sum keeps fp32 P) the weighted sum moves by <= 2^-8 max|V|, and
    rounding O to bf16 adds <= 2^-8 |O| <= 2^-8 max|V|, so |O - O_ref| is
    bounded by 2^-7 max|V|; N(0,1) inputs with moderate logits stay far below
    that, but a one-hot softmax comes near it."""
    spec = W.custom_spec("big", 16, 4, 128, 32, [64, 1], [700, 900])
    w = gen(spec, 23)
    w["q"] = (w["q"].float() * 30.0).to(torch.bfloat16)
    out, lse, _ = gpu_run(w)
    o_ref, l_ref = oracle_all(w)
    vmax = float(w["v_pool"].float().abs().max())
    # LSE: fp32 scores and an fp32 row sum give a relative error far below
    # 1e-3 of each row's own |LSE| (the bar of 1e-3 scaled per row, not by
    # the largest row of the batch)
    compare(out, lse, o_ref, l_ref, tol_o=2.0 ** -7 * vmax,
            tol_l=1e-3 * np.maximum(1.0, np.abs(l_ref)))


# ------------------------------------------------------------------ rows with few keys
def _vis_counts(w, causal=True):
    """Visible keys of every (token) row: [T]."""
    cu = w["cu_q_lens_cpu"].numpy()
    seq = w["seq_lens_cpu"].numpy()
    out = np.zeros(w["T"], dtype=np.int64)
    for b in range(w["B"]):
        qb = cu[b + 1] - cu[b]
        for i in range(qb):
            out[cu[b] + i] = seq[b] if not causal else min(seq[b], max(0, seq[b] - qb + i + 1))
    return out


@pytest.mark.parametrize("kind", ["one_stage", "two_stage", "decode_kernel", "d256", "d64",
                                  "decode_fp8"])
def test_few_key_rows_are_correctly_rounded(kind):
    """Rows that see fewer than 64 keys in total take the compensated P V
    (P_hi + P_lo, both 16-bit): their outputs equal the oracle's exact result
    correctly rounded to bf16, up to fp32 slack of 2^-14 max(|O|, 1) (the
    fp32 sums run over terms P_j V_j of magnitude up to max |V|, so the slack
    does not shrink with |O|) -- far inside the 2^-9 sum_j P_j |V_j| that
    rounding P alone would leave.  Rows with more keys meet the usual bar."""
    if kind in ("decode_kernel", "decode_fp8"):
        kv = [2, 3, 4, 5, 7, 8, 13, 31, 63, 64, 2, 3, 9]
        spec = W.custom_spec("few_dec", 16, 4, 128, 16, [1] * len(kv), kv, decode_only=True)
    elif kind == "d256":
        spec = W.custom_spec("few256", 8, 2, 256, 32, [40, 70, 3], [40, 70, 90])
    elif kind == "d64":
        spec = W.custom_spec("few64", 16, 2, 64, 16, [64, 100, 33], [64, 100, 50])
    else:
        spec = W.custom_spec("few", 16, 4, 128, 16, [64] * 6 + [150], [64] * 6 + [150])
    w = gen(spec, 60 + len(kind))
    plan = make_plan(w)
    use_cu = not spec.decode_only
    if kind == "two_stage":
        plan.set_two_stage_prefill(True)
    if kind == "decode_fp8":
        k8 = (w["k_pool"].float() * 4).to(torch.float8_e4m3fn)
        v8 = (w["v_pool"].float() * 4).to(torch.float8_e4m3fn)
        plan.set_kv_fp8(True, 0.25, 0.25)
        out, lse = plan.run(w["q"], k8.view(torch.uint8), v8.view(torch.uint8),
                            w["page_table"], w["seq_lens"], None)
        torch.cuda.synchronize()
        o_ref, l_ref = O.paged_attention_fp8(
            W.bf16_bits(w["q"]), k8.view(torch.uint8).cpu().numpy(),
            v8.view(torch.uint8).cpu().numpy(), 0.25, 0.25, w["page_table_cpu"].numpy(),
            w["seq_lens_cpu"].numpy(), w["cu_q_lens_cpu"].numpy(), w["scale"])
    else:
        out, lse, _ = gpu_run(w, plan, use_cu=use_cu)
        o_ref, l_ref = oracle_all(w)
    assert plan.status() == 0
    compare(out, lse, o_ref, l_ref)
    few = _vis_counts(w) < 64
    o = out.float().cpu().numpy().astype(np.float64)[few]
    x = o_ref[few]
    rounded = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    slack = 2.0 ** -14 * np.maximum(np.abs(x), 1.0)
    excess = np.abs(o - x) - (np.abs(rounded - x) + slack)
    assert np.all(excess <= 0), "few-key row off its correctly rounded value by %g" % excess.max()


# ------------------------------------------------------------------ full-size configs, every element
# Each of the five workloads at its full size, in the launch configuration
# bench.py times (default plan), and the opt-in two-stage kernel where it
# applies: every element of O and LSE against the oracle over the whole
# output, plus a count of non-finite elements (must be 0).  The oracle runs
# once per workload on all host cores.
FULL_SIZE = [("tiny_decode", ()), ("llama8b_decode", ()),
             ("llama8b_causal_prefill", ("two_stage",)), ("unified_mixed", ("two_stage",)),
             ("long_gqa32_decode", ("decode_kernel",))]


@pytest.mark.slow
@pytest.mark.parametrize("name,extra", FULL_SIZE, ids=[n for n, _ in FULL_SIZE])
def test_full_size_config_every_element(name, extra):
    spec = W.CONFIGS[name]
    w = gen(spec, W.default_seed(name))
    use_cu = not spec.decode_only
    runs = []
    plan = make_plan(w)
    out, lse, _ = gpu_run(w, plan, use_cu=use_cu)
    assert plan.status() == 0
    runs.append(("default", out.cpu(), lse.cpu()))
    if "two_stage" in extra:
        plan.set_two_stage_prefill(True)
        out, lse, _ = gpu_run(w, plan, use_cu=use_cu)
        assert plan.status() == 0
        runs.append(("two_stage", out.cpu(), lse.cpu()))
        plan.set_two_stage_prefill(False)
    if "decode_kernel" in extra:
        plan.set_decode_kernel(True)
        out, lse, _ = gpu_run(w, plan, use_cu=use_cu)
        assert plan.status() == 0
        runs.append(("decode_kernel", out.cpu(), lse.cpu()))
    plan.close()
    del out, lse
    o_ref, l_ref = oracle_all(w)
    for label, o, l in runs:
        err_o, err_l = compare(o, l, o_ref, l_ref)
        print("%s/%s: %d elements, max|O-oracle| %.3e, max|LSE-oracle| %.3e, non-finite 0"
              % (name, label, o.numel(), err_o, err_l))


# ------------------------------------------------------------------ mask mode, table stride
@pytest.mark.parametrize("D,ps,G,pairs,splits", [(128, 16, 4, False, 0), (64, 32, 8, False, 0),
                                                 (256, 64, 2, False, 3), (128, 64, 1, True, 0),
                                                 (64, 16, 3, True, 0)])
def test_non_causal_mode(D, ps, G, pairs, splits):
    """pa_set_causal(plan, 0): every row sees its request's whole KV, on the
    one-stage kernel (with and without splits) and the two-stage kernel."""
    spec = W.custom_spec("nc", 2 * G, 2, D, ps, [300, 1, 129, 77, 0], [300, 700, 400, 500, 90])
    w = gen(spec, 80 + D + ps + G)
    plan = make_plan(w, num_splits=splits)
    plan.set_causal(False)
    if pairs:
        plan.set_two_stage_prefill(True)
    out, lse, _ = gpu_run(w, plan)
    assert plan.status() == 0
    o_ref, l_ref = O.paged_attention(W.bf16_bits(w["q"]), W.bf16_bits(w["k_pool"]),
                                     W.bf16_bits(w["v_pool"]), w["page_table_cpu"].numpy(),
                                     w["seq_lens_cpu"].numpy(), w["cu_q_lens_cpu"].numpy(),
                                     w["scale"], causal=False)
    compare(out, lse, o_ref, l_ref)


@pytest.mark.parametrize("decode_only", [False, True])
def test_page_table_row_stride(decode_only):
    """The K plane of a [B, 2, C] table (row stride 2C) passed without a copy;
    plane 1 holds garbage that must never be read."""
    q = [1] * 6 if decode_only else [40, 1, 300, 1, 17, 1]
    spec = W.custom_spec("stride", 32, 8, 128, 16, q, [900, 1500, 300, 64, 1200, 7],
                         decode_only=decode_only)
    w = gen(spec, 90 + int(decode_only))
    B, C = w["page_table_cpu"].shape
    t3 = torch.full((B, 2, C), -12345, dtype=torch.int32)
    t3[:, 0, :] = w["page_table_cpu"]
    t3 = t3.cuda()
    plan = make_plan(w)
    out, lse, _ = gpu_run(w, plan, use_cu=not decode_only, page_table=t3[:, 0, :])
    assert plan.status() == 0
    compare(out, lse, *oracle_all(w))


# ------------------------------------------------------------------ bounded waits
@pytest.mark.parametrize("limit_us", [500, 5000])
def test_wait_timeout_sets_status_and_releases_other_roles(limit_us):
    """A wait on an mbarrier that nothing arrives at gives up after its limit
    and sets PA_STATUS_TIMEOUT; a second wait with the production limit (2 s)
    leaves through the abort flag right after; the context stays usable."""
    from paged_kv_gqa_fmha_b200 import binding
    status, t_short, t_long = binding.selftest_wait_timeout(limit_us)
    assert status & binding.STATUS_TIMEOUT
    assert limit_us <= t_short < limit_us + 50000
    assert t_long < t_short + 50000          # far below the 2 s production limit
    spec = W.custom_spec("after_timeout", 8, 2, 128, 16, [1, 1], [100, 300])
    w = gen(spec, 19)
    out, lse, plan = gpu_run(w, use_cu=False)
    assert plan.status() == 0
    compare(out, lse, *oracle_all(w))


def test_batch_larger_than_scheduler_cache():
    """More requests (3 200) than the scheduler keeps unit offsets for in shared
    memory (3 072), so its later requests' offsets come from global memory:
    decode rows, multi-block prefill requests and a few long-KV rows that split,
    every element against the oracle."""
    rng = np.random.default_rng(3200)
    B = 3200
    q_lens = [1] * B
    kv_lens = [int(x) for x in rng.integers(1, 120, size=B)]
    for b in range(0, B, 97):          # prefill requests of two or more blocks
        q_lens[b] = kv_lens[b] = int(rng.integers(40, 160))
    for b in range(5, B, 401):         # long decode rows
        kv_lens[b] = 3000
    spec = W.custom_spec("big_batch", 8, 2, 128, 16, q_lens, kv_lens)
    w = gen(spec, 3200)
    out, lse, _ = gpu_run(w)
    compare(out, lse, *oracle_all(w))

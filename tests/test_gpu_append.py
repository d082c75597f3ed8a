"""GPU parity of the paged KV append (pa_append_kv, through the C ABI) with
the oracle: the pools must match bit for bit, the status word must flag what
was skipped, and attention over the appended pools must match the oracle's
attention over its own appended pools."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from paged_kv_gqa_fmha_b200 import binding
from tests.gpu_common import TOL_LSE, o_tolerance
from tests.test_append_pins import _case

pytestmark = pytest.mark.gpu


def _t(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def _plan(c, num_pages=None):
    B, C = c["table"].shape
    return binding.Plan(B, c["Hkv"] * c["G"], c["Hkv"], c["D"], c["ps"], C,
                        num_pages=c["P"] if num_pages is None else num_pages)


_DEFAULT = object()


def _gpu_append(c, table=None, kv=None, cu=_DEFAULT, num_pages=None):
    table = c["table"] if table is None else table
    kv = c["kv"] if kv is None else kv
    cu = c["cu"] if cu is _DEFAULT else cu
    plan = _plan(c, num_pages)
    kp = _t(c["k_pool"], torch.bfloat16)
    vp = _t(c["v_pool"], torch.bfloat16)
    plan.append_kv(_t(c["k_new"], torch.bfloat16), _t(c["v_new"], torch.bfloat16), kp, vp,
                   _t(table), _t(kv), None if cu is None else _t(cu))
    st = plan.status()
    return kp.view(torch.int16).cpu().numpy().view(np.uint16), \
        vp.view(torch.int16).cpu().numpy().view(np.uint16), st, plan


@pytest.mark.parametrize("seed,Hkv,D,ps,decode", [(1, 2, 64, 16, False), (2, 8, 128, 32, False),
                                                  (3, 2, 256, 128, False), (4, 4, 128, 16, True),
                                                  (5, 1, 64, 64, False)])
def test_append_matches_oracle(seed, Hkv, D, ps, decode):
    c = _case(seed, B=5, Hkv=Hkv, D=D, ps=ps, decode=decode)
    cu = None if decode else c["cu"]
    k_ref, v_ref, flags = O.append_kv(c["k_new"], c["v_new"], c["k_pool"], c["v_pool"],
                                      c["table"], c["kv"], cu)
    assert flags == 0
    k_out, v_out, st, _ = _gpu_append(c, cu=cu)
    assert st == 0
    assert np.array_equal(k_out, k_ref) and np.array_equal(v_out, v_ref)


def test_append_skips_and_flags_like_the_oracle():
    c = _case(21, B=4, Hkv=2, D=64, ps=16)
    rb = next(b for b in range(4) if c["q"][b] > 0)
    table = c["table"].copy()
    table[rb, (int(c["kv"][rb]) - 1) // 16] = c["P"] + 3           # bad page on new rows
    k_ref, v_ref, flags = O.append_kv(c["k_new"], c["v_new"], c["k_pool"], c["v_pool"], table,
                                      c["kv"], c["cu"], num_pages=c["P"])
    k_out, v_out, st, _ = _gpu_append(c, table=table)
    assert flags & 1 and st & binding.STATUS_BAD_PAGE
    assert np.array_equal(k_out, k_ref) and np.array_equal(v_out, v_ref)
    kv = c["kv"].copy()
    kv[rb] = c["q"][rb] - 1                                        # q > kv
    k_ref, v_ref, flags = O.append_kv(c["k_new"], c["v_new"], c["k_pool"], c["v_pool"],
                                      c["table"], kv, c["cu"])
    k_out, v_out, st, _ = _gpu_append(c, kv=kv)
    assert flags & 2 and st & binding.STATUS_Q_GT_KV
    assert np.array_equal(k_out, k_ref) and np.array_equal(v_out, v_ref)
    bad_cu = c["cu"].copy()
    bad_cu[1] = bad_cu[2] + 1                                      # decreasing
    k_out, v_out, st, _ = _gpu_append(c, cu=bad_cu)
    assert st & binding.STATUS_BAD_CU_Q
    assert np.array_equal(k_out, c["k_pool"]) and np.array_equal(v_out, c["v_pool"])


def test_append_then_attention():
    """Append on the GPU, then attend over the same pools with pa_run: the
    result matches the oracle's attention over the oracle-appended pools."""
    c = _case(31, B=6, Hkv=2, G=4, D=128, ps=16)
    k_ref, v_ref, _ = O.append_kv(c["k_new"], c["v_new"], c["k_pool"], c["v_pool"], c["table"],
                                  c["kv"], c["cu"])
    plan = _plan(c)
    kp = _t(c["k_pool"], torch.bfloat16)
    vp = _t(c["v_pool"], torch.bfloat16)
    table, kv, cu = _t(c["table"]), _t(c["kv"]), _t(c["cu"])
    plan.append_kv(_t(c["k_new"], torch.bfloat16), _t(c["v_new"], torch.bfloat16), kp, vp,
                   table, kv, cu)
    T = int(c["cu"][-1])
    rng = np.random.default_rng(7)
    qb = (rng.standard_normal((T, c["Hkv"] * c["G"], c["D"])).astype(np.float32)
          .view(np.uint32) >> 16).astype(np.uint16)
    out, lse = plan.run(_t(qb, torch.bfloat16), kp, vp, table, kv, cu)
    torch.cuda.synchronize()
    assert plan.status() == 0
    o_ref, l_ref = O.paged_attention(qb, k_ref, v_ref, c["table"], c["kv"], c["cu"],
                                     1.0 / np.sqrt(c["D"]))
    o = out.float().cpu().numpy()
    l = lse.cpu().numpy()
    fin = np.isfinite(l_ref)
    assert np.all(np.abs(o - o_ref) <= o_tolerance(o_ref))
    assert np.max(np.abs(l[fin] - l_ref[fin])) <= TOL_LSE


def test_append_full_prefill_size():
    """32 requests x 1024 new tokens (the causal-prefill shape), bit for bit."""
    rng = np.random.default_rng(41)
    B, Hkv, D, ps, kvl = 32, 8, 128, 64, 1024
    C = kvl // ps
    P = B * C + 64
    perm = rng.permutation(P).astype(np.int32)
    table = perm[: B * C].reshape(B, C)
    kv = np.full(B, kvl, dtype=np.int32)
    cu = np.arange(0, (B + 1) * kvl, kvl, dtype=np.int32)
    k_new = rng.integers(0, 1 << 16, size=(B * kvl, Hkv, D), dtype=np.uint16)
    v_new = rng.integers(0, 1 << 16, size=(B * kvl, Hkv, D), dtype=np.uint16)
    k_pool = rng.integers(0, 1 << 16, size=(P, ps, Hkv, D), dtype=np.uint16)
    v_pool = rng.integers(0, 1 << 16, size=(P, ps, Hkv, D), dtype=np.uint16)
    k_ref, v_ref, flags = O.append_kv(k_new, v_new, k_pool, v_pool, table, kv, cu)
    assert flags == 0
    plan = binding.Plan(B, 4 * Hkv, Hkv, D, ps, C, num_pages=P)
    kp, vp = _t(k_pool, torch.bfloat16), _t(v_pool, torch.bfloat16)
    plan.append_kv(_t(k_new, torch.bfloat16), _t(v_new, torch.bfloat16), kp, vp, _t(table),
                   _t(kv), _t(cu))
    assert plan.status() == 0
    assert np.array_equal(kp.view(torch.int16).cpu().numpy().view(np.uint16), k_ref)
    assert np.array_equal(vp.view(torch.int16).cpu().numpy().view(np.uint16), v_ref)


def test_append_with_strided_table():
    """pa_append_kv through the K plane of a [B, 2, C] table (row stride 2C)."""
    c = _case(51, B=5, Hkv=2, D=64, ps=16)
    k_ref, v_ref, flags = O.append_kv(c["k_new"], c["v_new"], c["k_pool"], c["v_pool"],
                                      c["table"], c["kv"], c["cu"])
    assert flags == 0
    B, C = c["table"].shape
    t3 = np.full((B, 2, C), -777, dtype=np.int32)
    t3[:, 0, :] = c["table"]
    t3 = _t(t3)
    plan = _plan(c)
    kp = _t(c["k_pool"], torch.bfloat16)
    vp = _t(c["v_pool"], torch.bfloat16)
    plan.append_kv(_t(c["k_new"], torch.bfloat16), _t(c["v_new"], torch.bfloat16), kp, vp,
                   t3[:, 0, :], _t(c["kv"]), _t(c["cu"]))
    assert plan.status() == 0
    assert np.array_equal(kp.view(torch.int16).cpu().numpy().view(np.uint16), k_ref)
    assert np.array_equal(vp.view(torch.int16).cpu().numpy().view(np.uint16), v_ref)

"""Pins of the oracle's FP8 (E4M3) KV path.

The decoder is checked code by code against torch's float8_e4m3fn (an
implementation written elsewhere), and attention over fp8 pools against the
brute-force dense attention run on pools dequantized by torch.  The descales
are pinned by their closed-form effect: k_scale multiplies every score (the
same as multiplying the softmax scale), v_scale multiplies O and leaves LSE
unchanged.  A planted mistake in the decoder is caught."""
import os
import subprocess

import numpy as np
import pytest
import torch

from oracle import oracle as O
from paged_kv_gqa_fmha_b200 import workloads as W
from tests.brute import bits_to_f64, dense_attention_values


def _torch_decode(codes):
    return torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(
        torch.float8_e4m3fn).to(torch.float64).numpy()


def test_every_code_decodes_like_torch():
    c = np.arange(256, dtype=np.uint8)
    a, b = O.e4m3_decode(c), _torch_decode(c)
    assert np.array_equal(np.isnan(a), np.isnan(b))
    assert np.array_equal(a[~np.isnan(a)], b[~np.isnan(b)])
    assert np.nanmax(a) == 448.0 and np.nanmin(a) == -448.0


def _fp8_case(seed, decode=True):
    rng = np.random.default_rng(seed)
    spec = W.random_small(rng, prefill=not decode, max_kv=220, D=128)
    w = W.generate(spec, seed, device="cpu")
    # fp8 codes of values N(0,1) * 4 (torch's round-to-nearest quantisation)
    def codes(shape):
        x = torch.from_numpy(rng.standard_normal(shape).astype(np.float32) * 4)
        return x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    k8 = codes(tuple(w["k_pool"].shape))
    v8 = codes(tuple(w["v_pool"].shape))
    return w, k8, v8


@pytest.mark.parametrize("seed,decode", [(1, True), (2, True), (3, False), (4, False)])
def test_fp8_attention_matches_brute_force(seed, decode):
    w, k8, v8 = _fp8_case(seed, decode)
    ks, vs = 0.37, 1.9
    q = W.bf16_bits(w["q"])
    table, seq, cu = (w["page_table_cpu"].numpy(), w["seq_lens_cpu"].numpy(),
                      w["cu_q_lens_cpu"].numpy())
    o, l = O.paged_attention_fp8(q, k8, v8, ks, vs, table, seq, cu, w["scale"])
    ob, lb = dense_attention_values(bits_to_f64(q), _torch_decode(k8) * ks,
                                    _torch_decode(v8) * vs, table, seq, cu, w["scale"])
    assert np.max(np.abs(o - ob)) < 1e-10
    fin = np.isfinite(lb)
    assert np.max(np.abs(l[fin] - lb[fin])) < 1e-10


def test_descales_act_as_stated():
    w, k8, v8 = _fp8_case(11)
    q = W.bf16_bits(w["q"])
    table, seq, cu = (w["page_table_cpu"].numpy(), w["seq_lens_cpu"].numpy(),
                      w["cu_q_lens_cpu"].numpy())
    o1, l1 = O.paged_attention_fp8(q, k8, v8, 0.5, 1.0, table, seq, cu, w["scale"])
    o2, l2 = O.paged_attention_fp8(q, k8, v8, 1.0, 1.0, table, seq, cu, w["scale"] * 0.5)
    assert np.max(np.abs(o1 - o2)) < 1e-12 and np.max(np.abs(l1 - l2)) < 1e-12
    o3, l3 = O.paged_attention_fp8(q, k8, v8, 0.5, 3.0, table, seq, cu, w["scale"])
    assert np.max(np.abs(o3 - 3.0 * o1)) < 1e-12 and np.max(np.abs(l3 - l1)) < 1e-12


def test_pin_catches_a_wrong_exponent_bias(tmp_path):
    src = open(os.path.join(os.path.dirname(O.__file__), "oracle.c")).read()
    old = "else v = (1.0 + m / 8.0) * ldexp(1.0, e - 7);"
    assert src.count(old) == 1
    c = tmp_path / "f8.c"
    so = tmp_path / "f8.so"
    c.write_text(src.replace(old, "else v = (1.0 + m / 8.0) * ldexp(1.0, e - 8);", 1))
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread", "-o",
                           str(so), str(c), "-lm"])
    lib = O.load_library(str(so))
    codes = np.arange(256, dtype=np.uint8)
    out = np.zeros(256)
    lib.oracle_e4m3_decode(O._ptr(codes), 256, O._ptr(out))
    ok = np.isnan(out) | (out == _torch_decode(codes))
    assert not ok.all()

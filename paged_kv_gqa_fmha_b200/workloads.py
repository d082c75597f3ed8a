"""Seeded synthetic inputs for paged-KV attention.

This module only draws inputs: request lengths, a shuffled page pool, the
page table and N(0,1) bf16 tensors.  It contains no attention arithmetic, so
both the CUDA path's tests/benchmark and the CPU oracle can be fed from it.

Draw order for one workload (one ``torch.Generator`` seeded with ``seed``):
request lengths, the page permutation, then q, k_pool, v_pool.  Lengths and
the permutation are always drawn on the CPU so that the metadata is the same
whatever device the values are drawn on.  Values are drawn as fp32 N(0,1)
and rounded to bf16 (round to nearest even).

Layouts (the flash-attention paged "NHD" layout):
    q          bf16  [T, Hq, D]       packed varlen queries
    k_pool     bf16  [P, ps, Hkv, D]
    v_pool     bf16  [P, ps, Hkv, D]
    page_table int32 [B, C]           -1 in columns past the live pages
    seq_lens   int32 [B]              whole KV length, this step's tokens included
    cu_q_lens  int32 [B+1]            query offsets (cu_q_lens[0] = 0)
"""
from __future__ import annotations

import dataclasses
import math
from typing import Callable, Optional, Sequence

import numpy as np
import torch


@dataclasses.dataclass
class Spec:
    """Shape of one workload.  ``lens`` draws (q_lens, kv_lens) from a CPU
    generator; ``pool_pages`` maps the number of live pages to the pool size."""
    name: str
    Hq: int
    Hkv: int
    D: int
    ps: int
    C: int
    lens: Callable[[torch.Generator], tuple]
    pool_pages: Callable[[int], int]
    decode_only: bool = False   # cu_q_lens may be passed as NULL (every q_b = 1)


def _pool_125(n_live: int) -> int:
    return int(math.ceil(1.25 * n_live))


def _uniform(g: torch.Generator, lo: int, hi: int, n: int) -> list:
    """Integers uniform in [lo, hi], inclusive."""
    return torch.randint(lo, hi + 1, (n,), generator=g).tolist()


def _tiny_decode_lens(g):
    return [1, 1], [37, 64]


def _llama_decode_lens(g):
    kv = _uniform(g, 1024, 2048, 256)
    return [1] * 256, kv


def _causal_prefill_lens(g):
    return [1024] * 32, [1024] * 32


def _mixed_lens(g):
    ctx = _uniform(g, 1000, 1100, 248)
    q = [1000] * 8 + [1] * 248
    kv = [1000] * 8 + [c + 1 for c in ctx]
    return q, kv


def _long_decode_lens(g):
    kv = _uniform(g, 32768, 131072, 8)
    return [1] * 8, kv


CONFIGS = {
    "tiny_decode": Spec("tiny_decode", 4, 2, 64, 16, 4, _tiny_decode_lens, lambda n: 12,
                        decode_only=True),
    "llama8b_decode": Spec("llama8b_decode", 32, 8, 128, 16, 128, _llama_decode_lens, _pool_125,
                           decode_only=True),
    "llama8b_causal_prefill": Spec("llama8b_causal_prefill", 32, 8, 128, 64, 16,
                                   _causal_prefill_lens, _pool_125),
    "unified_mixed": Spec("unified_mixed", 32, 8, 128, 16, 69, _mixed_lens, _pool_125),
    "long_gqa32_decode": Spec("long_gqa32_decode", 64, 2, 256, 128, 1024, _long_decode_lens,
                              _pool_125, decode_only=True),
}
CONFIG_IDS = {name: i + 1 for i, name in enumerate(CONFIGS)}   # seed = 1000 + id


def default_seed(name: str) -> int:
    return 1000 + CONFIG_IDS[name]


def custom_spec(name, Hq, Hkv, D, ps, q_lens: Sequence[int], kv_lens: Sequence[int],
                C: Optional[int] = None, pool_extra: float = 1.25, decode_only=False) -> Spec:
    q_lens, kv_lens = list(q_lens), list(kv_lens)
    if C is None:
        C = max(1, max((k + ps - 1) // ps for k in kv_lens))
    return Spec(name, Hq, Hkv, D, ps, C, lambda g: (q_lens, kv_lens),
                lambda n: max(1, int(math.ceil(pool_extra * n))), decode_only=decode_only)


def generate(spec: Spec, seed: int, device="cpu", values: bool = True) -> dict:
    """Draw one workload.  Returns a dict of tensors (values on ``device``,
    metadata always also on the CPU under the ``*_cpu`` keys)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    q_lens, kv_lens = spec.lens(g)
    B = len(q_lens)
    n_pages = [(k + spec.ps - 1) // spec.ps for k in kv_lens]
    n_live = sum(n_pages)
    P = spec.pool_pages(n_live)
    if P < n_live:
        raise ValueError("pool of %d pages cannot hold %d live pages" % (P, n_live))
    if max(n_pages) > spec.C:
        raise ValueError("capacity %d columns < %d live pages" % (spec.C, max(n_pages)))
    perm = torch.randperm(P, generator=g).to(torch.int32)
    table = torch.full((B, spec.C), -1, dtype=torch.int32)
    off = 0
    for b, n in enumerate(n_pages):
        table[b, :n] = perm[off:off + n]
        off += n
    cu = torch.zeros(B + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(q_lens, dtype=torch.int64), 0).to(torch.int32)
    T = int(cu[-1])
    seq = torch.tensor(kv_lens, dtype=torch.int32)

    out = dict(spec=spec, seed=seed, B=B, T=T, P=P, Hq=spec.Hq, Hkv=spec.Hkv, D=spec.D,
               ps=spec.ps, C=spec.C, scale=1.0 / math.sqrt(spec.D),
               q_lens=q_lens, kv_lens=kv_lens,
               page_table_cpu=table, seq_lens_cpu=seq, cu_q_lens_cpu=cu)
    dev = torch.device(device)
    out["page_table"] = table.to(dev)
    out["seq_lens"] = seq.to(dev)
    out["cu_q_lens"] = cu.to(dev)
    if values:
        gv = g if dev.type == "cpu" else torch.Generator(device=dev)
        if dev.type != "cpu":
            gv.manual_seed(seed)
        out["q"] = _normal_bf16((T, spec.Hq, spec.D), gv, dev)
        out["k_pool"] = _normal_bf16((P, spec.ps, spec.Hkv, spec.D), gv, dev)
        out["v_pool"] = _normal_bf16((P, spec.ps, spec.Hkv, spec.D), gv, dev)
    return out


def _normal_bf16(shape, g, dev, chunk=1 << 26):
    """N(0,1) drawn in fp32 and rounded to bf16, in chunks to bound memory."""
    n = int(np.prod(shape))
    out = torch.empty(n, dtype=torch.bfloat16, device=dev)
    for a in range(0, n, chunk):
        e = min(n, a + chunk)
        out[a:e] = torch.randn(e - a, generator=g, device=dev, dtype=torch.float32).to(
            torch.bfloat16)
    return out.view(shape)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (CPU copy)."""
    assert t.dtype == torch.bfloat16
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def random_small(rng: np.random.Generator, name="rand", D=None, ps=None, G=None, Hkv=None,
                 B=None, max_kv=300, prefill=None) -> Spec:
    """A small random geometry for parity and pin tests."""
    D = D or int(rng.choice([64, 128, 256]))
    ps = ps or int(rng.choice([16, 32, 64, 128]))
    G = G or int(rng.choice([1, 2, 4, 8]))
    Hkv = Hkv or int(rng.choice([1, 2]))
    B = B or int(rng.integers(1, 5))
    kv = [int(rng.integers(1, max_kv + 1)) for _ in range(B)]
    if prefill is None:
        prefill = bool(rng.integers(0, 2))
    q = [int(rng.integers(1, k + 1)) if prefill else 1 for k in kv]
    return custom_spec(name, G * Hkv, Hkv, D, ps, q, kv)

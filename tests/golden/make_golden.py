"""Writes tests/golden/tiny_decode.txt: the oracle's outputs for the tiny
decode workload (B=2, 4 query heads, 2 KV heads, head_dim 64, page size 16,
seq_lens {37, 64}, capacity 4, a 12-page pool assigned by a seeded
permutation, seed 1001).  Calls only the CPU oracle and the seeded input
generator; never the CUDA path.

    python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import oracle as O                      # noqa: E402
from paged_kv_gqa_fmha_b200 import workloads as W   # noqa: E402


def main():
    name = "tiny_decode"
    w = W.generate(W.CONFIGS[name], W.default_seed(name))
    out, lse = O.paged_attention(W.bf16_bits(w["q"]), W.bf16_bits(w["k_pool"]),
                                 W.bf16_bits(w["v_pool"]), w["page_table_cpu"].numpy(),
                                 w["seq_lens_cpu"].numpy(), None, w["scale"],
                                 num_pages=w["P"], nthreads=1)
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), name + ".txt")
    with open(path, "w") as f:
        f.write("# oracle output, tiny decode workload, seed %d\n" % w["seed"])
        f.write("# page_table %s\n" % w["page_table_cpu"].numpy().tolist())
        f.write("# seq_lens %s\n" % w["seq_lens_cpu"].numpy().tolist())
        f.write("# lse [T=2, Hq=4]\n")
        for v in lse.reshape(-1):
            f.write("%.17g\n" % v)
        f.write("# out [T=2, Hq=4, D=64]\n")
        for v in out.reshape(-1):
            f.write("%.17g\n" % v)
    print("wrote", path)


if __name__ == "__main__":
    main()

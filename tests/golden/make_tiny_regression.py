"""Writes tests/golden/tiny_regression.json from the fp64 CPU oracle alone.

Regression values for the tiny fp32 workload (64 docs x 512 tokens): chunk
CSR, a sample of pooled vectors, routing indices and scores, and a sample of
decode outputs.  Run:  python tests/golden/make_tiny_regression.py
"""
import json
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
import oracle  # noqa: E402
from workloads import TINY_F32, gen  # noqa: E402


def compute():
    w = TINY_F32
    x = gen.generate(w)
    kp, vp, krp = oracle.encode(x["doc_tok_off"], x["k_tok"], x["v_tok"], x["kr_tok"], w.chunk,
                                w.rope_theta)
    coff = oracle.chunk_offsets(x["doc_tok_off"], w.chunk)
    kpt, vpt, krt = (torch.from_numpy(a).float() for a in (kp, vp, krp))
    idx, sc = oracle.route(x["qr"], coff, krt, w.top_k, w.n_kv_heads)
    out = oracle.decode(x["q"], idx, coff, kpt, vpt, x["local_off"], x["local_k"], x["local_v"],
                        w.top_k, w.rope_theta, w.n_kv_heads)
    rows = [0, 7, 100, 511]
    return {
        "workload": w.name,
        "chunk_off_last": int(coff[-1]),
        "k_pool_rows": {str(r): kp[r, 1, :8].tolist() for r in rows},
        "v_pool_rows": {str(r): vp[r, 2, :8].tolist() for r in rows},
        "kr_pool_rows": {str(r): krp[r, 3, :8].tolist() for r in rows},
        "route_idx": idx[0].tolist(),
        "route_score": sc[0].tolist(),
        "decode_out_t0_h0": out[0, 0, 0].tolist(),
        "decode_out_t3_h3": out[0, 3, 3].tolist(),
    }


if __name__ == "__main__":
    res = compute()
    res["about"] = ("Oracle-only regression values for the tiny fp32 workload; written by "
                    "tests/golden/make_tiny_regression.py, which calls nothing but the oracle "
                    "and the seeded input generator.")
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_regression.json"), "w") as f:
        json.dump(res, f, indent=1)

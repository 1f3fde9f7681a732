"""The pages' block-size ablation, restated on the synthetic 64K workload with the oracle.

Step 5 Preview pages (mo.ai.kr, "Step 5 Preview agentic work design", section "model structure
and training stability"): compressing the shared index keys into blocks of 8 makes indexing and
selection eightfold cheaper, and the block version (k = 4096 tokens, 512 blocks) kept slightly
more of the relevant tokens than token-level selection (k = 2048). This script computes, for both
settings on the same seeded inputs and a strided sample of query rows:

  * scored candidates per row (sum over t of the candidates j < floor(t/B));
  * selected tokens per (row, group) (|U|);
  * token coverage: the fraction of each (row, head)'s top-2048 keys by exact q.k (ties to the
    lower position) that the selection contains (oracle_coverage), averaged over rows with
    t >= 4096 where it is not trivially 1.

Test infrastructure: runs the fp64 oracle only (no GPU). The inputs are synthetic: q and k are
independent of the index keys' topics, so coverage here measures how much of the dense top-2048
a random-looking selection of the right size holds, not the pages' trained model.

Usage: python oracle/ablation_coverage.py [--stride 2048] [--threads 0]
"""
import argparse
import os
import sys
import time

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import oracle  # noqa: E402
from sgqa_inputs import CONFIGS, gen_full, gen_rows  # noqa: E402


def run(stride: int, threads: int) -> dict:
    oracle.build()
    res = {}
    rows_t = np.arange(4096 + stride // 2, CONFIGS["64k_b8"].T, stride)
    for name in ("64k_b8", "64k_b1"):
        cfg = CONFIGS[name]
        dm = oracle.dims_of(cfg)
        t0 = time.time()
        k_idx = gen_full(cfg, "k_idx")
        k = gen_full(cfg, "k")
        rows = np.stack([np.zeros_like(rows_t), rows_t], axis=1).astype(np.int32)
        qi = gen_rows(cfg, "q_idx", 0, rows_t).reshape(len(rows), -1)
        q = gen_rows(cfg, "q", 0, rows_t).reshape(len(rows), -1)
        kbar = oracle.compress(dm, k_idx, threads)
        sel, _, _ = oracle.select(dm, kbar, rows, qi, threads)
        cov = oracle.coverage(dm, rows, q, k, sel, 2048, threads)
        u = []
        for i, t in enumerate(rows_t):
            for g in range(cfg.G):
                blocks = sel[i, g][sel[i, g] >= 0]
                u.append(sum(min(cfg.B, t + 1 - j * cfg.B) for j in blocks))
        scored = sum(t // cfg.B for t in range(cfg.T))
        res[name] = {"B": cfg.B, "k": cfg.k, "rows": len(rows), "coverage": float(cov.mean()),
                     "selected_tokens_mean": float(np.mean(u)), "scored_candidates_per_group": scored,
                     "seconds": time.time() - t0}
    res["scored_ratio_b1_over_b8"] = res["64k_b1"]["scored_candidates_per_group"] / res["64k_b8"][
        "scored_candidates_per_group"]
    return res


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--stride", type=int, default=2048)
    ap.add_argument("--threads", type=int, default=0)
    a = ap.parse_args()
    import json
    print(json.dumps(run(a.stride, a.threads), indent=1))

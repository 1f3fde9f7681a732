"""The benchmark's analytic work counts (the numerators of its roofline fractions) against a direct
count over the oracle's selection, and against the per-launch figures of the 128K workload."""
import numpy as np
import pytest

import bench
import oracle
from sgqa_inputs import CONFIGS, Config, gen_full


def test_counts_match_a_direct_count(oracle_lib):
    cfg = Config("counts", 2, 301, 8, 2, 64, 32, 4, 64, 40, 5)
    dm = oracle.dims_of(cfg)
    k_idx = gen_full(cfg, "k_idx")
    q_idx = gen_full(cfg, "q_idx")
    rows = np.array([[b, t] for b in range(cfg.batch) for t in range(cfg.T)], dtype=np.int32)
    kbar = oracle.compress(dm, k_idx)
    sel, _, _ = oracle.select(dm, kbar, rows, q_idx.reshape(len(rows), -1))
    visits = 0
    scored = 0
    for i, (_, t) in enumerate(rows):
        scored += (t // cfg.B) * cfg.G
        for g in range(cfg.G):
            for j in sel[i, g]:
                if j >= 0:
                    visits += sum(1 for u in range(j * cfg.B, (j + 1) * cfg.B) if u <= t)
    wc = bench.work_counts(cfg)
    assert wc["scored"] == scored
    assert wc["visits"] == visits
    assert wc["attn_flops"] == 4 * cfg.d * (cfg.Hq // cfg.G) * visits
    assert wc["gather_bytes"] == visits * 2 * cfg.d * 2


def test_counts_at_128k():
    wc = bench.work_counts(CONFIGS["128k"])
    assert wc["scored"] == pytest.approx(4.295e9, rel=1e-3)
    assert wc["index_flops"] == pytest.approx(5.50e11, rel=1e-3)
    assert wc["visits"] == pytest.approx(2.11e9, rel=2e-3)
    assert wc["attn_flops"] == pytest.approx(8.65e12, rel=2e-3)
    assert wc["gather_bytes"] == pytest.approx(1.08e12, rel=3e-3)
    # compulsory DRAM bytes of the attention: q, gate, out; the selection; K and V once
    assert wc["qgo_bytes"] + wc["sel_bytes"] + wc["kv_bytes"] == 4563402752


def test_decode_launch_counts():
    """Decode steps at the 1M workload: bf16 caches split each (sequence, group) over two CTAs
    and merge (8 launches: 3 appends, K4, K5, union, K6, merge); FP8 caches run one CTA per unit
    with no merge (7: 2 quantizing appends, the k_idx append, K4, K5, union, K6). The ncu launch
    list of the bench shows the merge kernel once per bf16 step only. A step whose new rows
    complete a block adds the block means."""
    cfg = CONFIGS["decode_1m"]
    assert bench.decode_launches(cfg, 4, cfg.T, fp8=False) == 8
    assert bench.decode_launches(cfg, 4, cfg.T, fp8=True) == 7
    assert bench.decode_launches(cfg, 4, cfg.T + 4, fp8=True) == 8  # completes block (T + 8) / 8 - 1
    one = cfg.replace(batch=1)
    assert bench.decode_launches(one, 4, cfg.T, fp8=True) == 8      # 4 units: K6 splits, merge

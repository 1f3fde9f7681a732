"""Shared test helpers: moving bf16 bit patterns between numpy and torch, workload inputs on
the device, and the comparisons the parity tests make against the oracle."""
from __future__ import annotations

import numpy as np

import oracle
from sgqa_inputs import Config, gen_device, gen_full, bf16_bits_to_f64

NAMES = ("q", "k", "v", "gate", "q_idx", "k_idx")
# output tolerances for bf16 inputs, outputs computed with the oracle's selection replayed
MAX_ABS = 1e-2
MEAN_ABS = 1e-3
NEAR_TIE_REL = 1e-4


def shape_of(cfg: Config, name: str, T=None, batch=None):
    return cfg.shape(name, T=T, batch=batch)


def to_dev(u16: np.ndarray, shape=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16)
    if shape is not None:
        t = t.reshape(shape)
    return t.cuda()


def to_host(t) -> np.ndarray:
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def host_inputs(cfg: Config):
    return {n: gen_full(cfg, n).reshape(shape_of(cfg, n)) for n in NAMES}


def device_inputs(cfg: Config, names=NAMES):
    import torch
    out = {}
    for n in names:
        t = torch.empty(shape_of(cfg, n), dtype=torch.bfloat16, device="cuda")
        gen_device(cfg, n, t)
        out[n] = t
    return out


def all_rows(cfg: Config):
    bb, tt = np.meshgrid(np.arange(cfg.batch), np.arange(cfg.T), indexing="ij")
    return np.stack([bb.ravel(), tt.ravel()], axis=1).astype(np.int32)


def sample_rows(cfg: Config, n: int, seed: int = 0, T=None):
    """Seeded sample of (b, t) rows: the first and last rows of every sequence plus random ones."""
    T = cfg.T if T is None else T
    rng = np.random.default_rng(seed)
    rows = set()
    for b in range(cfg.batch):
        for t in (0, 1, cfg.B - 1, cfg.B, T - 2, T - 1):
            if 0 <= t < T:
                rows.add((b, t))
    while len(rows) < n:
        rows.add((int(rng.integers(cfg.batch)), int(rng.integers(T))))
    return np.array(sorted(rows), dtype=np.int32)


def compare_selection(dm, kbar64, rows, qidx_rows, gpu_sel, orc_sel, s_m):
    """Selections must be identical except at near-ties: a row may differ from the oracle only
    if every swapped block's fp64 score is within NEAR_TIE_REL * |s_m| of the oracle's m-th best
    score s_m. Returns the number of (row, group) pairs that differ (all of them near-ties)."""
    gpu_sel = np.asarray(gpu_sel).reshape(orc_sel.shape)
    diff = np.nonzero((gpu_sel != orc_sel).any(axis=2))
    n_tie = 0
    for r, g in zip(*diff):
        b, t = int(rows[r, 0]), int(rows[r, 1])
        A = [int(j) for j in gpu_sel[r, g] if j >= 0]
        O = [int(j) for j in orc_sel[r, g] if j >= 0]
        assert len(A) == len(O), f"row {(b, t, g)}: set sizes differ {len(A)} vs {len(O)}"
        assert A == sorted(set(A)), f"row {(b, t, g)}: gpu selection not ascending/unique"
        c = t // dm.B
        assert A[-1] == c, f"row {(b, t, g)}: own block missing"
        swapped = set(A) ^ set(O)
        s = oracle.scores(dm, kbar64, b, qidx_rows[r].reshape(dm.G, dm.d_idx)[g], c)
        thr = NEAR_TIE_REL * abs(s_m[r, g])
        for j in swapped:
            assert j < c, f"row {(b, t, g)}: block {j} is not a candidate"
            assert abs(s[j] - s_m[r, g]) <= thr, (
                f"row {(b, t, g)}: block {j} score {s[j]} vs s_m {s_m[r, g]} beyond near-tie {thr}")
        n_tie += 1
    return n_tie


def output_errors(gpu_out_u16, ref64):
    g = bf16_bits_to_f64(gpu_out_u16).reshape(ref64.shape)
    d = np.abs(g - ref64)
    rel_rms = float(np.sqrt((d ** 2).sum() / max((ref64 ** 2).sum(), 1e-300)))
    return float(d.max()), float(d.mean()), rel_rms


def assert_outputs_close(gpu_out_u16, ref64, what=""):
    mx, mean, rel = output_errors(gpu_out_u16, ref64)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, f"{what}: max-abs {mx:.3g} mean-abs {mean:.3g} rel-rms {rel:.3g}"
    return mx, mean, rel

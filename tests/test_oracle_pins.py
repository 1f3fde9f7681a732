"""Pins of the fp64 oracle against things other than itself.

Each test fixes the oracle to something the definition or mathematics determines, chosen so that
a plausible mistake (a dropped term, a wrong sign or index, a transposed operand, an off-by-one
in the causal limit or the budget) fails at least one of them:

* brute force on T <= 64 (full Python sort, dense masked T x T softmax), B in {1, 2, 4, 8},
  every budget k in {B, 2B, ..., >= T};
* dense reduction: with k >= T every past block fits, and the layer equals dense causal gated
  GQA, checked against torch's scaled_dot_product_attention in fp64;
* a hand-derived worked example (tests/golden/hand_example.json);
* closed forms: block means of constant / arithmetic blocks, t = 0 gives v_0 * sigmoid(gate);
* invariants: set size min(k/B, c+1), own block kept, ascending and unique, causality,
  positive scaling of q_idx, exact ties to the lower block, B = 1 is the top-(k-1) tokens
  plus self, the page's 8x indexing ratio.

Definition: Step 5 Preview pages (mo.ai.kr "Step 5 Preview agentic work design", section
"model structure and training stability"; ai.info "StepFun illustrates the 92-block architecture
of Step 5 Preview", section "Sparse GQA aims at a 1 million token context").
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from sgqa_inputs import Config, bf16_bits_to_f64, f64_to_bf16_bits, gen_full

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_case(T, B, k, Hq=4, G=2, d=8, d_idx=4, seed=0, span=None, batch=1):
    span = span or max(B * 2, 8)
    cfg = Config("t", batch, T, Hq, G, d, d_idx, B, k, span, seed)
    x = {n: gen_full(cfg, n) for n in ("q", "k", "v", "gate", "q_idx", "k_idx")}
    return cfg, x


def _f(u):
    return bf16_bits_to_f64(u)


def brute_force(cfg, x):
    """Independent restatement: Python sort of every candidate, dense masked T x T softmax."""
    T, B, G, Hq, d, d_idx = cfg.T, cfg.B, cfg.G, cfg.Hq, cfg.d, cfg.d_idx
    R, Kb = Hq // G, cfg.k // cfg.B
    outs, sels = [], []
    for b in range(cfg.batch):
        kidx = _f(x["k_idx"][b]).reshape(T, d_idx)
        qidx = _f(x["q_idx"][b]).reshape(T, G, d_idx)
        q = _f(x["q"][b]).reshape(T, Hq, d)
        k = _f(x["k"][b]).reshape(T, G, d)
        v = _f(x["v"][b]).reshape(T, G, d)
        gate = _f(x["gate"][b]).reshape(T, Hq, d)
        nblk = T // B
        kbar = [[sum(kidx[j * B + r, i] for r in range(B)) / B for i in range(d_idx)] for j in range(nblk)]
        sel = np.full((T, G, Kb), -1, dtype=np.int32)
        mask = np.zeros((G, T, T), dtype=bool)
        for t in range(T):
            c = t // B
            for g in range(G):
                sc = []
                for j in range(c):
                    acc = 0.0
                    for i in range(d_idx):
                        acc += qidx[t, g, i] * kbar[j][i]
                    sc.append((-acc, j))
                sc.sort()
                m = min(Kb - 1, c)
                S = sorted([j for _, j in sc[:m]] + [c])
                sel[t, g, :len(S)] = S
                for u in range(t + 1):
                    if u // B in S:
                        mask[g, t, u] = True
        out = np.zeros((T, Hq, d))
        for h in range(Hq):
            g = h // R
            z = q[:, h, :] @ k[:, g, :].T / math.sqrt(d)
            z = np.where(mask[g], z, -np.inf)
            z = z - z.max(axis=1, keepdims=True)
            p = np.exp(z)
            p /= p.sum(axis=1, keepdims=True)
            out[:, h, :] = (p @ v[:, g, :]) / (1.0 + np.exp(-gate[:, h, :]))
        outs.append(out)
        sels.append(sel)
    return np.stack(sels), np.stack(outs)


def run_oracle(cfg, x, rows=None):
    dm = oracle.dims_of(cfg)
    sel, out, s_m, s_m1, r = oracle.forward(dm, x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], x["gate"],
                                            rows_bt=rows)
    return sel, out, s_m, s_m1, r


@pytest.mark.parametrize("B", [1, 2, 4, 8])
@pytest.mark.parametrize("T", [13, 40, 64])
def test_brute_force_small(oracle_lib, B, T):
    ks = list(range(B, T + 2 * B, B))
    for k in ks:
        cfg, x = _rand_case(T, B, k, seed=T * 100 + B, span=max(2 * B, 6))
        sel, out, _, _, _ = run_oracle(cfg, x)
        bsel, bout = brute_force(cfg, x)
        Kb = k // B
        np.testing.assert_array_equal(sel.reshape(cfg.batch, T, cfg.G, Kb), bsel)
        np.testing.assert_allclose(out.reshape(bout.shape), bout, rtol=1e-11, atol=1e-12)


def test_brute_force_batch2_uneven(oracle_lib):
    cfg, x = _rand_case(37, 4, 12, Hq=6, G=3, d=16, d_idx=8, seed=11, batch=2)
    sel, out, _, _, _ = run_oracle(cfg, x)
    bsel, bout = brute_force(cfg, x)
    np.testing.assert_array_equal(sel.reshape(bsel.shape), bsel)
    np.testing.assert_allclose(out.reshape(bout.shape), bout, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("T,B,Hq,G,d", [(96, 8, 8, 2, 16), (77, 4, 6, 3, 8), (50, 1, 4, 4, 32)])
def test_dense_reduction_matches_sdpa(oracle_lib, T, B, Hq, G, d):
    k = ((T + B - 1) // B) * B  # every block fits the budget
    cfg, x = _rand_case(T, B, k, Hq=Hq, G=G, d=d, d_idx=8, seed=5)
    _, out, _, _, _ = run_oracle(cfg, x)
    q = torch.from_numpy(_f(x["q"][0]).reshape(T, Hq, d)).permute(1, 0, 2)[None]
    kk = torch.from_numpy(_f(x["k"][0]).reshape(T, G, d)).permute(1, 0, 2)[None]
    vv = torch.from_numpy(_f(x["v"][0]).reshape(T, G, d)).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(q, kk, vv, is_causal=True, enable_gqa=True)
    ref = ref[0].permute(1, 0, 2).numpy() * torch.sigmoid(torch.from_numpy(_f(x["gate"][0]).reshape(T, Hq, d))).numpy()
    np.testing.assert_allclose(out.reshape(T, Hq, d), ref, rtol=1e-10, atol=1e-12)


def test_hand_worked_example(oracle_lib):
    ex = json.load(open(os.path.join(GOLDEN, "hand_example.json")))
    D = ex["dims"]
    T, Hq, d = D["T"], D["Hq"], D["d"]
    dm = oracle.dims(**D)
    k_idx = f64_to_bf16_bits(np.array(ex["k_idx"], dtype=np.float64)).reshape(1, T, D["d_idx"])
    q_idx = f64_to_bf16_bits(np.array(ex["q_idx"], dtype=np.float64)).reshape(1, T, 1, D["d_idx"])
    kbar = oracle.compress(dm, k_idx)
    np.testing.assert_array_equal(kbar[0], np.array(ex["kbar"], dtype=np.float64))
    q = np.zeros((1, T, Hq, d), np.uint16)
    kk = np.zeros((1, T, 1, d), np.uint16)
    v = f64_to_bf16_bits(np.array([[t, t * t] for t in range(T)], dtype=np.float64)).reshape(1, T, 1, d)
    gate = np.zeros((1, T, Hq, d), np.float64)
    gate[:, :, 1, :] = 100.0
    gate = f64_to_bf16_bits(gate)
    sel, out, _, _, _ = oracle.forward(dm, q, kk, v, q_idx, k_idx, gate)
    np.testing.assert_array_equal(sel.reshape(T, 2), np.array(ex["sel"]))
    mean_v = np.array(ex["mean_v"])
    np.testing.assert_allclose(out[:, 0, :], 0.5 * mean_v, rtol=1e-15, atol=0)
    np.testing.assert_allclose(out[:, 1, :], mean_v, rtol=1e-15, atol=0)


def test_compress_closed_forms(oracle_lib):
    T, B, d_idx = 32, 8, 4
    dm = oracle.dims(1, T, 2, 1, 4, d_idx, B, 16)
    vals = np.zeros((T, d_idx))
    for t in range(T):
        vals[t, 0] = 3.0                  # constant block -> 3
        vals[t, 1] = t % B + 1            # 1..8 -> 4.5
        vals[t, 2] = (-1.0) ** t * 0.25   # alternating -> 0
        vals[t, 3] = t // B * 2.0 - 1.0   # per-block constant -> itself
    kbar = oracle.compress(dm, f64_to_bf16_bits(vals).reshape(1, T, d_idx))
    np.testing.assert_array_equal(kbar[0, :, 0], 3.0)
    np.testing.assert_array_equal(kbar[0, :, 1], 4.5)
    np.testing.assert_array_equal(kbar[0, :, 2], 0.0)
    np.testing.assert_array_equal(kbar[0, :, 3], np.arange(T // B) * 2.0 - 1.0)
    # a trailing partial block is never compressed
    dm2 = oracle.dims(1, 35, 2, 1, 4, d_idx, B, 16)
    vals2 = np.vstack([vals, np.full((3, d_idx), 100.0)])
    kbar2 = oracle.compress(dm2, f64_to_bf16_bits(vals2).reshape(1, 35, d_idx))
    assert kbar2.shape == (1, 4, d_idx)
    np.testing.assert_array_equal(kbar2, kbar)


def test_first_token_is_gated_v0(oracle_lib):
    cfg, x = _rand_case(24, 8, 16, seed=3)
    _, out, _, _, rows = run_oracle(cfg, x)
    R = cfg.R
    v0 = _f(x["v"][0, 0]).reshape(cfg.G, cfg.d)
    g0 = _f(x["gate"][0, 0]).reshape(cfg.Hq, cfg.d)
    for h in range(cfg.Hq):
        np.testing.assert_allclose(out[0, h], v0[h // R] / (1 + np.exp(-g0[h])), rtol=1e-15, atol=0)


@pytest.mark.parametrize("B,k", [(8, 64), (8, 24), (4, 32), (1, 16)])
def test_selection_invariants(oracle_lib, B, k):
    cfg, x = _rand_case(200, B, k, Hq=4, G=2, d=8, d_idx=8, seed=21, span=40)
    sel, _, _, _, rows = run_oracle(cfg, x)
    Kb = k // B
    for r, (b, t) in enumerate(rows):
        c = t // B
        for g in range(cfg.G):
            S = sel[r, g]
            n = int((S >= 0).sum())
            assert n == min(Kb, c + 1)
            assert (S[n:] == -1).all()
            assert S[n - 1] == c                       # own block kept (and it is the largest)
            assert (np.diff(S[:n]) > 0).all()          # ascending, unique
            assert S[:n].max() <= c and S[:n].min() >= 0


def test_causality(oracle_lib):
    cfg, x = _rand_case(120, 8, 32, Hq=4, G=2, d=8, d_idx=8, seed=8, span=24)
    sel, out, _, _, _ = run_oracle(cfg, x)
    cut = 70
    y = {n: a.copy() for n, a in x.items()}
    rng = np.random.default_rng(0)
    for n in y:
        y[n][:, cut + 1:] = rng.integers(0, 2 ** 15, size=y[n][:, cut + 1:].shape, dtype=np.uint16) & 0x7F7F
    sel2, out2, _, _, _ = run_oracle(cfg, y)
    np.testing.assert_array_equal(sel2[:cut + 1], sel[:cut + 1])
    np.testing.assert_array_equal(out2[:cut + 1], out[:cut + 1])
    assert not np.array_equal(out2[cut + 1:], out[cut + 1:])


@pytest.mark.parametrize("alpha", [2.0, 0.5, 4.0])
def test_positive_scaling_of_index_queries_keeps_selection(oracle_lib, alpha):
    cfg, x = _rand_case(160, 8, 40, Hq=4, G=2, d=8, d_idx=8, seed=4, span=32)
    sel, _, _, _, _ = run_oracle(cfg, x)
    y = dict(x)
    y["q_idx"] = f64_to_bf16_bits(_f(x["q_idx"]) * alpha)  # exact: power-of-two scale
    sel2, _, _, _, _ = run_oracle(cfg, y)
    np.testing.assert_array_equal(sel2, sel)
    y["q_idx"] = f64_to_bf16_bits(_f(x["q_idx"]) * -1.0)   # a sign flip must change it
    sel3, _, _, _, _ = run_oracle(cfg, y)
    assert not np.array_equal(sel3, sel)


def test_exact_ties_go_to_lower_block(oracle_lib):
    T, B, k, d_idx = 64, 8, 24, 4  # Kb = 3 -> pick 2 candidates
    cfg, x = _rand_case(T, B, k, Hq=2, G=1, d=8, d_idx=d_idx, seed=9)
    base = _f(x["k_idx"][0]).reshape(T, d_idx)
    kid = base.copy()
    for j in range(T // B):            # all blocks identical -> all scores equal
        kid[j * B:(j + 1) * B] = base[0:B]
    y = dict(x)
    y["k_idx"] = f64_to_bf16_bits(kid).reshape(1, T, d_idx)
    sel, _, _, _, _ = run_oracle(cfg, y)
    for t in range(T):
        c = t // B
        S = [j for j in sel[t, 0] if j >= 0]
        assert S == sorted(list(range(min(2, c))) + [c])
    # partial tie: blocks 1 and 4 duplicate the best block 6; with 2 picks, 1 and 4 win over 6
    kid2 = base.copy()
    rng = np.random.default_rng(1)
    kid2[:] = rng.normal(size=kid2.shape) * 0.01
    kid2[6 * B:7 * B] = 5.0
    kid2[1 * B:2 * B] = 5.0
    kid2[4 * B:5 * B] = 5.0
    y["k_idx"] = f64_to_bf16_bits(kid2).reshape(1, T, d_idx)
    y["q_idx"] = f64_to_bf16_bits(np.ones((1, T, 1, d_idx)))
    sel, _, s_m, s_m1, _ = run_oracle(cfg, y)
    assert [j for j in sel[63, 0] if j >= 0] == [1, 4, 7]
    assert s_m[63, 0] == s_m1[63, 0]   # the boundary is an exact tie


def test_b1_is_topk_tokens_plus_self(oracle_lib):
    T, k = 90, 12
    cfg, x = _rand_case(T, 1, k, Hq=2, G=2, d=8, d_idx=8, seed=12, span=16)
    sel, _, _, _, _ = run_oracle(cfg, x)
    kid = _f(x["k_idx"][0]).reshape(T, 8)
    qid = _f(x["q_idx"][0]).reshape(T, 2, 8)
    for t in range(T):
        for g in range(2):
            s = [(-(float(np.dot(qid[t, g], kid[u]))), u) for u in range(t)]
            s.sort()
            want = sorted([u for _, u in s[:k - 1]] + [t])
            assert [j for j in sel[t, g] if j >= 0] == want


def test_row_subset_equals_full_run(oracle_lib):
    cfg, x = _rand_case(150, 8, 32, Hq=4, G=2, d=16, d_idx=8, seed=13, span=24, batch=2)
    sel, out, _, _, rows = run_oracle(cfg, x)
    pick = np.array([[1, 149], [0, 0], [1, 77], [0, 148], [1, 8]])
    sel2, out2, _, _, _ = run_oracle(cfg, x, rows=pick)
    idx = [b * cfg.T + t for b, t in pick]
    np.testing.assert_array_equal(sel2, sel[idx])
    np.testing.assert_array_equal(out2, out[idx])


def test_page_constants_and_eightfold_indexing(oracle_lib):
    pc = json.load(open(os.path.join(GOLDEN, "page_constants.json")))
    assert pc["topk_tokens_k"] // pc["block_size_B"] == pc["topk_blocks"]
    # scored (query, candidate) pairs: sum_t floor(t / B); B = 1 vs B = 8 -> (T-1)/(T/8-1) -> 8
    T = 8192
    pairs = {B: sum(t // B for t in range(T)) for B in (1, 8)}
    ratio = pairs[1] / pairs[8]
    assert abs(ratio - (T - 1) / (T / 8 - 1)) < 1e-12
    assert abs(ratio - pc["indexing_cost_reduction_from_B8"]) < 0.01
    # the oracle scores exactly floor(t/B) candidates: a row's scores stop at its own block
    cfg, x = _rand_case(64, 8, 16, seed=2)
    dm = oracle.dims_of(cfg)
    kbar = oracle.compress(dm, x["k_idx"])
    assert kbar.shape[1] == 64 // 8
    s = oracle.scores(dm, kbar, 0, x["q_idx"][0, 63, :cfg.d_idx], 63 // 8)
    assert s.shape == (7,)


def test_coverage_closed_forms(oracle_lib):
    cfg, x = _rand_case(100, 4, 400, Hq=2, G=1, d=8, d_idx=4, seed=6)
    sel, _, _, _, rows = run_oracle(cfg, x)
    dm = oracle.dims_of(cfg)
    qr = np.ascontiguousarray(x["q"].reshape(cfg.T, -1))
    cov = oracle.coverage(dm, rows, qr, x["k"], sel, ktop=10)
    np.testing.assert_array_equal(cov, 1.0)          # everything selected -> full coverage
    only_own = np.full_like(sel, -1)
    only_own[:, 0, 0] = rows[:, 1] // 4
    cov2 = oracle.coverage(dm, rows, qr, x["k"], only_own, ktop=1000)
    want = np.array([((t % 4) + 1) / (t + 1) for t in rows[:, 1]])
    np.testing.assert_allclose(cov2[:, 0], want, rtol=1e-15)


def _coverage_brute_force(cfg, q, k, rows, sel, ktop):
    """Token coverage written out directly: every (row, head) sorts all tokens u <= t by
    (exact score desc, u asc) with a Python sort, keeps the first min(ktop, t + 1), and counts
    those whose block the row's group selected. Scores are sums of exact products taken with
    math.fsum (correctly rounded), so they do not depend on a summation order."""
    T, G, Hq, d, B = cfg.T, cfg.G, cfg.Hq, cfg.d, cfg.B
    R, Kb = Hq // G, cfg.k // cfg.B
    qf = _f(q).reshape(len(rows), Hq, d)
    kf = _f(k).reshape(cfg.batch, T, G, d)
    cov = np.zeros((len(rows), Hq))
    for i, (b, t) in enumerate(rows):
        for h in range(Hq):
            g = h // R
            S = {int(j) for j in sel[i, g] if j >= 0}
            order = sorted(range(t + 1), key=lambda u: (-math.fsum(qf[i, h] * kf[b, u, g]), u))
            top = order[:min(ktop, t + 1)]
            cov[i, h] = sum(1 for u in top if u // B in S) / len(top)
    return cov


def _random_selection(cfg, rows, seed):
    """A valid selection per (row, group) that is neither empty nor everything: the own block plus
    a seeded random subset of the complete past blocks, at most k/B - 1 of them, ascending."""
    rng = np.random.default_rng(seed)
    Kb = cfg.k // cfg.B
    sel = np.full((len(rows), cfg.G, Kb), -1, dtype=np.int32)
    for i, (_, t) in enumerate(rows):
        c = t // cfg.B
        for g in range(cfg.G):
            past = [j for j in range(c) if rng.random() < 0.5][:Kb - 1]
            S = sorted(past + [c])
            sel[i, g, :len(S)] = S
    return sel


@pytest.mark.parametrize("integer_valued", [False, True])
def test_coverage_brute_force(oracle_lib, integer_valued):
    """oracle_coverage against the brute force with ktop < t + 1 (the top set really has to be
    chosen), two groups of two heads (so h // R and h % G differ), and a selection that covers
    about half of every row. The integer-valued case has scores in [-72, 72] with many exact
    ties at the ktop boundary, which only the (score desc, u asc) rule orders correctly."""
    cfg, x = _rand_case(56, 4, 16, Hq=4, G=2, d=8, d_idx=4, seed=31)
    q, k = x["q"], x["k"]
    if integer_valued:
        rng = np.random.default_rng(5)
        q = f64_to_bf16_bits(rng.integers(-3, 4, size=q.shape).astype(np.float64))
        k = f64_to_bf16_bits(rng.integers(-3, 4, size=k.shape).astype(np.float64))
    rows = np.array([[0, t] for t in range(cfg.T)], dtype=np.int32)
    sel = _random_selection(cfg, rows, seed=3)
    dm = oracle.dims_of(cfg)
    qr = np.ascontiguousarray(q.reshape(cfg.T, -1))
    for ktop in (1, 5, 12):
        got = oracle.coverage(dm, rows, qr, k, sel, ktop=ktop)
        want = _coverage_brute_force(cfg, q, k, rows, sel, ktop)
        np.testing.assert_array_equal(got, want)
        assert 0.0 < got[ktop + 8:].mean() < 1.0


def test_coverage_all_scores_tied_takes_lowest_tokens(oracle_lib):
    """Every key equal, so every score ties: the top-ktop set is the ktop lowest tokens u < ktop
    (ties to the lower index), and coverage is the closed form |{u < ktop : u // B in S}| / ktop."""
    cfg, x = _rand_case(48, 4, 16, Hq=4, G=2, d=8, d_idx=4, seed=32)
    k = np.broadcast_to(x["k"][:, :1], x["k"].shape).copy()
    rows = np.array([[0, t] for t in range(cfg.T)], dtype=np.int32)
    sel = _random_selection(cfg, rows, seed=4)
    dm = oracle.dims_of(cfg)
    ktop = 9
    cov = oracle.coverage(dm, rows, np.ascontiguousarray(x["q"].reshape(cfg.T, -1)), k, sel, ktop=ktop)
    for i, (_, t) in enumerate(rows):
        n = min(ktop, t + 1)
        for h in range(cfg.Hq):
            S = {int(j) for j in sel[i, h // cfg.R] if j >= 0}
            assert cov[i, h] == sum(1 for u in range(n) if u // cfg.B in S) / n

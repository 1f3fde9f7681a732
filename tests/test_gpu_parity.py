"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the same seeded inputs.

* kbar: bit-exact against the oracle's fp64 block mean rounded once to fp32.
* selection: identical block sets, except near-ties (every swapped block's oracle score within
  1e-4 * |s_m| of the oracle's m-th best score s_m), which are counted.
* outputs with the oracle's selection replayed (sgqa_attend): max-abs <= 1e-2, mean-abs <= 1e-3.
* the whole layer (sgqa_forward) and a decode step (sgqa_decode) likewise.

Small workloads are compared in full (several tiles and a ragged tail); the full-size
workloads, in the launch configuration the benchmark times, on seeded samples of rows.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
import block_sparse_long_kbar_b200 as sg
import sgqa_inputs as sgi
from sgqa_inputs import CONFIGS, DECODE_NEW, Config, gen_device, gen_full, gen_rows
from tests._helpers import (NAMES, all_rows, assert_outputs_close, compare_selection, device_inputs, host_inputs,
                            output_errors, sample_rows, shape_of, to_dev, to_host)

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": CONFIGS["tiny"],
    "ragged_g4": Config("ragged_g4", 2, 3001, 32, 4, 128, 64, 8, 512, 400, 7),
    "b1": Config("b1", 1, 1500, 8, 2, 64, 32, 1, 128, 200, 8),
    "b16_r16": Config("b16_r16", 1, 1000, 16, 1, 128, 64, 16, 256, 160, 9),
    "g8_r1": Config("g8_r1", 1, 777, 8, 8, 64, 32, 4, 64, 100, 10),
    "dense": Config("dense", 1, 300, 8, 2, 64, 32, 8, 304, 64, 11),
    "t9": Config("t9", 3, 9, 8, 2, 64, 32, 8, 16, 4, 12),
    "t1": Config("t1", 2, 1, 4, 4, 128, 64, 8, 64, 4, 13),
    "r3_rowkernel": Config("r3_rowkernel", 1, 1200, 12, 4, 64, 32, 8, 256, 150, 19),
    "g4_r2": Config("g4_r2", 1, 1300, 8, 4, 64, 32, 8, 256, 150, 23),
}


def _ws(dims):
    ws = sg.alloc_workspace(sg.sgqa_workspace_size(dims))
    sg.sgqa_reset_device_status(ws)
    return ws


def _status_ok(ws):
    torch.cuda.synchronize()
    assert sg.sgqa_get_device_status(ws) == 0


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    sg.load_library()
    oracle.build()


@pytest.fixture(scope="module")
def small_cases():
    cache = {}

    def get(name):
        if name not in cache:
            cfg = SMALL[name]
            h = host_inputs(cfg)
            d = {n: to_dev(h[n], shape_of(cfg, n)) for n in NAMES}
            dm = oracle.dims_of(cfg)
            kbar64 = oracle.compress(dm, h["k_idx"])
            rows = all_rows(cfg)
            qi = h["q_idx"].reshape(cfg.batch * cfg.T, -1)
            sel_o, s_m, s_m1 = oracle.select(dm, kbar64, rows, qi)
            cache[name] = (cfg, h, d, dm, kbar64, rows, sel_o, s_m)
        return cache[name]
    return get


@pytest.mark.parametrize("name", list(SMALL))
def test_compress_bit_exact(small_cases, name):
    cfg, h, d, dm, kbar64, *_ = small_cases(name)
    dims = sg.sgqa_dims.of(cfg)
    kbar = torch.full((cfg.batch, cfg.T // cfg.B, cfg.d_idx), float("nan"), device="cuda")
    sg.sgqa_compress_keys(dims, d["k_idx"], kbar, None)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(kbar.cpu().numpy().view(np.uint32), kbar64.astype(np.float32).view(np.uint32))


@pytest.mark.parametrize("name", list(SMALL))
def test_select_matches_oracle(small_cases, name):
    cfg, h, d, dm, kbar64, rows, sel_o, s_m = small_cases(name)
    dims = sg.sgqa_dims.of(cfg)
    ws = _ws(dims)
    kbar = torch.empty((cfg.batch, cfg.T // cfg.B, cfg.d_idx), device="cuda")
    sg.sgqa_compress_keys(dims, d["k_idx"], kbar, None)
    sel = torch.full((cfg.batch, cfg.T, cfg.G, cfg.Kb), -7, dtype=torch.int32, device="cuda")
    sg.sgqa_select(dims, d["q_idx"], kbar, sel, ws)
    _status_ok(ws)
    gsel = sel.cpu().numpy().reshape(-1, cfg.G, cfg.Kb)
    n_tie = compare_selection(dm, kbar64, rows, h["q_idx"].reshape(len(rows), -1), gsel, sel_o, s_m)
    assert n_tie <= max(2, len(rows) * cfg.G // 100), f"{n_tie} near-tie rows"


@pytest.mark.parametrize("name", list(SMALL))
def test_attend_with_oracle_selection(small_cases, name):
    cfg, h, d, dm, kbar64, rows, sel_o, s_m = small_cases(name)
    dims = sg.sgqa_dims.of(cfg)
    ws = _ws(dims)
    sel = torch.from_numpy(sel_o.reshape(cfg.batch, cfg.T, cfg.G, cfg.Kb)).cuda()
    out = torch.full(shape_of(cfg, "q"), float("nan"), dtype=torch.bfloat16, device="cuda")
    sg.sgqa_attend(dims, d["q"], d["k"], d["v"], d["gate"], sel, out, ws)
    _status_ok(ws)
    ref = oracle.attend(dm, rows, h["q"].reshape(len(rows), -1), h["k"], h["v"], h["gate"].reshape(len(rows), -1),
                        sel_o)
    assert_outputs_close(to_host(out), ref.reshape(shape_of(cfg, "q")), name)


def test_attend_rows_far_above_their_reference_max(small_cases):
    """Rows whose scores exceed their own block's maximum by far more than the fp32 exponent range
    allows to keep unscaled: the keys of block 0 are scaled by 64 and every row selects block 0,
    so the tile is streamed again with exact maxima for those rows (the kernel's fallback).
    Such rows attend almost to one token, so their outputs are as large as single values of v;
    v is scaled by 1/4 so that the bf16 rounding of the output alone (half an ulp, 2^-6 at
    |y| >= 4) stays well inside the max-abs bound."""
    cfg, h, d, dm, kbar64, rows, sel_o, s_m = small_cases("ragged_g4")
    k = h["k"].copy()
    kf = sgi.bf16_bits_to_f64(k[:, :cfg.B]) * 64.0  # exact: a power of two
    k[:, :cfg.B] = sgi.f64_to_bf16_bits(kf)
    v = sgi.f64_to_bf16_bits(sgi.bf16_bits_to_f64(h["v"]) * 0.25)
    sel = sel_o.reshape(-1, cfg.Kb).copy()
    for i in range(sel.shape[0]):
        t = int(rows[i // cfg.G][1])
        c = t // cfg.B
        s = [int(j) for j in sel[i] if j >= 0]
        if 0 not in s:
            if len(s) >= cfg.Kb:
                s.remove(next(j for j in s if j != c))
            s = sorted(s + [0])
        sel[i] = s + [-1] * (cfg.Kb - len(s))
    sel = sel.reshape(sel_o.shape)
    # the case is really exercised: some row's block-0 score is far above its own block's
    qf = sgi.bf16_bits_to_f64(h["q"].reshape(len(rows), cfg.Hq, cfg.d))
    kk = sgi.bf16_bits_to_f64(k.reshape(cfg.batch, cfg.T, cfg.G, cfg.d))
    sc = np.log2(np.e) / np.sqrt(cfg.d)
    gap = 0.0
    for i in range(100, len(rows), 997):
        b, t = int(rows[i][0]), int(rows[i][1])
        c = t // cfg.B
        for hq in range(0, cfg.Hq, 5):
            g = hq // cfg.R
            s0 = kk[b, :cfg.B, g] @ qf[i, hq]
            so = kk[b, c * cfg.B:t + 1, g] @ qf[i, hq]
            gap = max(gap, (s0.max() - so.max()) * sc)
    assert gap > 80, gap
    dims = sg.sgqa_dims.of(cfg)
    ws = _ws(dims)
    out = torch.full(shape_of(cfg, "q"), float("nan"), dtype=torch.bfloat16, device="cuda")
    sg.sgqa_attend(dims, d["q"], to_dev(k, shape_of(cfg, "k")), to_dev(v, shape_of(cfg, "v")), d["gate"],
                   torch.from_numpy(sel.reshape(cfg.batch, cfg.T, cfg.G, cfg.Kb)).cuda(), out, ws)
    _status_ok(ws)
    ref = oracle.attend(dm, rows, h["q"].reshape(len(rows), -1), k, v, h["gate"].reshape(len(rows), -1), sel)
    assert_outputs_close(to_host(out), ref.reshape(shape_of(cfg, "q")), "far above reference")


@pytest.mark.parametrize("name", list(SMALL))
def test_forward_matches_oracle(small_cases, name):
    cfg, h, d, dm, kbar64, rows, sel_o, s_m = small_cases(name)
    dims = sg.sgqa_dims.of(cfg)
    ws = _ws(dims)
    out = torch.full(shape_of(cfg, "q"), float("nan"), dtype=torch.bfloat16, device="cuda")
    sel = torch.full((cfg.batch, cfg.T, cfg.G, cfg.Kb), -7, dtype=torch.int32, device="cuda")
    sg.sgqa_forward(dims, d["q"], d["k"], d["v"], d["q_idx"], d["k_idx"], d["gate"], out, ws, sel_out=sel)
    _status_ok(ws)
    gsel = sel.cpu().numpy().reshape(-1, cfg.G, cfg.Kb)
    compare_selection(dm, kbar64, rows, h["q_idx"].reshape(len(rows), -1), gsel, sel_o, s_m)
    ref = oracle.attend(dm, rows, h["q"].reshape(len(rows), -1), h["k"], h["v"], h["gate"].reshape(len(rows), -1),
                        gsel)
    assert_outputs_close(to_host(out), ref.reshape(shape_of(cfg, "q")), name)
    # same result without sel_out (selection kept in the workspace) and run to run
    out2 = torch.empty_like(out)
    sg.sgqa_forward(dims, d["q"], d["k"], d["v"], d["q_idx"], d["k_idx"], d["gate"], out2, ws)
    _status_ok(ws)
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))


def test_forward_chunked_selection_is_identical():
    # T above the 32768-row selection chunk: the chunked path must give the same bits
    cfg = Config("chunked", 1, 40000, 4, 1, 64, 32, 8, 256, 3000, 14)
    dims = sg.sgqa_dims.of(cfg)
    d = device_inputs(cfg)
    ws = _ws(dims)
    out1 = torch.empty(shape_of(cfg, "q"), dtype=torch.bfloat16, device="cuda")
    out2 = torch.empty_like(out1)
    sel = torch.empty((1, cfg.T, cfg.G, cfg.Kb), dtype=torch.int32, device="cuda")
    sg.sgqa_forward(dims, d["q"], d["k"], d["v"], d["q_idx"], d["k_idx"], d["gate"], out1, ws, sel_out=sel)
    sg.sgqa_forward(dims, d["q"], d["k"], d["v"], d["q_idx"], d["k_idx"], d["gate"], out2, ws)
    _status_ok(ws)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


def test_exact_ties_go_to_lower_blocks():
    """All index keys equal, so every candidate block has exactly the same score: the selection
    must be the lowest m = min(k/B - 1, c) blocks plus the own block (ties to the lower index)."""
    cfg = Config("ties", 2, 1500, 8, 2, 64, 32, 8, 256, 100, 24)
    dims = sg.sgqa_dims.of(cfg)
    one = gen_rows(cfg, "k_idx", 0, np.array([5]))[0]
    k_idx = np.broadcast_to(one, (cfg.batch, cfg.T, cfg.d_idx)).copy()
    q_idx = to_dev(gen_full(cfg, "q_idx").reshape(shape_of(cfg, "q_idx")), shape_of(cfg, "q_idx"))
    kbar = torch.empty((cfg.batch, cfg.T // cfg.B, cfg.d_idx), device="cuda")
    sg.sgqa_compress_keys(dims, to_dev(k_idx, shape_of(cfg, "k_idx")), kbar, None)
    ws = _ws(dims)
    sel = torch.full((cfg.batch, cfg.T, cfg.G, cfg.Kb), -7, dtype=torch.int32, device="cuda")
    sg.sgqa_select(dims, q_idx, kbar, sel, ws)
    _status_ok(ws)
    got = sel.cpu().numpy()
    want = np.full((cfg.T, cfg.Kb), -1, dtype=np.int32)
    for t in range(cfg.T):
        c = t // cfg.B
        m = min(cfg.Kb - 1, c)
        want[t, :m] = np.arange(m)
        want[t, m] = c
    for b in range(cfg.batch):
        for g in range(cfg.G):
            np.testing.assert_array_equal(got[b, :, g], want)


def test_zero_scores_tie_to_lower_blocks():
    """Nine blocks in ten have all-zero index keys, so most scores are exactly zero (the tensor
    cores may give +0.0 or -0.0, depending on the signs of the products) and many rows' m-th best
    score is 0: the zeros are one score, tied, and go to the lower block indices. The selections
    must equal the oracle's exactly (at s_m = 0 the near-tie rule would excuse any order)."""
    cfg = Config("zeros", 1, 2048, 8, 2, 64, 32, 8, 512, 256, 25)
    dims = sg.sgqa_dims.of(cfg)
    k_idx = gen_full(cfg, "k_idx").reshape(shape_of(cfg, "k_idx")).copy()
    blocks = np.arange(cfg.T) // cfg.B
    k_idx[:, blocks % 10 != 0] = 0  # bf16 +0.0
    q_h = gen_full(cfg, "q_idx").reshape(shape_of(cfg, "q_idx"))
    kbar = torch.empty((cfg.batch, cfg.T // cfg.B, cfg.d_idx), device="cuda")
    sg.sgqa_compress_keys(dims, to_dev(k_idx, shape_of(cfg, "k_idx")), kbar, None)
    ws = _ws(dims)
    sel = torch.full((cfg.batch, cfg.T, cfg.G, cfg.Kb), -7, dtype=torch.int32, device="cuda")
    sg.sgqa_select(dims, to_dev(q_h, shape_of(cfg, "q_idx")), kbar, sel, ws)
    _status_ok(ws)
    dm = oracle.dims_of(cfg)
    kbar64 = oracle.compress(dm, k_idx)
    rows = all_rows(cfg)
    sel_o, s_m, _ = oracle.select(dm, kbar64, rows, q_h.reshape(len(rows), -1))
    chosen = np.asarray(rows)[:, 1] // cfg.B > cfg.Kb - 1  # rows that choose among their candidates
    assert np.sum(s_m[chosen] == 0) > 500  # the case is exercised
    np.testing.assert_array_equal(sel.cpu().numpy().reshape(sel_o.shape), sel_o)


def test_causality_on_gpu():
    cfg = Config("causal", 1, 2500, 8, 2, 64, 32, 8, 256, 300, 15)
    dims = sg.sgqa_dims.of(cfg)
    h = host_inputs(cfg)
    cut = 1234
    h2 = {n: a.copy() for n, a in h.items()}
    rng = np.random.default_rng(1)
    for n in NAMES:
        h2[n][:, cut + 1:] = rng.integers(0, 2 ** 15, size=h2[n][:, cut + 1:].shape, dtype=np.uint16) & 0x3F7F
    outs = []
    for hh in (h, h2):
        d = {n: to_dev(hh[n], shape_of(cfg, n)) for n in NAMES}
        ws = _ws(dims)
        out = torch.empty(shape_of(cfg, "q"), dtype=torch.bfloat16, device="cuda")
        sg.sgqa_forward(dims, d["q"], d["k"], d["v"], d["q_idx"], d["k_idx"], d["gate"], out, ws)
        _status_ok(ws)
        outs.append(to_host(out))
    np.testing.assert_array_equal(outs[0][:, :cut + 1], outs[1][:, :cut + 1])
    assert not np.array_equal(outs[0][:, cut + 1:], outs[1][:, cut + 1:])


def test_invalid_selection_is_reported_not_faulted():
    cfg = SMALL["tiny"]
    dims = sg.sgqa_dims.of(cfg)
    d = device_inputs(cfg)
    ws = _ws(dims)
    sel = torch.full((1, cfg.T, cfg.G, cfg.Kb), -1, dtype=torch.int32, device="cuda")
    t = torch.arange(cfg.T, device="cuda")
    sel[0, :, :, 0] = (t // cfg.B)[:, None].int()
    sel[0, 100, 1, 1] = 10 ** 6          # a block far beyond row 100's own block
    out = torch.empty(shape_of(cfg, "q"), dtype=torch.bfloat16, device="cuda")
    sg.sgqa_attend(dims, d["q"], d["k"], d["v"], d["gate"], sel, out, ws)
    torch.cuda.synchronize()
    assert sg.sgqa_get_device_status(ws) == 6
    sg.sgqa_reset_device_status(ws)
    torch.cuda.synchronize()
    assert sg.sgqa_get_device_status(ws) == 0
    assert torch.isfinite(out.float()).all()


def test_duplicate_selection_entry_is_reported_on_the_row_kernel(small_cases):
    """R = 3 runs on the per-row attention kernel. A selection row that names a block twice breaks
    the format (strictly ascending ids): the device check flags it (status 6) and skips the
    repeated entry instead of weighting that block twice; every other row is unchanged."""
    cfg, h, d, dm, kbar64, rows, sel_o, s_m = small_cases("r3_rowkernel")
    assert cfg.Hq // cfg.G == 3
    dims = sg.sgqa_dims.of(cfg)
    sel_ok = torch.from_numpy(sel_o.reshape(cfg.batch, cfg.T, cfg.G, cfg.Kb)).cuda()
    t_bad, g_bad = 777, 1
    row = sel_o.reshape(cfg.batch, cfg.T, cfg.G, cfg.Kb)[0, t_bad, g_bad].copy()
    n = int((row >= 0).sum())
    assert n >= 3
    dup = row.copy()
    dup[1] = dup[0]  # block dup[0] named twice; the block that was second is dropped
    sel_dup = sel_ok.clone()
    sel_dup[0, t_bad, g_bad] = torch.from_numpy(dup).cuda()
    outs = []
    for s_, want in ((sel_ok, 0), (sel_dup, 6)):
        ws = _ws(dims)
        out = torch.full(shape_of(cfg, "q"), float("nan"), dtype=torch.bfloat16, device="cuda")
        sg.sgqa_attend(dims, d["q"], d["k"], d["v"], d["gate"], s_, out, ws)
        torch.cuda.synchronize()
        assert sg.sgqa_get_device_status(ws) == want
        outs.append(out)
    a, b = outs[0].view(torch.int16), outs[1].view(torch.int16)
    R = cfg.Hq // cfg.G
    heads = slice(g_bad * R, (g_bad + 1) * R)
    other = torch.ones(a.shape[:3], dtype=torch.bool, device="cuda")
    other[0, t_bad, heads] = False
    assert torch.equal(a[other], b[other])
    # the flagged row attends to its selection without the repeated entry
    kept = np.array([j for i, j in enumerate(dup) if j >= 0 and i != 1], dtype=np.int32)
    sel_kept = np.full((1, cfg.G, cfg.Kb), -1, dtype=np.int32)
    sel_kept[0] = sel_o.reshape(cfg.batch, cfg.T, cfg.G, cfg.Kb)[0, t_bad]
    sel_kept[0, g_bad] = -1
    sel_kept[0, g_bad, :len(kept)] = kept
    r1 = np.array([[0, t_bad]], dtype=np.int32)
    ref = oracle.attend(dm, r1, h["q"][0, t_bad].reshape(1, -1), h["k"], h["v"], h["gate"][0, t_bad].reshape(1, -1),
                        sel_kept)
    assert_outputs_close(to_host(outs[1][0, t_bad]), ref.reshape(cfg.Hq, cfg.d), "duplicate entry skipped")
    assert torch.isfinite(outs[1].float()).all()


def test_device_generator_matches_host_generator():
    cfg = CONFIGS["128k"]
    for name in NAMES:
        t = torch.empty(shape_of(cfg, name, T=4096), dtype=torch.bfloat16, device="cuda")
        c4 = cfg.replace(T=4096)
        gen_device(c4, name, t)
        got = to_host(t).reshape(4096, -1)
        want = gen_rows(cfg, name, 0, np.arange(4096))
        np.testing.assert_array_equal(got, want)


def _decode_case(cfg, cache_len, n_new, check_seqs):
    """Run one decode step after a cache of cache_len tokens and check sequences check_seqs."""
    n_seq = cfg.batch
    T_cap = ((cache_len + n_new + cfg.B - 1) // cfg.B) * cfg.B
    dims = sg.sgqa_dims(n_seq, T_cap, cfg.Hq, cfg.G, cfg.d, cfg.d_idx, cfg.B, cfg.k)
    caches = {}
    for n in ("k", "v", "k_idx"):
        caches[n] = torch.zeros(shape_of(cfg, n, T=T_cap, batch=n_seq), dtype=torch.bfloat16, device="cuda")
        gen_device(cfg, n, caches[n], t0=0, n_t=cache_len)
    kbar = torch.zeros((n_seq, T_cap // cfg.B, cfg.d_idx), device="cuda")
    sg.sgqa_compress_keys(dims, caches["k_idx"], kbar, None)
    new = {}
    for n in NAMES:
        new[n] = torch.empty((n_seq, n_new) + shape_of(cfg, n)[2:], dtype=torch.bfloat16, device="cuda")
        gen_device(cfg, n, new[n], t0=cache_len, n_t=n_new, dst_t0=0)
    ws = sg.alloc_workspace(sg.sgqa_decode_workspace_size(dims, n_new))
    sg.sgqa_reset_device_status(ws)
    out = torch.full((n_seq, n_new, cfg.Hq, cfg.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    sel = torch.full((n_seq, n_new, cfg.G, cfg.Kb), -7, dtype=torch.int32, device="cuda")
    sg.sgqa_decode(dims, cache_len, n_new, caches["k"], caches["v"], caches["k_idx"], kbar, new["q"], new["k"],
                   new["v"], new["q_idx"], new["k_idx"], new["gate"], out, ws, sel_out=sel)
    _status_ok(ws)
    # idempotent at a fixed cache_len
    out2 = torch.empty_like(out)
    sg.sgqa_decode(dims, cache_len, n_new, caches["k"], caches["v"], caches["k_idx"], kbar, new["q"], new["k"],
                   new["v"], new["q_idx"], new["k_idx"], new["gate"], out2, ws)
    _status_ok(ws)
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
    Tn = cache_len + n_new
    dm = oracle.dims(1, Tn, cfg.Hq, cfg.G, cfg.d, cfg.d_idx, cfg.B, cfg.k)
    errs = []
    for b in check_seqs:
        kh = to_host(caches["k"][b:b + 1, :Tn])
        vh = to_host(caches["v"][b:b + 1, :Tn])
        kih = to_host(caches["k_idx"][b:b + 1, :Tn])
        # the caches hold exactly the generator's rows (append included)
        np.testing.assert_array_equal(kih[0, cache_len:], gen_rows(cfg, "k_idx", b, np.arange(cache_len, Tn)))
        kbar64 = oracle.compress(dm, kih)
        # the decode step's kbar update matches for the blocks it completed
        j0, j1 = cache_len // cfg.B, Tn // cfg.B
        if j1 > j0:
            np.testing.assert_array_equal(kbar[b, j0:j1].cpu().numpy(), kbar64[0, j0:j1].astype(np.float32))
        rows = np.array([[0, cache_len + i] for i in range(n_new)], dtype=np.int32)
        qi = to_host(new["q_idx"][b]).reshape(n_new, -1)
        sel_o, s_m, _ = oracle.select(dm, kbar64, rows, qi)
        gsel = sel[b].cpu().numpy()
        compare_selection(dm, kbar64, rows, qi, gsel, sel_o, s_m)
        ref = oracle.attend(dm, rows, to_host(new["q"][b]).reshape(n_new, -1), kh, vh,
                            to_host(new["gate"][b]).reshape(n_new, -1), gsel)
        errs.append(assert_outputs_close(to_host(out[b]), ref.reshape(n_new, cfg.Hq, cfg.d), f"decode seq {b}"))
    return errs


def test_decode_small_matches_oracle():
    cfg = Config("dec_small", 3, 5000, 32, 4, 128, 64, 8, 512, 600, 16)
    _decode_case(cfg, 4996, 4, [0, 2])          # new tokens complete block 624
    _decode_case(cfg, 4000, 4, [1])             # all new tokens in one partial block
    _decode_case(cfg, 3, 4, [0])                # tiny cache: fewer candidates than the budget


def test_decode_n1_and_b1():
    _decode_case(Config("dec_b1", 2, 3000, 8, 2, 64, 32, 1, 64, 300, 17), 2500, 3, [1])
    _decode_case(Config("dec_n1", 2, 3000, 8, 2, 64, 32, 8, 128, 300, 18), 2999, 1, [0])


@pytest.mark.parametrize("cfg,cache_len,n_new,seqs", [
    (Config("dec_b16", 2, 4000, 32, 4, 128, 64, 16, 512, 500, 26), 3990, 4, [1]),      # blocks of 16
    (Config("dec_r16", 2, 3000, 64, 4, 128, 64, 8, 256, 300, 27), 2996, 4, [0]),       # 64 query-head columns
    (Config("dec_q1", 3, 3000, 32, 4, 128, 64, 8, 512, 300, 28), 2777, 1, [2]),        # one new token
    (Config("dec_q3", 1, 3000, 16, 2, 128, 64, 8, 1024, 300, 29), 2600, 3, [0]),       # R = 8, G = 2, splits
])
def test_decode_tensor_core_shapes(cfg, cache_len, n_new, seqs):
    _decode_case(cfg, cache_len, n_new, seqs)


def test_decode_rows_far_above_their_reference_max():
    """Decode rows whose scores exceed their own block's maximum far beyond the fp32 exponent range
    (block 0's keys scaled by 64; every block is selected since k covers the whole cache): the
    decode attention must stream its tiles again with exact maxima for those columns. v is scaled
    by 1/4 so the bf16 rounding of the near-one-hot outputs stays inside the bound."""
    cfg = Config("dec_risky", 2, 600, 32, 4, 128, 64, 8, 640, 100, 30)
    cache_len, n_new = 596, 4
    T_cap = 600
    dims = sg.sgqa_dims(cfg.batch, T_cap, cfg.Hq, cfg.G, cfg.d, cfg.d_idx, cfg.B, cfg.k)
    caches = {}
    for n in ("k", "v", "k_idx"):
        caches[n] = torch.zeros(shape_of(cfg, n, T=T_cap), dtype=torch.bfloat16, device="cuda")
        gen_device(cfg, n, caches[n], t0=0, n_t=cache_len)
    caches["k"][:, :cfg.B] *= 64.0
    caches["v"] *= 0.25
    kbar = torch.zeros((cfg.batch, T_cap // cfg.B, cfg.d_idx), device="cuda")
    sg.sgqa_compress_keys(dims, caches["k_idx"], kbar, None)
    new = {}
    for n in NAMES:
        new[n] = torch.empty((cfg.batch, n_new) + shape_of(cfg, n)[2:], dtype=torch.bfloat16, device="cuda")
        gen_device(cfg, n, new[n], t0=cache_len, n_t=n_new, dst_t0=0)
    new["v"] *= 0.25
    ws = sg.alloc_workspace(sg.sgqa_decode_workspace_size(dims, n_new))
    sg.sgqa_reset_device_status(ws)
    out = torch.full((cfg.batch, n_new, cfg.Hq, cfg.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    sel = torch.full((cfg.batch, n_new, cfg.G, cfg.Kb), -7, dtype=torch.int32, device="cuda")
    sg.sgqa_decode(dims, cache_len, n_new, caches["k"], caches["v"], caches["k_idx"], kbar, new["q"], new["k"],
                   new["v"], new["q_idx"], new["k_idx"], new["gate"], out, ws, sel_out=sel)
    _status_ok(ws)
    Tn = cache_len + n_new
    dm = oracle.dims(1, Tn, cfg.Hq, cfg.G, cfg.d, cfg.d_idx, cfg.B, cfg.k)
    sc = np.log2(np.e) / np.sqrt(cfg.d)
    gap = 0.0
    for b in range(cfg.batch):
        kh, vh = to_host(caches["k"][b:b + 1, :Tn]), to_host(caches["v"][b:b + 1, :Tn])
        gsel = sel[b].cpu().numpy()
        assert (gsel[:, :, 0] == 0).all()  # every row selected block 0
        rows = np.array([[0, cache_len + i] for i in range(n_new)], dtype=np.int32)
        qh = to_host(new["q"][b]).reshape(n_new, -1)
        kf = sgi.bf16_bits_to_f64(kh.reshape(Tn, cfg.G, cfg.d))
        qf = sgi.bf16_bits_to_f64(qh.reshape(n_new, cfg.Hq, cfg.d))
        for i in range(n_new):
            t = cache_len + i
            c = t // cfg.B
            for h in range(cfg.Hq):
                g = h // cfg.R
                gap = max(gap, ((kf[:cfg.B, g] @ qf[i, h]).max() - (kf[c * cfg.B:t + 1, g] @ qf[i, h]).max()) * sc)
        ref = oracle.attend(dm, rows, qh, kh, vh, to_host(new["gate"][b]).reshape(n_new, -1), gsel)
        assert_outputs_close(to_host(out[b]), ref.reshape(n_new, cfg.Hq, cfg.d), f"risky decode seq {b}")
    assert gap > 130, gap


def test_decode_selection_matches_forward():
    """Decode and forward compute the same definition on different kernels: on the same
    sequence, decode's selection for the new rows equals forward's for those rows except at
    near-ties (both are also checked against the oracle), and the outputs agree within the
    parity bounds."""
    cfg = Config("dec_fwd", 2, 6000, 32, 4, 128, 64, 8, 512, 500, 25)
    cache_len, n_new = 5996, 4
    Tn = cache_len + n_new
    T_cap = Tn
    # forward over the concatenated sequence
    fcfg = cfg.replace(T=Tn)
    fdims = sg.sgqa_dims.of(fcfg)
    d = device_inputs(fcfg)
    ws = _ws(fdims)
    fout = torch.empty(shape_of(fcfg, "q"), dtype=torch.bfloat16, device="cuda")
    fsel = torch.empty((fcfg.batch, Tn, cfg.G, cfg.Kb), dtype=torch.int32, device="cuda")
    sg.sgqa_forward(fdims, d["q"], d["k"], d["v"], d["q_idx"], d["k_idx"], d["gate"], fout, ws, sel_out=fsel)
    _status_ok(ws)
    # decode of the last n_new rows after a cache of cache_len
    dims = sg.sgqa_dims(cfg.batch, T_cap, cfg.Hq, cfg.G, cfg.d, cfg.d_idx, cfg.B, cfg.k)
    caches = {n: torch.zeros(shape_of(cfg, n, T=T_cap), dtype=torch.bfloat16, device="cuda") for n in ("k", "v", "k_idx")}
    for n in caches:
        caches[n][:, :cache_len] = d[n][:, :cache_len]
    kbar = torch.zeros((cfg.batch, T_cap // cfg.B, cfg.d_idx), device="cuda")
    sg.sgqa_compress_keys(dims, caches["k_idx"], kbar, None)
    new = {n: d[n][:, cache_len:].contiguous() for n in NAMES}
    dws = sg.alloc_workspace(sg.sgqa_decode_workspace_size(dims, n_new))
    sg.sgqa_reset_device_status(dws)
    dout = torch.empty((cfg.batch, n_new, cfg.Hq, cfg.d), dtype=torch.bfloat16, device="cuda")
    dsel = torch.empty((cfg.batch, n_new, cfg.G, cfg.Kb), dtype=torch.int32, device="cuda")
    sg.sgqa_decode(dims, cache_len, n_new, caches["k"], caches["v"], caches["k_idx"], kbar, new["q"], new["k"],
                   new["v"], new["q_idx"], new["k_idx"], new["gate"], dout, dws, sel_out=dsel)
    _status_ok(dws)
    dm = oracle.dims(1, Tn, cfg.Hq, cfg.G, cfg.d, cfg.d_idx, cfg.B, cfg.k)
    differ = 0
    for b in range(cfg.batch):
        kbar64 = oracle.compress(dm, to_host(d["k_idx"][b:b + 1]))
        rows = np.array([[0, t] for t in range(cache_len, Tn)], dtype=np.int32)
        qi = to_host(new["q_idx"][b]).reshape(n_new, -1)
        sel_o, s_m, _ = oracle.select(dm, kbar64, rows, qi)
        ds = dsel[b].cpu().numpy()
        fs = fsel[b, cache_len:].cpu().numpy()
        compare_selection(dm, kbar64, rows, qi, ds, sel_o, s_m)
        compare_selection(dm, kbar64, rows, qi, fs, sel_o, s_m)
        differ += int((ds != fs).any(axis=2).sum())
        ref = oracle.attend(dm, rows, to_host(new["q"][b]).reshape(n_new, -1), to_host(d["k"][b:b + 1]),
                            to_host(d["v"][b:b + 1]), to_host(new["gate"][b]).reshape(n_new, -1), ds)
        assert_outputs_close(to_host(dout[b]), ref.reshape(n_new, cfg.Hq, cfg.d), "decode")
        same = (ds == fs).all(axis=2).all(axis=1)
        if same.any():
            sm = torch.from_numpy(same).cuda()
            assert_outputs_close(to_host(dout[b][sm]), sgi.bf16_bits_to_f64(to_host(fout[b, cache_len:][sm])),
                                 "decode vs forward")
    print(f"decode vs forward: {differ} of {cfg.batch * n_new * cfg.G} rows differ (near-ties)")


# ---- full-size workloads, sampled rows, the benchmark's launch configuration ----------------

def _full_size_forward(cfg, n_rows, seed):
    dims = sg.sgqa_dims.of(cfg)
    d = device_inputs(cfg)
    ws = _ws(dims)
    out = torch.full(shape_of(cfg, "q"), float("nan"), dtype=torch.bfloat16, device="cuda")
    sel = torch.full((cfg.batch, cfg.T, cfg.G, cfg.Kb), -7, dtype=torch.int32, device="cuda")
    sg.sgqa_forward(dims, d["q"], d["k"], d["v"], d["q_idx"], d["k_idx"], d["gate"], out, ws, sel_out=sel)
    _status_ok(ws)
    rows = sample_rows(cfg, n_rows, seed)
    dm = oracle.dims_of(cfg)
    kih, kh, vh = to_host(d["k_idx"]), to_host(d["k"]), to_host(d["v"])
    kbar64 = oracle.compress(dm, kih)
    pick = lambda n: to_host(d[n][rows[:, 0], rows[:, 1]]).reshape(len(rows), -1)
    qi, qh, gh = pick("q_idx"), pick("q"), pick("gate")
    sel_o, s_m, _ = oracle.select(dm, kbar64, rows, qi)
    gsel = sel[rows[:, 0], rows[:, 1]].cpu().numpy()
    n_tie = compare_selection(dm, kbar64, rows, qi, gsel, sel_o, s_m)
    ref = oracle.attend(dm, rows, qh, kh, vh, gh, gsel)
    err = assert_outputs_close(to_host(out[rows[:, 0], rows[:, 1]]), ref.reshape(len(rows), cfg.Hq, cfg.d), cfg.name)
    # replay the oracle's selection through sgqa_attend
    sel[rows[:, 0], rows[:, 1]] = torch.from_numpy(sel_o).cuda()
    out2 = torch.empty_like(out)
    sg.sgqa_attend(dims, d["q"], d["k"], d["v"], d["gate"], sel, out2, ws)
    _status_ok(ws)
    ref2 = oracle.attend(dm, rows, qh, kh, vh, gh, sel_o)
    assert_outputs_close(to_host(out2[rows[:, 0], rows[:, 1]]), ref2.reshape(len(rows), cfg.Hq, cfg.d), cfg.name)
    del d, out, out2, sel, ws
    torch.cuda.empty_cache()
    return n_tie, err


# near-tie (row, group) pairs allowed in a sample: the 32K workload's topic spans (128 blocks)
# put the 511th place inside a cluster of similar scores in about a tenth of its rows
NEAR_TIE_FRACTION = {"32k": 0.25, "128k": 0.05, "64k_b8": 0.15, "64k_b1": 0.15}


@pytest.mark.parametrize("name", ["32k", "128k", "64k_b8", "64k_b1"])
def test_full_size_prefill_sampled(name):
    cfg = CONFIGS[name]
    n_rows = 2048
    n_tie, err = _full_size_forward(cfg, n_rows, 100)
    print(f"{name}: near-tie (row, group) pairs {n_tie} of {n_rows * cfg.G}; max-abs/mean-abs/rel-rms {err}")
    assert n_tie <= NEAR_TIE_FRACTION[name] * n_rows * cfg.G
    assert err[2] < 1e-2, f"rel-rms {err[2]}"


def test_largest_budget_sampled():
    """The largest supported budget, k/B = 16384 blocks (B = 1, so up to 16383 picks per row):
    selections far longer than a tile, nearly every candidate taken in the early rows."""
    n_tie, err = _full_size_forward(Config("max_budget", 1, 17000, 8, 2, 64, 32, 1, 16384, 1000, 21), 40, 7)
    print(f"max budget: near-tie rows {n_tie}; max-abs/mean-abs/rel-rms {err}")


def test_full_size_decode_1m_sampled():
    cfg = CONFIGS["decode_1m"]
    errs = _decode_case(cfg, cfg.T, DECODE_NEW, [0, 5, 9, 14, 18, 23, 27, 31])
    print(f"decode 1M: {errs}")


def test_decode_cache_beyond_4096_candidate_groups():
    """A cache of 1.2M tokens (B = 8): rows of more than 4096 groups of 32 candidates, which the
    decode select lists in several chunks."""
    cfg = CONFIGS["decode_1m"].replace(batch=2)
    cache_len = 1258288
    assert (cache_len // cfg.B + 31) // 32 > 4096
    errs = _decode_case(cfg, cache_len, DECODE_NEW, [0, 1])
    print(f"decode 1.2M: {errs}")

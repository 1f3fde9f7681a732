"""GPU parity of the FP8 KV-cache decode (sgqa_quantize_kv_fp8, sgqa_decode_fp8) against the oracle.

* quantization: codes and row scales bit-exact against the oracle's quantizer (its e4m3
  rounding is pinned against torch's float8_e4m3fn cast in test_oracle_fp8_pins.py);
* a decode step over FP8 caches: the caches it appends to equal the oracle's quantization of the
  sequence, bit for bit (on the new rows, every token the step attends to and a seeded sample); the selection equals sgqa_decode's on the bf16 caches (the index
  keys are not quantized); outputs match the oracle's attention over the dequantized values
  (exact in bf16) within max-abs 1e-2 / mean-abs 1e-3;
* the 1M-context decode workload on sampled sequences.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
import block_sparse_long_kbar_b200 as sg
from sgqa_inputs import CONFIGS, DECODE_NEW, Config, f64_to_bf16_bits, gen_device, gen_rows
from tests._helpers import NAMES, assert_outputs_close, compare_selection, shape_of, to_dev, to_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    sg.load_library()
    oracle.build()


def _u8(t):
    return t.cpu().numpy().astype(np.uint8)


def test_quantize_matches_oracle_bit_exact():
    rng = np.random.default_rng(7)
    batch, T, G, d = 2, 300, 4, 128
    x = rng.standard_normal((batch, T, G, d)) * np.exp2(rng.integers(-30, 30, size=(batch, T, G, 1)))
    x[:, ::5, :, ::3] *= 1e-3
    x[0, 7, 1] = 0.0                      # an all-zero row
    xb = f64_to_bf16_bits(x)
    dims = sg.sgqa_dims(batch, T + 20, 8, G, d, 64, 8, 64)
    dst8 = torch.full((batch, T + 20, G, d), 0xAB, dtype=torch.uint8, device="cuda")
    dsc = torch.full((batch, T + 20, G), -1.0, dtype=torch.float32, device="cuda")
    sg.sgqa_quantize_kv_fp8(dims, 10, T, to_dev(xb), dst8, dsc)
    torch.cuda.synchronize()
    q, s = oracle.quantize_fp8(xb)
    np.testing.assert_array_equal(_u8(dst8[:, 10:10 + T]), q)
    np.testing.assert_array_equal(dsc[:, 10:10 + T].cpu().numpy().astype(np.float64), s)
    assert (_u8(dst8[:, :10]) == 0xAB).all() and (_u8(dst8[:, 10 + T:]) == 0xAB).all()


def _fp8_caches(cfg, T_cap, cache_len, chunk=65536):
    """FP8 K/V caches of the first cache_len tokens, quantized on the GPU chunk by chunk from the
    generator's bf16 rows; bf16 index-key cache and block means."""
    dims = sg.sgqa_dims(cfg.batch, T_cap, cfg.Hq, cfg.G, cfg.d, cfg.d_idx, cfg.B, cfg.k)
    c8 = {n: torch.zeros(shape_of(cfg, n, T=T_cap), dtype=torch.uint8, device="cuda") for n in ("k", "v")}
    csc = {n: torch.zeros((cfg.batch, T_cap, cfg.G), dtype=torch.float32, device="cuda") for n in ("k", "v")}
    for t0 in range(0, cache_len, chunk):
        n = min(chunk, cache_len - t0)
        for name in ("k", "v"):
            tmp = torch.empty((cfg.batch, n, cfg.G, cfg.d), dtype=torch.bfloat16, device="cuda")
            gen_device(cfg, name, tmp, t0=t0, n_t=n, dst_t0=0)
            sg.sgqa_quantize_kv_fp8(dims, t0, n, tmp, c8[name], csc[name])
            del tmp
    kidx = torch.zeros(shape_of(cfg, "k_idx", T=T_cap), dtype=torch.bfloat16, device="cuda")
    gen_device(cfg, "k_idx", kidx, t0=0, n_t=cache_len)
    kbar = torch.zeros((cfg.batch, T_cap // cfg.B, cfg.d_idx), device="cuda")
    sg.sgqa_compress_keys(dims, kidx, kbar, None)
    return dims, c8, csc, kidx, kbar


def _dequant_bf16_bits(q, s):
    y = oracle.dequantize_fp8(q, s)
    b = f64_to_bf16_bits(y)
    return b


def _fp8_decode_case(cfg, cache_len, n_new, check_seqs, compare_bf16=True, T_cap=None):
    if T_cap is None:
        T_cap = ((cache_len + n_new + cfg.B - 1) // cfg.B) * cfg.B
    dims, c8, csc, kidx, kbar = _fp8_caches(cfg, T_cap, cache_len)
    new = {}
    for n in NAMES:
        new[n] = torch.empty((cfg.batch, n_new) + shape_of(cfg, n)[2:], dtype=torch.bfloat16, device="cuda")
        gen_device(cfg, n, new[n], t0=cache_len, n_t=n_new, dst_t0=0)
    ws = sg.alloc_workspace(sg.sgqa_decode_workspace_size(dims, n_new))
    sg.sgqa_reset_device_status(ws)
    out = torch.full((cfg.batch, n_new, cfg.Hq, cfg.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    sel = torch.full((cfg.batch, n_new, cfg.G, cfg.Kb), -7, dtype=torch.int32, device="cuda")
    sg.sgqa_decode_fp8(dims, cache_len, n_new, c8["k"], csc["k"], c8["v"], csc["v"], kidx, kbar, new["q"], new["k"],
                       new["v"], new["q_idx"], new["k_idx"], new["gate"], out, ws, sel_out=sel)
    torch.cuda.synchronize()
    assert sg.sgqa_get_device_status(ws) == 0
    # run-to-run identical
    out2 = torch.empty_like(out)
    sg.sgqa_decode_fp8(dims, cache_len, n_new, c8["k"], csc["k"], c8["v"], csc["v"], kidx, kbar, new["q"], new["k"],
                       new["v"], new["q_idx"], new["k_idx"], new["gate"], out2, ws)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
    Tn = cache_len + n_new
    dm = oracle.dims(1, Tn, cfg.Hq, cfg.G, cfg.d, cfg.d_idx, cfg.B, cfg.k)
    rng = np.random.default_rng(cfg.seed)
    errs = []
    for b in check_seqs:
        gsel = sel[b].cpu().numpy()
        # the tokens the step attends to (every group's selection), the new rows, and a sample
        blocks = np.unique(gsel[gsel >= 0])
        toks = (blocks[:, None] * cfg.B + np.arange(cfg.B)[None, :]).ravel()
        toks = toks[toks < Tn]
        sample = rng.integers(0, Tn, size=min(2048, Tn))
        check = np.unique(np.concatenate([toks, np.arange(cache_len, Tn), sample]))
        ti = torch.from_numpy(check.astype(np.int64)).cuda()
        got = {n: (_u8(c8[n][b].index_select(0, ti)), csc[n][b].index_select(0, ti).cpu().numpy().astype(np.float64))
               for n in ("k", "v")}
        # the caches hold exactly the oracle's quantization of the sequence (checked rows)
        for n in ("k", "v"):
            q, sc_ = oracle.quantize_fp8(gen_rows(cfg, n, b, check).reshape(len(check), cfg.G, cfg.d))
            np.testing.assert_array_equal(got[n][0], q)
            np.testing.assert_array_equal(got[n][1], sc_)
        # the oracle attends over the dequantized values (exact in bf16) of the tokens it needs
        kh = np.zeros((1, Tn, cfg.G, cfg.d), dtype=np.uint16)
        vh = np.zeros((1, Tn, cfg.G, cfg.d), dtype=np.uint16)
        kh[0, check] = _dequant_bf16_bits(*got["k"])
        vh[0, check] = _dequant_bf16_bits(*got["v"])
        kbar64 = oracle.compress(dm, to_host(kidx[b:b + 1, :Tn]))
        rows = np.array([[0, cache_len + i] for i in range(n_new)], dtype=np.int32)
        qi = to_host(new["q_idx"][b]).reshape(n_new, -1)
        sel_o, s_m, _ = oracle.select(dm, kbar64, rows, qi)
        compare_selection(dm, kbar64, rows, qi, gsel, sel_o, s_m)
        ref = oracle.attend(dm, rows, to_host(new["q"][b]).reshape(n_new, -1), kh, vh,
                            to_host(new["gate"][b]).reshape(n_new, -1), gsel)
        errs.append(assert_outputs_close(to_host(out[b]), ref.reshape(n_new, cfg.Hq, cfg.d), f"fp8 decode seq {b}"))
    if compare_bf16:
        # the selection is the bf16 decode's (same index keys, same kernels)
        bf = {n: torch.zeros(shape_of(cfg, n, T=T_cap), dtype=torch.bfloat16, device="cuda") for n in ("k", "v")}
        for n in bf:
            gen_device(cfg, n, bf[n], t0=0, n_t=cache_len)
        kidx2 = kidx.clone()
        kbar2 = torch.zeros_like(kbar)
        sg.sgqa_compress_keys(dims, kidx2, kbar2, None)
        sel2 = torch.full_like(sel, -7)
        out3 = torch.empty_like(out)
        sg.sgqa_decode(dims, cache_len, n_new, bf["k"], bf["v"], kidx2, kbar2, new["q"], new["k"], new["v"],
                       new["q_idx"], new["k_idx"], new["gate"], out3, ws, sel_out=sel2)
        torch.cuda.synchronize()
        assert torch.equal(sel, sel2)
    return errs


@pytest.mark.parametrize("cfg,cache_len,n_new,seqs", [
    (Config("f8_small", 3, 5000, 32, 4, 128, 64, 8, 512, 600, 40), 4996, 4, [0, 2]),   # splits + merge
    (Config("f8_b16", 2, 4000, 32, 4, 128, 64, 16, 512, 500, 41), 3990, 4, [1]),
    (Config("f8_q1", 2, 3000, 16, 2, 128, 64, 8, 1024, 300, 42), 2777, 1, [0]),
    (Config("f8_tiny_cache", 2, 64, 32, 4, 128, 64, 8, 512, 16, 43), 3, 4, [1]),        # fewer blocks than the budget
])
def test_fp8_decode_matches_oracle(cfg, cache_len, n_new, seqs):
    _fp8_decode_case(cfg, cache_len, n_new, seqs)


def test_fp8_decode_capacity_ending_inside_a_block():
    """The caches hold exactly cache_len + n_new tokens and that count is not a multiple of B:
    the last block is partial, and its missing tokens (past the capacity) have no scale to read."""
    cfg = Config("f8_ragged_cap", 2, 5000, 32, 4, 128, 64, 8, 512, 600, 44)
    _fp8_decode_case(cfg, 4993, 4, [0, 1], T_cap=4997)


def test_fp8_decode_rejects_shapes_without_the_tensor_core_path():
    cfg = Config("f8_d64", 1, 600, 8, 2, 64, 32, 8, 128, 100, 44)
    dims = sg.sgqa_dims(1, 600, 8, 2, 64, 32, 8, 128)
    x = torch.zeros(1 << 16, dtype=torch.bfloat16, device="cuda")
    u8 = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    f = torch.zeros(1 << 14, dtype=torch.float32, device="cuda")
    ws = sg.alloc_workspace(max(sg.sgqa_decode_workspace_size(dims, 4), 256))
    with pytest.raises(sg.SgqaError) as e:
        sg.sgqa_decode_fp8(dims, 500, 4, u8, f, u8, f, x, f, x, x, x, x, x, x, x, ws)
    assert e.value.code == 2


def test_fp8_decode_1m_sampled():
    cfg = CONFIGS["decode_1m"]
    errs = _fp8_decode_case(cfg, cfg.T, DECODE_NEW, [0, 17, 31], compare_bf16=False)
    print(f"fp8 decode 1M: {errs}")

"""Failure detection on the GPU without a fault: a bounded wait that runs out.

The test hook sgqa_test_stall_decode_cta makes one decode-attention CTA issue no loads, so the
wait of its tensor-core issuer for the first tile is never satisfied (a flag that nothing sets).
That wait gives up after its 2 s bound: the kernel records SGQA_ERR_TIMEOUT in the status word,
stops its other roles, frees TMEM and returns with nothing in flight, so the context stays
usable. Every tensor-core kernel then sees the recorded timeout (at CTA start, and while polling
inside its waits) and stops early instead of running or waiting out its own bound: a second
call without a reset leaves its output unwritten and returns at once. After
sgqa_reset_device_status the same step runs normally and matches the oracle.
"""
import time

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
import block_sparse_long_kbar_b200 as sg
from sgqa_inputs import Config, gen_device
from tests._helpers import NAMES, assert_outputs_close, compare_selection, shape_of, to_host

pytestmark = pytest.mark.gpu


def test_decode_wait_that_runs_out_is_reported_and_stops_later_work():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    cfg = Config("timeout", 2, 3000, 32, 4, 128, 64, 8, 512, 300, 50)
    cache_len, n_new = 2996, 4
    T_cap = 3000
    dims = sg.sgqa_dims(cfg.batch, T_cap, cfg.Hq, cfg.G, cfg.d, cfg.d_idx, cfg.B, cfg.k)
    caches = {}
    for n in ("k", "v", "k_idx"):
        caches[n] = torch.zeros(shape_of(cfg, n, T=T_cap), dtype=torch.bfloat16, device="cuda")
        gen_device(cfg, n, caches[n], t0=0, n_t=cache_len)
    kbar = torch.zeros((cfg.batch, T_cap // cfg.B, cfg.d_idx), device="cuda")
    sg.sgqa_compress_keys(dims, caches["k_idx"], kbar, None)
    new = {}
    for n in NAMES:
        new[n] = torch.empty((cfg.batch, n_new) + shape_of(cfg, n)[2:], dtype=torch.bfloat16, device="cuda")
        gen_device(cfg, n, new[n], t0=cache_len, n_t=n_new, dst_t0=0)
    ws = sg.alloc_workspace(sg.sgqa_decode_workspace_size(dims, n_new))
    sg.sgqa_reset_device_status(ws)
    torch.cuda.synchronize()

    def step(out, sel=None):
        sg.sgqa_decode(dims, cache_len, n_new, caches["k"], caches["v"], caches["k_idx"], kbar, new["q"], new["k"],
                       new["v"], new["q_idx"], new["k_idx"], new["gate"], out, ws, sel_out=sel)
        t0 = time.perf_counter()
        torch.cuda.synchronize()
        return time.perf_counter() - t0

    fill = lambda: torch.full((cfg.batch, n_new, cfg.Hq, cfg.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    sg.sgqa_test_stall_decode_cta(0)
    try:
        dt = step(fill())
    finally:
        sg.sgqa_test_stall_decode_cta(-1)
    assert sg.sgqa_get_device_status(ws) == 5, "the wait that ran out is recorded as SGQA_ERR_TIMEOUT"
    assert dt < 15.0, dt
    # without a reset, the tensor-core kernels stop at once: the output stays unwritten
    out2 = fill()
    dt2 = step(out2)
    assert sg.sgqa_get_device_status(ws) == 5
    assert torch.isnan(out2.float()).all()
    assert dt2 < 1.0, dt2
    # after a reset, the same step runs normally and matches the oracle
    sg.sgqa_reset_device_status(ws)
    out3 = fill()
    sel = torch.full((cfg.batch, n_new, cfg.G, cfg.Kb), -7, dtype=torch.int32, device="cuda")
    step(out3, sel)
    assert sg.sgqa_get_device_status(ws) == 0
    Tn = cache_len + n_new
    dm = oracle.dims(1, Tn, cfg.Hq, cfg.G, cfg.d, cfg.d_idx, cfg.B, cfg.k)
    b = 1
    kbar64 = oracle.compress(dm, to_host(caches["k_idx"][b:b + 1, :Tn]))
    rows = np.array([[0, cache_len + i] for i in range(n_new)], dtype=np.int32)
    qi = to_host(new["q_idx"][b]).reshape(n_new, -1)
    sel_o, s_m, _ = oracle.select(dm, kbar64, rows, qi)
    gsel = sel[b].cpu().numpy()
    compare_selection(dm, kbar64, rows, qi, gsel, sel_o, s_m)
    ref = oracle.attend(dm, rows, to_host(new["q"][b]).reshape(n_new, -1), to_host(caches["k"][b:b + 1, :Tn]),
                        to_host(caches["v"][b:b + 1, :Tn]), to_host(new["gate"][b]).reshape(n_new, -1), gsel)
    assert_outputs_close(to_host(out3[b]), ref.reshape(n_new, cfg.Hq, cfg.d), "after reset")

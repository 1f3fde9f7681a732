"""GPU parity of the backward (sgqa_attend_backward) against the oracle's fp64 gradients.

For each workload the selection comes from the GPU forward (sel_out); the oracle differentiates
the same selection. fp32 gradients against fp64: every element within 2e-3 of the largest
magnitude of its tensor, and the mean error within 1e-4 of it; the bits are the same run to run.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
import block_sparse_long_kbar_b200 as sg
from sgqa_inputs import Config, f64_to_bf16_bits
from tests._helpers import NAMES, all_rows, host_inputs, shape_of, to_dev

pytestmark = pytest.mark.gpu

CASES = [
    Config("bw_tiny", 1, 1536, 8, 2, 64, 32, 8, 512, 256, 70),
    Config("bw_g4", 1, 1200, 32, 4, 128, 64, 8, 256, 200, 71),
    Config("bw_b4", 2, 700, 8, 2, 128, 32, 4, 128, 100, 72),
    Config("bw_b16_r1", 1, 900, 4, 4, 64, 32, 16, 256, 150, 73),
]


def _grads(cfg, d, sel, dy):
    dims = sg.sgqa_dims.of(cfg)
    ws = sg.alloc_workspace(sg.sgqa_backward_workspace_size(dims))
    sg.sgqa_reset_device_status(ws)
    out = {n: torch.full(shape_of(cfg, "q" if n in ("dq", "dgate") else "k"), float("nan"), device="cuda")
           for n in ("dq", "dk", "dv", "dgate")}
    sg.sgqa_attend_backward(dims, d["q"], d["k"], d["v"], d["gate"], sel, dy, out["dq"], out["dk"], out["dv"],
                            out["dgate"], ws)
    torch.cuda.synchronize()
    assert sg.sgqa_get_device_status(ws) == 0
    return out


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_backward_matches_oracle(cfg):
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    h = host_inputs(cfg)
    d = {n: to_dev(h[n], shape_of(cfg, n)) for n in NAMES}
    dims = sg.sgqa_dims.of(cfg)
    ws = sg.alloc_workspace(sg.sgqa_workspace_size(dims))
    sg.sgqa_reset_device_status(ws)
    out = torch.empty(shape_of(cfg, "q"), dtype=torch.bfloat16, device="cuda")
    sel = torch.empty((cfg.batch, cfg.T, cfg.G, cfg.Kb), dtype=torch.int32, device="cuda")
    sg.sgqa_forward(dims, d["q"], d["k"], d["v"], d["q_idx"], d["k_idx"], d["gate"], out, ws, sel_out=sel)
    dy_h = f64_to_bf16_bits(np.random.default_rng(cfg.seed).standard_normal(shape_of(cfg, "q")))
    dy = to_dev(dy_h, shape_of(cfg, "q"))
    g1 = _grads(cfg, d, sel, dy)
    g2 = _grads(cfg, d, sel, dy)
    for n in g1:
        assert torch.equal(g1[n], g2[n]), f"{n} differs run to run"
    rows = all_rows(cfg)
    dm = oracle.dims_of(cfg)
    gsel = sel.cpu().numpy().reshape(len(rows), cfg.G, cfg.Kb)
    dq, dk, dv, dgate = oracle.attend_backward(dm, rows, h["q"].reshape(len(rows), -1), h["k"], h["v"],
                                               h["gate"].reshape(len(rows), -1), gsel, dy_h.reshape(len(rows), -1))
    ref = {"dq": dq.reshape(shape_of(cfg, "q")), "dk": dk.reshape(shape_of(cfg, "k")),
           "dv": dv.reshape(shape_of(cfg, "k")), "dgate": dgate.reshape(shape_of(cfg, "q"))}
    for n in ref:
        got = g1[n].double().cpu().numpy()
        scale = np.abs(ref[n]).max()
        err = np.abs(got - ref[n])
        assert err.max() <= 2e-3 * scale, (n, err.max(), scale)
        assert err.mean() <= 1e-4 * scale, (n, err.mean(), scale)


def test_backward_rejects_unsupported_block_size():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    dims = sg.sgqa_dims(1, 100, 8, 2, 64, 32, 1, 16)
    assert sg.sgqa_backward_workspace_size(dims) == 0
    x = torch.zeros(1 << 16, dtype=torch.bfloat16, device="cuda")
    s = torch.zeros(1 << 12, dtype=torch.int32, device="cuda")
    f = torch.zeros(1 << 16, dtype=torch.float32, device="cuda")
    ws = sg.alloc_workspace(1 << 20)
    with pytest.raises(sg.SgqaError) as e:
        sg.sgqa_attend_backward(dims, x, x, x, x, s, x, f, f, f, f, ws)
    assert e.value.code == 2

"""GPU parity of sgqa_gated_swa (Gated SWA, the efficient layer that alternates 3:1 with Sparse
GQA; mo.ai.kr, "Step 5 Preview agentic work design", section "model structure and training
stability") against the oracle's fp64 definition: the gated softmax attention over the keys
t - window < u <= t.

* the window selection written to sel_out: exact (the blocks max(0, t - window + 1) / B .. t / B);
* outputs: max-abs <= 1e-2, mean-abs <= 1e-3 against oracle.swa, every row of small workloads
  (windows of one block, unaligned windows, windows longer than the sequence; R in {4, 8, 16};
  B in {1, 8, 16}) and sampled rows of the 128K workload with the bench's 4096-token window.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
import block_sparse_long_kbar_b200 as sg
from sgqa_inputs import CONFIGS, Config
from tests._helpers import all_rows, assert_outputs_close, device_inputs, sample_rows, shape_of, to_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    sg.load_library()
    oracle.build()


def _capacity(window, B):
    return ((window + B + B - 1) // B) * B


def _run(cfg, window, rows=None):
    cfg = cfg.replace(k=_capacity(window, cfg.B))
    dims = sg.sgqa_dims.of(cfg)
    d = device_inputs(cfg, ("q", "k", "v", "gate"))
    ws = sg.alloc_workspace(sg.sgqa_workspace_size(dims))
    sg.sgqa_reset_device_status(ws)
    out = torch.full(shape_of(cfg, "q"), float("nan"), dtype=torch.bfloat16, device="cuda")
    sel = torch.full((cfg.batch, cfg.T, cfg.G, cfg.Kb), -7, dtype=torch.int32, device="cuda")
    sg.sgqa_gated_swa(dims, window, d["q"], d["k"], d["v"], d["gate"], out, ws, sel_out=sel)
    torch.cuda.synchronize()
    assert sg.sgqa_get_device_status(ws) == 0
    rows = all_rows(cfg) if rows is None else rows
    # the selection: the blocks the window overlaps, ascending, -1 padded
    gsel = sel[rows[:, 0], rows[:, 1]].cpu().numpy()
    for i, (_, t) in enumerate(rows):
        first, c = max(0, t - window + 1) // cfg.B, t // cfg.B
        want = np.full(cfg.Kb, -1, dtype=np.int32)
        want[:c - first + 1] = np.arange(first, c + 1)
        for g in range(cfg.G):
            np.testing.assert_array_equal(gsel[i, g], want)
    dm = oracle.dims_of(cfg)
    pick = lambda n: to_host(d[n][rows[:, 0], rows[:, 1]]).reshape(len(rows), -1)
    ref = oracle.swa(dm, rows, pick("q"), to_host(d["k"]), to_host(d["v"]), pick("gate"), window)
    assert_outputs_close(to_host(out[rows[:, 0], rows[:, 1]]), ref.reshape(len(rows), cfg.Hq, cfg.d),
                         f"{cfg.name} window {window}")
    # without sel_out (selection in the workspace, in chunks): the same bits
    out2 = torch.empty_like(out)
    sg.sgqa_gated_swa(dims, window, d["q"], d["k"], d["v"], d["gate"], out2, ws)
    torch.cuda.synchronize()
    assert sg.sgqa_get_device_status(ws) == 0
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))


@pytest.mark.parametrize("window", [8, 100, 512, 5000])
def test_swa_tiny(window):
    _run(CONFIGS["tiny"], window)


@pytest.mark.parametrize("window", [64, 700])
def test_swa_ragged_r8(window):
    _run(Config("swa_ragged_g4", 2, 3001, 32, 4, 128, 64, 8, 512, 400, 7), window)


def test_swa_b16_r16():
    _run(Config("swa_b16_r16", 1, 1000, 16, 1, 128, 64, 16, 256, 160, 9), 300)


def test_swa_b1_r4():
    _run(Config("swa_b1", 1, 1500, 8, 2, 64, 32, 1, 128, 200, 8), 50)


def test_swa_128k_sampled():
    cfg = CONFIGS["128k"]
    _run(cfg, 4096, sample_rows(cfg.replace(k=_capacity(4096, cfg.B)), 24, seed=5))

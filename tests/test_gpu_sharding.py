"""GPU: the query-sharded prefill, emulated on one GPU. Each of four ranks runs
sgqa_forward_rows on its zig-zag ranges with only its own rows of q, gate and q_idx (and the whole
sequence's k, v, k_idx, as the all-gather leaves them); put together, the outputs and selections
are bit-identical to a single sgqa_forward over the sequence."""
import pytest

torch = pytest.importorskip("torch")

import block_sparse_long_kbar_b200 as sg
from block_sparse_long_kbar_b200.sharding import prefill_rows, zigzag_ranges
from sgqa_inputs import Config
from tests._helpers import device_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg,world", [
    (Config("shard_tiny", 1, 2048, 8, 2, 64, 32, 8, 512, 256, 60), 4),
    (Config("shard_g4", 2, 4096, 32, 4, 128, 64, 8, 512, 400, 61), 4),
    (Config("shard_r2", 1, 1600, 8, 4, 64, 32, 8, 256, 150, 62), 2),
])
def test_query_sharded_prefill_equals_single_gpu_forward(cfg, world):
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    dims = sg.sgqa_dims.of(cfg)
    d = device_inputs(cfg)
    ws = sg.alloc_workspace(sg.sgqa_workspace_size(dims))
    sg.sgqa_reset_device_status(ws)
    out = torch.empty(cfg.shape("q"), dtype=torch.bfloat16, device="cuda")
    sel = torch.empty((cfg.batch, cfg.T, cfg.G, cfg.Kb), dtype=torch.int32, device="cuda")
    sg.sgqa_forward(dims, d["q"], d["k"], d["v"], d["q_idx"], d["k_idx"], d["gate"], out, ws, sel_out=sel)
    out_s = torch.full_like(out, float("nan"))
    sel_s = torch.full_like(sel, -7)
    for rank in range(world):
        ranges = zigzag_ranges(cfg.T, world, rank)
        rows = lambda n: [d[n][:, t0:t1].contiguous() for t0, t1 in ranges]
        outs = [torch.empty_like(x) for x in rows("q")]
        sels = [torch.empty((cfg.batch, t1 - t0, cfg.G, cfg.Kb), dtype=torch.int32, device="cuda") for t0, t1 in ranges]
        prefill_rows(dims, ranges, rows("q"), rows("gate"), rows("q_idx"), d["k"], d["v"], d["k_idx"], outs, ws,
                     sel_rows=sels)
        for (t0, t1), o, s_ in zip(ranges, outs, sels):
            out_s[:, t0:t1] = o
            sel_s[:, t0:t1] = s_
    torch.cuda.synchronize()
    assert sg.sgqa_get_device_status(ws) == 0
    assert torch.equal(sel_s, sel)
    assert torch.equal(out_s.view(torch.int16), out.view(torch.int16))


def test_forward_from_host_equals_forward():
    """The host-buffer entry point (chunked copies overlapped with sgqa_forward_rows) gives
    sgqa_forward's bits, for two sequences and a ragged last chunk."""
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    cfg = Config("from_host", 2, 3000, 32, 4, 128, 64, 8, 512, 400, 63)
    dims = sg.sgqa_dims.of(cfg)
    d = device_inputs(cfg)
    ws = sg.alloc_workspace(sg.sgqa_workspace_size(dims))
    sg.sgqa_reset_device_status(ws)
    out = torch.empty(cfg.shape("q"), dtype=torch.bfloat16, device="cuda")
    sg.sgqa_forward(dims, d["q"], d["k"], d["v"], d["q_idx"], d["k_idx"], d["gate"], out, ws)
    host = {n: torch.empty(d[n].shape, dtype=torch.bfloat16, pin_memory=True).copy_(d[n]) for n in d}
    dev = {n: torch.zeros_like(d[n]) for n in d}
    dev["out"] = torch.zeros_like(out)
    out_h = torch.empty(out.shape, dtype=torch.bfloat16, pin_memory=True)
    for _ in range(2):
        out_h.zero_()
        sg.sgqa_forward_from_host(dims, host, dev, out_h, ws, chunks=5)
        torch.cuda.synchronize()
        assert sg.sgqa_get_device_status(ws) == 0
        assert torch.equal(out_h.view(torch.int16), out.cpu().view(torch.int16))

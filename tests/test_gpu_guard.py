"""Guard bands: every output is written inside its own extent and nowhere else.

Each output tensor (and the decode caches, whose rows past cache_len + n_new must stay
untouched) is a view into a larger buffer filled with a canary pattern; after the call, the
bytes before and after the view must still hold the canary."""
import numpy as np
import pytest
import torch

import block_sparse_long_kbar_b200 as sg
from sgqa_inputs import CONFIGS, f64_to_bf16_bits
from tests._helpers import NAMES, device_inputs, shape_of

pytestmark = pytest.mark.gpu
GUARD = 4096  # elements on each side


def guarded(shape, dtype, fill):
    n = int(np.prod(shape))
    buf = torch.empty(n + 2 * GUARD, dtype=dtype, device="cuda")
    buf.view(torch.uint8).fill_(fill)
    return buf, buf[GUARD:GUARD + n].view(shape)


def assert_guard(buf, fill):
    torch.cuda.synchronize()
    u8 = buf.view(torch.uint8)
    e = buf.element_size()
    head, tail = u8[:GUARD * e], u8[u8.numel() - GUARD * e:]
    assert bool((head == fill).all()) and bool((tail == fill).all()), "a write left the tensor's extent"


@pytest.mark.parametrize("T,batch", [(2048, 1), (1000, 2)])
def test_forward_swa_and_backward_write_only_their_outputs(T, batch):
    cfg = CONFIGS["tiny"].replace(T=T, batch=batch)
    d = device_inputs(cfg)
    dims = sg.sgqa_dims.of(cfg)
    ws = sg.alloc_workspace(sg.sgqa_workspace_size(dims))
    sg.sgqa_reset_device_status(ws)
    ob, out = guarded(shape_of(cfg, "q"), torch.bfloat16, 0xA5)
    sb, sel = guarded((cfg.batch, cfg.T, cfg.G, cfg.Kb), torch.int32, 0x5A)
    sg.sgqa_forward(dims, d["q"], d["k"], d["v"], d["q_idx"], d["k_idx"], d["gate"], out, ws, sel_out=sel)
    assert_guard(ob, 0xA5)
    assert_guard(sb, 0x5A)
    wb, swa = guarded(shape_of(cfg, "q"), torch.bfloat16, 0x3C)
    sg.sgqa_gated_swa(dims, 256, d["q"], d["k"], d["v"], d["gate"], swa, ws)
    assert_guard(wb, 0x3C)
    assert sg.sgqa_get_device_status(ws) == 0
    bws = sg.alloc_workspace(sg.sgqa_backward_workspace_size(dims))
    sg.sgqa_reset_device_status(bws)
    dy = torch.from_numpy(f64_to_bf16_bits(np.random.default_rng(1).standard_normal(shape_of(cfg, "q"))).view(
        np.int16)).view(torch.bfloat16).cuda()
    grads = {}
    for n, like in (("dq", "q"), ("dk", "k"), ("dv", "k"), ("dgate", "q")):
        grads[n] = guarded(shape_of(cfg, like), torch.float32, 0xC3)
    sg.sgqa_attend_backward(dims, d["q"], d["k"], d["v"], d["gate"], sel, dy, *[grads[n][1] for n in
                                                                                  ("dq", "dk", "dv", "dgate")], bws)
    for n in grads:
        assert_guard(grads[n][0], 0xC3)
    assert sg.sgqa_get_device_status(bws) == 0


def test_decode_writes_only_the_new_cache_rows_and_its_outputs():
    cfg = CONFIGS["tiny"]
    n_new, cache_len = 4, 1500
    dims = sg.sgqa_dims.of(cfg)
    full = device_inputs(cfg)
    caches, before = {}, {}
    for n in ("k", "v", "k_idx"):
        buf, c = guarded(shape_of(cfg, n), torch.bfloat16, 0x99)
        c.copy_(full[n])
        caches[n] = (buf, c)
        before[n] = c.clone()
    kbar = torch.zeros((cfg.batch, cfg.T // cfg.B, cfg.d_idx), device="cuda")
    sg.sgqa_compress_keys(sg.sgqa_dims(cfg.batch, cache_len, cfg.Hq, cfg.G, cfg.d, cfg.d_idx, cfg.B, cfg.k),
                          caches["k_idx"][1], kbar, None)
    new = {n: full[n][:, cache_len:cache_len + n_new].contiguous() for n in NAMES}
    ob, out = guarded(new["q"].shape, torch.bfloat16, 0x77)
    sb, sel = guarded((cfg.batch, n_new, cfg.G, cfg.Kb), torch.int32, 0x66)
    ws = sg.alloc_workspace(sg.sgqa_decode_workspace_size(dims, n_new))
    sg.sgqa_reset_device_status(ws)
    sg.sgqa_decode(dims, cache_len, n_new, caches["k"][1], caches["v"][1], caches["k_idx"][1], kbar, new["q"],
                   new["k"], new["v"], new["q_idx"], new["k_idx"], new["gate"], out, ws, sel_out=sel)
    assert_guard(ob, 0x77)
    assert_guard(sb, 0x66)
    for n in caches:
        assert_guard(caches[n][0], 0x99)
        c = caches[n][1]
        # rows before the cache end and after the appended ones are unchanged; the appended rows
        # hold the new tokens
        assert torch.equal(c[:, :cache_len], before[n][:, :cache_len]), n
        assert torch.equal(c[:, cache_len + n_new:], before[n][:, cache_len + n_new:]), n
        assert torch.equal(c[:, cache_len:cache_len + n_new], new[n]), n
    assert sg.sgqa_get_device_status(ws) == 0

"""sgqa_decode_noalloc: the decode step for callers that cannot allocate device memory.

Such callers (a plugin inside a server whose allocator owns all device memory, code that may
not touch the CUDA allocator, an embedder with a fixed memory budget) get a decode entry point
that takes no workspace and uses the library's fixed device scratch array instead. This test
calls it through the C ABI twice in a row and checks each result against sgqa_decode with a
caller-allocated workspace on the same inputs, within the parity tolerances used throughout
(max-abs 1e-2, mean-abs 1e-3), plus identical selections. The file is named so that pytest
collects it last.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import block_sparse_long_kbar_b200 as sg
from sgqa_inputs import Config, gen_device
from tests._helpers import NAMES, assert_outputs_close, to_host
from sgqa_inputs import bf16_bits_to_f64

pytestmark = pytest.mark.gpu


def test_decode_noalloc_matches_decode_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    cfg = Config("noalloc", 2, 5000, 32, 4, 128, 64, 8, 512, 600, 21)
    cache_len, n_new = 4996, 4
    T_cap = 5008
    dims = sg.sgqa_dims(cfg.batch, T_cap, cfg.Hq, cfg.G, cfg.d, cfg.d_idx, cfg.B, cfg.k)
    assert 0 < sg.sgqa_decode_workspace_size(dims, n_new) <= sg.NOALLOC_SCRATCH_BYTES
    caches = {}
    for n in ("k", "v", "k_idx"):
        caches[n] = torch.zeros(cfg.shape(n, T=T_cap), dtype=torch.bfloat16, device="cuda")
        gen_device(cfg, n, caches[n], t0=0, n_t=cache_len)
    kbar = torch.zeros((cfg.batch, T_cap // cfg.B, cfg.d_idx), device="cuda")
    sg.sgqa_compress_keys(dims, caches["k_idx"], kbar, None)
    new = {}
    for n in NAMES:
        new[n] = torch.empty((cfg.batch, n_new) + cfg.shape(n)[2:], dtype=torch.bfloat16, device="cuda")
        gen_device(cfg, n, new[n], t0=cache_len, n_t=n_new, dst_t0=0)

    def run(fn, with_sel=True, **kw):
        out = torch.full((cfg.batch, n_new, cfg.Hq, cfg.d), float("nan"), dtype=torch.bfloat16, device="cuda")
        sel = torch.full((cfg.batch, n_new, cfg.G, cfg.Kb), -7, dtype=torch.int32, device="cuda")
        fn(dims, cache_len, n_new, caches["k"], caches["v"], caches["k_idx"], kbar, new["q"], new["k"], new["v"],
           new["q_idx"], new["k_idx"], new["gate"], out, sel_out=sel if with_sel else None, **kw)
        torch.cuda.synchronize()
        return out, sel

    ws = sg.alloc_workspace(sg.sgqa_decode_workspace_size(dims, n_new))
    sg.sgqa_reset_device_status(ws)
    ref_out, ref_sel = run(sg.sgqa_decode, ws=ws)
    assert sg.sgqa_get_device_status(ws) == 0
    ref = bf16_bits_to_f64(to_host(ref_out))
    # two calls in a row, the second without sel_out (the selection then lives in the scratch
    # array); both run the same kernels on the same inputs as sgqa_decode, so the bits agree too
    for with_sel in (True, False):
        out, sel = run(sg.sgqa_decode_noalloc, with_sel=with_sel)
        if with_sel:
            assert torch.equal(sel, ref_sel)
        assert_outputs_close(to_host(out), ref, "sgqa_decode_noalloc vs sgqa_decode")
        assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16))


def test_decode_noalloc_rejects_sizes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    dims = sg.sgqa_dims(32, (1 << 20) + 8, 32, 4, 128, 64, 8, 4096)
    assert sg.sgqa_decode_workspace_size(dims, 4) > sg.NOALLOC_SCRATCH_BYTES
    x = torch.zeros(8, dtype=torch.bfloat16, device="cuda")
    f = torch.zeros(8, dtype=torch.float32, device="cuda")
    with pytest.raises(sg.SgqaError) as e:
        sg.sgqa_decode_noalloc(dims, 1 << 20, 4, x, x, x, f, x, x, x, x, x, x, x)
    assert e.value.code == 3

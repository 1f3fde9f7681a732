"""Runs the layer's entry points on one small seeded workload and saves every result.

Used by the bounds-check tests: run once with the normal library and once (in a child process
with SGQA_LIBRARY=checks) with the bounds-checking build, then the two result files are compared
bit for bit. Usage: python tests/_layer_runner.py OUT.npz
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def run(path: str) -> None:
    import numpy as np
    import torch

    import block_sparse_long_kbar_b200 as sg
    from sgqa_inputs import CONFIGS, f64_to_bf16_bits
    from tests._helpers import NAMES, device_inputs, shape_of

    torch.cuda.set_device(0)
    res = {}
    for name, T in (("tiny", None), ("tiny", 1000)):  # whole tiles, then two ragged sequences
        cfg = CONFIGS[name]
        if T is not None:
            cfg = cfg.replace(T=T, batch=2)
        d = device_inputs(cfg)
        dims = sg.sgqa_dims.of(cfg)
        ws = sg.alloc_workspace(sg.sgqa_workspace_size(dims))
        sg.sgqa_reset_device_status(ws)
        out = torch.empty(shape_of(cfg, "q"), dtype=torch.bfloat16, device="cuda")
        sel = torch.empty((cfg.batch, cfg.T, cfg.G, cfg.Kb), dtype=torch.int32, device="cuda")
        sg.sgqa_forward(dims, d["q"], d["k"], d["v"], d["q_idx"], d["k_idx"], d["gate"], out, ws, sel_out=sel)
        swa = torch.empty_like(out)
        sg.sgqa_gated_swa(dims, 256, d["q"], d["k"], d["v"], d["gate"], swa, ws)
        torch.cuda.synchronize()
        tag = f"{name}_{cfg.T}"
        res[f"{tag}_status_fwd"] = np.array(sg.sgqa_get_device_status(ws))
        res[f"{tag}_out"] = out.view(torch.int16).cpu().numpy()
        res[f"{tag}_sel"] = sel.cpu().numpy()
        res[f"{tag}_swa"] = swa.view(torch.int16).cpu().numpy()
        # backward through the selection
        bdims = dims
        bws = sg.alloc_workspace(sg.sgqa_backward_workspace_size(bdims))
        sg.sgqa_reset_device_status(bws)
        dy = torch.from_numpy(f64_to_bf16_bits(np.random.default_rng(7).standard_normal(shape_of(cfg, "q"))).view(
            np.int16)).view(torch.bfloat16).cuda()
        g = {n: torch.empty(shape_of(cfg, "q" if n in ("dq", "dgate") else "k"), dtype=torch.float32, device="cuda")
             for n in ("dq", "dk", "dv", "dgate")}
        sg.sgqa_attend_backward(bdims, d["q"], d["k"], d["v"], d["gate"], sel, dy, g["dq"], g["dk"], g["dv"],
                                g["dgate"], bws)
        torch.cuda.synchronize()
        res[f"{tag}_status_bwd"] = np.array(sg.sgqa_get_device_status(bws))
        for n in g:
            res[f"{tag}_{n}"] = g[n].cpu().numpy()
    # decode: 4 new tokens after a 2044-token cache
    cfg = CONFIGS["tiny"]
    n_new, cache_len = 4, cfg.T - 4
    dims = sg.sgqa_dims.of(cfg)
    full = device_inputs(cfg)
    caches = {n: full[n].clone() for n in ("k", "v", "k_idx")}
    kbar = torch.zeros((cfg.batch, cfg.T // cfg.B, cfg.d_idx), device="cuda")
    sg.sgqa_compress_keys(sg.sgqa_dims(cfg.batch, cache_len, cfg.Hq, cfg.G, cfg.d, cfg.d_idx, cfg.B, cfg.k),
                          caches["k_idx"], kbar, None)
    new = {n: full[n][:, cache_len:].contiguous() for n in NAMES}
    out = torch.empty_like(new["q"])
    sel = torch.empty((cfg.batch, n_new, cfg.G, cfg.Kb), dtype=torch.int32, device="cuda")
    ws = sg.alloc_workspace(sg.sgqa_decode_workspace_size(dims, n_new))
    sg.sgqa_reset_device_status(ws)
    sg.sgqa_decode(dims, cache_len, n_new, caches["k"], caches["v"], caches["k_idx"], kbar, new["q"], new["k"],
                   new["v"], new["q_idx"], new["k_idx"], new["gate"], out, ws, sel_out=sel)
    torch.cuda.synchronize()
    res["decode_status"] = np.array(sg.sgqa_get_device_status(ws))
    res["decode_out"] = out.view(torch.int16).cpu().numpy()
    res["decode_sel"] = sel.cpu().numpy()
    res["library"] = np.array(os.path.basename(sg.SO_PATH))
    np.savez(path, **res)


if __name__ == "__main__":
    run(sys.argv[1])

"""Pins of the oracle's Gated SWA (the efficient layer that alternates 3:1 with Sparse GQA;
mo.ai.kr, "Step 5 Preview agentic work design", section "model structure and training
stability"): the gated softmax attention over the keys t - window < u <= t.

* brute force: a dense T x T score matrix with a band mask, softmax by numpy, gate;
* window >= T: dense causal gated GQA, against torch's scaled_dot_product_attention in fp64;
* window a multiple of B at the last token of a block: the oracle's selection-based attention
  over the window's whole blocks;
* locality: keys outside the window do not change the row.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from sgqa_inputs import Config, bf16_bits_to_f64, gen_full


def _case(T, B, Hq=4, G=2, d=8, seed=0, batch=1, k=None):
    cfg = Config("swa", batch, T, Hq, G, d, 4, B, k or B, max(2 * B, 8), seed)
    x = {n: gen_full(cfg, n) for n in ("q", "k", "v", "gate")}
    return cfg, x


def _rows(cfg):
    bb, tt = np.meshgrid(np.arange(cfg.batch), np.arange(cfg.T), indexing="ij")
    return np.stack([bb.ravel(), tt.ravel()], axis=1).astype(np.int32)


def _swa(cfg, x, window, rows=None):
    rows = _rows(cfg) if rows is None else rows
    n = len(rows)
    q = np.stack([x["q"][b].reshape(cfg.T, -1)[t] for b, t in rows])
    gate = np.stack([x["gate"][b].reshape(cfg.T, -1)[t] for b, t in rows])
    return oracle.swa(oracle.dims_of(cfg), rows, q, x["k"], x["v"], gate, window).reshape(n, cfg.Hq, cfg.d)


def _brute(cfg, x, window):
    T, Hq, G, d = cfg.T, cfg.Hq, cfg.G, cfg.d
    R = Hq // G
    outs = []
    for b in range(cfg.batch):
        q = bf16_bits_to_f64(x["q"][b]).reshape(T, Hq, d)
        k = bf16_bits_to_f64(x["k"][b]).reshape(T, G, d)
        v = bf16_bits_to_f64(x["v"][b]).reshape(T, G, d)
        gate = bf16_bits_to_f64(x["gate"][b]).reshape(T, Hq, d)
        tt, uu = np.meshgrid(np.arange(T), np.arange(T), indexing="ij")
        band = (uu <= tt) & (uu > tt - window)
        out = np.zeros((T, Hq, d))
        for h in range(Hq):
            z = q[:, h, :] @ k[:, h // R, :].T / math.sqrt(d)
            z = np.where(band, z, -np.inf)
            p = np.exp(z - z.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            out[:, h, :] = (p @ v[:, h // R, :]) / (1.0 + np.exp(-gate[:, h, :]))
        outs.append(out)
    return np.concatenate(outs)


@pytest.mark.parametrize("T,B,window", [(40, 8, 8), (40, 8, 13), (64, 4, 24), (33, 1, 5), (50, 8, 1)])
def test_swa_brute_force(oracle_lib, T, B, window):
    cfg, x = _case(T, B, seed=T + window, batch=2)
    np.testing.assert_allclose(_swa(cfg, x, window), _brute(cfg, x, window), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("T,Hq,G,d", [(70, 8, 2, 16), (45, 6, 3, 8)])
def test_swa_full_window_is_dense_causal(oracle_lib, T, Hq, G, d):
    cfg, x = _case(T, 8, Hq=Hq, G=G, d=d, seed=7)
    out = _swa(cfg, x, window=T)
    q = torch.from_numpy(bf16_bits_to_f64(x["q"][0]).reshape(T, Hq, d)).permute(1, 0, 2)[None]
    kk = torch.from_numpy(bf16_bits_to_f64(x["k"][0]).reshape(T, G, d)).permute(1, 0, 2)[None]
    vv = torch.from_numpy(bf16_bits_to_f64(x["v"][0]).reshape(T, G, d)).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(q, kk, vv, is_causal=True, enable_gqa=True)
    gate = torch.from_numpy(bf16_bits_to_f64(x["gate"][0]).reshape(T, Hq, d))
    ref = ref[0].permute(1, 0, 2).numpy() * torch.sigmoid(gate).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


def test_swa_block_aligned_window_equals_block_selection(oracle_lib):
    """At t = cB + B - 1 a window of nB tokens is exactly the blocks c-n+1 .. c."""
    T, B, n = 96, 8, 3
    cfg, x = _case(T, B, seed=3, k=n * B)
    rows = np.array([[0, t] for t in range(B - 1, T, B)], dtype=np.int32)
    out = _swa(cfg, x, n * B, rows)
    sel = np.full((len(rows), cfg.G, n), -1, dtype=np.int32)
    for i, (_, t) in enumerate(rows):
        c = t // B
        blocks = list(range(max(0, c - n + 1), c + 1))
        sel[i, :, :len(blocks)] = blocks
    q = np.stack([x["q"][0].reshape(T, -1)[t] for _, t in rows])
    gate = np.stack([x["gate"][0].reshape(T, -1)[t] for _, t in rows])
    ref = oracle.attend(oracle.dims_of(cfg), rows, q, x["k"], x["v"], gate, sel).reshape(out.shape)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_swa_locality(oracle_lib):
    T, B, window, t = 60, 4, 10, 37
    cfg, x = _case(T, B, seed=9)
    rows = np.array([[0, t]], dtype=np.int32)
    base = _swa(cfg, x, window, rows)
    y = {n: v.copy() for n, v in x.items()}
    far = [u for u in range(T) if u <= t - window or u > t]
    y["k"][0].reshape(T, -1)[far] ^= 0x00FF
    y["v"][0].reshape(T, -1)[far] ^= 0x00FF
    np.testing.assert_array_equal(_swa(cfg, y, window, rows), base)
    # and a key inside the window does change it
    y["k"][0].reshape(T, -1)[t - window + 1] ^= 0x00FF
    assert not np.array_equal(_swa(cfg, y, window, rows), base)

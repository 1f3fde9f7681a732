"""Pins of the oracle's backward (gradients of the gated attention through a fixed selection).

* dense reduction: with every block selected, the layer is causal gated GQA, so its gradients
  are torch autograd's through scaled_dot_product_attention(is_causal=True, enable_gqa=True) in
  fp64, times sigmoid(gate);
* a sparse selection: torch autograd through a dense softmax masked to the selected tokens (the
  derivative is autograd's, not a hand formula);
* central finite differences of the oracle's own forward (oracle.attend) on single elements of
  q, k, v and gate, stepped by one bf16 ulp either way.
"""
import numpy as np
import pytest
import torch

import oracle
from sgqa_inputs import Config, bf16_bits_to_f64, f64_to_bf16_bits, gen_full


def _case(T, B, k, Hq=4, G=2, d=8, seed=0):
    cfg = Config("bw", 1, T, Hq, G, d, 4, B, k, max(2 * B, 8), seed)
    x = {n: gen_full(cfg, n) for n in ("q", "k", "v", "gate", "q_idx", "k_idx")}
    dy = f64_to_bf16_bits(np.random.default_rng(seed + 100).standard_normal((1, T, Hq * d)))
    return cfg, x, dy


def _oracle_grads(cfg, x, dy, sel):
    dm = oracle.dims_of(cfg)
    rows = np.array([[0, t] for t in range(cfg.T)], dtype=np.int32)
    return oracle.attend_backward(dm, rows, x["q"].reshape(cfg.T, -1), x["k"], x["v"], x["gate"].reshape(cfg.T, -1),
                                  sel, dy.reshape(cfg.T, -1))


def _torch_inputs(cfg, x, dy):
    f = lambda n: torch.from_numpy(bf16_bits_to_f64(x[n])).double()
    q = f("q").reshape(cfg.T, cfg.Hq, cfg.d).requires_grad_()
    k = f("k").reshape(cfg.T, cfg.G, cfg.d).requires_grad_()
    v = f("v").reshape(cfg.T, cfg.G, cfg.d).requires_grad_()
    gl = f("gate").reshape(cfg.T, cfg.Hq, cfg.d).requires_grad_()
    g = torch.from_numpy(bf16_bits_to_f64(dy)).double().reshape(cfg.T, cfg.Hq, cfg.d)
    return q, k, v, gl, g


def _check(cfg, grads, q, k, v, gl):
    dq, dk, dv, dgate = grads
    np.testing.assert_allclose(dq.reshape(q.shape), q.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dk.reshape(k.shape), k.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dv.reshape(v.shape), v.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dgate.reshape(gl.shape), gl.grad.numpy(), rtol=1e-9, atol=1e-11)


@pytest.mark.parametrize("T,B", [(40, 8), (33, 4), (24, 1)])
def test_backward_dense_reduction_matches_sdpa_autograd(oracle_lib, T, B):
    cfg, x, dy = _case(T, B, ((T + B - 1) // B) * B, seed=T + B)
    dm = oracle.dims_of(cfg)
    rows = np.array([[0, t] for t in range(T)], dtype=np.int32)
    kbar = oracle.compress(dm, x["k_idx"])
    sel, _, _ = oracle.select(dm, kbar, rows, x["q_idx"].reshape(T, -1))
    assert (sel >= 0).sum(axis=2).min() >= 1
    q, k, v, gl, g = _torch_inputs(cfg, x, dy)
    o = torch.nn.functional.scaled_dot_product_attention(q.transpose(0, 1)[None], k.transpose(0, 1)[None],
                                                         v.transpose(0, 1)[None], is_causal=True, enable_gqa=True)
    y = o[0].transpose(0, 1) * torch.sigmoid(gl)
    (y * g).sum().backward()
    _check(cfg, _oracle_grads(cfg, x, dy, sel), q, k, v, gl)


def test_backward_sparse_selection_matches_masked_autograd(oracle_lib):
    T, B = 48, 4
    cfg, x, dy = _case(T, B, 12, seed=7)
    dm = oracle.dims_of(cfg)
    rows = np.array([[0, t] for t in range(T)], dtype=np.int32)
    kbar = oracle.compress(dm, x["k_idx"])
    sel, _, _ = oracle.select(dm, kbar, rows, x["q_idx"].reshape(T, -1))
    mask = np.zeros((cfg.G, T, T), dtype=bool)
    for t in range(T):
        for g in range(cfg.G):
            for j in sel[t, g]:
                if j >= 0:
                    mask[g, t, j * B:min((j + 1) * B, t + 1)] = True
    assert not mask[:, T - 1].all()  # the selection really is sparse
    q, k, v, gl, g = _torch_inputs(cfg, x, dy)
    R = cfg.Hq // cfg.G
    outs = []
    for h in range(cfg.Hq):
        gg = h // R
        z = q[:, h] @ k[:, gg].T / np.sqrt(cfg.d)
        z = z.masked_fill(~torch.from_numpy(mask[gg]), float("-inf"))
        outs.append(torch.softmax(z, dim=1) @ v[:, gg])
    y = torch.stack(outs, dim=1) * torch.sigmoid(gl)
    (y * g).sum().backward()
    _check(cfg, _oracle_grads(cfg, x, dy, sel), q, k, v, gl)


def test_backward_matches_finite_differences_of_the_forward(oracle_lib):
    T, B = 30, 4
    cfg, x, dy = _case(T, B, 8, seed=11)
    dm = oracle.dims_of(cfg)
    rows = np.array([[0, t] for t in range(T)], dtype=np.int32)
    kbar = oracle.compress(dm, x["k_idx"])
    sel, _, _ = oracle.select(dm, kbar, rows, x["q_idx"].reshape(T, -1))
    dq, dk, dv, dgate = _oracle_grads(cfg, x, dy, sel)
    dyf = bf16_bits_to_f64(dy).reshape(T, cfg.Hq, cfg.d)

    def loss(xx):
        out = oracle.attend(dm, rows, xx["q"].reshape(T, -1), xx["k"], xx["v"], xx["gate"].reshape(T, -1), sel)
        return float((out.reshape(T, cfg.Hq, cfg.d) * dyf).sum())

    rng = np.random.default_rng(3)
    grads = {"q": dq.reshape(x["q"].shape), "k": dk.reshape(x["k"].shape), "v": dv.reshape(x["v"].shape),
             "gate": dgate.reshape(x["gate"].shape)}
    for name in ("q", "k", "v", "gate"):
        flat = x[name].reshape(-1)
        for idx in rng.integers(0, flat.size, size=6):
            bits = int(flat[idx])
            up, dn = x[name].copy(), x[name].copy()
            # one bf16 ulp up and down in magnitude (same sign), the exact step taken from the values
            up.reshape(-1)[idx] = bits + 1
            dn.reshape(-1)[idx] = bits - 1
            xu, xd = dict(x), dict(x)
            xu[name], xd[name] = up, dn
            a = bf16_bits_to_f64(np.array([bits + 1], dtype=np.uint16))[0]
            c = bf16_bits_to_f64(np.array([bits - 1], dtype=np.uint16))[0]
            fd = (loss(xu) - loss(xd)) / (a - c)
            gval = grads[name].reshape(-1)[idx]
            assert abs(fd - gval) <= 2e-3 * max(1.0, abs(gval)) + 1e-6, (name, idx, fd, gval)

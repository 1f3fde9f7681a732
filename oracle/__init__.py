"""Sparse GQA oracle (fp64, CPU): ctypes wrapper over sgqa_oracle.cpp.

TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline
and reference legs may import this package. The product library never calls it, and it
shares no code with the CUDA path.

Definition followed (Step 5 Preview pages; mo.ai.kr "Step 5 Preview agentic work design",
section "model structure and training stability", and ai.info "StepFun illustrates the 92-block
architecture of Step 5 Preview", section "Sparse GQA aims at a 1 million token context"):
block-mean index keys (B tokens per block), per-KV-group top-(k/B) block selection that always
keeps the query's own block, causal softmax attention of every head of the group over the
selected tokens scaled by 1/sqrt(d), and an elementwise sigmoid output gate. Also the Gated SWA
layer that alternates 3:1 with it (same section): the gated attention over a sliding window of
keys, the window size being a parameter (the pages give none). And the FP8 storage of the KV
cache (section "long-horizon RL and run cost"): e4m3 values with a power-of-two scale per
(token, group) row; decode over an FP8 cache is attention over the dequantized values. And the
backward of the gated attention through a fixed selection (dq, dk, dv, dgate).

Parity pins: every function here is pinned by tests/test_oracle_pins.py (brute force on
T <= 64, dense reduction against torch's SDPA in fp64, closed forms and invariants).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(_HERE, "liboracle.so")
SRC = os.path.join(_HERE, "sgqa_oracle.cpp")
_lib = None


class Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("batch", "T", "Hq", "G", "d", "d_idx", "B", "k")]


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (plain -O2, OpenMP, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(SO) or os.path.getmtime(SO) < os.path.getmtime(SRC):
        cmd = ["g++", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
               "-o", SO, SRC]
        subprocess.run(cmd, check=True)
    return SO


def load(path: str):
    """Load and configure an oracle shared object (the default one, or a test's mutant)."""
    L = ctypes.CDLL(path)
    P = ctypes.c_void_p
    L.oracle_compress.argtypes = [ctypes.POINTER(Dims), P, P, ctypes.c_int]
    L.oracle_scores.argtypes = [ctypes.POINTER(Dims), P, P, ctypes.c_int, P]
    L.oracle_select.argtypes = [ctypes.POINTER(Dims), P, ctypes.c_int, P, P, P, P, P, ctypes.c_int]
    L.oracle_attend.argtypes = [ctypes.POINTER(Dims), ctypes.c_int, P, P, P, P, P, P, P, ctypes.c_int]
    L.oracle_coverage.argtypes = [ctypes.POINTER(Dims), ctypes.c_int, P, P, P, P, ctypes.c_int, P,
                                  ctypes.c_int]
    L.oracle_swa.argtypes = [ctypes.POINTER(Dims), ctypes.c_int, P, P, P, P, P, ctypes.c_int, P, ctypes.c_int]
    L.oracle_quantize_fp8.argtypes = [ctypes.c_int, ctypes.c_int, P, P, P]
    L.oracle_attend_backward.argtypes = [ctypes.POINTER(Dims), ctypes.c_int, P, P, P, P, P, P, P, P, P, P, P]
    L.oracle_dequantize_fp8.argtypes = [ctypes.c_int, ctypes.c_int, P, P, P]
    for f in (L.oracle_compress, L.oracle_scores, L.oracle_select, L.oracle_attend, L.oracle_coverage,
              L.oracle_swa, L.oracle_max_threads, L.oracle_quantize_fp8, L.oracle_dequantize_fp8,
              L.oracle_attend_backward):
        f.restype = ctypes.c_int
    return L


def lib():
    global _lib
    if _lib is None:
        build()
        _lib = load(SO)
    return _lib


def max_threads() -> int:
    return lib().oracle_max_threads()


def dims(batch, T, Hq, G, d, d_idx, B, k) -> Dims:
    return Dims(batch, T, Hq, G, d, d_idx, B, k)


def dims_of(cfg, T=None) -> Dims:
    return Dims(cfg.batch, cfg.T if T is None else T, cfg.Hq, cfg.G, cfg.d, cfg.d_idx, cfg.B, cfg.k)


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


def compress(dm: Dims, k_idx: np.ndarray, n_threads: int = 0) -> np.ndarray:
    """kbar [batch, T//B, d_idx] fp64 from k_idx [batch, T, d_idx] (bf16 bits)."""
    k_idx = _u16(k_idx)
    assert k_idx.size == dm.batch * dm.T * dm.d_idx
    kbar = np.zeros((dm.batch, dm.T // dm.B, dm.d_idx), dtype=np.float64)
    rc = lib().oracle_compress(ctypes.byref(dm), _p(k_idx), _p(kbar), n_threads)
    if rc != 0:
        raise ValueError(f"oracle_compress: {rc}")
    return kbar


def scores(dm: Dims, kbar: np.ndarray, b: int, q_idx_row: np.ndarray, n: int) -> np.ndarray:
    """fp64 indexer scores of one (token, group) row against blocks j < n of sequence b."""
    q_idx_row = _u16(q_idx_row).reshape(-1)
    assert q_idx_row.size == dm.d_idx
    kb = np.ascontiguousarray(kbar[b])
    s = np.zeros(max(n, 1), dtype=np.float64)
    rc = lib().oracle_scores(ctypes.byref(dm), _p(kb), _p(q_idx_row), n, _p(s))
    if rc != 0:
        raise ValueError(f"oracle_scores: {rc}")
    return s[:n]


def _rows(rows_bt) -> np.ndarray:
    r = np.ascontiguousarray(np.asarray(rows_bt, dtype=np.int32).reshape(-1, 2))
    return r


def select(dm: Dims, kbar: np.ndarray, rows_bt, q_idx_rows: np.ndarray, n_threads: int = 0):
    """Returns (sel [n, G, Kb] int32, s_m [n, G], s_m1 [n, G]) for query rows (b, t)."""
    rows = _rows(rows_bt)
    n = rows.shape[0]
    q_idx_rows = _u16(q_idx_rows)
    assert q_idx_rows.size == n * dm.G * dm.d_idx
    kbar = np.ascontiguousarray(kbar, dtype=np.float64)
    Kb = dm.k // dm.B
    sel = np.full((n, dm.G, Kb), -7, dtype=np.int32)
    s_m = np.zeros((n, dm.G))
    s_m1 = np.zeros((n, dm.G))
    rc = lib().oracle_select(ctypes.byref(dm), _p(kbar), n, _p(rows), _p(q_idx_rows), _p(sel), _p(s_m),
                             _p(s_m1), n_threads)
    if rc != 0:
        raise ValueError(f"oracle_select: {rc}")
    return sel, s_m, s_m1


def attend(dm: Dims, rows_bt, q_rows, k, v, gate_rows, sel, n_threads: int = 0) -> np.ndarray:
    """out [n, Hq, d] fp64 for query rows (b, t) given a selection sel [n, G, Kb]."""
    rows = _rows(rows_bt)
    n = rows.shape[0]
    q_rows, gate_rows, k, v = _u16(q_rows), _u16(gate_rows), _u16(k), _u16(v)
    assert q_rows.size == n * dm.Hq * dm.d and gate_rows.size == q_rows.size
    assert k.size == dm.batch * dm.T * dm.G * dm.d and v.size == k.size
    sel = np.ascontiguousarray(sel, dtype=np.int32)
    assert sel.size == n * dm.G * (dm.k // dm.B)
    out = np.zeros((n, dm.Hq, dm.d), dtype=np.float64)
    rc = lib().oracle_attend(ctypes.byref(dm), n, _p(rows), _p(q_rows), _p(k), _p(v), _p(gate_rows), _p(sel),
                             _p(out), n_threads)
    if rc != 0:
        raise ValueError(f"oracle_attend: {rc}")
    return out


def swa(dm: Dims, rows_bt, q_rows, k, v, gate_rows, window: int, n_threads: int = 0) -> np.ndarray:
    """Gated SWA: out [n, Hq, d] fp64 for query rows (b, t) over the keys t - window < u <= t."""
    rows = _rows(rows_bt)
    n = rows.shape[0]
    q_rows, gate_rows, k, v = _u16(q_rows), _u16(gate_rows), _u16(k), _u16(v)
    assert q_rows.size == n * dm.Hq * dm.d and gate_rows.size == q_rows.size
    assert k.size == dm.batch * dm.T * dm.G * dm.d and v.size == k.size
    out = np.zeros((n, dm.Hq, dm.d), dtype=np.float64)
    rc = lib().oracle_swa(ctypes.byref(dm), n, _p(rows), _p(q_rows), _p(k), _p(v), _p(gate_rows), int(window),
                          _p(out), n_threads)
    if rc != 0:
        raise ValueError(f"oracle_swa: {rc}")
    return out


def coverage(dm: Dims, rows_bt, q_rows, k, sel, ktop: int = 2048, n_threads: int = 0) -> np.ndarray:
    """cov [n, Hq]: fraction of the top-ktop dense-score tokens that the selection covers."""
    rows = _rows(rows_bt)
    n = rows.shape[0]
    q_rows, k = _u16(q_rows), _u16(k)
    sel = np.ascontiguousarray(sel, dtype=np.int32)
    cov = np.zeros((n, dm.Hq), dtype=np.float64)
    rc = lib().oracle_coverage(ctypes.byref(dm), n, _p(rows), _p(q_rows), _p(k), _p(sel), ktop, _p(cov),
                               n_threads)
    if rc != 0:
        raise ValueError(f"oracle_coverage: {rc}")
    return cov


def attend_backward(dm: Dims, rows_bt, q_rows, k, v, gate_rows, sel, dy_rows):
    """Gradients of the gated attention through a fixed selection, for query rows (b, t):
    returns (dq [n, Hq, d], dk [batch, T, G, d], dv [batch, T, G, d], dgate [n, Hq, d]) in fp64,
    dk and dv summed over the listed rows."""
    rows = _rows(rows_bt)
    n = rows.shape[0]
    q_rows, gate_rows, k, v, dy_rows = _u16(q_rows), _u16(gate_rows), _u16(k), _u16(v), _u16(dy_rows)
    assert q_rows.size == n * dm.Hq * dm.d and gate_rows.size == q_rows.size and dy_rows.size == q_rows.size
    assert k.size == dm.batch * dm.T * dm.G * dm.d and v.size == k.size
    sel = np.ascontiguousarray(sel, dtype=np.int32)
    assert sel.size == n * dm.G * (dm.k // dm.B)
    dq = np.zeros((n, dm.Hq, dm.d))
    dgate = np.zeros((n, dm.Hq, dm.d))
    dk = np.zeros((dm.batch, dm.T, dm.G, dm.d))
    dv = np.zeros((dm.batch, dm.T, dm.G, dm.d))
    rc = lib().oracle_attend_backward(ctypes.byref(dm), n, _p(rows), _p(q_rows), _p(k), _p(v), _p(gate_rows),
                                      _p(sel), _p(dy_rows), _p(dq), _p(dk), _p(dv), _p(dgate))
    if rc != 0:
        raise ValueError(f"oracle_attend_backward: {rc}")
    return dq, dk, dv, dgate


def quantize_fp8(x) -> tuple:
    """FP8 KV storage of bf16 rows x [..., d]: (codes uint8 [..., d] e4m3, scale fp64 [...]),
    one power-of-two scale per row (the smallest with max |x| <= 448 * scale)."""
    x = _u16(x)
    d = x.shape[-1]
    n = x.size // d
    q = np.zeros(x.shape, dtype=np.uint8)
    sc = np.zeros(x.shape[:-1], dtype=np.float64)
    rc = lib().oracle_quantize_fp8(n, d, _p(x), _p(q), _p(sc))
    if rc != 0:
        raise ValueError(f"oracle_quantize_fp8: {rc}")
    return q, sc


def dequantize_fp8(q, scale) -> np.ndarray:
    """fp64 values of FP8 rows: e4m3 value * row scale."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    scale = np.ascontiguousarray(scale, dtype=np.float64)
    d = q.shape[-1]
    out = np.zeros(q.shape, dtype=np.float64)
    rc = lib().oracle_dequantize_fp8(q.size // d, d, _p(q), _p(scale), _p(out))
    if rc != 0:
        raise ValueError(f"oracle_dequantize_fp8: {rc}")
    return out


def forward(dm: Dims, q, k, v, q_idx, k_idx, gate, rows_bt=None, n_threads: int = 0):
    """Whole layer for rows (b, t) (all rows when None). Full tensors in the natural layouts:
    q, gate [batch, T, Hq, d]; k, v [batch, T, G, d]; q_idx [batch, T, G, d_idx];
    k_idx [batch, T, d_idx]. Returns (sel, out, s_m, s_m1, rows)."""
    if rows_bt is None:
        bb, tt = np.meshgrid(np.arange(dm.batch), np.arange(dm.T), indexing="ij")
        rows_bt = np.stack([bb.ravel(), tt.ravel()], axis=1)
    rows = _rows(rows_bt)
    kbar = compress(dm, k_idx, n_threads)
    qi = _u16(np.asarray(q_idx).reshape(dm.batch, dm.T, -1)[rows[:, 0], rows[:, 1]])
    sel, s_m, s_m1 = select(dm, kbar, rows, qi, n_threads)
    qr = _u16(np.asarray(q).reshape(dm.batch, dm.T, -1)[rows[:, 0], rows[:, 1]])
    gr = _u16(np.asarray(gate).reshape(dm.batch, dm.T, -1)[rows[:, 0], rows[:, 1]])
    out = attend(dm, rows, qr, k, v, gr, sel, n_threads)
    return sel, out, s_m, s_m1, rows

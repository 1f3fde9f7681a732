"""Seeded synthetic inputs for Sparse GQA (Step 5 Preview's full-context attention layer).

This module is shared by the oracle side and the CUDA side and holds none of the
method's arithmetic: it only defines, element by element, the bf16 input tensors
of the workloads, as a pure function of (seed, tensor, position).

Workloads (Step 5 Preview pages, "model structure & training stability": blocks of
B=8, top-k of k=4096 tokens = 512 blocks, 1M-token context):

    q, k, v, gate_logits ~ N(0, 1)
    k_idx[b, t]    = N(0, 1) + 2 * topic[b, t // span]
    q_idx[b, t, g] = N(0, 1) + 2 * topic[b, r],  r uniform over {0 .. t // span}
    topic[b, s]    ~ N(0, I)  (fp64, never rounded)

Counter-based generator (our own definition; "seed n" means this generator's seed n):

    splitmix64(x): x += 0x9E3779B97F4A7C15; z = x;
                   z = (z ^ z>>30) * 0xBF58476D1CE4E5B9; z = (z ^ z>>27) * 0x94D049BB133111EB;
                   return z ^ z>>31                                   (all mod 2^64)
    key(seed, stream) = splitmix64(splitmix64(seed) ^ (stream * 0xD1B54A32D192ED03))
    word(key, i)      = splitmix64(key + i)
    u1 = ((word(key, 2i) >> 11) + 0.5) * 2^-53,  u2 = (word(key, 2i+1) >> 11) * 2^-53
    normal(key, i)    = sqrt(-2 ln u1) * cos(6.283185307179586 * u2)   (fp64 Box-Muller)

Element (b, t, w) of a tensor whose rows are W wide has counter i = (b * 2^32 + t) * W + w,
so a token's values do not depend on the sequence length: a decode step at position t
sees exactly the values a longer prefill would. Values are rounded fp64 -> fp32 (RNE)
-> bf16 (RNE) and handled as uint16 bit patterns.

The CUDA twin of this generator (for inputs too large to make on the host) is
``gen.cu`` in this directory; it implements the same definition.
"""
from __future__ import annotations

import dataclasses
import os
import ctypes
import numpy as np

M64 = (1 << 64) - 1
GOLDEN_GAMMA = 0x9E3779B97F4A7C15
STREAM_MUL = 0xD1B54A32D192ED03
TWO_PI = 6.283185307179586

STREAMS = {"q": 1, "k": 2, "v": 3, "gate": 4, "q_idx": 5, "k_idx": 6, "topic": 7, "r": 8}
KIND_CODES = {"q": 0, "k": 1, "v": 2, "gate": 3, "q_idx": 4, "k_idx": 5}


@dataclasses.dataclass(frozen=True)
class Config:
    """One Sparse GQA workload: shapes (b, T, Hq, G, d, d_idx, B, k), topic span and seed."""
    name: str
    batch: int
    T: int
    Hq: int
    G: int
    d: int
    d_idx: int
    B: int
    k: int
    span: int
    seed: int

    @property
    def Kb(self) -> int:
        return self.k // self.B

    @property
    def R(self) -> int:
        return self.Hq // self.G

    def width(self, name: str) -> int:
        return {"q": self.Hq * self.d, "gate": self.Hq * self.d, "k": self.G * self.d,
                "v": self.G * self.d, "q_idx": self.G * self.d_idx, "k_idx": self.d_idx}[name]

    def replace(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)

    def shape(self, name: str, T: int | None = None, batch: int | None = None) -> tuple:
        """Natural layout of tensor `name`: q/gate [b,T,Hq,d], k/v [b,T,G,d], q_idx [b,T,G,d_idx],
        k_idx [b,T,d_idx]."""
        T = self.T if T is None else T
        b = self.batch if batch is None else batch
        return {"q": (b, T, self.Hq, self.d), "gate": (b, T, self.Hq, self.d), "k": (b, T, self.G, self.d),
                "v": (b, T, self.G, self.d), "q_idx": (b, T, self.G, self.d_idx), "k_idx": (b, T, self.d_idx)}[name]


# The five workloads of the hot path (prefill tiny / 32K / 128K, the B=1 vs B=8 ablation at
# 64K, and MTP-style decode at 1M context with 4 new tokens per sequence).
CONFIGS = {
    "tiny": Config("tiny", 1, 2048, 8, 2, 64, 32, 8, 512, 256, 0),
    "32k": Config("32k", 2, 32768, 32, 4, 128, 64, 8, 4096, 1024, 1),
    "128k": Config("128k", 1, 131072, 32, 4, 128, 64, 8, 4096, 4096, 2),
    "64k_b8": Config("64k_b8", 1, 65536, 32, 4, 128, 64, 8, 4096, 2048, 3),
    "64k_b1": Config("64k_b1", 1, 65536, 32, 4, 128, 64, 1, 2048, 2048, 3),
    # decode: batch = sequences, T = cached tokens before the step; 4 new tokens per step
    "decode_1m": Config("decode_1m", 32, 1 << 20, 32, 4, 128, 64, 8, 4096, 8192, 4),
}
DECODE_NEW = 4


def _splitmix64(x: np.ndarray) -> np.ndarray:
    x = x + np.uint64(GOLDEN_GAMMA)
    z = x
    z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
    return z ^ (z >> np.uint64(31))


def _splitmix64_int(x: int) -> int:
    x = (x + GOLDEN_GAMMA) & M64
    z = x
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
    return z ^ (z >> 31)


def stream_key(seed: int, stream: int) -> int:
    return _splitmix64_int(_splitmix64_int(seed & M64) ^ ((stream * STREAM_MUL) & M64))


def words(key: int, idx: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return _splitmix64(np.uint64(key) + idx.astype(np.uint64))


def normals(key: int, idx: np.ndarray) -> np.ndarray:
    """fp64 N(0,1) at counters idx (uint64 array)."""
    idx = idx.astype(np.uint64)
    with np.errstate(over="ignore"):
        w1 = words(key, idx * np.uint64(2))
        w2 = words(key, idx * np.uint64(2) + np.uint64(1))
    u1 = ((w1 >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)
    u2 = (w2 >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(TWO_PI * u2)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp64 -> fp32 (RNE) -> bf16 (RNE), returned as uint16 bit patterns."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f64(u: np.ndarray) -> np.ndarray:
    return (np.asarray(u, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def topics(cfg: Config, b: int, n_topics: int) -> np.ndarray:
    """topic[b, s, :] for s < n_topics, fp64 [n_topics, d_idx]."""
    key = stream_key(cfg.seed, STREAMS["topic"])
    s = np.arange(n_topics, dtype=np.uint64)[:, None]
    i = np.arange(cfg.d_idx, dtype=np.uint64)[None, :]
    idx = (np.uint64(b) * np.uint64(1 << 32) + s) * np.uint64(cfg.d_idx) + i
    return normals(key, idx)


def topic_draw(cfg: Config, b: int, t: np.ndarray) -> np.ndarray:
    """r[b, t, g] uniform over {0 .. t // span}; int64 [len(t), G]."""
    key = stream_key(cfg.seed, STREAMS["r"])
    t = np.asarray(t, dtype=np.uint64)
    g = np.arange(cfg.G, dtype=np.uint64)[None, :]
    idx = (np.uint64(b) * np.uint64(1 << 32) + t[:, None]) * np.uint64(cfg.G) + g
    w = words(key, idx)
    n = (t // np.uint64(cfg.span) + np.uint64(1))[:, None]
    return (w % n).astype(np.int64)


def gen_rows(cfg: Config, name: str, b: int, t) -> np.ndarray:
    """bf16 bits of tensor `name` at tokens t of sequence b: uint16 [len(t), W]."""
    t = np.asarray(t, dtype=np.int64)
    W = cfg.width(name)
    key = stream_key(cfg.seed, STREAMS[name])
    idx = ((np.uint64(b) * np.uint64(1 << 32) + t.astype(np.uint64))[:, None] * np.uint64(W)
           + np.arange(W, dtype=np.uint64)[None, :])
    val = normals(key, idx)
    if name == "k_idx":
        top = topics(cfg, b, int(t.max()) // cfg.span + 1 if len(t) else 1)
        val = val + 2.0 * top[t // cfg.span]
    elif name == "q_idx":
        r = topic_draw(cfg, b, t)  # [n, G]
        top = topics(cfg, b, int(t.max()) // cfg.span + 1 if len(t) else 1)
        val = val.reshape(len(t), cfg.G, cfg.d_idx) + 2.0 * top[r]
        val = val.reshape(len(t), W)
    return f64_to_bf16_bits(val)


def gen_full(cfg: Config, name: str, T: int | None = None, chunk: int = 4096) -> np.ndarray:
    """Whole tensor on the host: uint16 [batch, T, W]. Meant for small workloads."""
    T = cfg.T if T is None else T
    out = np.empty((cfg.batch, T, cfg.width(name)), dtype=np.uint16)
    for b in range(cfg.batch):
        for t0 in range(0, T, chunk):
            t1 = min(T, t0 + chunk)
            out[b, t0:t1] = gen_rows(cfg, name, b, np.arange(t0, t1))
    return out


# ---------------------------------------------------------------------------------------------
# CUDA twin (device-side fill for workloads too large to generate on the host)

_HERE = os.path.dirname(os.path.abspath(__file__))
GEN_SO = os.path.join(_HERE, "libsgqa_gen.so")
_gen_lib = None


def build_gen(force: bool = False) -> str:
    import subprocess
    src = os.path.join(_HERE, "gen.cu")
    if force or not os.path.exists(GEN_SO) or os.path.getmtime(GEN_SO) < os.path.getmtime(src):
        cmd = ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
               "-shared", "-Xcompiler", "-fPIC", "-o", GEN_SO, src]
        subprocess.run(cmd, check=True)
    return GEN_SO


def _lib():
    global _gen_lib
    if _gen_lib is None:
        if not os.path.exists(GEN_SO):
            raise RuntimeError("sgqa_inputs: libsgqa_gen.so is not built (run __graft_entry__.build())")
        _gen_lib = ctypes.CDLL(GEN_SO)
        _gen_lib.sgqa_gen_fill.restype = ctypes.c_int
        _gen_lib.sgqa_gen_fill.argtypes = [
            ctypes.c_int, ctypes.c_uint64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
    return _gen_lib


def gen_device(cfg: Config, name: str, out, t0: int = 0, n_t: int | None = None, dst_t0: int | None = None,
               stream=None):
    """Fill a torch CUDA tensor `out` laid out [batch, T_alloc, W] (bf16 or int16) with the values
    of positions [t0, t0 + n_t) of tensor `name`, written at rows dst_t0.. (default t0)."""
    import torch
    n_t = cfg.T - t0 if n_t is None else n_t
    dst_t0 = t0 if dst_t0 is None else dst_t0
    W = cfg.width(name)
    assert out.is_cuda and out.is_contiguous() and out.element_size() == 2
    T_alloc = out.numel() // (cfg.batch * W)
    assert out.numel() == cfg.batch * T_alloc * W and dst_t0 + n_t <= T_alloc
    s = torch.cuda.current_stream().cuda_stream if stream is None else stream
    rc = _lib().sgqa_gen_fill(KIND_CODES[name], cfg.seed, cfg.span, cfg.G, cfg.d_idx, W,
                              cfg.batch, t0, n_t, dst_t0, T_alloc * W, ctypes.c_void_p(out.data_ptr()),
                              ctypes.c_void_p(s))
    if rc != 0:
        raise RuntimeError(f"sgqa_gen_fill failed with CUDA error {rc}")

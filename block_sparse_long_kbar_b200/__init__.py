"""Sparse GQA (Step 5 Preview's full-context attention layer) on B200: Python binding.

A thin ctypes layer over the C ABI in include/sgqa.h (libsgqa.so, built in-tree for sm_100a).
Every function has the C entry point's name and does argument marshalling only — torch
tensors in, raw device pointers and sizes out; every step of the layer runs in the library's
CUDA kernels. There is no CPU fallback: without the built library or a GPU the calls raise.

The layer (mo.ai.kr, "Step 5 Preview agentic work design", section "model structure and training
stability"; ai.info, "StepFun illustrates the 92-block architecture of Step 5 Preview", section
"Sparse GQA aims at a 1 million token context"): block-mean index keys over B = 8 tokens,
per-KV-group top-(k/B) block selection keeping the own block, causal softmax attention over
the selected tokens scaled by 1/sqrt(d), and an elementwise sigmoid gate.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# SGQA_LIBRARY=checks selects the debug build with device-side bounds checks (libsgqa_checks.so)
SO_PATH = os.path.join(_HERE, "libsgqa_checks.so" if os.environ.get("SGQA_LIBRARY") == "checks" else "libsgqa.so")

SGQA_OK = 0
STATUS_NAMES = {0: "SGQA_OK", 1: "SGQA_ERR_INVALID_ARG", 2: "SGQA_ERR_UNSUPPORTED", 3: "SGQA_ERR_WORKSPACE",
                4: "SGQA_ERR_CUDA", 5: "SGQA_ERR_TIMEOUT", 6: "SGQA_ERR_DEVICE_CHECK"}

# every symbol include/sgqa.h declares
EXPORTS = ["sgqa_status_string", "sgqa_version", "sgqa_workspace_size", "sgqa_decode_workspace_size",
           "sgqa_reset_device_status", "sgqa_get_device_status", "sgqa_compress_keys", "sgqa_select",
           "sgqa_attend", "sgqa_forward", "sgqa_decode", "sgqa_decode_noalloc", "sgqa_gated_swa",
           "sgqa_quantize_kv_fp8", "sgqa_decode_fp8", "sgqa_test_stall_decode_cta", "sgqa_forward_rows",
           "sgqa_backward_workspace_size", "sgqa_attend_backward"]


class SgqaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(code, code)} ({status_string(code)})")


class sgqa_dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("batch", "T", "Hq", "G", "d", "d_idx", "B", "k")]

    @classmethod
    def of(cls, cfg, T=None, batch=None) -> "sgqa_dims":
        return cls(cfg.batch if batch is None else batch, cfg.T if T is None else T, cfg.Hq, cfg.G, cfg.d,
                   cfg.d_idx, cfg.B, cfg.k)


_lib = None


def load_library():
    """Load libsgqa.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(SO_PATH):
        raise RuntimeError(f"{os.path.basename(SO_PATH)} is not built at {SO_PATH}: run __graft_entry__.build()")
    L = ctypes.CDLL(SO_PATH)
    P, S, I = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    D = ctypes.POINTER(sgqa_dims)
    L.sgqa_status_string.restype = ctypes.c_char_p
    L.sgqa_status_string.argtypes = [I]
    L.sgqa_version.restype = ctypes.c_char_p
    L.sgqa_version.argtypes = []
    L.sgqa_workspace_size.restype = S
    L.sgqa_workspace_size.argtypes = [D]
    L.sgqa_decode_workspace_size.restype = S
    L.sgqa_decode_workspace_size.argtypes = [D, I]
    L.sgqa_reset_device_status.argtypes = [P, S, P]
    L.sgqa_get_device_status.argtypes = [P, S, ctypes.POINTER(I)]
    L.sgqa_compress_keys.argtypes = [D, P, P, P, S, P]
    L.sgqa_select.argtypes = [D, P, P, P, P, S, P]
    L.sgqa_attend.argtypes = [D, P, P, P, P, P, P, P, S, P]
    L.sgqa_forward.argtypes = [D, P, P, P, P, P, P, P, P, P, S, P]
    L.sgqa_decode.argtypes = [D, I, I] + [P] * 13 + [S, P]
    L.sgqa_decode_noalloc.argtypes = [D, I, I] + [P] * 12 + [P]
    L.sgqa_gated_swa.argtypes = [D, I, P, P, P, P, P, P, P, S, P]
    L.sgqa_quantize_kv_fp8.argtypes = [D, I, I, P, P, P, P]
    L.sgqa_decode_fp8.argtypes = [D, I, I] + [P] * 15 + [S, P]
    L.sgqa_test_stall_decode_cta.argtypes = [I]
    L.sgqa_forward_rows.argtypes = [D, I, I, P, P, P, P, P, P, P, P, P, S, P]
    L.sgqa_backward_workspace_size.restype = S
    L.sgqa_backward_workspace_size.argtypes = [D]
    L.sgqa_attend_backward.argtypes = [D] + [P] * 11 + [S, P]
    for n in ("sgqa_reset_device_status", "sgqa_get_device_status", "sgqa_compress_keys", "sgqa_select",
              "sgqa_attend", "sgqa_forward", "sgqa_decode", "sgqa_decode_noalloc", "sgqa_gated_swa",
              "sgqa_quantize_kv_fp8", "sgqa_decode_fp8", "sgqa_test_stall_decode_cta", "sgqa_forward_rows", "sgqa_attend_backward"):
        getattr(L, n).restype = I
    _lib = L
    return L


def status_string(code: int) -> str:
    return load_library().sgqa_status_string(code).decode()


def sgqa_version() -> str:
    return load_library().sgqa_version().decode()


def _ptr(t, name):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn, rc):
    if rc != SGQA_OK:
        raise SgqaError(fn, rc)


def sgqa_workspace_size(dims: sgqa_dims) -> int:
    return int(load_library().sgqa_workspace_size(ctypes.byref(dims)))


def sgqa_decode_workspace_size(dims: sgqa_dims, n_new: int) -> int:
    return int(load_library().sgqa_decode_workspace_size(ctypes.byref(dims), n_new))


def alloc_workspace(nbytes: int, device=None):
    """A zeroed uint8 device buffer usable as ws (torch allocations are 512-byte aligned)."""
    import torch
    if nbytes <= 0:
        raise ValueError("workspace size is 0: dims invalid or unsupported")
    return torch.zeros(nbytes, dtype=torch.uint8, device=device or "cuda")


def sgqa_reset_device_status(ws, stream=None):
    _check("sgqa_reset_device_status", load_library().sgqa_reset_device_status(_ptr(ws, "ws"), ws.numel(),
                                                                               _stream(stream)))


def sgqa_get_device_status(ws) -> int:
    v = ctypes.c_int(0)
    _check("sgqa_get_device_status", load_library().sgqa_get_device_status(_ptr(ws, "ws"), ws.numel(),
                                                                            ctypes.byref(v)))
    return v.value


def sgqa_compress_keys(dims, k_idx, kbar, ws, stream=None):
    _check("sgqa_compress_keys", load_library().sgqa_compress_keys(
        ctypes.byref(dims), _ptr(k_idx, "k_idx"), _ptr(kbar, "kbar"), _ptr(ws, "ws"),
        0 if ws is None else ws.numel(), _stream(stream)))


def sgqa_select(dims, q_idx, kbar, sel, ws, stream=None):
    _check("sgqa_select", load_library().sgqa_select(
        ctypes.byref(dims), _ptr(q_idx, "q_idx"), _ptr(kbar, "kbar"), _ptr(sel, "sel"), _ptr(ws, "ws"), ws.numel(),
        _stream(stream)))


def sgqa_attend(dims, q, k, v, gate, sel, out, ws, stream=None):
    _check("sgqa_attend", load_library().sgqa_attend(
        ctypes.byref(dims), _ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), _ptr(gate, "gate"), _ptr(sel, "sel"),
        _ptr(out, "out"), _ptr(ws, "ws"), ws.numel(), _stream(stream)))


def sgqa_gated_swa(dims, window, q, k, v, gate, out, ws, sel_out=None, stream=None):
    _check("sgqa_gated_swa", load_library().sgqa_gated_swa(
        ctypes.byref(dims), int(window), _ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), _ptr(gate, "gate"),
        _ptr(out, "out"), _ptr(sel_out, "sel_out"), _ptr(ws, "ws"), ws.numel(), _stream(stream)))


def sgqa_forward(dims, q, k, v, q_idx, k_idx, gate, out, ws, sel_out=None, stream=None):
    _check("sgqa_forward", load_library().sgqa_forward(
        ctypes.byref(dims), _ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), _ptr(q_idx, "q_idx"), _ptr(k_idx, "k_idx"),
        _ptr(gate, "gate"), _ptr(out, "out"), _ptr(sel_out, "sel_out"), _ptr(ws, "ws"), ws.numel(),
        _stream(stream)))


def sgqa_forward_rows(dims, t_begin, t_end, q_rows, k, v, q_idx_rows, k_idx, gate_rows, out_rows, ws,
                      sel_out_rows=None, stream=None):
    """The layer for query rows [t_begin, t_end) only (q, gate, q_idx, out hold those rows; k, v,
    k_idx whole sequences): the per-GPU unit of a query-sharded prefill."""
    _check("sgqa_forward_rows", load_library().sgqa_forward_rows(
        ctypes.byref(dims), int(t_begin), int(t_end), _ptr(q_rows, "q_rows"), _ptr(k, "k"), _ptr(v, "v"),
        _ptr(q_idx_rows, "q_idx_rows"), _ptr(k_idx, "k_idx"), _ptr(gate_rows, "gate_rows"), _ptr(out_rows, "out_rows"),
        _ptr(sel_out_rows, "sel_out_rows"), _ptr(ws, "ws"), ws.numel(), _stream(stream)))


def sgqa_backward_workspace_size(dims: sgqa_dims) -> int:
    return int(load_library().sgqa_backward_workspace_size(ctypes.byref(dims)))


def sgqa_attend_backward(dims, q, k, v, gate, sel, dout, dq, dk, dv, dgate, ws, stream=None):
    """Gradients (fp32) of the gated attention through the given selection: dq, dk, dv, dgate."""
    _check("sgqa_attend_backward", load_library().sgqa_attend_backward(
        ctypes.byref(dims), _ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), _ptr(gate, "gate"), _ptr(sel, "sel"),
        _ptr(dout, "dout"), _ptr(dq, "dq"), _ptr(dk, "dk"), _ptr(dv, "dv"), _ptr(dgate, "dgate"), _ptr(ws, "ws"),
        ws.numel(), _stream(stream)))


INPUTS = ("q", "k", "v", "q_idx", "k_idx", "gate")


def sgqa_forward_from_host(dims, host, dev, out_host, ws, chunks=32, streams=None):
    """The whole layer (sgqa_forward's result) from pinned host buffers, with the host<->device
    copies overlapped with the computation.

    host: pinned CPU tensors q, k, v, q_idx, k_idx, gate in their natural layouts; dev: device
    tensors of the same shapes (the staging copies) plus dev["out"]; out_host: pinned CPU tensor
    for the output. The layer is causal, so the query rows [t0, t1) of a chunk need only the first
    t1 rows of k, v and k_idx: for every sequence and every chunk of rows, in order, one stream
    copies the chunk's rows of all inputs, the compute stream runs sgqa_forward_rows on the chunk
    once they have landed, and a third stream copies the chunk's output back while later chunks
    run. The outputs are bit-identical to sgqa_forward's. streams = (h2d, compute, d2h); by default
    two new streams around the current one. The compute stream waits for the last copy back."""
    import torch
    h2d, comp, d2h = streams if streams is not None else (torch.cuda.Stream(), torch.cuda.current_stream(),
                                                           torch.cuda.Stream())
    T, B = dims.T, dims.B
    one = sgqa_dims(1, T, dims.Hq, dims.G, dims.d, dims.d_idx, dims.B, dims.k)
    h2d.wait_stream(comp)  # the device inputs may still be in use by work queued before this call
    step = max(B, ((T + chunks - 1) // chunks + 127) // 128 * 128)
    bounds = list(range(0, T, step)) + [T]
    for b in range(dims.batch):
        for t0, t1 in zip(bounds[:-1], bounds[1:]):
            with torch.cuda.stream(h2d):
                for n in INPUTS:
                    dev[n][b, t0:t1].copy_(host[n][b, t0:t1], non_blocking=True)
                ready = torch.cuda.Event()
                ready.record(h2d)
            comp.wait_event(ready)
            sgqa_forward_rows(one, t0, t1, dev["q"][b, t0:t1], dev["k"][b], dev["v"][b], dev["q_idx"][b, t0:t1],
                              dev["k_idx"][b], dev["gate"][b, t0:t1], dev["out"][b, t0:t1], ws, stream=comp)
            done = torch.cuda.Event()
            done.record(comp)
            d2h.wait_event(done)
            with torch.cuda.stream(d2h):
                out_host[b, t0:t1].copy_(dev["out"][b, t0:t1], non_blocking=True)
    comp.wait_stream(d2h)
    comp.wait_stream(h2d)


def sgqa_decode(dims, cache_len, n_new, k_cache, v_cache, kidx_cache, kbar_cache, q_new, k_new, v_new, qidx_new,
                kidx_new, gate_new, out, ws, sel_out=None, stream=None):
    _check("sgqa_decode", load_library().sgqa_decode(
        ctypes.byref(dims), int(cache_len), int(n_new), _ptr(k_cache, "k_cache"), _ptr(v_cache, "v_cache"),
        _ptr(kidx_cache, "kidx_cache"), _ptr(kbar_cache, "kbar_cache"), _ptr(q_new, "q_new"), _ptr(k_new, "k_new"),
        _ptr(v_new, "v_new"), _ptr(qidx_new, "qidx_new"), _ptr(kidx_new, "kidx_new"), _ptr(gate_new, "gate_new"),
        _ptr(out, "out"), _ptr(sel_out, "sel_out"), _ptr(ws, "ws"), ws.numel(), _stream(stream)))


def sgqa_quantize_kv_fp8(dims, t0, n_t, src, dst8, dst_scale, stream=None):
    """FP8 (e4m3 + power-of-two row scale) storage of rows [t0, t0 + n_t) of a K or V cache."""
    _check("sgqa_quantize_kv_fp8", load_library().sgqa_quantize_kv_fp8(
        ctypes.byref(dims), int(t0), int(n_t), _ptr(src, "src"), _ptr(dst8, "dst8"), _ptr(dst_scale, "dst_scale"),
        _stream(stream)))


def sgqa_decode_fp8(dims, cache_len, n_new, k8_cache, k_scale, v8_cache, v_scale, kidx_cache, kbar_cache, q_new,
                    k_new, v_new, qidx_new, kidx_new, gate_new, out, ws, sel_out=None, stream=None):
    _check("sgqa_decode_fp8", load_library().sgqa_decode_fp8(
        ctypes.byref(dims), int(cache_len), int(n_new), _ptr(k8_cache, "k8_cache"), _ptr(k_scale, "k_scale"),
        _ptr(v8_cache, "v8_cache"), _ptr(v_scale, "v_scale"), _ptr(kidx_cache, "kidx_cache"),
        _ptr(kbar_cache, "kbar_cache"), _ptr(q_new, "q_new"), _ptr(k_new, "k_new"), _ptr(v_new, "v_new"),
        _ptr(qidx_new, "qidx_new"), _ptr(kidx_new, "kidx_new"), _ptr(gate_new, "gate_new"), _ptr(out, "out"),
        _ptr(sel_out, "sel_out"), _ptr(ws, "ws"), ws.numel(), _stream(stream)))


def sgqa_test_stall_decode_cta(cta: int):
    """Failure-detection test hook: decode attention CTA `cta` issues no loads (-1: off)."""
    _check("sgqa_test_stall_decode_cta", load_library().sgqa_test_stall_decode_cta(int(cta)))


NOALLOC_SCRATCH_BYTES = 16 << 20


def sgqa_decode_noalloc(dims, cache_len, n_new, k_cache, v_cache, kidx_cache, kbar_cache, q_new, k_new, v_new,
                        qidx_new, kidx_new, gate_new, out, sel_out=None, stream=None):
    """sgqa_decode without a workspace: the library's fixed device scratch array is used instead
    (for callers that cannot allocate device memory; see include/sgqa.h)."""
    _check("sgqa_decode_noalloc", load_library().sgqa_decode_noalloc(
        ctypes.byref(dims), int(cache_len), int(n_new), _ptr(k_cache, "k_cache"), _ptr(v_cache, "v_cache"),
        _ptr(kidx_cache, "kidx_cache"), _ptr(kbar_cache, "kbar_cache"), _ptr(q_new, "q_new"), _ptr(k_new, "k_new"),
        _ptr(v_new, "v_new"), _ptr(qidx_new, "qidx_new"), _ptr(kidx_new, "kidx_new"), _ptr(gate_new, "gate_new"),
        _ptr(out, "out"), _ptr(sel_out, "sel_out"), _stream(stream)))

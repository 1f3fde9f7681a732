"""The C-ABI library loads without a GPU, exports every symbol include/sgqa.h declares, and its
host-side validation answers bad arguments with the documented status codes before touching
the device (no compute call is made here: the pointers below are never dereferenced)."""
import ctypes
import os
import re
import subprocess

import pytest

import block_sparse_long_kbar_b200 as sg
from block_sparse_long_kbar_b200 import build as sg_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sgqa.h")


@pytest.fixture(scope="module")
def lib():
    sg_build.build()
    return sg.load_library()


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sgqa_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_expected_api():
    syms = declared_symbols()
    for name in ("sgqa_compress_keys", "sgqa_select", "sgqa_attend", "sgqa_forward", "sgqa_decode",
                 "sgqa_gated_swa"):
        assert name in syms
    assert sorted(sg.EXPORTS) == syms


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", sg.SO_PATH], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\b(sgqa_[a-z_0-9]+)\b", out))
    for s in declared_symbols():
        assert s in exported, s
        assert hasattr(lib, s)


def test_bounds_checking_build_exports_every_declared_symbol():
    """libsgqa_checks.so (-DSGQA_CHECKS) is the same library with device-side index checks."""
    so = sg_build.build(variant="checks")
    out = subprocess.run(["nm", "-D", "--defined-only", so], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\b(sgqa_[a-z_0-9]+)\b", out))
    for s in declared_symbols():
        assert s in exported, s


def test_header_compiles_as_c(tmp_path):
    src = tmp_path / "t.c"
    src.write_text('#include "sgqa.h"\nint main(void){ sgqa_dims d = {1,8,2,1,64,32,8,8}; '
                   'return (int)sgqa_workspace_size(&d) * 0; }\n')
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-c", "-I", os.path.join(ROOT, "include"), str(src),
                    "-o", str(tmp_path / "t.o")], check=True)


def D(**kw):
    base = dict(batch=1, T=2048, Hq=8, G=2, d=64, d_idx=32, B=8, k=512)
    base.update(kw)
    return sg.sgqa_dims(*[base[n] for n in ("batch", "T", "Hq", "G", "d", "d_idx", "B", "k")])


@pytest.mark.parametrize("kw,ok", [
    ({}, True), ({"d": 128, "d_idx": 64, "G": 4, "Hq": 32}, True), ({"B": 1, "k": 2048}, True),
    ({"d": 96}, False), ({"d_idx": 48}, False), ({"B": 3, "k": 12}, False), ({"k": 500}, False),
    ({"Hq": 7}, False), ({"Hq": 34, "G": 2}, False), ({"G": 3, "Hq": 9}, False), ({"T": 0}, False),
    ({"batch": -1}, False), ({"T": 1 << 28}, False),
])
def test_workspace_size_validation(lib, kw, ok):
    n = sg.sgqa_workspace_size(D(**kw))
    assert (n > 0) == ok


def test_workspace_size_formula(lib):
    d = D(batch=2, T=32768, Hq=32, G=4, d=128, d_idx=64, B=8, k=4096)
    nblk = 32768 // 8
    al = lambda x: (x + 255) // 256 * 256
    units = 2 * 32768 * 4
    plan = 4 * al(units * 4) + al(8 * 256 * ((32768 + 2047) // 2048) * 4)
    # taken-candidate bitmaps: 4 words per 128 blocks per (token, group), query ranges within 256 MiB
    bstride = 4 * ((nblk + 127) // 128)
    bits_q = min(32768, (256 << 20) // (2 * 4 * bstride * 4) // 128 * 128)
    want = (256 + plan + al(2 * nblk * 64 * 4) + 2 * al(2 * nblk * 64 * 2) + al(2 * bits_q * 4 * bstride * 4)
            + al(2 * 32768 * 4 * 512 * 4))
    assert sg.sgqa_workspace_size(d) == want
    assert sg.sgqa_decode_workspace_size(D(batch=32, T=(1 << 20) + 8, Hq=32, G=4, d=128, d_idx=64, B=8, k=4096), 4) > 0
    assert sg.sgqa_decode_workspace_size(D(), 0) == 0
    assert sg.sgqa_decode_workspace_size(D(G=16, Hq=16), 4) == 0   # more than 32 rows per sequence


def _call_forward(lib, dims, ptr, ws, ws_bytes):
    P = ctypes.c_void_p
    return lib.sgqa_forward(ctypes.byref(dims), P(ptr), P(ptr), P(ptr), P(ptr), P(ptr), P(ptr), P(ptr), None,
                            P(ws), ws_bytes, None)


def test_host_validation_codes(lib):
    d = D()
    good = 0x7F0000000000  # never dereferenced: each call below fails validation first
    need = sg.sgqa_workspace_size(d)
    assert _call_forward(lib, D(d=96), good, good, need) == 2          # unsupported
    assert _call_forward(lib, D(T=0), good, good, need) == 1           # invalid
    assert _call_forward(lib, D(batch=64, T=(1 << 27) - 8, Hq=32, G=4), good, good, need) == 2  # 2^31 rows
    assert _call_forward(lib, d, good + 8, good, need) == 1            # misaligned tensor
    assert _call_forward(lib, d, 0, good, need) == 1                   # null tensor
    assert _call_forward(lib, d, good, good, need - 1) == 3            # workspace too small
    assert _call_forward(lib, d, good, good + 16, need) == 3           # workspace misaligned
    P = ctypes.c_void_p
    assert lib.sgqa_attend(ctypes.byref(d), P(good), P(good), P(good), P(good), P(good), P(good), P(good), 16,
                           None) == 3
    assert lib.sgqa_select(ctypes.byref(D(k=500)), P(good), P(good), P(good), P(good), need, None) == 2
    # decode: cache overflow and too many rows
    args = [P(good)] * 12
    assert lib.sgqa_decode(ctypes.byref(D(T=64)), 62, 4, *args, P(good), 1 << 30, None) == 1
    assert lib.sgqa_decode(ctypes.byref(D(T=64)), 0, 0, *args, P(good), 1 << 30, None) == 1
    assert lib.sgqa_decode(ctypes.byref(D(T=64, G=16, Hq=16)), 0, 4, *args, P(good), 1 << 30, None) == 1
    assert lib.sgqa_decode(ctypes.byref(D(T=64)), 0, 4, *args, P(good), 1024, None) == 3
    # Gated SWA: window below one block, selection capacity below window + B, heads per group
    # outside the tcgen05 attention, workspace too small
    swa = lambda dims, w, ws_bytes: lib.sgqa_gated_swa(ctypes.byref(dims), w, *[P(good)] * 5, None, P(good),
                                                       ws_bytes, None)
    ds = D(k=512)
    ws_swa = sg.sgqa_workspace_size(ds)
    assert swa(ds, ds.B - 1, ws_swa) == 1
    assert swa(ds, ds.k - ds.B + 1, ws_swa) == 1
    assert swa(D(k=512, Hq=8, G=8), 64, sg.sgqa_workspace_size(D(k=512, Hq=8, G=8))) == 2
    assert swa(ds, 64, ws_swa - 1) == 3
    v = ctypes.c_int(0)
    assert lib.sgqa_get_device_status(None, 256, ctypes.byref(v)) == 1
    assert lib.sgqa_reset_device_status(None, 256, None) == 3


def test_status_strings(lib):
    for code in range(7):
        assert sg.status_string(code)
    assert sg.status_string(99) == "unknown status"
    assert "sm_100a" in sg.sgqa_version()


def test_binding_fails_loudly_without_cuda_tensors(lib):
    import torch
    x = torch.zeros(16, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        sg.sgqa_compress_keys(D(T=8), x, x, None)

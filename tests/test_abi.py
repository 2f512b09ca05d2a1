"""The C-ABI library loads on a machine without a GPU, exports every entry
point include/nf4lora.h declares, sizes buffers as the storage accounting
says, and rejects bad arguments on the host before touching a device."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def nf():
    import nf4_base_lora_b200 as nf
    return nf


def header_functions():
    text = open(os.path.join(ROOT, "include", "nf4lora.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^[A-Za-z_][\w \*]*?\b(\w+)\s*\(", text, flags=re.M)


def test_every_declared_symbol_is_exported(nf):
    names = header_functions()
    assert set(names) == set(nf.ABI_SYMBOLS), names
    for name in names:
        assert hasattr(nf.lib, name), name


def test_version(nf):
    assert nf.version().startswith("nf4lora")


@pytest.mark.parametrize("d_out,d_in", [(512, 512), (4096, 4096), (11008, 4096), (4096, 11008),
                                        (22016, 8192), (8, 64), (3, 128)])
def test_packed_bytes_cover_the_unpadded_storage(nf, d_out, d_in):
    n = d_out * d_in
    unpadded = oracle.packed_bytes(n)            # n/2 + n_b + 4 n_g + 4
    got = nf.nf4_packed_bytes(d_out, d_in)
    assert unpadded <= got <= unpadded + 4 * 256
    assert got % 256 == 0


def test_sizing_rejects_bad_shapes(nf):
    assert nf.nf4_packed_bytes(4, 96) == 0        # d_in % 64 != 0
    assert nf.nf4_packed_bytes(0, 64) == 0
    assert nf.qlora_fwd_workspace_bytes(0, 64, 64, 8) == 0
    assert nf.qlora_fwd_workspace_bytes(4, 64, 64, 300) == 0


def test_tensor_from_buffer_layout(nf):
    s = nf.Nf4TensorStruct()
    base = 1 << 20                                 # any 256-aligned address; never dereferenced
    need = nf.nf4_packed_bytes(128, 256)
    assert nf.lib.nf4_tensor_from_buffer(ctypes.byref(s), ctypes.c_void_p(base), need, 128, 256) == 0
    assert s.codes == base and s.d_out == 128 and s.d_in == 256
    assert s.qscale == base + 128 * 256 // 2
    assert s.scale2 == s.qscale + 512                  # 512 blocks, 256-aligned
    assert s.scale_mean == s.scale2 + 256
    assert nf.lib.nf4_tensor_from_buffer(ctypes.byref(s), ctypes.c_void_p(base + 16), need, 128, 256) == -3
    assert nf.lib.nf4_tensor_from_buffer(ctypes.byref(s), ctypes.c_void_p(base), need - 1, 128, 256) == -1


def fake_tensor(nf, d_out=128, d_in=256):
    s = nf.Nf4TensorStruct()
    assert nf.lib.nf4_tensor_from_buffer(ctypes.byref(s), ctypes.c_void_p(1 << 20),
                                         nf.nf4_packed_bytes(d_out, d_in), d_out, d_in) == 0
    return s


P = ctypes.c_void_p


def test_host_validation_without_device(nf):
    s = fake_tensor(nf)
    A = P(1 << 24); B = P(1 << 25); X = P(1 << 26); Y = P(1 << 27); ws = P(1 << 28)
    L = nf.lib
    f = ctypes.c_float(2.0)
    # NULL X
    assert L.qlora_linear_fwd(ctypes.byref(s), A, B, 8, f, None, 16, Y, None, ws, 1 << 30, None) == -1
    # any rank in [1, 256] passes the host checks (r = 12 runs padded to 16): here, without a
    # device, the call then stops at the device check
    assert L.qlora_linear_fwd(ctypes.byref(s), A, B, 12, f, X, 16, Y, None, ws, 1 << 30, None) == -5
    # r out of range
    assert L.qlora_linear_fwd(ctypes.byref(s), A, B, 0, f, X, 16, Y, None, ws, 1 << 30, None) == -1
    assert L.qlora_linear_fwd(ctypes.byref(s), A, B, 257, f, X, 16, Y, None, ws, 1 << 30, None) == -1
    # misaligned X
    assert L.qlora_linear_fwd(ctypes.byref(s), A, B, 8, f, P((1 << 26) + 2), 16, Y, None, ws, 1 << 30, None) == -3
    # workspace too small / NULL
    assert L.qlora_linear_fwd(ctypes.byref(s), A, B, 8, f, X, 16, Y, None, ws, 16, None) == -4
    assert L.qlora_linear_fwd(ctypes.byref(s), A, B, 8, f, X, 16, Y, None, None, 0, None) == -4
    # non-finite scaling
    assert L.qlora_linear_fwd(ctypes.byref(s), A, B, 8, ctypes.c_float(float("inf")), X, 16, Y, None, ws,
                              1 << 30, None) == -1
    # M out of range
    assert L.qlora_linear_fwd(ctypes.byref(s), A, B, 8, f, X, -1, Y, None, ws, 1 << 30, None) == -1
    assert b"M = -1" in L.nf4lora_last_error_string()
    assert L.qlora_linear_fwd(ctypes.byref(s), A, B, 8, f, X, 1 << 31, Y, None, ws, 1 << 30, None) == -1
    # an empty batch is a no-op (no device access: X, Y and the workspace may be NULL)
    assert L.qlora_linear_fwd(ctypes.byref(s), A, B, 8, f, None, 0, None, None, None, 0, None) == 0
    # ... and so is its backward when the gradients accumulate
    assert L.qlora_linear_bwd(ctypes.byref(s), A, B, 8, f, None, None, None, 0, None, P(1 << 29), P(1 << 28), 1,
                              None, 0, None) == 0
    # backward: dA needs X
    assert L.qlora_linear_bwd(ctypes.byref(s), A, B, 8, f, None, None, Y, 16, None, P(1 << 29), None, 0, ws,
                              1 << 30, None) == -1
    # backward with nothing to compute is a no-op
    assert L.qlora_linear_bwd(ctypes.byref(s), A, B, 8, f, None, None, Y, 16, None, None, None, 0, None, 0,
                              None) == 0
    # quantize: shape mismatch, misaligned W, unsupported shape
    assert L.nf4_quantize(P(1 << 24), 128, 128, ctypes.byref(s), ws, 1 << 30, None) == -1
    assert L.nf4_quantize(P((1 << 24) + 4), 128, 256, ctypes.byref(s), ws, 1 << 30, None) == -3
    bad = nf.Nf4TensorStruct(128, 96, 1 << 20, 1 << 21, 1 << 22, 1 << 23)
    assert L.nf4_dequantize(ctypes.byref(bad), Y, None) == -2
    assert L.nf4_dequantize(None, Y, None) == -1


def test_merge_host_validation_without_device(nf):
    L = nf.lib
    s = fake_tensor(nf)
    A = P(1 << 24); B = P(1 << 25); out = P(1 << 26); ws = P(1 << 28)
    f = ctypes.c_float(0.5)
    assert nf.nf4_merge_workspace_bytes(128, 256) >= 128 * 256 * 4
    assert nf.nf4_merge_workspace_bytes(128, 100) == 0                       # d_in % 64 != 0
    assert L.nf4_merge_lora(ctypes.byref(s), A, B, 8, f, None, None) == -1    # no output
    assert L.nf4_merge_lora(ctypes.byref(s), A, B, 8, f, P((1 << 26) + 4), None) == -3
    assert L.nf4_merge_lora(ctypes.byref(s), A, B, 0, f, out, None) == -1     # r out of range
    assert L.nf4_merge_lora(ctypes.byref(s), A, B, 257, f, out, None) == -1
    assert L.nf4_merge_lora(ctypes.byref(s), None, B, 8, f, out, None) == -1
    assert L.nf4_merge_lora(ctypes.byref(s), A, B, 8, ctypes.c_float(float("nan")), out, None) == -1
    other = fake_tensor(nf, 64, 256)
    assert L.nf4_merge_requantize(ctypes.byref(s), A, B, 8, f, ctypes.byref(other), ws, 1 << 30, None) == -1
    assert L.nf4_merge_requantize(ctypes.byref(s), A, B, 8, f, ctypes.byref(s), ws, 1024, None) == -4
    assert L.nf4_merge_requantize(ctypes.byref(s), A, B, 8, f, ctypes.byref(s), None, 0, None) == -4


def test_adamw_host_validation_without_device(nf):
    L = nf.lib
    T = nf.AdamwTensorStruct
    h = nf.AdamwHparamsStruct(1e-3, 0.9, 0.999, 1e-8, 0.0, 1)
    good = (T * 1)(T(1 << 24, None, 1 << 25, 1 << 26, 1 << 27, 64))
    assert L.lora_adamw_step(good, 0, ctypes.byref(h), None) == -1          # count
    assert L.lora_adamw_step(None, 1, ctypes.byref(h), None) == -1          # no tensors
    assert L.lora_adamw_step(good, 1, None, None) == -1                     # no hyper-parameters
    bad = (T * 1)(T(1 << 24, None, None, 1 << 26, 1 << 27, 64))
    assert L.lora_adamw_step(bad, 1, ctypes.byref(h), None) == -1           # NULL gradient
    mis = (T * 1)(T((1 << 24) + 4, None, 1 << 25, 1 << 26, 1 << 27, 64))
    assert L.lora_adamw_step(mis, 1, ctypes.byref(h), None) == -3           # misaligned master
    neg = (T * 1)(T(1 << 24, None, 1 << 25, 1 << 26, 1 << 27, -1))
    assert L.lora_adamw_step(neg, 1, ctypes.byref(h), None) == -1           # n < 0
    for hp in [(1e-3, 1.0, 0.999, 1e-8, 0.0, 1), (1e-3, 0.9, 0.999, 0.0, 0.0, 1),
               (-1e-3, 0.9, 0.999, 1e-8, 0.0, 1), (1e-3, 0.9, 0.999, 1e-8, 0.0, 0),
               (float("nan"), 0.9, 0.999, 1e-8, 0.0, 1), (1e-3, 0.9, 0.999, 1e-8, -0.1, 1)]:
        bh = nf.AdamwHparamsStruct(*hp)
        assert L.lora_adamw_step(good, 1, ctypes.byref(bh), None) == -1, hp
    assert b"hyper-parameters" in L.nf4lora_last_error_string()


def test_workspace_grows_with_tokens(nf):
    a = nf.qlora_fwd_workspace_bytes(16, 4096, 4096, 64)
    b = nf.qlora_fwd_workspace_bytes(4096, 4096, 4096, 64)
    assert 0 < a < b
    assert nf.qlora_bwd_workspace_bytes(4096, 11008, 4096, 64) > 0
    assert nf.nf4_quantize_workspace_bytes(4096, 4096) >= 4096 * 4096 // 64 * 4

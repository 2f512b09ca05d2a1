"""The allocation-free encoder entry point against the regular one.

nf4_quantize_noalloc serves callers that may not allocate device memory (a
host framework that owns all device memory, or code where a cudaMalloc would
break a capture or a budget): its scratch is a fixed array inside the library.
Called through the C ABI twice in a row, it must give exactly what
nf4_quantize gives -- the encoding is integer-exact, so the tolerance is zero.
This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes on its own in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nf():
    import nf4_base_lora_b200 as nf
    return nf


def test_noalloc_quantize_matches_workspace_version(nf):
    torch.cuda.set_device(0)
    shapes = [(512, 512), (300, 448)]
    for d_out, d_in in shapes:
        W = torch.from_numpy(workloads.weight(d_out, d_in, outliers=True, index=d_out % 5)).cuda()
        ref = nf.nf4_quantize(W)
        for _ in range(2):                       # two calls in a row share the scratch
            got = nf.NF4Tensor(d_out, d_in, W.device)
            got.buffer.fill_(0xAB)               # catch anything left unwritten
            status = nf.lib.nf4_quantize_noalloc(ctypes.c_void_p(W.data_ptr()), d_out, d_in,
                                                 ctypes.byref(got.struct),
                                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
            assert status == 0
            torch.cuda.synchronize()
            assert torch.equal(got.codes, ref.codes)
            assert torch.equal(got.qscale, ref.qscale)
            assert torch.equal(got.scale2.view(torch.int32), ref.scale2.view(torch.int32))
            assert torch.equal(got.scale_mean.view(torch.int32), ref.scale_mean.view(torch.int32))


def test_noalloc_rejects_sizes_beyond_its_scratch(nf):
    d_out, d_in = 65536, 4160                    # 4,259,840 blocks > 4,194,304
    s = nf.Nf4TensorStruct(d_out, d_in, 1 << 20, 1 << 21, 1 << 22, 1 << 23)
    status = nf.lib.nf4_quantize_noalloc(ctypes.c_void_p(1 << 24), d_out, d_in, ctypes.byref(s), None)
    assert status == -2


def test_noalloc_quantize_fp32_scales(nf):
    """The fp32-block-scale format needs no scratch: the same bytes as
    nf4_quantize into that format."""
    d_out, d_in = 300, 448
    W = torch.from_numpy(workloads.weight(d_out, d_in, outliers=True, index=1)).cuda()
    ref = nf.nf4_quantize(W, double_quant=False)
    got = nf.NF4Tensor(d_out, d_in, W.device, double_quant=False)
    got.buffer.fill_(0xAB)
    status = nf.lib.nf4_quantize_noalloc(ctypes.c_void_p(W.data_ptr()), d_out, d_in, ctypes.byref(got.struct),
                                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert status == 0
    torch.cuda.synchronize()
    assert torch.equal(got.codes, ref.codes)
    assert torch.equal(got.absmax.view(torch.int32), ref.absmax.view(torch.int32))

"""GPU parity of the encoder and the materialising decoder: packed codes, int8
scale codes, group scales, mean and W_hat must equal the oracle's bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nf():
    import nf4_base_lora_b200 as nf
    return nf


def encode_both(nf, w):
    qt = oracle.quantize(w)
    dev = nf.nf4_quantize(torch.from_numpy(np.ascontiguousarray(w)).cuda())
    torch.cuda.synchronize()
    nf.device_status()
    return qt, dev


def assert_encoding_equal(qt, dev):
    assert np.array_equal(dev.codes.cpu().numpy(), qt["packed"])
    assert np.array_equal(dev.qscale.cpu().numpy(), qt["q"])
    assert np.array_equal(dev.scale2.cpu().numpy().view(np.uint32), qt["a2"].view(np.uint32))
    assert dev.scale_mean.cpu().numpy().view(np.uint32)[0] == np.float32(qt["mu"]).view(np.uint32)


@pytest.mark.parametrize("d_out,d_in,outliers,sigma", [
    (8, 64, False, 0.02), (3, 128, False, 0.02), (64, 256, True, 0.02),
    (512, 512, False, 0.02), (300, 448, True, 0.015), (257, 1088, True, 0.02)])
def test_quantize_bit_exact(nf, d_out, d_in, outliers, sigma):
    w = workloads.weight(d_out, d_in, sigma=sigma, outliers=outliers, index=d_out % 7)
    qt, dev = encode_both(nf, w)
    assert_encoding_equal(qt, dev)


def test_quantize_special_blocks_bit_exact(nf):
    w = workloads.special_blocks(16)
    qt, dev = encode_both(nf, w)
    assert_encoding_equal(qt, dev)


def test_quantize_constant_weight(nf):
    w = np.full((16, 512), 0.25, np.float32)          # every scale equal: a2 = 0, q = 0
    qt, dev = encode_both(nf, w)
    assert_encoding_equal(qt, dev)
    assert np.all(dev.qscale.cpu().numpy() == 0)


@pytest.mark.parametrize("d_out,d_in", [(4096, 4096), (11008, 4096)])
def test_quantize_llama_shapes_bit_exact(nf, d_out, d_in):
    w = workloads.weight(d_out, d_in, outliers=True, index=1)
    qt, dev = encode_both(nf, w)
    assert_encoding_equal(qt, dev)


@pytest.mark.parametrize("d_out,d_in", [(8, 64), (512, 512), (300, 448), (4096, 4096)])
def test_dequantize_bit_exact(nf, d_out, d_in):
    w = workloads.weight(d_out, d_in, outliers=True, index=2)
    qt, dev = encode_both(nf, w)
    got = nf.nf4_dequantize(dev)
    torch.cuda.synchronize()
    ref = oracle.dequantize_bits(qt["packed"], qt["q"], qt["a2"], float(qt["mu"]), d_out * d_in)
    assert np.array_equal(got.view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1), ref)


def test_dequantize_special_blocks_bit_exact(nf):
    w = workloads.special_blocks(16)
    qt, dev = encode_both(nf, w)
    got = nf.nf4_dequantize(dev)
    ref = oracle.dequantize_bits(qt["packed"], qt["q"], qt["a2"], float(qt["mu"]), w.size)
    assert np.array_equal(got.view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1), ref)


def test_quantize_is_deterministic(nf):
    w = torch.from_numpy(workloads.weight(1024, 1024, outliers=True)).cuda()
    a = nf.nf4_quantize(w).buffer.clone()
    for _ in range(2):
        assert torch.equal(nf.nf4_quantize(w).buffer, a)

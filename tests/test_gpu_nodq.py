"""GPU parity of the encoding without double quantisation (the codes with
one fp32 scale per block of 64, "第 04 篇：QLoRA 原理" §5.1) on every path that
reads an encoded weight: the encoder and the materialising decoder bit for
bit, the layer's forward and backward on the few-token and many-token paths
against the oracle, and the adapter merge with its re-encoding."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nf():
    import nf4_base_lora_b200 as nf
    return nf


def _encode(nf, w):
    dev = nf.nf4_quantize(torch.from_numpy(np.ascontiguousarray(w)).cuda(), double_quant=False)
    torch.cuda.synchronize()
    nf.device_status()
    return dev


def _assert_nodq_equal(dev, ref):
    assert not dev.double_quant
    assert np.array_equal(dev.codes.cpu().numpy(), ref["packed"])
    assert np.array_equal(dev.absmax.cpu().numpy().view(np.uint32), ref["absmax"].view(np.uint32))


@pytest.mark.parametrize("d_out,d_in,outliers", [(8, 64, False), (64, 256, True), (300, 448, True),
                                                 (4096, 4096, True)])
def test_quantize_nodq_bit_exact(nf, d_out, d_in, outliers):
    w = workloads.weight(d_out, d_in, outliers=outliers, index=d_out % 5)
    _assert_nodq_equal(_encode(nf, w), oracle.quantize_nodq(w))


def test_quantize_nodq_special_and_threshold_blocks(nf):
    from test_gpu_quantize import near_threshold_blocks
    for w in (workloads.special_blocks(16), near_threshold_blocks()):
        _assert_nodq_equal(_encode(nf, w), oracle.quantize_nodq(w))


def test_storage_is_4_5_bits_per_weight(nf):
    n = 4096 * 4096
    assert nf.nf4_packed_bytes_nodq(4096, 4096) == n // 2 + 4 * (n // 64)   # both parts 256-byte multiples
    enc = nf.NF4Tensor(4096, 4096, double_quant=False)
    assert enc.buffer.numel() * 8 / n == 4.5


@pytest.mark.parametrize("d_out,d_in", [(8, 64), (300, 448), (4096, 4096)])
def test_dequantize_nodq_bit_exact(nf, d_out, d_in):
    w = workloads.weight(d_out, d_in, outliers=True, index=1)
    qt = oracle.quantize_nodq(w)
    W_hat = nf.nf4_dequantize(_encode(nf, w))
    torch.cuda.synchronize()
    ref = oracle.dequantize_scales_bits(qt["packed"], qt["absmax"], w.size)
    assert np.array_equal(W_hat.view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1), ref)


LAYER_CASES = [
    # (d_out, d_in, M, r): few-token forward and dX, then the many-token kernels
    (384, 320, 16, 64),
    (136, 192, 3, 8),
    (4096, 11008, 3, 64),     # the few-token stage ring refilled
    (264, 320, 130, 64),      # many tokens, ragged tokens and d_out
    (512, 768, 300, 128),
]


@pytest.mark.parametrize("d_out,d_in,m,r", LAYER_CASES)
def test_layer_nodq_matches_oracle(nf, d_out, d_in, m, r):
    c = workloads.linear_case(d_out, d_in, m, r, 16.0, outliers=True, index=2, b_std=0.05)
    qt = oracle.quantize_nodq(c.W)
    W_hat = oracle.dequantize(qt, c.W.shape)
    w = _encode(nf, c.W)
    A, B, X, dY = (getattr(c, k).cuda() for k in ("A", "B", "X", "dY"))
    Y, T = nf.qlora_linear_fwd(w, A, B, c.scaling, X)
    dX, dA, dB = nf.qlora_linear_bwd(w, A, B, c.scaling, X, T, dY)
    torch.cuda.synchronize()
    nf.device_status()
    Y_ref, _ = oracle.forward(W_hat, c.A, c.B, c.X, c.scaling)
    dX_ref, dA_ref, dB_ref = oracle.backward(W_hat, c.A, c.B, c.X, c.dY, c.scaling)
    assert_close(Y, Y_ref, "Y")
    assert_close(dX, dX_ref, "dX")
    assert_close(dA, dA_ref, "dA")
    assert_close(dB, dB_ref, "dB")


def test_nodq_weight_is_more_accurate_on_average(nf):
    """Plain fp32 scales carry no second rounding: over a whole weight the
    mean |W - W_hat| is not larger than with double-quantised scales."""
    w = workloads.weight(512, 1024, outliers=True, index=0)
    Wt = torch.from_numpy(w).cuda()
    e_nodq = (nf.nf4_dequantize(nf.nf4_quantize(Wt, double_quant=False)).float() - Wt).abs().mean().item()
    e_dq = (nf.nf4_dequantize(nf.nf4_quantize(Wt)).float() - Wt).abs().mean().item()
    assert e_nodq <= e_dq


@pytest.mark.parametrize("src_dq,dst_dq", [(False, False), (True, False), (False, True)])
def test_merge_nodq_bit_exact(nf, src_dq, dst_dq):
    d_out, d_in, r, s = 300, 448, 12, 0.5
    w = workloads.weight(d_out, d_in, outliers=True, index=3)
    qt = oracle.quantize(w) if src_dq else oracle.quantize_nodq(w)
    enc = nf.nf4_quantize(torch.from_numpy(w).cuda(), double_quant=src_dq)
    A = workloads.lora_a(r, d_in, 1)
    B = workloads.lora_b(d_out, r, 1, std=0.05)
    ref = oracle.merge_lora(oracle.dequantize(qt, (d_out, d_in)), A, B, s)
    merged = nf.nf4_merge_lora(enc, A.cuda(), B.cuda(), s)
    out = nf.NF4Tensor(d_out, d_in, double_quant=dst_dq)
    nf.nf4_merge_requantize(enc, A.cuda(), B.cuda(), s, out=out)
    torch.cuda.synchronize()
    nf.device_status()
    assert np.array_equal(merged.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    if dst_dq:
        q = oracle.quantize(ref)
        assert np.array_equal(out.codes.cpu().numpy(), q["packed"])
        assert np.array_equal(out.qscale.cpu().numpy(), q["q"])
    else:
        _assert_nodq_equal(out, oracle.quantize_nodq(ref))


def test_requantize_nodq_in_place(nf):
    w = workloads.weight(256, 320, outliers=True, index=4)
    A = workloads.lora_a(16, 320, 2)
    B = workloads.lora_b(256, 16, 2, std=0.05)
    enc = nf.nf4_quantize(torch.from_numpy(w).cuda(), double_quant=False)
    ref = oracle.quantize_nodq(oracle.merge_lora(oracle.dequantize(oracle.quantize_nodq(w), w.shape), A, B, 0.5))
    out = nf.nf4_merge_requantize(enc, A.cuda(), B.cuda(), 0.5, out=enc)
    torch.cuda.synchronize()
    assert out is enc
    _assert_nodq_equal(enc, ref)

"""GPU parity of the adapter merge (nf4_merge_lora) and of the merged weight's
re-encoding (nf4_merge_requantize) with the oracle: the merged fp32 weight and
the new encoding must match bit for bit (every step of the merge is a fixed
sequence of IEEE operations, and the encoding is exact).  Cases cover a
ragged row tile (d_out not a multiple of 128), ranks that are not a multiple
of the 16-rank staging slice (with and without whole 16-byte pieces of B's
rows), the largest rank, products whose fp64 running
sum must round, re-encoding in place and the LLaMA-7B q_proj size."""
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


def _setup(nf, d_out, d_in, r, index=0):
    W = workloads.weight(d_out, d_in, outliers=True, index=index)
    qt = oracle.quantize(W)
    enc = nf.nf4_quantize(torch.from_numpy(W).cuda())
    A = workloads.lora_a(r, d_in, index)
    B = workloads.lora_b(d_out, r, index, std=0.05)
    return qt, enc, A, B


def _assert_encoding_equal(dev, ref):
    assert np.array_equal(dev.codes.cpu().numpy(), ref["packed"])
    assert np.array_equal(dev.qscale.cpu().numpy(), ref["q"])
    assert np.array_equal(dev.scale2.cpu().numpy().view(np.uint32), ref["a2"].view(np.uint32))
    assert dev.scale_mean.cpu().numpy().view(np.uint32)[0] == np.float32(ref["mu"]).view(np.uint32)


@pytest.mark.parametrize("d_out,d_in,r,s", [(512, 512, 8, 2.0), (300, 448, 16, 0.25), (136, 192, 5, 1.0),
                                            (200, 320, 24, 0.5), (64, 256, 256, 0.0625)])
def test_merge_bit_exact(nf, d_out, d_in, r, s):
    qt, enc, A, B = _setup(nf, d_out, d_in, r, index=d_out % 5)
    W_hat = oracle.dequantize(qt, (d_out, d_in))
    merged = nf.nf4_merge_lora(enc, A.cuda(), B.cuda(), s)
    torch.cuda.synchronize()
    nf.device_status()
    ref = oracle.merge_lora(W_hat, A, B, s)
    assert np.array_equal(merged.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    again = nf.nf4_merge_requantize(enc, A.cuda(), B.cuda(), s)
    torch.cuda.synchronize()
    _assert_encoding_equal(again, oracle.quantize(ref))


def test_merge_rounds_the_rank_sum_in_order(nf):
    """Products 2^60, 1, -2^60 per element: the ascending fp64 sum loses the 1."""
    d_out, d_in = 128, 128
    qt, enc, _, _ = _setup(nf, d_out, d_in, 3)
    W_hat = oracle.dequantize(qt, (d_out, d_in))
    B = torch.tensor([[2.0 ** 30, 1.0, -2.0 ** 30]] * d_out, dtype=torch.bfloat16)
    A = torch.tensor([[2.0 ** 30] * d_in, [1.0] * d_in, [2.0 ** 30] * d_in], dtype=torch.bfloat16)
    merged = nf.nf4_merge_lora(enc, A.cuda(), B.cuda(), 1.0)
    torch.cuda.synchronize()
    ref = oracle.merge_lora(W_hat, A, B, 1.0)
    assert np.array_equal(ref, W_hat)
    assert np.array_equal(merged.cpu().numpy().view(np.uint32), ref.view(np.uint32))


def test_requantize_in_place(nf):
    qt, enc, A, B = _setup(nf, 256, 320, 16, index=2)
    W_hat = oracle.dequantize(qt, (256, 320))
    ref = oracle.merge_requantize(qt, (256, 320), A, B, 0.5)
    out = nf.nf4_merge_requantize(enc, A.cuda(), B.cuda(), 0.5, out=enc)
    torch.cuda.synchronize()
    nf.device_status()
    assert out is enc
    _assert_encoding_equal(enc, ref)
    assert not np.array_equal(ref["packed"], qt["packed"])  # the merge changed the weight
    del W_hat


def test_merge_q_proj_size(nf):
    qt, enc, A, B = _setup(nf, 4096, 4096, 64, index=0)
    ref = oracle.merge_lora(oracle.dequantize(qt, (4096, 4096)), A, B, 0.25)
    merged = nf.nf4_merge_lora(enc, A.cuda(), B.cuda(), 0.25)
    torch.cuda.synchronize()
    assert np.array_equal(merged.cpu().numpy().view(np.uint32), ref.view(np.uint32))

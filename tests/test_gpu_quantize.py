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


def near_threshold_blocks(n_blocks: int = 256, seed: int = 11) -> np.ndarray:
    """[n_blocks / 4, 256] fp32: each 64-block attains its absmax a (random,
    some powers of two) at element 0 and puts w = fl(m_j a) moved by -2..+1
    ulp for every threshold m_j (j = 0..14) in the rest, half the blocks
    negated: fl(w / a) then lands on or within a few ulp of the thresholds,
    where the encoder's division-free test hands over to the exact division."""
    rng = np.random.default_rng(seed)
    m = oracle.midpoints().astype(np.float32)
    out = np.zeros((n_blocks, 64), np.float32)
    for b in range(n_blocks):
        a = np.float32(2.0 ** rng.integers(-8, 3)) if b % 4 == 0 else np.float32(rng.uniform(0.003, 4.0))
        blk = [a]
        for j in range(15):
            w = np.float32(m[j] * a)
            for step in (-2, -1, 0, 1):
                v = w
                for _ in range(abs(step)):
                    v = np.nextafter(v, np.float32(np.copysign(np.inf, step)))
                blk.append(np.float32(v))
        blk += list(rng.uniform(-1, 1, 64 - len(blk)).astype(np.float32) * a)
        out[b] = np.array(blk, np.float32)
        assert np.max(np.abs(out[b])) == a
        if b % 2:
            out[b] = -out[b]
    return out.reshape(n_blocks // 4, 256)


def test_quantize_near_thresholds_bit_exact(nf):
    w = near_threshold_blocks()
    qt, dev = encode_both(nf, w)
    assert_encoding_equal(qt, dev)


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

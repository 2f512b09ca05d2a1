"""GPU parity of the fused NF4-LoRA linear layer (forward and backward)
against the fp64 oracle, on seeded inputs at sizes that span several tiles
and ragged tails, for both the few-token (M <= 16) and the many-token paths."""
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


def setup(nf, d_out, d_in, m, r, alpha=16.0, b_std=0.05, outliers=True, index=0):
    c = workloads.linear_case(d_out, d_in, m, r, alpha, outliers=outliers, index=index, b_std=b_std)
    qt = oracle.quantize(c.W)
    W_hat = oracle.dequantize(qt, c.W.shape)
    w = nf.nf4_quantize(torch.from_numpy(c.W).cuda())
    dev = {k: getattr(c, k).cuda() for k in ("A", "B", "X", "dY")}
    return c, W_hat, w, dev


CASES = [
    # (d_out, d_in, M, r)
    (128, 64, 1, 8),
    (256, 512, 4, 16),
    (384, 320, 16, 64),
    (136, 192, 3, 8),         # ragged d_out vs the 128-row tile
    (512, 512, 16, 8),
    (256, 256, 17, 16),       # first many-token size
    (264, 320, 130, 64),      # ragged tokens and d_out
    (512, 768, 300, 128),
    (1024, 512, 256, 24),
    (384, 1024, 200, 192),
    (4736, 4800, 2000, 16),   # enough tiles for the 256-row CTA tile; ragged tokens
    (9472, 1408, 5, 16),      # few tokens: two splits of 11 blocks (a ragged block quad)
    (256, 256, 7, 256),       # largest rank, few tokens
    (384, 256, 40, 256),      # largest rank, many tokens
    (5120, 4096, 4096, 16),   # 320 CTA tiles of 256 x 256: more than two waves, compared whole
    (11008, 4096, 16, 64),    # few tokens, 19 weight octets per cluster: the stage ring is refilled
    (4096, 11008, 3, 64),     # few tokens, 22 block quads per CTA: the stage ring is refilled
    (256, 16384, 5, 16),      # few tokens, one octet per cluster: a ring of 24 stages, deeper than the 16 warps
    (256, 512, 4, 1),         # ranks that are not multiples of 8 (padded internally): few tokens
    (384, 320, 16, 5),
    (264, 320, 130, 12),      # and many tokens
    (512, 768, 300, 5),
    (384, 256, 40, 251),
]


@pytest.mark.parametrize("d_out,d_in,m,r", CASES)
def test_forward_matches_oracle(nf, d_out, d_in, m, r):
    c, W_hat, w, dev = setup(nf, d_out, d_in, m, r)
    Y, T = nf.qlora_linear_fwd(w, dev["A"], dev["B"], c.scaling, dev["X"])
    torch.cuda.synchronize()
    nf.device_status()
    Y_ref, T_ref = oracle.forward(W_hat, c.A, c.B, c.X, c.scaling)
    assert_close(Y, Y_ref, "Y")
    assert T.dtype == torch.float32
    assert_close(T, T_ref, "T", max_rel=1e-5, mean_rel=1e-6, round_ref=False)


@pytest.mark.parametrize("d_out,d_in,m,r", CASES)
def test_backward_matches_oracle(nf, d_out, d_in, m, r):
    c, W_hat, w, dev = setup(nf, d_out, d_in, m, r)
    _, T = nf.qlora_linear_fwd(w, dev["A"], dev["B"], c.scaling, dev["X"])
    dX, dA, dB = nf.qlora_linear_bwd(w, dev["A"], dev["B"], c.scaling, dev["X"], T, dev["dY"])
    torch.cuda.synchronize()
    nf.device_status()
    dX_ref, dA_ref, dB_ref = oracle.backward(W_hat, c.A, c.B, c.X, c.dY, c.scaling)
    assert_close(dX, dX_ref, "dX")
    assert_close(dA, dA_ref, "dA")
    assert_close(dB, dB_ref, "dB")


def test_backward_recomputes_t_when_not_saved(nf):
    c, W_hat, w, dev = setup(nf, 256, 256, 40, 16)
    dX, dA, dB = nf.qlora_linear_bwd(w, dev["A"], dev["B"], c.scaling, dev["X"], None, dev["dY"])
    torch.cuda.synchronize()
    dX_ref, dA_ref, dB_ref = oracle.backward(W_hat, c.A, c.B, c.X, c.dY, c.scaling)
    assert_close(dB, dB_ref, "dB")
    assert_close(dA, dA_ref, "dA")
    assert_close(dX, dX_ref, "dX")


def test_zero_b_gives_base_product_and_zero_da(nf):
    c, W_hat, w, dev = setup(nf, 256, 512, 64, 16)
    B0 = torch.zeros_like(dev["B"])
    Y, T = nf.qlora_linear_fwd(w, dev["A"], B0, c.scaling, dev["X"])
    dX, dA, dB = nf.qlora_linear_bwd(w, dev["A"], B0, c.scaling, dev["X"], T, dev["dY"])
    torch.cuda.synchronize()
    W_dev = nf.nf4_dequantize(w)
    ref = (dev["X"].float() @ W_dev.float().t())
    assert_close(Y, ref, "Y (B = 0)")
    assert torch.count_nonzero(dA) == 0
    assert_close(dX, dev["dY"].float() @ W_dev.float(), "dX (B = 0)")


def test_accumulate_and_skipped_outputs(nf):
    c, W_hat, w, dev = setup(nf, 256, 256, 32, 8)
    _, T = nf.qlora_linear_fwd(w, dev["A"], dev["B"], c.scaling, dev["X"])
    dX, dA, dB = nf.qlora_linear_bwd(w, dev["A"], dev["B"], c.scaling, dev["X"], T, dev["dY"])
    _, dA2, dB2 = nf.qlora_linear_bwd(w, dev["A"], dev["B"], c.scaling, dev["X"], T, dev["dY"],
                                      need_dx=False, dA=dA.clone(), dB=dB.clone(), accumulate=True)
    only_dx, none_a, none_b = nf.qlora_linear_bwd(w, dev["A"], dev["B"], c.scaling, None, None, dev["dY"],
                                                  need_da=False, need_db=False)
    torch.cuda.synchronize()
    assert none_a is None and none_b is None
    assert torch.equal(only_dx, dX)
    assert_close(dA2, 2 * dA.float(), "dA accumulated")
    assert_close(dB2, 2 * dB.float(), "dB accumulated")


@pytest.mark.parametrize("m,r", [(7, 5), (200, 12)])
def test_accumulate_with_a_rank_off_the_multiple_of_8(nf, m, r):
    """dA and dB are accumulated through their padded copies: 2x the single
    gradient, and T from the forward is the oracle's."""
    c, W_hat, w, dev = setup(nf, 256, 320, m, r)
    _, T = nf.qlora_linear_fwd(w, dev["A"], dev["B"], c.scaling, dev["X"])
    dX, dA, dB = nf.qlora_linear_bwd(w, dev["A"], dev["B"], c.scaling, dev["X"], T, dev["dY"])
    _, dA2, dB2 = nf.qlora_linear_bwd(w, dev["A"], dev["B"], c.scaling, dev["X"], None, dev["dY"],
                                      need_dx=False, dA=dA.clone(), dB=dB.clone(), accumulate=True)
    torch.cuda.synchronize()
    nf.device_status()
    _, T_ref = oracle.forward(W_hat, c.A, c.B, c.X, c.scaling)
    assert_close(T, T_ref, "T", max_rel=1e-5, mean_rel=1e-6, round_ref=False)
    _, dA_ref, dB_ref = oracle.backward(W_hat, c.A, c.B, c.X, c.dY, c.scaling)
    assert_close(dA2, 2 * dA_ref, "dA accumulated")
    assert_close(dB2, 2 * dB_ref, "dB accumulated")


def test_layer_is_deterministic(nf):
    c, W_hat, w, dev = setup(nf, 512, 512, 256, 64)
    outs = []
    for _ in range(3):
        Y, T = nf.qlora_linear_fwd(w, dev["A"], dev["B"], c.scaling, dev["X"])
        g = nf.qlora_linear_bwd(w, dev["A"], dev["B"], c.scaling, dev["X"], T, dev["dY"])
        outs.append([Y.clone(), T.clone()] + [t.clone() for t in g])
    for o in outs[1:]:
        for a, b in zip(outs[0], o):
            assert torch.equal(a, b)


def test_empty_batch(nf):
    """M = 0: the forward does nothing; the backward's adapter gradients are
    zero (the gradient of an empty sum), or left as they are when accumulating."""
    c, W_hat, w, dev = setup(nf, 256, 256, 1, 16)
    X0 = dev["X"][:0]
    Y0 = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    Y, T = nf.qlora_linear_fwd(w, dev["A"], dev["B"], c.scaling, X0, Y=Y0)
    assert Y.shape == (0, 256) and T.shape == (0, 16)
    dA = torch.full((16, 256), 3.0, dtype=torch.bfloat16, device="cuda")
    dB = torch.full((256, 16), 3.0, dtype=torch.bfloat16, device="cuda")
    dY0 = dev["dY"][:0]
    nf.qlora_linear_bwd(w, dev["A"], dev["B"], c.scaling, X0, None, dY0, dA=dA, dB=dB, accumulate=True)
    torch.cuda.synchronize()
    assert torch.all(dA == 3.0) and torch.all(dB == 3.0)
    nf.qlora_linear_bwd(w, dev["A"], dev["B"], c.scaling, X0, None, dY0, dA=dA, dB=dB, accumulate=False)
    torch.cuda.synchronize()
    nf.device_status()
    assert torch.all(dA == 0) and torch.all(dB == 0)

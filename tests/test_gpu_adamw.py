"""GPU parity of the adapter's AdamW step (lora_adamw_step) with the oracle.

Per step the oracle (fp64, decoupled-weight-decay AdamW with bias-corrected
moments) starts from the same fp32 state as the kernel, so the comparison
measures one step's fp32 rounding only.  The tolerance is the first-order
rounding bound of the fp32 evaluation, element by element, with u = 2^-24
and a factor 4 for the few roundings of each step:
    |dm| <= 4u (|b1 m| + |(1 - b1) g|)        (the two terms may cancel)
    |dv| <= 4u (|b2 v| + |(1 - b2) g^2|)
    |dp| <= 4u |p (1 - lr wd)| + 8u |u_p| + (lr / bc1) |dm| / den
            + |u_p| |dv| / (2 v)              (u_p the update, den its divisor)
The bf16 copy the layer reads must be exactly the round-to-nearest-even of
the fp32 master.  Sizes cover the vector body, a ragged tail (n % 4 != 0),
an empty tensor and more tensors than one launch takes."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nf():
    import nf4_base_lora_b200 as nf
    return nf


def _state(n, seed):
    g = torch.Generator().manual_seed(seed)
    master = (torch.randn(n, generator=g) * 0.05).float()
    grad = (torch.randn(n, generator=g) * 10.0 ** float(torch.empty(1).uniform_(-4, -1, generator=g))).bfloat16()
    m = (torch.randn(n, generator=g) * 1e-3).float()
    v = (torch.rand(n, generator=g) * 1e-5).float()
    return master, grad, m, v


def f32(x):
    """The hyper-parameters cross the C ABI as fp32: the oracle takes the same values."""
    return float(np.float32(x))


def _check_step(nf, sizes, step, lr, wd, with_param=True, seed=0):
    host = [_state(n, seed + i) for i, n in enumerate(sizes)]
    dev = [tuple(t.cuda() for t in h) for h in host]
    params = [torch.empty(n, dtype=torch.bfloat16, device="cuda") if with_param else None for n in sizes]
    nf.lora_adamw_step([(d[0], p, d[1], d[2], d[3]) for d, p in zip(dev, params)], lr=lr, beta1=0.9, beta2=0.999,
                       eps=1e-8, weight_decay=wd, step=step)
    torch.cuda.synchronize()
    nf.device_status()
    for (master, grad, m, v), d, p in zip(host, dev, params):
        rp, rm, rv = oracle.adamw_step(master.numpy(), grad.float().numpy(), m.numpy(), v.numpy(), step, f32(lr),
                                       f32(0.9), f32(0.999), f32(1e-8), f32(wd))
        gp, gm, gv = (t.cpu().numpy().astype(np.float64) for t in d[:1] + d[2:])
        p0, g0, m0, v0 = (t.float().numpy().astype(np.float64) for t in (master, grad, m, v))
        b1, b2, lr_, wd_, eps = f32(0.9), f32(0.999), f32(lr), f32(wd), f32(1e-8)
        u = 2.0 ** -24
        err_m = 4 * u * (np.abs(b1 * m0) + np.abs((1 - b1) * g0)) + 1e-38
        err_v = 4 * u * (np.abs(b2 * v0) + np.abs((1 - b2) * g0 * g0)) + 1e-38
        bc1, bc2 = 1 - b1 ** step, 1 - b2 ** step
        den = np.sqrt(rv) / np.sqrt(bc2) + eps
        upd = (lr_ / bc1) * rm / den
        err_p = (4 * u * np.abs(p0 * (1 - lr_ * wd_)) + 8 * u * np.abs(upd) + (lr_ / bc1) * err_m / den
                 + np.abs(upd) * err_v / (2 * np.maximum(rv, 1e-38)) + 1e-38)
        assert np.all(np.abs(gm - rm) <= err_m), np.max(np.abs(gm - rm) / err_m)
        assert np.all(np.abs(gv - rv) <= err_v), np.max(np.abs(gv - rv) / err_v)
        assert np.all(np.abs(gp - rp) <= err_p), np.max(np.abs(gp - rp) / err_p)
        if p is not None:
            assert torch.equal(p.cpu(), d[0].cpu().bfloat16())


@pytest.mark.parametrize("step,lr,wd", [(1, 2e-4, 0.0), (7, 1e-3, 0.01), (1000, 2e-4, 0.1)])
def test_adamw_step_matches_oracle(nf, step, lr, wd):
    _check_step(nf, [4096 * 64, 64 * 11008 + 4, 1021, 0, 8], step, lr, wd)


def test_adamw_many_tensors_and_no_bf16_copy(nf):
    _check_step(nf, [1000 + 37 * i for i in range(11)], 3, 5e-4, 0.0, with_param=False, seed=50)


def test_adamw_steps_track_the_oracle(nf):
    """Five consecutive steps on the GPU against five fp64 oracle steps."""
    n = 4100
    master, _, _, _ = _state(n, 9)
    m = torch.zeros(n)
    v = torch.zeros(n)
    d = [master.cuda(), m.cuda(), v.cuda()]
    rp, rm, rv = master.double().numpy(), np.zeros(n), np.zeros(n)
    rng = torch.Generator().manual_seed(10)
    for t in range(1, 6):
        grad = (torch.randn(n, generator=rng) * 1e-3).bfloat16()
        nf.lora_adamw_step([(d[0], None, grad.cuda(), d[1], d[2])], lr=1e-3, weight_decay=0.01, step=t)
        rp, rm, rv = oracle.adamw_step(rp, grad.float().numpy(), rm, rv, t, f32(1e-3), f32(0.9), f32(0.999),
                                       f32(1e-8), f32(0.01))
    torch.cuda.synchronize()
    # five steps of fp32 rounding, normwise (an entry can pass through zero or a
    # moment cancel to near zero, so element-wise ratios are not meaningful)
    for got, ref, tol in ((d[0], rp, 1e-6), (d[1], rm, 1e-5), (d[2], rv, 1e-5)):
        got = got.cpu().double().numpy()
        assert np.max(np.abs(got - ref)) <= tol * np.max(np.abs(ref))


@pytest.mark.parametrize("m", [4, 16, 64])
def test_layer_right_after_the_step_sees_the_new_adapter(nf, m):
    """The optimizer step rewrites the bf16 A and B the layer reads; the
    forward and backward enqueued right after it on the same stream (no
    synchronisation in between) must use the new values."""
    import workloads
    from parity import assert_close
    d_out, d_in, r, s = 512, 512, 16, 0.5
    W = workloads.weight(d_out, d_in, index=3)
    qt = oracle.quantize(W)
    enc = nf.nf4_quantize(torch.from_numpy(W).cuda())
    A0, B0 = workloads.lora_a(r, d_in, 3), workloads.lora_b(d_out, r, 3, std=0.05)
    X, dY = workloads.activations(m, d_in), workloads.grad_output(m, d_out, 3)
    params = []
    for p0 in (A0, B0):
        master = p0.float().reshape(-1).cuda()
        param = p0.clone().cuda()
        grad = (torch.randn(p0.numel(), generator=torch.Generator().manual_seed(p0.numel())) * 0.1).bfloat16().cuda()
        params.append((master, param.reshape(-1), grad, torch.zeros_like(master), torch.zeros_like(master), param))
    torch.cuda.synchronize()
    nf.lora_adamw_step([t[:5] for t in params], lr=0.05, step=1)  # moves every entry by about 0.05
    A, B = params[0][5], params[1][5]
    Y, T = nf.qlora_linear_fwd(enc, A, B, s, X.cuda())
    dX, dA, dB = nf.qlora_linear_bwd(enc, A, B, s, X.cuda(), T, dY.cuda())
    torch.cuda.synchronize()
    nf.device_status()
    A1, B1 = A.cpu(), B.cpu()
    assert not torch.equal(A1, A0)
    W_hat = oracle.dequantize(qt, (d_out, d_in))
    Y_ref, _ = oracle.forward(W_hat, A1, B1, X, s)
    assert_close(Y.cpu(), Y_ref, "Y after the step")
    dX_ref, dA_ref, dB_ref = oracle.backward(W_hat, A1, B1, X, dY, s)
    assert_close(dX.cpu(), dX_ref, "dX after the step")
    assert_close(dA.cpu(), dA_ref, "dA after the step")
    assert_close(dB.cpu(), dB_ref, "dB after the step")

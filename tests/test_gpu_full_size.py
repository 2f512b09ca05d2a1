"""GPU parity at the full sizes the benchmark times, through the same calls
the benchmark step makes (forward without saving T, backward recomputing T
from X, one shared workspace).

A full oracle product at these sizes takes minutes, so the check is sampled
where the outputs separate cleanly: rows of Y and dX depend only on their own
token row, so one row inside every 128-row tile, the rows on both sides of
every 256-row boundary, and the first and last row are compared against the
fp64 oracle computed for those rows alone (every column of each).  The rank-r gradients
dA and dB need no pass over the base weight and are compared whole.  The
weight the kernels decode is first checked to be, byte for byte, the oracle's
encoding of the same fp32 weight, so the sampled rows test the fused GEMMs
against an independent W_hat."""
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


def _unique_modules(wl):
    """(module index, module) of the first module of each distinct shape."""
    seen, out = set(), []
    for i, mod in enumerate(wl.modules):
        if (mod.d_out, mod.d_in) not in seen:
            seen.add((mod.d_out, mod.d_in))
            out.append((i, mod))
    return out


CASES = [(name, i, mod) for name, wl in workloads.WORKLOADS.items() if name != "linear512_r8_m16"
         for i, mod in _unique_modules(wl)]


def _sample_rows(m):
    """Token rows that reach every CTA tile of a launch: one row inside each
    128-row tile (at an offset that moves from tile to tile, 128 t + 37 t mod
    128), both rows on either side of every 256-row boundary (where the 256-
    and 128-row tile shapes split differently), and the first and last row."""
    rows = {0, m - 1}
    for t in range((m + 127) // 128):
        rows.add(min(m - 1, 128 * t + (37 * t) % 128))
    for b in range(256, m, 256):
        rows.update((b - 1, b))
    return np.array(sorted(rows))


def test_sample_rows_cover_every_tile():
    for m in (17, 300, 2048, 4096, 8192):
        rows = _sample_rows(m)
        assert rows[0] == 0 and rows[-1] == m - 1
        assert set(rows // 128) == set(range((m + 127) // 128))
        for b in range(256, m, 256):
            assert b - 1 in rows and b in rows


@pytest.mark.parametrize("name,index,mod", CASES,
                         ids=[f"{n}-{m.name}" for n, _, m in CASES])
def test_bench_workload_sampled(nf, name, index, mod):
    wl = workloads.WORKLOADS[name]
    W = workloads.weight(mod.d_out, mod.d_in, wl.sigma, wl.outliers, index)
    qt = oracle.quantize(W)
    enc = nf.nf4_quantize(torch.from_numpy(W).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(enc.codes.cpu().numpy(), qt["packed"])
    assert np.array_equal(enc.qscale.cpu().numpy(), qt["q"])
    del W
    W_hat = oracle.dequantize(qt, (mod.d_out, mod.d_in))
    del qt
    A = workloads.lora_a(wl.r, mod.d_in, index)
    B = workloads.lora_b(mod.d_out, wl.r, index)
    mmax = max(wl.tokens)
    X_all = workloads.activations(mmax, mod.d_in, workloads.x_seed(mod.d_in, wl.modules[0].d_in))
    dY_all = workloads.grad_output(mmax, mod.d_out, index)
    Ad, Bd = A.cuda(), B.cuda()
    ws_bytes = max(max(nf.qlora_fwd_workspace_bytes(m, mod.d_out, mod.d_in, wl.r),
                       nf.qlora_bwd_workspace_bytes(m, mod.d_out, mod.d_in, wl.r)) for m in wl.tokens)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    for m in wl.tokens:
        X, dY = X_all[:m], dY_all[:m]
        Xd, dYd = X.cuda(), dY.cuda()
        Y, _ = nf.qlora_linear_fwd(enc, Ad, Bd, wl.scaling, Xd, save_t=False, workspace=ws)
        if wl.backward == "dx":
            dX, dA, dB = nf.qlora_linear_bwd(enc, Ad, Bd, wl.scaling, None, None, dYd, need_da=False,
                                             need_db=False, workspace=ws)
        else:
            dX, dA, dB = nf.qlora_linear_bwd(enc, Ad, Bd, wl.scaling, Xd, None, dYd, workspace=ws)
        torch.cuda.synchronize()
        nf.device_status()
        rows = _sample_rows(m) if m > 16 else np.arange(m)
        Y_ref = oracle.output_rows(W_hat, A, B, X[rows], wl.scaling)
        assert_close(Y.cpu()[rows], Y_ref, f"Y[{m}]")
        dX_ref = oracle.input_grad_rows(W_hat, A, B, dY[rows], wl.scaling)
        assert_close(dX.cpu()[rows], dX_ref, f"dX[{m}]")
        if dA is not None:
            dA_ref, dB_ref = oracle.lora_grads(A, B, X, dY, wl.scaling)
            assert_close(dA, dA_ref, f"dA[{m}]")
            assert_close(dB, dB_ref, f"dB[{m}]")

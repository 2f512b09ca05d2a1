"""The failure detector every kernel shares, made to fire without a fault.

Each kernel bounds its waits on shared-memory barriers; a wait that runs out
sets the device status word, drains the copies in flight, frees tensor memory
and returns.  nf4lora_check_bounded_wait runs a kernel that holds tensor
memory and a bulk copy in flight like a layer kernel, then waits on a barrier
nothing arrives on with a 1 ms limit.  The test checks that the kernel
returns, that the status reads NF4_ERR_TIMEOUT exactly once, and that the
context is still fully usable: the many-token layer (which allocates tensor
memory) and the few-token layer still match the oracle afterwards."""
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


def test_wait_runs_out_and_is_reported_once(nf):
    torch.cuda.set_device(0)
    nf.device_status()                          # clean start
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    nf.check_bounded_wait(1_000_000)            # 1 ms
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    assert 0.9 <= ms < 200.0, ms                # it waited its limit, then returned
    with pytest.raises(nf.Nf4Error) as err:
        nf.device_status()
    assert err.value.status == -6               # NF4_ERR_TIMEOUT
    nf.device_status()                          # read and cleared: OK now


def test_layer_still_matches_after_a_timeout(nf):
    nf.check_bounded_wait(200_000)
    torch.cuda.synchronize()
    with pytest.raises(nf.Nf4Error):
        nf.device_status()
    for m in (300, 7):                          # many-token (tcgen05 + TMEM) and few-token paths
        c = workloads.linear_case(256, 512, m, 16, 16.0, outliers=True, b_std=0.05)
        qt = oracle.quantize(c.W)
        W_hat = oracle.dequantize(qt, c.W.shape)
        w = nf.nf4_quantize(torch.from_numpy(c.W).cuda())
        Y, T = nf.qlora_linear_fwd(w, c.A.cuda(), c.B.cuda(), c.scaling, c.X.cuda())
        dX, dA, dB = nf.qlora_linear_bwd(w, c.A.cuda(), c.B.cuda(), c.scaling, c.X.cuda(), T, c.dY.cuda())
        torch.cuda.synchronize()
        nf.device_status()
        Y_ref, _ = oracle.forward(W_hat, c.A, c.B, c.X, c.scaling)
        dX_ref, dA_ref, dB_ref = oracle.backward(W_hat, c.A, c.B, c.X, c.dY, c.scaling)
        assert_close(Y, Y_ref, "Y")
        assert_close(dX, dX_ref, "dX")
        assert_close(dA, dA_ref, "dA")
        assert_close(dB, dB_ref, "dB")


def test_limit_is_checked_on_the_host(nf):
    assert nf.lib.nf4lora_check_bounded_wait(10, None) == -1
    assert nf.lib.nf4lora_check_bounded_wait(2_000_000_000, None) == -1

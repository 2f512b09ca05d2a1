"""Ordering of the overlapped gradient exchange on one GPU (a process group
of one rank over NCCL: the all-reduce is then the identity, so any
difference is an ordering fault).  The backward that writes dA and dB is
held back behind a long device-side sleep; the exchange is launched right
after it is enqueued.  The buffer the exchange packs must hold the complete
gradients (it waited for the backward's event, not for the host), the host
must not have been blocked, and after finish() the gradients are the
backward's own."""
import datetime
import os
import socket
import time

import pytest
import torch
import torch.distributed as dist

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nf():
    import nf4_base_lora_b200 as nf
    return nf


@pytest.fixture(scope="module")
def group():
    torch.cuda.set_device(0)
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    yield
    dist.destroy_process_group()


def test_exchange_waits_for_the_backward_not_the_host(nf, group):
    from nf4_base_lora_b200 import dp
    c = workloads.linear_case(1024, 2048, 512, 16, 16.0, outliers=True, index=1)
    w = nf.nf4_quantize(torch.from_numpy(c.W).cuda())
    A, B, X, dY = (getattr(c, k).cuda() for k in ("A", "B", "X", "dY"))
    _, dA_ref, dB_ref = nf.qlora_linear_bwd(w, A, B, c.scaling, X, None, dY, need_dx=False)
    dA = torch.zeros_like(dA_ref)
    dB = torch.zeros_like(dB_ref)
    ex = dp.OverlappedGradExchange([[dA, dB]])
    ex.launch(0)                                  # a first exchange: the communicator's set-up
    ex.finish()
    dA.zero_()
    dB.zero_()
    torch.cuda.synchronize()
    torch.cuda._sleep(200_000_000)               # about 0.1 s of device time before the backward
    nf.qlora_linear_bwd(w, A, B, c.scaling, X, None, dY, need_dx=False, dA=dA, dB=dB)
    t0 = time.perf_counter()
    ex.launch(0)
    host_s = time.perf_counter() - t0
    pending = not ex.stream.query()
    ex.finish()
    torch.cuda.synchronize()
    nf.device_status()
    packed = ex.buckets[0].flat
    assert torch.equal(packed, torch.cat([dA_ref.float().reshape(-1), dB_ref.float().reshape(-1)]))
    assert torch.equal(dA, dA_ref) and torch.equal(dB, dB_ref)
    # the host went on while the exchange still waited for the backward
    assert host_s < 0.05 and pending, (host_s, pending)


def test_finish_orders_the_next_write_after_the_exchange(nf, group):
    """A write to the gradients enqueued after finish() lands after the
    exchange's write-back, so it is what remains."""
    from nf4_base_lora_b200 import dp
    dA = torch.zeros((16, 2048), dtype=torch.bfloat16, device="cuda")
    dB = torch.zeros((1024, 16), dtype=torch.bfloat16, device="cuda")
    ex = dp.OverlappedGradExchange([[dA, dB]])
    torch.cuda.synchronize()
    dA.fill_(1.0)
    dB.fill_(2.0)
    ex.launch(0)
    ex.finish()
    dA.fill_(3.0)                                 # the next step's backward, say
    torch.cuda.synchronize()
    assert torch.all(dA == 3.0) and torch.all(dB == 2.0)

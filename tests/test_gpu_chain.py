"""Back-to-back layer calls: the many-token kernels are chained as
programmatic dependents (the next kernel may start while the one before it
finishes), and consecutive calls share one workspace.  A training-step-like
sequence over three linears (forward of each, then the backward of each, the
next linear's input being the previous one's output) is run three ways —
with a device synchronisation after every call, back to back on one stream,
and replayed from a CUDA graph of the back-to-back sequence — and every
output must be bit-identical across the three (the kernels have a fixed
summation order, so any difference is an ordering fault)."""
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

SHAPES = [(512, 384), (640, 512), (384, 640)]   # (d_out, d_in): each d_in is the previous d_out
R = 24


@pytest.fixture(scope="module")
def nf():
    import nf4_base_lora_b200 as nf
    return nf


def _setup(nf, M):
    torch.cuda.set_device(0)
    mods = []
    for i, (d_out, d_in) in enumerate(SHAPES):
        W = torch.from_numpy(workloads.weight(d_out, d_in, outliers=True, index=i)).cuda()
        mods.append({"w": nf.nf4_quantize(W), "A": workloads.lora_a(R, d_in, i).cuda(),
                     "B": workloads.lora_b(d_out, R, i, std=0.05).cuda(),
                     "dY": workloads.grad_output(M, d_out, i).cuda()})
    X0 = workloads.activations(M, SHAPES[0][1]).cuda()
    ws = torch.empty(max(max(nf.qlora_fwd_workspace_bytes(M, o, k, R), nf.qlora_bwd_workspace_bytes(M, o, k, R))
                         for o, k in SHAPES), dtype=torch.uint8, device="cuda")
    outs = [{"Y": torch.empty((M, o), dtype=torch.bfloat16, device="cuda"),
             "T": torch.empty((M, R), dtype=torch.float32, device="cuda"),
             "dX": torch.empty((M, k), dtype=torch.bfloat16, device="cuda"),
             "dA": torch.empty((R, k), dtype=torch.bfloat16, device="cuda"),
             "dB": torch.empty((o, R), dtype=torch.bfloat16, device="cuda")} for o, k in SHAPES]
    return mods, X0, ws, outs


def _sequence(nf, mods, X0, ws, outs, sync):
    x = X0
    for d, o in zip(mods, outs):
        nf.qlora_linear_fwd(d["w"], d["A"], d["B"], 0.5, x, Y=o["Y"], T=o["T"], workspace=ws)
        if sync:
            torch.cuda.synchronize()
        x = o["Y"]
    xs = [X0] + [o["Y"] for o in outs[:-1]]
    for d, o, x in zip(reversed(mods), reversed(outs), reversed(xs)):
        nf.qlora_linear_bwd(d["w"], d["A"], d["B"], 0.5, x, o["T"], d["dY"], dX=o["dX"], dA=o["dA"], dB=o["dB"],
                            workspace=ws)
        if sync:
            torch.cuda.synchronize()


def _snapshot(outs):
    return [{k: v.clone() for k, v in o.items()} for o in outs]


@pytest.mark.parametrize("M", [300, 9])   # the many-token kernels and the few-token ones
def test_chained_calls_match_synchronised_calls(nf, M):
    mods, X0, ws, outs = _setup(nf, M)
    _sequence(nf, mods, X0, ws, outs, sync=True)
    ref = _snapshot(outs)
    for o in outs:
        for v in o.values():
            v.zero_()
    torch.cuda.synchronize()
    for _ in range(3):
        _sequence(nf, mods, X0, ws, outs, sync=False)
    torch.cuda.synchronize()
    nf.device_status()
    for o, r in zip(outs, ref):
        for k in o:
            assert torch.equal(o[k], r[k]), k

    # the same sequence captured once and replayed
    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        _sequence(nf, mods, X0, ws, outs, sync=False)  # warm-up on the capture stream
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=stream):
            _sequence(nf, mods, X0, ws, outs, sync=False)
    for o in outs:
        for v in o.values():
            v.zero_()
    torch.cuda.synchronize()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    nf.device_status()
    for o, r in zip(outs, ref):
        for k in o:
            assert torch.equal(o[k], r[k]), k

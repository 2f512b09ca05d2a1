"""Launch tracing: a layer call traced eagerly and the same call traced while
it is captured into a CUDA graph (then replayed) record the same kernels in
the same order, each with a positive device time; inside a capture the event
pairs are event-record nodes of the graph, so a replay records them again.
Tracing must not change the results either."""
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nf():
    import nf4_base_lora_b200 as nf
    return nf


@pytest.mark.parametrize("M", [16, 512])
def test_trace_eager_and_graph_replay(nf, M):
    torch.cuda.set_device(0)
    d_out, d_in, r = 1024, 512, 16
    w = nf.nf4_quantize(torch.from_numpy(workloads.weight(d_out, d_in, index=1)).cuda())
    A = workloads.lora_a(r, d_in, 1).cuda()
    B = workloads.lora_b(d_out, r, 1, std=0.05).cuda()
    X = workloads.activations(M, d_in).cuda()
    ws = torch.empty(nf.qlora_fwd_workspace_bytes(M, d_out, d_in, r), dtype=torch.uint8, device="cuda")
    Y = torch.empty((M, d_out), dtype=torch.bfloat16, device="cuda")
    T = torch.empty((M, r), dtype=torch.float32, device="cuda")
    stream = torch.cuda.Stream()

    def call():
        nf.qlora_linear_fwd(w, A, B, 0.5, X, Y=Y, T=T, workspace=ws)

    with torch.cuda.stream(stream):
        call()
    torch.cuda.synchronize()
    Y_plain = Y.clone()

    nf.trace_start(64)
    with torch.cuda.stream(stream):
        call()
    torch.cuda.synchronize()
    eager = nf.trace_records()
    nf.trace_stop()
    assert torch.equal(Y, Y_plain)

    nf.trace_start(64)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        call()
    Y.zero_()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        graph.replay()
    torch.cuda.synchronize()
    replayed = nf.trace_records()
    nf.trace_stop()
    del graph
    assert torch.equal(Y, Y_plain)

    assert len(eager) >= 2
    assert [n for n, _ in replayed] == [n for n, _ in eager]
    assert all(ms > 0.0 for _, ms in eager + replayed)
    nf.device_status()

"""CUDA-graph capture of the layer and shape edge cases (GPU)."""
import pytest
import torch

from sparse_moe_layer_warp_b200 import synth
from tests.helpers import compare_layer, make_layer

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kw", [
    {"dtype": "bf16", "T": 16, "d": 512, "E": 64, "k": 8, "f": 256},      # decode-like, fused routing
    {"dtype": "bf16", "T": 700, "d": 768, "E": 8, "k": 4, "f": 512},      # CTA-pair kernels
    {"dtype": "f32"},
])
def test_forward_captured_in_cuda_graph_matches_eager(cuda_ok, kw):
    w = synth.WORKLOADS["tiny_fp32"].replace(**kw)
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp)
    x = inp.x.clone()
    out = torch.empty_like(x)
    eager = layer.forward(x).clone()  # also allocates the workspace before capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        layer.forward(x, out=out)  # warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(s)
    with torch.cuda.graph(g):
        layer.forward(x, out=out)
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, eager)
    # a new input through the same graph
    x2 = synth.make_x(w, w.T, device="cuda", seed=5)
    x.copy_(x2)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, layer.forward(x2))
    assert layer.device_status() == 0


def test_forward_many_experts_k32(cuda_ok):
    # E = 1024 (the routing kernels' limit) and k = 32 (one slot per lane)
    w = synth.WORKLOADS["tiny_fp32"].replace(dtype="bf16", T=50, d=256, E=1024, k=32, f=128)
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp)
    out = layer.forward(inp.x)
    r = layer.route(x=inp.x)
    torch.cuda.synchronize()
    compare_layer(inp, out, r["idx"].cpu().numpy())


def test_forward_at_max_tokens_and_below(cuda_ok):
    w = synth.WORKLOADS["tiny_fp32"].replace(dtype="bf16", T=130, d=256, E=32, k=8, f=128)
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp, max_tokens=130)
    for T in (130, 129, 65, 64, 1):  # both routing paths, ragged tails
        sub = synth.LayerInputs(w.replace(T=T), inp.x[:T].contiguous(), inp.w_router, inp.bias,
                                inp.w_gate, inp.w_up, inp.w_down)
        out = layer.forward(sub.x)
        r = layer.route(x=sub.x)
        torch.cuda.synchronize()
        compare_layer(sub, out, r["idx"].cpu().numpy())


@pytest.mark.parametrize("kw,expected", [
    # decode: routing in one launch, rows gathered by the up GEMM -> route, up, down, combine
    ({"dtype": "bf16", "T": 16, "d": 256, "E": 64, "k": 8, "f": 128}, 4),
    # ~75 tokens per expert: router, top-k, scatter, row gather, up, down, combine
    ({"dtype": "bf16", "T": 300, "d": 512, "E": 32, "k": 8, "f": 256}, 7),
    # CTA pairs (350 tokens per expert; the shared expert's 6 up units are fewer than the
    # device's CTA pairs, so the sorted copy has its own launch): router, top-k, scatter,
    # row gather, up, down, combine
    ({"dtype": "bf16", "T": 700, "d": 768, "E": 8, "k": 4, "f": 512, "seed": 6}, 7),
    # fp32, 64 tokens: router, small-batch routing, up, down, combine
    ({"dtype": "f32"}, 5),
    # fp32, 65 tokens: router, top-k, scatter, up, down, combine
    ({"dtype": "f32", "T": 65}, 6),
])
def test_forward_launch_count_matches_captured_graph(cuda_ok, kw, expected):
    from cuda.bindings import runtime as rt
    from sparse_moe_layer_warp_b200 import moe_forward_launch_count
    w = synth.WORKLOADS["tiny_fp32"].replace(**kw)
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp)
    assert moe_forward_launch_count(layer.handle, w.T) == expected
    assert moe_forward_launch_count(layer.handle, 0) == 0
    assert moe_forward_launch_count(layer.handle, w.T + 10**6) == -1
    x = inp.x.clone()
    out = layer.forward(x).clone()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph(keep_graph=True)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        layer.forward(x, out=out)
    torch.cuda.current_stream().wait_stream(s)
    with torch.cuda.graph(g):
        layer.forward(x, out=out)
    graph = rt.cudaGraph_t(init_value=g.raw_cuda_graph())
    err, _, n = rt.cudaGraphGetNodes(graph, 0)
    assert err == rt.cudaError_t.cudaSuccess
    err, nodes, n = rt.cudaGraphGetNodes(graph, n)
    assert err == rt.cudaError_t.cudaSuccess
    kernels = 0
    for node in nodes[:n]:
        err, typ = rt.cudaGraphNodeGetType(node)
        assert err == rt.cudaError_t.cudaSuccess
        kernels += typ == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel
    assert kernels == expected


@pytest.mark.parametrize("kw", [
    {"dtype": "bf16", "T": 16, "d": 256, "E": 64, "k": 8, "f": 256},      # decode routing
    {"dtype": "bf16", "T": 300, "d": 256, "E": 8, "k": 4, "f": 512},      # CTA-pair kernels
    {"dtype": "f32", "T": 40},
])
def test_backward_captured_in_cuda_graph_matches_eager(cuda_ok, kw):
    """moe_backward records into a CUDA graph (no host synchronisation or allocation inside);
    replays equal the eager call bitwise, and the weight gradients accumulate per replay."""
    w = synth.WORKLOADS["tiny_fp32"].replace(**kw)
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp)
    dout = synth.make_x(w, w.T, device="cuda", seed=8)
    eager = layer.backward(inp.x, dout)  # also allocates the backward workspace
    torch.cuda.synchronize()
    names = ("dw_router", "dw_gate", "dw_up", "dw_down")
    grads = {n: torch.zeros_like(eager[n]) for n in names}
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        layer.backward(inp.x, dout, grads=grads)  # warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        out = layer.backward(inp.x, dout, grads=grads)
    for t in grads.values():
        t.zero_()
    g.replay()
    torch.cuda.synchronize()
    for n in eager:
        assert torch.equal(out[n], eager[n]), n
    g.replay()
    torch.cuda.synchronize()
    for n in names:
        assert torch.equal(out[n], 2 * eager[n]), n
    assert layer.device_status() == 0

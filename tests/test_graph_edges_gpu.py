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

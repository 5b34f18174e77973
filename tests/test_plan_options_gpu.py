"""Launch-plan options of a handle (moe_set_option).

MOE_OPTION_H_HANDOVER = 0 plans the bf16 forward's down-projection GEMM with a whole-grid
wait on the up GEMM instead of the per-group hand-over of h (the plan the forward also takes
when the init-time occupancy check finds an up grid that would not be co-resident).  Both
plans run the same arithmetic in the same order, so their outputs must be equal bit for bit,
and both must match the oracle.  MOE_OPTION_ROW_GATHER_IN_GEMM = 0 writes the expert-sorted
copy of x with a kernel of its own instead of the CTA-pair up GEMM's gather warps: same
bytes in the copy, same results bit for bit."""
import pytest
import torch

from sparse_moe_layer_warp_b200 import (MOE_OPTION_GEMM_CLOCK, MOE_OPTION_H_HANDOVER,
                                        MOE_OPTION_ROW_GATHER_IN_GEMM, MoEError, synth)
from tests.helpers import compare_layer, make_layer

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kw", [
    {"T": 16, "d": 512, "E": 64, "k": 8, "f": 256},               # one-CTA, rows gathered by TMA
    {"T": 300, "d": 512, "E": 32, "k": 8, "f": 256},              # one-CTA, sorted copy of x
    {"T": 700, "d": 768, "E": 8, "k": 4, "f": 512, "seed": 6},    # CTA pairs
    {"T": 600, "d": 256, "E": 16, "k": 4, "f": 256, "seed": 4, "bias": "zipf"},  # skewed pairs
])
def test_whole_grid_wait_plan_matches_handover_plan(cuda_ok, kw):
    w = synth.WORKLOADS["tiny_fp32"].replace(dtype="bf16", **kw)
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp)
    a = layer.forward(inp.x).clone()
    layer.set_option(MOE_OPTION_H_HANDOVER, 0)
    b = layer.forward(inp.x).clone()
    r = layer.route(x=inp.x)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    compare_layer(inp, b, r["idx"].cpu().numpy())
    layer.set_option(MOE_OPTION_H_HANDOVER, 1)
    c = layer.forward(inp.x)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), c.view(torch.int16))
    assert layer.device_status() == 0


def test_set_option_rejects_unknown(cuda_ok):
    w = synth.WORKLOADS["tiny_fp32"]
    layer = make_layer(synth.make_inputs(w, device="cuda"))
    with pytest.raises(MoEError):
        layer.set_option(99, 1)
    with pytest.raises(MoEError):
        layer.set_option(MOE_OPTION_H_HANDOVER, 2)


PAIR_CASES = [
    {"T": 700, "d": 768, "E": 8, "k": 4, "f": 512, "seed": 6},
    {"T": 600, "d": 256, "E": 16, "k": 4, "f": 256, "seed": 4, "bias": "zipf"},
    {"T": 1000, "d": 512, "E": 24, "k": 6, "f": 256, "seed": 8, "routed_scale": 1.5},
]


@pytest.mark.parametrize("kw", PAIR_CASES)
@pytest.mark.parametrize("sms", [2, 32, 148])
def test_shared_expert_on_side_stream_matches(cuda_ok, kw, sms):
    """MOE_OPTION_SHARED_SIDE_SMS: the shared expert's GEMMs on the handle's side stream
    during the routing give the same output bit for bit, eagerly and in a CUDA graph."""
    from sparse_moe_layer_warp_b200 import MOE_OPTION_SHARED_SIDE_SMS, moe_forward_launch_count

    w = synth.WORKLOADS["tiny_fp32"].replace(dtype="bf16", **kw)
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp)
    ref = layer.forward(inp.x).clone()
    layer.set_option(MOE_OPTION_ROW_GATHER_IN_GEMM, 0)
    n0 = moe_forward_launch_count(layer.handle, w.T)
    layer.set_option(MOE_OPTION_ROW_GATHER_IN_GEMM, 1)
    layer.set_option(MOE_OPTION_SHARED_SIDE_SMS, sms)
    # the two side GEMMs; the row gather has its own launch (the up GEMM gathers the rows
    # itself only while it runs the shared expert's units)
    assert moe_forward_launch_count(layer.handle, w.T) == n0 + 2
    a = layer.forward(inp.x).clone()
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), ref.view(torch.int16))
    # captured: the fork and join are recorded into the graph
    x = inp.x.clone()
    out = torch.empty_like(x)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        layer.forward(x, out=out)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        layer.forward(x, out=out)
    x2 = synth.make_x(w, w.T, device="cuda", seed=11)
    x.copy_(x2)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    layer.set_option(MOE_OPTION_SHARED_SIDE_SMS, 0)
    b = layer.forward(x2)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), b.view(torch.int16))
    del g
    assert layer.device_status() == 0


@pytest.mark.parametrize("kw", PAIR_CASES + [
    {"T": 900, "d": 512, "E": 16, "k": 4, "f": 256, "seed": 9, "n_shared": 0},  # no shared
])
def test_row_gather_in_up_gemm_matches_own_launch(cuda_ok, kw):
    """The CTA-pair up GEMM's own row gather (2: forced; these shapes have too few shared
    units for the default to choose it) against the gather kernel (0): outputs equal bit for
    bit, both equal to the oracle, one launch fewer with a shared expert; the in-GEMM gather
    replays from a CUDA graph."""
    from sparse_moe_layer_warp_b200 import moe_forward_launch_count

    w = synth.WORKLOADS["tiny_fp32"].replace(dtype="bf16", **kw)
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp)
    n1 = moe_forward_launch_count(layer.handle, w.T)
    layer.set_option(MOE_OPTION_ROW_GATHER_IN_GEMM, 2)
    n2 = moe_forward_launch_count(layer.handle, w.T)
    assert n2 == n1 - (1 if w.n_shared else 0)
    a = layer.forward(inp.x).clone()
    layer.set_option(MOE_OPTION_ROW_GATHER_IN_GEMM, 0)
    assert moe_forward_launch_count(layer.handle, w.T) == n1
    b = layer.forward(inp.x).clone()
    r = layer.route(x=inp.x)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    compare_layer(inp, a, r["idx"].cpu().numpy())
    # captured with the in-GEMM gather, replayed on another batch
    layer.set_option(MOE_OPTION_ROW_GATHER_IN_GEMM, 2)
    x = inp.x.clone()
    out = torch.empty_like(x)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        layer.forward(x, out=out)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        layer.forward(x, out=out)
    x.copy_(synth.make_x(w, w.T, device="cuda", seed=21))
    g.replay()
    layer.set_option(MOE_OPTION_ROW_GATHER_IN_GEMM, 0)
    d = layer.forward(x)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), d.view(torch.int16))
    del g
    assert layer.device_status() == 0
    with pytest.raises(MoEError):
        layer.set_option(MOE_OPTION_ROW_GATHER_IN_GEMM, 3)


@pytest.mark.parametrize("kw", [
    {"T": 16, "d": 512, "E": 64, "k": 8, "f": 256},               # one-CTA GEMMs
    {"T": 700, "d": 768, "E": 8, "k": 4, "f": 512, "seed": 6},    # CTA pairs
])
def test_gemm_clock_option(cuda_ok, kw):
    w = synth.WORKLOADS["tiny_fp32"].replace(dtype="bf16", **kw)
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp)
    a = layer.forward(inp.x).clone()
    assert layer.gemm_clock_mhz() == (0.0, 0.0)  # off by default: nothing recorded
    layer.set_option(MOE_OPTION_GEMM_CLOCK, 1)
    for _ in range(3):
        b = layer.forward(inp.x)
    up, down = layer.gemm_clock_mhz()
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert 100.0 < up < 3000.0 and 100.0 < down < 3000.0, (up, down)
    assert layer.gemm_clock_mhz() == (0.0, 0.0)  # read and cleared
    layer.set_option(MOE_OPTION_GEMM_CLOCK, 0)
    layer.forward(inp.x)
    assert layer.gemm_clock_mhz() == (0.0, 0.0)
    with pytest.raises(MoEError):
        layer.set_option(MOE_OPTION_GEMM_CLOCK, 2)

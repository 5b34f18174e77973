"""GPU parity for the layer backward (moe_backward) against the CPU oracle's chain rule, on
the GPU's own selection (the backward is defined for the forward's discrete choice of
experts): the oracle takes the GPU's idx, and computes the gates of that selection itself
from its own router logits."""
import numpy as np
import pytest
import torch

from oracle import oracle_gates, oracle_moe_backward, oracle_router_logits
from sparse_moe_layer_warp_b200 import synth
from tests.helpers import host_inputs, make_layer

pytestmark = pytest.mark.gpu

CASES = [
    {"dtype": "bf16", "T": 16, "d": 256, "E": 64, "k": 8, "f": 128},             # decode routing
    {"dtype": "bf16", "T": 40, "d": 256, "E": 16, "k": 4, "f": 128, "routed_scale": 2.0},
    {"dtype": "bf16", "T": 150, "d": 256, "E": 8, "k": 4, "f": 256, "seed": 3},  # 75 per expert
    {"dtype": "bf16", "T": 90, "d": 128, "E": 24, "k": 3, "f": 128, "bias": "zipf",
     "n_shared": 0},                                                               # empty experts
    {"dtype": "bf16", "T": 400, "d": 128, "E": 8, "k": 4, "f": 128, "seed": 5},   # 256-row tiles
    {"dtype": "bf16", "T": 16, "d": 256, "E": 64, "k": 8, "f": 256, "seed": 6},   # 1-CTA 128x256
    {"dtype": "bf16", "T": 75, "d": 512, "E": 12, "k": 2, "f": 256, "seed": 7,    # small groups,
     "routed_scale": 0.5},                                                       # ragged 16-row pads
    {"dtype": "bf16", "T": 200, "d": 256, "E": 16, "k": 4, "f": 256, "seed": 8,   # pair wgrad,
     "bias": "zipf"},                                                               # skewed groups
    {"dtype": "bf16", "T": 256, "d": 256, "E": 8, "k": 4, "f": 256, "seed": 9},   # pair dgrad
    {"dtype": "bf16", "T": 300, "d": 256, "E": 8, "k": 4, "f": 512, "seed": 10,   # pair dgrad,
     "bias": "zipf", "routed_scale": 1.5},                                          # skewed
    {"dtype": "bf16", "T": 1, "d": 256, "E": 16, "k": 4, "f": 128, "seed": 11},   # one token
    {"dtype": "bf16", "T": 17, "d": 128, "E": 8, "k": 2, "f": 128, "seed": 12,    # odd T, no
     "n_shared": 0},                                                               # shared expert
    {"dtype": "f32"},
    {"dtype": "f32", "T": 3, "seed": 13},
    {"dtype": "f32", "T": 100, "seed": 14},                                       # chunked routing
]


def tolerance(dtype):
    """Largest |error| allowed, relative to the largest |reference| entry of a gradient.

    fp32 layer: fp32 sums of products of exactly decoded inputs, far inside 2e-4.
    bf16 layer (tensor cores): the second-stage products take da, db and s*h rounded to bf16
    (unit roundoff u = 2^-8), each product with one rounded operand, so every term of a
    weight-gradient or dx sum carries a relative error of at most u; with independent rounding
    signs the largest error stays below u * max|ref| (a float64 simulation of exactly these
    roundings at the sizes below gives 1.4e-3 .. 2.4e-3).  The bound is 2u = 2^-7; dgate and
    the router terms are computed from fp32 values and sit far inside it."""
    return 2.0 ** -7 if dtype == "bf16" else 2e-4


@pytest.mark.parametrize("kw", CASES)
def test_backward_matches_oracle(cuda_ok, kw):
    w = synth.WORKLOADS["tiny_fp32"].replace(**kw)
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp)
    dout = synth.make_x(w, w.T, device="cuda", seed=77)
    g = layer.backward(inp.x, dout)
    r = layer.route(x=inp.x)
    torch.cuda.synchronize()
    x, wr, _, wg, wu, wd = host_inputs(inp)
    idx = r["idx"].cpu().numpy()
    gates = oracle_gates(oracle_router_logits(x, wr), idx)
    ref = oracle_moe_backward(x, synth.to_numpy_bits(dout), wr, wg, wu, wd, idx, gates,
                              w.routed_scale, w.n_shared)
    counts = r["counts"].cpu().numpy()
    for name, want in ref.items():
        got = g[name].cpu().numpy().astype(np.float64)
        assert got.shape == want.shape, name
        scale = np.abs(want).max()
        err = np.abs(got - want).max()
        assert err <= tolerance(kw["dtype"]) * scale, (name, err, scale)
    # experts no token chose keep their (zero) weight gradients
    unchosen = np.nonzero(counts == 0)[0]
    for name in ("dw_gate", "dw_up", "dw_down"):
        assert (g[name][unchosen] == 0).all()
    assert (g["dw_router"][unchosen] == 0).all()
    # deterministic
    g2 = layer.backward(inp.x, dout)
    torch.cuda.synchronize()
    for name in g:
        assert torch.equal(g[name], g2[name]), name
    # weight gradients accumulate: a second call into the same buffers adds the same amount
    once = {n: g[n].clone() for n in g}
    g3 = layer.backward(inp.x, dout, grads=g)
    torch.cuda.synchronize()
    for name in ("dw_router", "dw_gate", "dw_up", "dw_down"):
        assert torch.equal(g3[name], 2 * once[name]), name
    assert layer.device_status() == 0


def test_backward_of_zero_dout_is_zero(cuda_ok):
    w = synth.WORKLOADS["tiny_fp32"].replace(dtype="bf16", T=20, d=128, E=8, k=2, f=128)
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp)
    g = layer.backward(inp.x, torch.zeros_like(inp.x))
    torch.cuda.synchronize()
    for name, t in g.items():
        assert (t == 0).all(), name


@pytest.mark.parametrize("kw", [
    {"dtype": "bf16", "T": 16, "d": 256, "E": 64, "k": 8, "f": 128},             # decode path
    {"dtype": "bf16", "T": 150, "d": 256, "E": 8, "k": 4, "f": 256, "seed": 3},  # 1-CTA / pair wgrad
    {"dtype": "bf16", "T": 300, "d": 256, "E": 8, "k": 4, "f": 512, "seed": 10,  # CTA pairs
     "bias": "zipf"},
])
def test_training_pair_matches_forward_and_backward(cuda_ok, kw):
    """forward_save returns moe_forward's output; backward from its saved pre-activations
    returns moe_backward's gradients (the kept a, b are the recompute's values)."""
    w = synth.WORKLOADS["tiny_fp32"].replace(**kw)
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp)
    dout = synth.make_x(w, w.T, device="cuda", seed=78)
    out_ref = layer.forward(inp.x).clone()
    g_ref = layer.backward(inp.x, dout)
    out, saved = layer.forward_save(inp.x)
    g = layer.backward(inp.x, dout, saved=saved)
    torch.cuda.synchronize()
    assert torch.equal(out, out_ref)
    for name in g_ref:
        ref = g_ref[name]
        # same arithmetic on the same values: equal up to the MMA accumulation order of a
        # and b in the two token tilings (the forward's rows are not padded)
        err = (g[name] - ref).abs().max().item()
        assert err <= 1e-5 * ref.abs().max().item() + 1e-30, (name, err)
    assert layer.device_status() == 0


@pytest.mark.parametrize("kw", [
    {"dtype": "bf16", "T": 16, "d": 256, "E": 64, "k": 8, "f": 128},             # 1-CTA, unchosen
    {"dtype": "bf16", "T": 40, "d": 256, "E": 16, "k": 4, "f": 256},             # 1-CTA 128 x 256
    {"dtype": "bf16", "T": 300, "d": 256, "E": 8, "k": 4, "f": 512, "seed": 10,  # fused pair tail,
     "bias": "zipf"},                                                              # empty experts
    {"dtype": "bf16", "T": 90, "d": 128, "E": 24, "k": 3, "f": 128, "bias": "zipf",
     "n_shared": 0},
    {"dtype": "f32"},
])
def test_backward_overwrite_sets_gradients(cuda_ok, kw):
    """MOE_BACKWARD_OVERWRITE sets the weight gradients (whatever the buffers held, NaN here)
    to exactly what an accumulating call adds to zeros, zeros for unchosen experts; with the
    kept pre-activations as well."""
    w = synth.WORKLOADS["tiny_fp32"].replace(**kw)
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp)
    dout = synth.make_x(w, w.T, device="cuda", seed=79)
    ref = layer.backward(inp.x, dout)
    torch.cuda.synchronize()
    names = ("dw_router", "dw_gate", "dw_up", "dw_down")
    runs = [None]
    if w.dtype == "bf16":
        runs.append(layer.forward_save(inp.x)[1])
    for saved in runs:
        grads = {n: torch.full_like(ref[n], float("nan")) for n in names}
        g = layer.backward(inp.x, dout, grads=grads, saved=saved, overwrite=True)
        torch.cuda.synchronize()
        for n in names:
            if saved is None:
                assert torch.equal(g[n], ref[n]), n
            else:  # as the saved-activation backward: within the recompute's rounding
                assert not torch.isnan(g[n]).any(), n
                err = (g[n] - ref[n]).abs().max().item()
                assert err <= 1e-5 * ref[n].abs().max().item() + 1e-30, (n, err)
        assert torch.equal(g["dx"], ref["dx"]) or saved is not None
    assert layer.device_status() == 0

"""GPU parity of the layer backward at the benchmark's full sizes, on sampled outputs the
oracle can compute one by one (oracle_moe_backward_sampled): dx rows of a few tokens, the
three weight gradients of a few experts (the shared one, touched routed ones, an untouched
one), router-gradient rows of a few experts.  Same launch configuration as
`bench.py --pass backward` (the workload's own T as max_tokens)."""
import numpy as np
import pytest
import torch

from oracle import oracle_moe_backward_sampled
from sparse_moe_layer_warp_b200 import synth
from tests.helpers import host_inputs, make_layer

pytestmark = pytest.mark.gpu

U_BF16 = 2.0 ** -8   # bf16 unit roundoff; bound 2u * max |ref| (see test_backward_gpu.py)


@pytest.mark.parametrize("name,toks,n_routed,router", [
    ("decode_t16", [0, 9, 15], 2, True),
    ("prefill_t8192", [0, 4097], 1, False),   # router rows would need ~228 whole tokens
    ("skew_t4096", [0, 2047], 2, False),      # Zipf-skewed groups (the two smallest)
    ("dense_ffn_t4096", [0, 4095], 0, False),  # one 4096-row expert: dx rows only
])
def test_backward_full_size_sampled(cuda_ok, name, toks, n_routed, router):
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp)
    dout = synth.make_x(w, w.T, device="cuda", seed=77)
    g = layer.backward(inp.x, dout)
    r = layer.route(x=inp.x)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    idx = r["idx"].cpu().numpy()
    gates = r["gates"].cpu().numpy()
    counts = r["counts"].cpu().numpy()
    touched = np.nonzero(counts)[0]
    # routed experts with the fewest rows (the oracle evaluates every row of a sampled expert)
    routed = [int(e) for e in touched[np.argsort(counts[touched], kind="stable")][:n_routed]]
    untouched = [int(e) for e in np.nonzero(counts == 0)[0][:1]]
    exps = routed + ([w.E] if w.n_shared and w.T <= 64 else []) + untouched
    rexps = routed if router else []
    x, wr, _, wg, wu, wd = host_inputs(inp)
    ref = oracle_moe_backward_sampled(x, synth.to_numpy_bits(dout), wr, wg, wu, wd, idx,
                                      gates, toks, exps, rexps, w.routed_scale, w.n_shared)
    got = {"dx": g["dx"][toks], "dw_gate": g["dw_gate"][exps], "dw_up": g["dw_up"][exps],
           "dw_down": g["dw_down"][exps]}
    if rexps:
        got["dw_router"] = g["dw_router"][rexps]
    for key, t in got.items():
        t = t.cpu().numpy().astype(np.float64)
        want = ref[key]
        blocks = range(len(want))
        for i in blocks:
            if key in ("dw_gate", "dw_up", "dw_down") and exps[i] in untouched:
                assert (t[i] == 0).all(), (key, i)   # experts no token chose are untouched
                continue
            scale = np.abs(want[i]).max()
            err = np.abs(t[i] - want[i]).max()
            assert err <= 2 * U_BF16 * scale, (key, i, err, scale)

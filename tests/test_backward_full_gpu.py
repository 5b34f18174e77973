"""GPU parity of the layer backward at the benchmark's full sizes, on sampled outputs the
oracle can compute one by one (oracle_moe_backward_sampled):

* dx rows of a token set whose selections together touch every touched expert group (a
  greedy cover of the oracle's own routing, plus the last token of the largest groups: their
  last, ragged token tiles); every token also goes through the shared expert;
* the three weight gradients of the routed experts with the fewest rows (all of an expert's
  rows enter its gradient), of an untouched expert (must stay zero), and at decode of the
  shared expert; router-gradient rows at decode.

The backward is defined for the forward's own selection, so the oracle takes the GPU's idx;
the gates of that selection come from the oracle's own router logits.  Same launch
configuration as `bench.py --pass backward` (the workload's own T as max_tokens)."""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

from oracle import oracle_gates, oracle_moe_backward_sampled
from sparse_moe_layer_warp_b200 import synth
from tests.helpers import check_full_routing, greedy_group_cover, host_inputs, make_layer, \
    oracle_routing

pytestmark = pytest.mark.gpu

U_BF16 = 2.0 ** -8   # bf16 unit roundoff; bound 2u * max |ref| (see test_backward_gpu.py)


@pytest.mark.slow
@pytest.mark.parametrize("name,n_routed,router", [
    ("decode_t16", 2, True),
    ("prefill_t8192", 1, False),    # router rows would need ~228 whole tokens
    ("skew_t4096", 2, False),       # Zipf-skewed groups (the two smallest)
    ("dense_ffn_t4096", 0, False),  # one 4096-row expert: dx rows only
])
def test_backward_full_size_sampled(cuda_ok, name, n_routed, router):
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp)
    dout = synth.make_x(w, w.T, device="cuda", seed=77)
    g = layer.backward(inp.x, dout)
    r = layer.route(x=inp.x)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    idx = r["idx"].cpu().numpy()
    counts = r["counts"].cpu().numpy()
    orc = oracle_routing(inp)
    check_full_routing(orc, idx, w.k)
    gates = oracle_gates(orc["logits"], idx)
    toks = greedy_group_cover(orc, w.T, w.k)
    touched = np.nonzero(counts)[0]
    assert set(idx[toks].ravel().tolist()) >= set(np.nonzero(orc["counts"])[0].tolist())
    # routed experts with the fewest rows (the oracle evaluates every row of a sampled expert)
    routed = [int(e) for e in touched[np.argsort(counts[touched], kind="stable")][:n_routed]]
    untouched = [int(e) for e in np.nonzero(counts == 0)[0][:1]]
    exps = routed + ([w.E] if w.n_shared and w.T <= 64 else []) + untouched
    rexps = routed if router else []
    x, wr, _, wg, wu, wd = host_inputs(inp)
    o = synth.to_numpy_bits(dout)
    none = np.zeros(0, np.int32)

    def one(t):  # the oracle releases the GIL: tokens run in parallel threads
        return oracle_moe_backward_sampled(x, o, wr, wg, wu, wd, idx, gates, [t], none, none,
                                           w.routed_scale, w.n_shared)["dx"][0]

    with ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as pool:
        dx_ref = np.stack(list(pool.map(one, [int(t) for t in toks])))
    ref = oracle_moe_backward_sampled(x, o, wr, wg, wu, wd, idx, gates, none, exps, rexps,
                                      w.routed_scale, w.n_shared)
    ref["dx"] = dx_ref
    got = {"dx": g["dx"][toks], "dw_gate": g["dw_gate"][exps], "dw_up": g["dw_up"][exps],
           "dw_down": g["dw_down"][exps]}
    if rexps:
        got["dw_router"] = g["dw_router"][rexps]
    for key, t in got.items():
        t = t.cpu().numpy().astype(np.float64)
        want = ref[key]
        for i in range(len(want)):
            if key in ("dw_gate", "dw_up", "dw_down") and exps[i] in untouched:
                assert (t[i] == 0).all(), (key, i)   # experts no token chose are untouched
                continue
            scale = np.abs(want[i]).max()
            err = np.abs(t[i] - want[i]).max()
            assert err <= 2 * U_BF16 * scale, (key, i, err, scale)
    print(name, "dx rows checked:", len(toks), "groups covered:", len(touched))

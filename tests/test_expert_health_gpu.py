"""GPU parity for the expert health signals (per-expert activation RMS, parameter Frobenius
norms, their cross-expert ratios) against the CPU oracle."""
import numpy as np
import pytest
import torch

from oracle import oracle_expert_act_rms, oracle_expert_param_norms, oracle_health_ratios
from sparse_moe_layer_warp_b200 import synth
from tests.helpers import host_inputs, make_layer

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kw,act_rtol", [
    # bf16: h is rounded to bf16 before its squares are summed
    ({"dtype": "bf16", "T": 16, "d": 256, "E": 64, "k": 8, "f": 128}, 4e-3),
    ({"dtype": "bf16", "T": 300, "d": 512, "E": 32, "k": 8, "f": 256}, 4e-3),
    ({"dtype": "bf16", "T": 700, "d": 768, "E": 8, "k": 4, "f": 512}, 4e-3),    # CTA pairs
    ({"dtype": "bf16", "T": 200, "d": 256, "E": 48, "k": 4, "f": 128, "bias": "zipf",
      "n_shared": 0}, 4e-3),                                                      # empty experts
    ({"dtype": "f32"}, 1e-5),
])
def test_expert_health_matches_oracle(cuda_ok, kw, act_rtol):
    w = synth.WORKLOADS["tiny_fp32"].replace(**kw)
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp)
    layer.forward(inp.x)
    act, par, ratios = layer.expert_health(w.T)
    r = layer.route(x=inp.x)
    torch.cuda.synchronize()
    idx = r["idx"].cpu().numpy()
    x, _, _, wg, wu, wd = host_inputs(inp)
    act0 = oracle_expert_act_rms(x, wg, wu, idx, w.E, w.n_shared)
    par0 = oracle_expert_param_norms(wg, wu, wd)
    a = act.cpu().numpy().astype(np.float64)
    p = par.cpu().numpy().astype(np.float64)
    counts = r["counts"].cpu().numpy()
    assert (a[:w.E][counts == 0] == 0).all()
    np.testing.assert_allclose(a, act0, rtol=act_rtol, atol=0)
    np.testing.assert_allclose(p, par0, rtol=1e-6, atol=0)  # fp64 sums, one fp32 rounding
    ra0, rp0 = oracle_health_ratios(a, p, idx, w.E)  # the same definition on the GPU values
    got = ratios.cpu().numpy()
    assert abs(got[0] - ra0) <= 1e-6 * max(ra0, 1e-30)
    assert abs(got[1] - rp0) <= 1e-6 * max(rp0, 1e-30)
    ra1, rp1 = oracle_health_ratios(act0, par0, idx, w.E)  # and on the oracle's values
    assert abs(got[0] - ra1) <= 2 * act_rtol * ra1
    assert abs(got[1] - rp1) <= 1e-5 * rp1
    # deterministic
    act2, par2, ratios2 = layer.expert_health(w.T)
    torch.cuda.synchronize()
    assert torch.equal(act, act2) and torch.equal(par, par2) and torch.equal(ratios, ratios2)

"""GPU parity for the router's balancing by-products (EP-group balance loss, routing
confidence, selection frequency, mean routing probability) and the bias step, against the
CPU oracle on the same logits and selections."""
import numpy as np
import pytest
import torch

from oracle import oracle_bias_update, oracle_route, oracle_router_stats
from sparse_moe_layer_warp_b200 import moe_update_router_bias, synth
from tests.helpers import make_layer

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,E,k,G", [(100, 40, 5, 8), (16, 288, 8, 8), (8192, 288, 8, 8),
                                     (67, 1000, 32, 10), (1, 16, 2, 1), (4096, 288, 8, 36)])
def test_router_stats_match_oracle(cuda_ok, T, E, k, G):
    w = synth.Workload("stats", T=T, d=128, E=E, k=k, f=128)
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp)
    logits = synth.make_logits(T, E, seed=T + 3 * E, device="cuda")
    r = layer.route(logits=logits)
    pm, fs, sc = layer.router_stats(logits, r["idx"], G)
    torch.cuda.synchronize()
    lg = logits.cpu().numpy()
    idx = r["idx"].cpu().numpy()
    ref_idx, _ = oracle_route(lg, inp.bias.cpu().numpy(), k)
    assert (idx == ref_idx).all()
    pm0, fs0, lep0, conf0 = oracle_router_stats(lg, idx, G)
    # fp32 softmax per token and fp32 sums over <= 8192 tokens: relative error ~1e-6..1e-5
    np.testing.assert_allclose(pm.cpu().numpy(), pm0, rtol=2e-5, atol=1e-9)
    np.testing.assert_array_equal(fs.cpu().numpy(), fs0)  # integer counts, exact
    lep, conf = sc.cpu().numpy().tolist()
    assert abs(lep - lep0) <= 2e-5 * abs(lep0)
    assert abs(conf - conf0) <= 2e-5 * abs(conf0)


def test_router_stats_balanced_closed_form(cuda_ok):
    # equal logits and a perfectly balanced selection: L_EP = 1 for every grouping
    T, E, k = 64, 32, 4
    w = synth.Workload("stats", T=T, d=128, E=E, k=k, f=128)
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp)
    logits = torch.zeros((T, E), device="cuda")
    idx = torch.tensor([[(4 * t + j) % E for j in range(k)] for t in range(T)],
                       dtype=torch.int32, device="cuda")
    for G in (1, 2, 4, 8, 16, 32):
        pm, fs, sc = layer.router_stats(logits, idx, G)
        torch.cuda.synchronize()
        assert abs(float(sc[0]) - 1.0) < 1e-5
        assert abs(float(sc[1]) - k / E) < 1e-6
        assert torch.allclose(pm, torch.full_like(pm, 1.0 / E))


def test_bias_update_matches_oracle(cuda_ok):
    T, E, k = 300, 48, 6
    w = synth.Workload("stats", T=T, d=128, E=E, k=k, f=128, bias="zipf")
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp)
    r = layer.route(logits=synth.make_logits(T, E, seed=11, device="cuda"))
    bias = inp.bias.clone()
    before = bias.cpu().numpy()
    moe_update_router_bias(layer.handle, r["counts"], T, 0.01, bias)
    torch.cuda.synchronize()
    ref = oracle_bias_update(r["counts"].cpu().numpy(), T * k, 0.01, before)
    np.testing.assert_array_equal(bias.cpu().numpy(), ref)

"""Pins for the CPU oracle (no GPU): closed forms, special cases that reduce to library
routines, brute force on tiny inputs, invariants, and the independent NumPy restatement.

Each pin is chosen so a plausible slip in the oracle fails it:
  * dropped/transposed term in the expert FFN  -> textbook SwiGLU via torch (E = k = 1)
  * wrong silu, wrong gate normalisation, sign -> silu antisymmetry closed form (golden)
  * bias leaking into the gates                 -> topk_ties golden case 4 and 6
  * wrong tie / NaN rule, wrong slot order      -> topk_ties golden + torch.topk
  * permutation index slip                      -> numpy stable argsort + invariants
  * routed/shared mix-up, missing routed scale  -> identical-experts invariance, zero W_down
"""
import json
import math
import os

import numpy as np
import pytest
import torch
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle import (oracle_expert_ffn, oracle_moe_forward, oracle_permute, oracle_route,
                    oracle_router_logits)
from oracle import moe_numpy as onp
from sparse_moe_layer_warp_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f(v):
    return {"nan": math.nan, "-inf": -math.inf, "inf": math.inf}.get(v, v) if isinstance(v, str) else v


def _small_inputs(name="tiny_fp32", **kw):
    w = synth.WORKLOADS[name].replace(**kw)
    inp = synth.make_inputs(w)
    cv = synth.to_numpy_bits
    return w, [cv(t) for t in (inp.x, inp.w_router, inp.bias, inp.w_gate, inp.w_up, inp.w_down)]


# ----------------------------------------------------------------------------- golden
def test_golden_silu_antisymmetry_closed_form():
    g = json.load(open(os.path.join(GOLDEN, "silu_antisymmetry.json")))
    arr = lambda k: np.array(g[k], np.float32)  # noqa: E731
    for case in g["cases"]:
        out, idx, gates, _ = oracle_moe_forward(arr("x"), arr("w_router"), arr("bias"),
                                                arr("w_gate"), arr("w_up"), arr("w_down"),
                                                k=g["k"], n_shared=1,
                                                routed_scale=case["routed_scale"])
        np.testing.assert_allclose(out, np.array(case["out"]), rtol=0, atol=1e-12)
        assert (idx == np.array(case["idx"])[None, :]).all()
        np.testing.assert_array_equal(gates, np.broadcast_to(np.float32(case["gates"]), gates.shape))


def test_golden_topk_ties_nan_signed_zero():
    g = json.load(open(os.path.join(GOLDEN, "topk_ties.json")))
    for case in g["cases"]:
        logits = np.array([[_f(v) for v in case["logits"]]], np.float32)
        bias = np.array(case["bias"], np.float32)
        idx, gates = oracle_route(logits, bias, case["k"])
        assert idx[0].tolist() == case["idx"], case
        np.testing.assert_allclose(gates[0], case["gates"], rtol=2e-7, atol=1e-30)
        idx2, gates2, _ = onp.np_select(logits, bias, case["k"])
        assert idx2[0].tolist() == case["idx"], case


# ------------------------------------------------------------------- library reductions
def test_topk_matches_torch_topk_without_ties():
    logits = synth.make_logits(300, 288, seed=3).numpy()
    bias = synth.make_bias(synth.WORKLOADS["decode_t16"], torch.Generator().manual_seed(1), "cpu").numpy()
    s = torch.from_numpy(logits) + torch.from_numpy(bias)
    ref = torch.topk(s, 8, dim=1, largest=True, sorted=True).indices.numpy()
    idx, gates = oracle_route(logits, bias, 8)
    assert (idx == ref).all()
    # gates: softmax of the UNBIASED logits of the selection (torch.softmax as the library routine)
    sel = np.take_along_axis(logits, idx.astype(np.int64), axis=1)
    ref_g = torch.softmax(torch.from_numpy(sel).double(), dim=1).numpy()
    np.testing.assert_allclose(gates, ref_g, rtol=1e-6, atol=0)


def test_gates_of_a_given_selection():
    """oracle_gates (gates of a selection made elsewhere) against torch.softmax over the
    selected unbiased logits, in any slot order, with repeated ids allowed by the softmax
    definition; and exactly oracle_route's gates on oracle_route's own selection."""
    from oracle import oracle_gates

    logits = synth.make_logits(120, 288, seed=11).numpy()
    bias = synth.make_bias(synth.WORKLOADS["skew_t4096"], torch.Generator().manual_seed(2),
                           "cpu").numpy()
    idx, gates = oracle_route(logits, bias, 8)
    assert np.array_equal(oracle_gates(logits, idx), gates)
    rng = np.random.default_rng(4)
    sel = np.stack([rng.choice(288, 8, replace=False) for _ in range(120)]).astype(np.int32)
    got = oracle_gates(logits, sel)
    lg = np.take_along_axis(logits, sel.astype(np.int64), axis=1)
    ref = torch.softmax(torch.from_numpy(lg).double(), dim=1).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-6, atol=0)
    # permuting the slots permutes the gates
    rev = np.ascontiguousarray(sel[:, ::-1])
    assert np.array_equal(oracle_gates(logits, rev), got[:, ::-1])
    # the bias does not enter: two selections with equal logits get equal gates
    two = np.zeros((1, 4), np.float32)
    assert (oracle_gates(two, np.array([[0, 3]], np.int32)) == 0.5).all()


def test_gates_k_equals_E_zero_bias_is_full_softmax():
    logits = synth.make_logits(40, 16, seed=5).numpy()
    idx, gates = oracle_route(logits, np.zeros(16, np.float32), 16)
    full = torch.softmax(torch.from_numpy(logits).double(), dim=1).numpy()
    got = np.zeros_like(full)
    np.put_along_axis(got, idx.astype(np.int64), gates.astype(np.float64), axis=1)
    np.testing.assert_allclose(got, full, rtol=1e-6, atol=1e-12)


def test_gates_k1_is_one_and_sum_to_one():
    logits = synth.make_logits(50, 24, seed=6).numpy()
    _, g1 = oracle_route(logits, None, 1)
    assert (g1 == 1.0).all()
    idx, g = oracle_route(logits, None, 5)
    assert np.abs(g.astype(np.float64).sum(1) - 1).max() < 1e-6
    assert (g > 0).all()
    for row in idx:
        assert len(set(row.tolist())) == 5


def test_router_logits_match_library_matmul():
    w, (x, wr, *_rest) = _small_inputs()
    got = oracle_router_logits(x, wr)
    ref = (x.astype(np.float64) @ wr.astype(np.float64).T).astype(np.float32)
    # double accumulation in either order rounds to the same fp32 except at most 1 ulp
    assert np.max(np.abs(got.view(np.int32).astype(np.int64) - ref.view(np.int32))) <= 1


def test_expert_ffn_E1_k1_is_textbook_swiglu():
    """E = k = 1: gate = 1 and the layer is FFN_0(x) + FFN_shared(x) (textbook SwiGLU)."""
    w, (x, wr, b, wg, wu, wd) = _small_inputs(E=1, k=1)
    wr = wr[:1]
    b = b[:1]
    out, idx, gates, _ = oracle_moe_forward(x, wr, b, wg[:2], wu[:2], wd[:2], k=1)
    assert (idx == 0).all() and (gates == 1.0).all()
    X = torch.from_numpy(x).double()
    ref = torch.zeros_like(X)
    for e in range(2):
        Wg, Wu, Wd = (torch.from_numpy(a[e]).double() for a in (wg, wu, wd))
        ref += (torch.nn.functional.silu(X @ Wg.T) * (X @ Wu.T)) @ Wd.T
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)
    y = oracle_expert_ffn(x[3], wg[0], wu[0], wd[0])
    Wg, Wu, Wd = (torch.from_numpy(a[0]).double() for a in (wg, wu, wd))
    y_ref = (torch.nn.functional.silu(X[3] @ Wg.T) * (X[3] @ Wu.T)) @ Wd.T
    np.testing.assert_allclose(y, y_ref.numpy(), rtol=1e-12, atol=1e-12)


def test_identical_experts_make_routing_irrelevant():
    """All routed experts equal => sum_j g_j y = y (gates sum to 1): closed form."""
    w, (x, wr, b, wg, wu, wd) = _small_inputs()
    E = w.E
    for a in (wg, wu, wd):
        a[:E] = a[0]
    scale = 1.75
    out, *_ = oracle_moe_forward(x, wr, b, wg, wu, wd, k=w.k, routed_scale=scale)
    X = torch.from_numpy(x).double()

    def ffn(e):
        Wg, Wu, Wd = (torch.from_numpy(a[e]).double() for a in (wg, wu, wd))
        return (torch.nn.functional.silu(X @ Wg.T) * (X @ Wu.T)) @ Wd.T

    ref = (scale * ffn(0) + ffn(E)).numpy()
    # the gates are fp32 outputs, so they sum to 1 only within k * 2^-24
    np.testing.assert_allclose(out, ref, rtol=0, atol=w.k * 2.0**-23 * scale * np.abs(ref).max())


def test_zero_routed_down_gives_shared_only():
    w, (x, wr, b, wg, wu, wd) = _small_inputs()
    wd = wd.copy()
    wd[: w.E] = 0
    out, *_ = oracle_moe_forward(x, wr, b, wg, wu, wd, k=w.k)
    X = torch.from_numpy(x).double()
    Wg, Wu, Wd = (torch.from_numpy(a[w.E]).double() for a in (wg, wu, wd))
    ref = (torch.nn.functional.silu(X @ Wg.T) * (X @ Wu.T)) @ Wd.T
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------------- permutation
@pytest.mark.parametrize("T,E,k,seed", [(64, 16, 2, 0), (37, 288, 8, 1), (1, 5, 5, 2), (300, 7, 3, 3)])
def test_permute_is_stable_argsort_and_invariants(T, E, k, seed):
    logits = synth.make_logits(T, E, seed=seed, ties=(seed % 2 == 1)).numpy()
    idx, _ = oracle_route(logits, None, k)
    counts, offsets, perm, slot_row = oracle_permute(idx, E)
    flat = idx.reshape(-1)
    assert (perm == np.argsort(flat, kind="stable")).all()
    assert counts.sum() == T * k and offsets[0] == 0 and offsets[-1] == T * k
    assert (np.diff(offsets) == counts).all()
    assert sorted(perm.tolist()) == list(range(T * k))
    assert (perm[slot_row.reshape(-1)] == np.arange(T * k)).all()
    for e in range(E):
        toks = perm[offsets[e]:offsets[e + 1]] // k
        assert (np.diff(toks) > 0).all()
        assert (flat[perm[offsets[e]:offsets[e + 1]]] == e).all()


def test_route_k_distinct_and_brute_force_rank():
    """Brute force: e is selected iff fewer than k experts rank before it."""
    logits = synth.make_logits(30, 12, seed=9, ties=True).numpy()
    bias = np.linspace(-0.2, 0.2, 12).astype(np.float32)
    idx, _ = oracle_route(logits, bias, 4)
    s = logits + bias
    for t in range(30):
        sel = set()
        for e in range(12):
            before = sum(1 for o in range(12) if s[t, o] > s[t, e] or (s[t, o] == s[t, e] and o < e))
            if before < 4:
                sel.add(e)
        assert sel == set(idx[t].tolist())
        assert len(set(idx[t].tolist())) == 4


# ----------------------------------------------------------------- NumPy restatement
@pytest.mark.parametrize("name,kw", [("tiny_fp32", {}),
                                     ("tiny_fp32", {"dtype": "bf16", "E": 9, "k": 3, "T": 21}),
                                     ("tiny_fp32", {"bias": "zipf", "seed": 4})])
def test_c_oracle_matches_numpy_brute_force(name, kw):
    w, (x, wr, b, wg, wu, wd) = _small_inputs(name, **kw)
    out, idx, gates, logits = oracle_moe_forward(x, wr, b, wg, wu, wd, k=w.k, routed_scale=1.0)
    out2, idx2, gates2, logits2 = onp.np_moe_forward(x, wr, b, wg, wu, wd, k=w.k, logits=logits)
    assert (idx == idx2).all()
    np.testing.assert_allclose(gates, gates2, rtol=2e-7, atol=0)
    np.testing.assert_allclose(out, out2, rtol=1e-9, atol=1e-9 * np.abs(out2).max())
    # the oracle's own logits agree with the NumPy matmul to 1 ulp
    assert np.max(np.abs(logits.view(np.int32).astype(np.int64) -
                         onp.np_logits(x, wr).view(np.int32))) <= 1
    c, o, p, s = oracle_permute(idx, w.E)
    c2, o2, p2, s2 = onp.np_permute(idx, w.E)
    assert (c == c2).all() and (o == o2).all() and (p == p2).all() and (s == s2).all()


def test_sampled_tokens_equal_full_run():
    w, (x, wr, b, wg, wu, wd) = _small_inputs()
    full, idx, gates, _ = oracle_moe_forward(x, wr, b, wg, wu, wd, k=w.k)
    toks = np.array([5, 0, 63, 17], np.int32)
    part, idx2, gates2, _ = oracle_moe_forward(x, wr, b, wg, wu, wd, k=w.k, tokens=toks)
    np.testing.assert_array_equal(part, full[toks])
    np.testing.assert_array_equal(idx2, idx[toks])


# ------------------------------------------------------------------- router statistics
from oracle import oracle_bias_update, oracle_router_stats  # noqa: E402


def test_router_stats_closed_forms():
    T, E, k = 48, 12, 3
    # equal logits -> p = 1/E; a balanced selection (each expert chosen T*k/E times) -> L_EP = 1
    logits = np.zeros((T, E), np.float32)
    idx = np.array([[(3 * t + j) % E for j in range(k)] for t in range(T)], np.int32)
    for G in (1, 2, 3, 4, 6, 12):
        pm, fs, lep, conf = oracle_router_stats(logits, idx, G)
        np.testing.assert_allclose(pm, 1.0 / E, rtol=1e-6)
        np.testing.assert_allclose(fs, 1.0 / E, rtol=1e-6)
        assert abs(lep - 1.0) < 1e-6
        assert abs(conf - k / E) < 1e-6
    # all mass and all selections inside group 0 of G groups -> L_EP = G
    G = 4
    logits2 = np.full((T, E), -60.0, np.float32)
    logits2[:, :3] = 5.0
    idx2 = np.tile(np.arange(3, dtype=np.int32), (T, 1))
    _, _, lep2, conf2 = oracle_router_stats(logits2, idx2, G)
    assert abs(lep2 - G) < 1e-5
    assert abs(conf2 - 1.0) < 1e-5
    # G = 1: L_EP = (sum f)(sum p) = 1 for any routing
    lg = synth.make_logits(T, E, seed=4).numpy()
    ix, _ = oracle_route(lg, None, k)
    assert abs(oracle_router_stats(lg, ix, 1)[2] - 1.0) < 1e-6
    # k = E: every expert is active, confidence = 1
    ixe, _ = oracle_route(lg, None, E)
    assert abs(oracle_router_stats(lg, ixe, 3)[3] - 1.0) < 1e-6


def test_router_stats_match_library_softmax_and_bincount():
    lg = synth.make_logits(70, 40, seed=8).numpy()
    ix, _ = oracle_route(lg, np.linspace(-0.3, 0.3, 40).astype(np.float32), 5)
    pm, fs, lep, conf = oracle_router_stats(lg, ix, 8)
    P = torch.softmax(torch.from_numpy(lg).double(), dim=1).numpy()
    np.testing.assert_allclose(pm, P.mean(0), rtol=1e-6)
    np.testing.assert_allclose(fs, np.bincount(ix.reshape(-1), minlength=40) / (70 * 5), rtol=1e-6)
    pg = P.mean(0).reshape(8, 5).sum(1)
    fg = (np.bincount(ix.reshape(-1), minlength=40) / (70 * 5)).reshape(8, 5).sum(1)
    assert abs(lep - 8 * float((pg * fg).sum())) < 1e-6
    assert abs(conf - float(np.take_along_axis(P, ix.astype(np.int64), 1).sum(1).mean())) < 1e-6


def test_bias_update_sign_rule():
    counts = np.array([10, 2, 6, 6], np.int32)  # T*k = 24, mean 6
    b = oracle_bias_update(counts, 24, 0.5, np.zeros(4, np.float32))
    assert b.tolist() == [-0.5, 0.5, 0.0, 0.0]
    b2 = oracle_bias_update(counts, 24, 0.25, b)
    assert b2.tolist() == [-0.75, 0.75, 0.0, 0.0]


# ------------------------------------------------------------------ expert health signals
from oracle import (oracle_expert_act_rms, oracle_expert_param_norms,  # noqa: E402
                    oracle_health_ratios)


def _expert_inputs(T=7, d=12, f=6, E=4, k=2, seed=3):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, d)).astype(np.float32)
    wg = rng.standard_normal((E + 1, f, d)).astype(np.float32) / math.sqrt(d)
    wu = rng.standard_normal((E + 1, f, d)).astype(np.float32) / math.sqrt(d)
    wd = rng.standard_normal((E + 1, d, f)).astype(np.float32) / math.sqrt(f)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    return x, wg, wu, wd, idx


def test_act_rms_matches_library_swiglu():
    # torch matmul + silu on the tokens each expert was chosen by (the shared expert: all)
    x, wg, wu, wd, idx = _expert_inputs()
    E = wg.shape[0] - 1
    got = oracle_expert_act_rms(x, wg, wu, idx, E, 1)
    X = torch.from_numpy(x).double()
    for g in range(E + 1):
        rows = np.arange(len(x)) if g == E else np.nonzero((idx == g).any(1))[0]
        if len(rows) == 0:
            assert got[g] == 0.0
            continue
        h = torch.nn.functional.silu(X[rows] @ torch.from_numpy(wg[g]).double().T) * \
            (X[rows] @ torch.from_numpy(wu[g]).double().T)
        assert abs(got[g] - float(h.pow(2).mean().sqrt())) <= 1e-12 * float(h.abs().max())


def test_act_rms_closed_form_constant_weights_and_down_invariance():
    # x = 1, W_g = W_u = c: every h = silu(c d) * c d; W_down plays no part
    T, d, f, E, k, c = 5, 8, 4, 3, 1, 0.3
    x = np.ones((T, d), np.float32)
    wg = np.full((E + 1, f, d), c, np.float32)
    wu = np.full((E + 1, f, d), c, np.float32)
    idx = np.array([[0], [0], [2], [0], [2]], np.int32)  # expert 1 never chosen
    got = oracle_expert_act_rms(x, wg, wu, idx, E, 1)
    z = float(np.float32(c)) * d
    want = abs(z / (1 + math.exp(-z)) * z)
    assert got[1] == 0.0
    for g in (0, 2, 3):
        assert abs(got[g] - want) <= 1e-12 * want


def test_param_norms_closed_form_and_library_norm():
    d, f, G, c = 8, 4, 3, 0.5
    wg = np.full((G, f, d), c, np.float32)
    wu = np.full((G, f, d), -c, np.float32)
    wd = np.full((G, d, f), 2 * c, np.float32)
    got = oracle_expert_param_norms(wg, wu, wd)
    want = math.sqrt(d * f * (c * c + c * c + 4 * c * c))  # all three matrices
    assert np.allclose(got, want, rtol=1e-14, atol=0)
    x, wg, wu, wd, idx = _expert_inputs()
    got = oracle_expert_param_norms(wg, wu, wd)
    for g in range(wg.shape[0]):
        ref = torch.linalg.vector_norm(torch.cat([torch.from_numpy(a[g]).double().ravel()
                                                  for a in (wg, wu, wd)]))
        assert abs(got[g] - float(ref)) <= 1e-12 * float(ref)


def test_health_ratios_identical_experts_and_library_median():
    x, wg, wu, wd, idx = _expert_inputs(E=4)
    same_g = np.repeat(wg[:1], 5, 0)
    same_u = np.repeat(wu[:1], 5, 0)
    same_d = np.repeat(wd[:1], 5, 0)
    act = oracle_expert_act_rms(x, same_g, same_u, idx, 4, 1)
    pn = oracle_expert_param_norms(same_g, same_u, same_d)
    ra, rp = oracle_health_ratios(act, pn, idx, 4)
    # every chosen expert sees different tokens, so only the parameter ratio is exactly 1
    assert rp == 1.0
    act = np.array([1.0, 4.0, 2.0, 0.0, 9.0])
    pn = np.array([3.0, 1.0, 5.0, 2.0, 7.0])
    ra, rp = oracle_health_ratios(act, pn, np.array([[0, 1], [2, 1]]), 4)
    assert ra == 2.0 / 4.0  # chosen experts 0, 1, 2: median 2, max 4 (expert 3 not chosen)
    assert rp == 1.0 / 2.5  # routed experts 0..3: min 1, median (2 + 3) / 2


# ------------------------------------------------------------------ backward
from oracle import oracle_moe_backward  # noqa: E402


def _torch_layer_grads(x, dout, wr, wg, wu, wd, idx, rs, n_shared):
    """The layer in float64 torch autograd for a fixed selection: gates = softmax of the
    selected router logits; returns the gradients of <out, dout>."""
    X = torch.tensor(x, dtype=torch.float64, requires_grad=True)
    WR = torch.tensor(wr, dtype=torch.float64, requires_grad=True)
    WG = torch.tensor(wg, dtype=torch.float64, requires_grad=True)
    WU = torch.tensor(wu, dtype=torch.float64, requires_grad=True)
    WD = torch.tensor(wd, dtype=torch.float64, requires_grad=True)
    E = wr.shape[0]
    rows = []
    for t in range(x.shape[0]):
        sel = torch.tensor(idx[t], dtype=torch.long)
        g = torch.softmax((X[t] @ WR.T)[sel], dim=0)
        o = torch.zeros(x.shape[1], dtype=torch.float64)
        for j, e in enumerate(idx[t]):
            h = torch.nn.functional.silu(WG[e] @ X[t]) * (WU[e] @ X[t])
            o = o + rs * g[j] * (WD[e] @ h)
        if n_shared:
            h = torch.nn.functional.silu(WG[E] @ X[t]) * (WU[E] @ X[t])
            o = o + WD[E] @ h
        rows.append(o)
    out = torch.stack(rows)
    (out * torch.tensor(dout, dtype=torch.float64)).sum().backward()
    gates = np.stack([torch.softmax(torch.tensor(x[t] @ wr.T.astype(np.float64))[idx[t]], 0)
                      .numpy() for t in range(x.shape[0])]).astype(np.float32)
    return dict(dx=X.grad.numpy(), dw_router=WR.grad.numpy(), dw_gate=WG.grad.numpy(),
                dw_up=WU.grad.numpy(), dw_down=WD.grad.numpy()), gates


@pytest.mark.parametrize("n_shared,rs", [(1, 1.0), (0, 2.5)])
def test_backward_matches_torch_autograd(n_shared, rs):
    rng = np.random.default_rng(11)
    T, d, f, E, k = 5, 12, 6, 5, 2
    x = rng.standard_normal((T, d)).astype(np.float32)
    dout = rng.standard_normal((T, d)).astype(np.float32)
    wr = (rng.standard_normal((E, d)) / math.sqrt(d)).astype(np.float32)
    wg = (rng.standard_normal((E + n_shared, f, d)) / math.sqrt(d)).astype(np.float32)
    wu = (rng.standard_normal((E + n_shared, f, d)) / math.sqrt(d)).astype(np.float32)
    wd = (rng.standard_normal((E + n_shared, d, f)) / math.sqrt(f)).astype(np.float32)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    want, gates = _torch_layer_grads(x, dout, wr, wg, wu, wd, idx, rs, n_shared)
    got = oracle_moe_backward(x, dout, wr, wg, wu, wd, idx, gates, rs, n_shared)
    for name in want:
        scale = np.abs(want[name]).max()
        # the oracle takes the gates as fp32 (as the GPU does): relative error ~1e-7
        assert np.abs(got[name] - want[name]).max() <= 2e-6 * scale, name


def test_backward_matches_finite_differences():
    # central differences of <forward(x), dout> through oracle_moe_forward itself (its own
    # routing; the perturbation is far too small to change the selection)
    w = synth.WORKLOADS["tiny_fp32"].replace(T=3, d=16, E=6, k=2, f=8, seed=4)
    inp = synth.make_inputs(w)
    x, wr, b, wg, wu, wd = [t.numpy() for t in (inp.x, inp.w_router, inp.bias, inp.w_gate,
                                                 inp.w_up, inp.w_down)]
    rng = np.random.default_rng(2)
    dout = rng.standard_normal(x.shape).astype(np.float32)
    _, idx, gates, _ = oracle_moe_forward(x, wr, b, wg, wu, wd, w.k)
    got = oracle_moe_backward(x, dout, wr, wg, wu, wd, idx, gates)
    eps = 1e-3

    def loss(**over):
        a = dict(x=x, wr=wr, wg=wg, wu=wu, wd=wd)
        a.update(over)
        out, idx2, _, _ = oracle_moe_forward(a["x"], a["wr"], b, a["wg"], a["wu"], a["wd"],
                                             w.k)
        assert (idx2 == idx).all()
        return float((out * dout).sum())

    for (name, arr, key, pos) in (("dx", x, "x", (1, 3)), ("dw_router", wr, "wr", (2, 5)),
                                  ("dw_gate", wg, "wg", (6, 1, 2)),
                                  ("dw_up", wu, "wu", (idx[0, 0], 3, 7)),
                                  ("dw_down", wd, "wd", (idx[1, 1], 4, 5))):
        p, m = arr.copy(), arr.copy()
        p[pos] += eps
        m[pos] -= eps
        fd = (loss(**{key: p}) - loss(**{key: m})) / (2 * eps)
        assert abs(got[name][pos] - fd) <= 2e-3 * max(1.0, abs(fd)), (name, got[name][pos], fd)


# ------------------------------------------------------------ sampled backward
from oracle import oracle_moe_backward_sampled  # noqa: E402


@pytest.mark.parametrize("n_shared,rs,dtype", [(1, 1.0, "f32"), (0, 1.5, "f32"), (1, 1.0, "bf16")])
def test_sampled_backward_equals_full_backward(n_shared, rs, dtype):
    """The sampled entry point returns exactly the selected rows / experts of the full
    (autograd- and finite-difference-pinned) oracle backward."""
    w = synth.WORKLOADS["tiny_fp32"].replace(T=9, d=16, E=6, k=2, f=8, seed=12, dtype=dtype,
                                             n_shared=n_shared)
    inp = synth.make_inputs(w)
    x, wr, b, wg, wu, wd = [synth.to_numpy_bits(t) for t in (inp.x, inp.w_router, inp.bias,
                                                             inp.w_gate, inp.w_up, inp.w_down)]
    dout = synth.to_numpy_bits(synth.make_x(w, w.T, seed=21))
    _, idx, gates, _ = oracle_moe_forward(x, wr, b, wg, wu, wd, w.k, n_shared=n_shared,
                                          routed_scale=rs)
    full = oracle_moe_backward(x, dout, wr, wg, wu, wd, idx, gates, rs, n_shared)
    toks = [0, 4, 8]
    exps = sorted({int(idx[1, 0]), int(idx[5, 1])} | ({w.E} if n_shared else set()))
    unchosen = [e for e in range(w.E) if e not in set(idx.ravel().tolist())]
    exps = exps + unchosen[:1]
    rexps = sorted({int(idx[2, 1]), int(idx[7, 0])})
    got = oracle_moe_backward_sampled(x, dout, wr, wg, wu, wd, idx, gates, toks, exps, rexps,
                                      rs, n_shared)
    assert np.array_equal(got["dx"], full["dx"][toks])
    for name in ("dw_gate", "dw_up", "dw_down"):
        assert np.array_equal(got[name], full[name][exps]), name
    assert np.array_equal(got["dw_router"], full["dw_router"][rexps])


# ------------------------------------------------------------ selection order, fuzzed
_GRID = [float("nan"), float("inf"), float("-inf"), 0.0, -0.0, 0.5, -0.5, 1.0, 0.25, -2.0]


@settings(max_examples=300, deadline=None)
@given(st.data())
def test_route_slot_order_equals_a_full_sort(data):
    """Slot j holds the expert of rank j in one full sort of the biased scores: larger score
    first, equal scores (-0.0 == +0.0) by lower id, NaN scores after every number (by id)."""
    T = data.draw(st.integers(1, 5))
    E = data.draw(st.integers(1, 20))
    k = data.draw(st.integers(1, E))
    vals = st.sampled_from(_GRID)
    logits = np.array(data.draw(st.lists(vals, min_size=T * E, max_size=T * E)),
                      dtype=np.float32).reshape(T, E)
    bias = np.array(data.draw(st.lists(st.sampled_from([0.0, -0.0, 0.5, -0.25]),
                                       min_size=E, max_size=E)), dtype=np.float32)
    idx, _ = oracle_route(logits, bias, k)
    s = logits + bias  # float32 add, as the selection rule states
    for t in range(T):
        def key(e):
            v = float(s[t, e])
            return (1, 0.0, e) if v != v else (0, -v, e)
        want = sorted(range(E), key=key)[:k]
        assert idx[t].tolist() == want, (logits[t], bias, k)

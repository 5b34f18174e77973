"""Shared test helpers: run the CUDA layer and the CPU oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

from oracle import oracle_moe_forward, oracle_permute, oracle_route
from sparse_moe_layer_warp_b200 import MoELayer, synth

BF16_TOL = 2e-2   # max |err| <= 2e-2 * RMS(out) for bf16 weights/activations, fp32 accumulation
F32_TOL = 1e-5    # max |err| <= 1e-5 * RMS(out) for the fp32 workload


def make_layer(inp: synth.LayerInputs, max_tokens=None) -> MoELayer:
    w = inp.w
    return MoELayer(inp.w_router, inp.bias, inp.w_gate, inp.w_up, inp.w_down, top_k=w.k,
                    max_tokens=max_tokens or inp.x.shape[0], n_shared=w.n_shared,
                    routed_scale=w.routed_scale)


def host_inputs(inp: synth.LayerInputs):
    cv = synth.to_numpy_bits
    return [cv(t) for t in (inp.x, inp.w_router, inp.bias, inp.w_gate, inp.w_up, inp.w_down)]


def selection_margin(logits, bias, k):
    """Gap between the k-th and (k+1)-th fp32 score of each token (inf if k == E)."""
    s = np.sort(logits.astype(np.float64) + bias.astype(np.float64), axis=1)[:, ::-1]
    if k >= s.shape[1]:
        return np.full(s.shape[0], np.inf)
    return s[:, k - 1] - s[:, k]


def compare_layer(inp: synth.LayerInputs, gpu_out: torch.Tensor, gpu_idx: np.ndarray,
                  tokens=None, tol=None):
    """Oracle on `tokens` (default all) vs the GPU output rows.

    Tokens whose GPU selection differs from the oracle's must be genuine near-ties (the
    oracle's k-th / (k+1)-th score gap below 1e-4, the size of fp32 logit rounding across
    accumulation orders); they are excluded from the value comparison.  Returns a dict of
    statistics; raises AssertionError on a failure."""
    w = inp.w
    x, wr, b, wg, wu, wd = host_inputs(inp)
    T = x.shape[0]
    toks = np.arange(T, dtype=np.int32) if tokens is None else np.asarray(tokens, np.int32)
    ref, idx, gates, logits = oracle_moe_forward(x, wr, b, wg, wu, wd, k=w.k,
                                                 n_shared=w.n_shared,
                                                 routed_scale=w.routed_scale, tokens=toks)
    gi = gpu_idx[toks]
    same = (np.sort(gi, axis=1) == np.sort(idx, axis=1)).all(axis=1)
    if not same.all():
        margin = selection_margin(logits[~same], b, w.k)
        assert (margin < 1e-4).all(), f"routing differs away from a tie: margins {margin}"
    got = gpu_out.float().cpu().numpy().astype(np.float64)[toks]
    rms = float(np.sqrt(np.mean(ref[same] ** 2))) if same.any() else 1.0
    err = np.abs(got[same] - ref[same])
    tol = (BF16_TOL if w.dtype == "bf16" else F32_TOL) if tol is None else tol
    stats = dict(max_err=float(err.max()) if err.size else 0.0, rms=rms,
                 rel=float(err.max() / rms) if err.size else 0.0,
                 n_tokens=int(len(toks)), n_tie_excluded=int((~same).sum()))
    assert stats["rel"] <= tol, stats
    return stats


def check_routing_exact(layer: MoELayer, logits: torch.Tensor, bias_np, k, E):
    """GPU routing from given fp32 logits vs the oracle's: integers bit-exact."""
    r = layer.route(logits=logits)
    torch.cuda.synchronize()
    lg = logits.cpu().numpy()
    idx, gates = oracle_route(lg, bias_np, k)
    counts, offsets, perm, slot_row = oracle_permute(idx, E)
    g = {kk: v.cpu().numpy() for kk, v in r.items()}
    assert (g["idx"] == idx).all()
    assert (g["counts"] == counts).all()
    assert (g["offsets"] == offsets).all()
    assert (g["perm"] == perm).all()
    assert (g["slot_row"] == slot_row).all()
    np.testing.assert_allclose(g["gates"], gates, rtol=2e-6, atol=1e-30)
    return g

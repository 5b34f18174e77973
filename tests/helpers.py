"""Shared test helpers: run the CUDA layer and the CPU oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

from oracle import (oracle_gates, oracle_moe_forward, oracle_permute, oracle_route,
                    oracle_router_logits)
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


def oracle_routing(inp: synth.LayerInputs):
    """The oracle's own routing of the whole batch: logits [T, E], idx, gates [T, k],
    counts [E], offsets [E + 1], perm [T*k], slot_row [T, k]."""
    w = inp.w
    x, wr, b, *_ = host_inputs(inp)
    logits = oracle_router_logits(x, wr)
    idx, gates = oracle_route(logits, b, w.k)
    counts, offsets, perm, slot_row = oracle_permute(idx, w.E)
    return dict(logits=logits, idx=idx, gates=gates, counts=counts, offsets=offsets,
                perm=perm, slot_row=slot_row, bias=b)


def check_full_routing(orc, gpu_idx, k):
    """GPU selection of every token against the oracle's: identical slot by slot, except at
    genuine near-ties (the oracle's k-th / (k+1)-th score gap below 1e-4), where the two
    sides' fp32 logits (different accumulation orders) may order the scores differently.
    Returns the number of such tokens."""
    diff = ~(gpu_idx == orc["idx"]).all(axis=1)
    if diff.any():
        lg = orc["logits"][diff]
        s = np.sort(lg.astype(np.float64) + orc["bias"].astype(np.float64), axis=1)[:, ::-1]
        # a swap inside the selection needs a near-tie among the k selected scores, a
        # different set one at the boundary: the smallest adjacent gap among the top k + 1
        gaps = -np.diff(s[:, :min(k + 1, s.shape[1])], axis=1)
        assert (gaps.min(axis=1) < 1e-4).all(), "routing differs away from a near-tie"
    return int(diff.sum())


def covering_tokens(orc, T, k, tile=128, extra=0, seed=7):
    """Tokens whose outputs check every touched expert group of the oracle's routing: for
    each group the first and last row (the last, ragged token tile), and both rows at every
    multiple of `tile` inside it (the edges of the token tiles of 128 and 256 rows); the
    shared group's first and last tokens and its first tile edges; plus `extra` random
    tokens.  Returns sorted unique token ids."""
    offs, perm = orc["offsets"], orc["perm"]
    rows = []
    for e in range(len(offs) - 1):
        lo, hi = int(offs[e]), int(offs[e + 1])
        if hi == lo:
            continue
        rows += [lo, hi - 1]
        for m in range(tile, hi - lo, tile):
            rows += [lo + m - 1, lo + m]
    toks = set(int(perm[r]) // k for r in rows)
    toks |= {t for t in (0, T - 1, tile - 1, tile, 2 * tile - 1, 2 * tile) if t < T}
    if extra:
        rng = np.random.default_rng(seed)
        toks |= set(int(t) for t in rng.choice(T, min(extra, T), replace=False))
    return np.array(sorted(toks), np.int32)


def greedy_group_cover(orc, T, k, n_largest=8):
    """A small token set whose selections together touch every touched routed expert (each
    token covers its k experts; greedy set cover), plus the last token of each of the
    `n_largest` largest groups (their last, ragged token tiles).  Every token also covers
    the shared expert."""
    idx = orc["idx"]
    counts = orc["counts"]
    touched = set(np.nonzero(counts)[0].tolist())
    big = np.argsort(-counts, kind="stable")[:n_largest]
    chosen = {int(orc["perm"][int(orc["offsets"][e + 1]) - 1]) // k for e in big
              if counts[e] > 0}
    covered = set()
    for t in chosen:
        covered |= set(idx[t].tolist())
    while covered != touched:
        gain = np.array([len(set(r.tolist()) - covered) for r in idx])
        t = int(gain.argmax())
        chosen.add(t)
        covered |= set(idx[t].tolist())
    return np.array(sorted(chosen), np.int32)

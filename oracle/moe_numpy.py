"""Vectorised NumPy restatement of the sparse-MoE layer -- test infrastructure only.

Written independently of ``moe_oracle.c`` (different algorithms for every step) so that the
two can pin each other on small inputs:

* selection: a lexicographic sort over (NaN flag, -score, expert id) instead of the C
  insertion sort;
* gates: a masked softmax over all experts (unselected -> -inf) instead of a softmax over
  the k picked logits;
* permutation: NumPy's stable argsort of the flattened expert ids instead of a counting sort;
* layer: dense evaluation of EVERY expert on EVERY token, then a [T, E] gate matrix that is
  zero off the selection (brute force), instead of visiting only the selected experts.

Sources: "Step 3.5 Flash: Open Frontier-Level Intelligence with 11B Active Parameters",
section 2.2 (288 routed + 1 shared expert, top-8) and 2.2.2 (S_t, s_{t,e}, p_{t,e}); the
parameter table and load-balancing note of "Step 3.5 Flash 技术论文深度解读" architecture
item 1 (bias adjustment for selection); its training-stability item on SwiGLU experts.
"""
from __future__ import annotations

import numpy as np


def decode(a) -> np.ndarray:
    """fp32 array or bf16 bit patterns (uint16) -> float64, exactly."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def np_logits(x, w_r) -> np.ndarray:
    return (decode(x) @ decode(w_r).T).astype(np.float32)


def np_select(logits, bias, k):
    """Top-k by (score desc, id asc), NaN last; scores are fp32 l + b."""
    logits = np.asarray(logits, np.float32)
    T, E = logits.shape
    s = logits + (np.zeros(E, np.float32) if bias is None else np.asarray(bias, np.float32))
    ids = np.broadcast_to(np.arange(E), (T, E))
    nan = np.isnan(s)
    key_score = np.where(nan, 0.0, -s.astype(np.float64))  # -0.0 and +0.0 compare equal
    # lexsort: last key is primary
    order = np.lexsort((ids, key_score, nan), axis=-1)
    idx = order[:, :k].astype(np.int32)
    sel = np.zeros((T, E), bool)
    np.put_along_axis(sel, idx.astype(np.int64), True, axis=1)
    masked = np.where(sel, logits.astype(np.float64), -np.inf)
    m = masked.max(axis=1, keepdims=True)
    p = np.exp(masked - m)
    p /= p.sum(axis=1, keepdims=True)
    gates = np.take_along_axis(p, idx.astype(np.int64), axis=1).astype(np.float32)
    return idx, gates, p  # p: [T, E] renormalised probabilities, zero off S_t


def np_permute(idx, E):
    idx = np.asarray(idx)
    T, k = idx.shape
    flat = idx.reshape(-1)
    counts = np.bincount(flat, minlength=E).astype(np.int32)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    perm = np.argsort(flat, kind="stable").astype(np.int32)
    slot_row = np.empty(T * k, np.int32)
    slot_row[perm] = np.arange(T * k, dtype=np.int32)
    return counts, offsets, perm, slot_row.reshape(T, k)


def np_swiglu_all(x, w_gate, w_up, w_down) -> np.ndarray:
    """Every expert on every token: [T, G, d] in float64 (G = number of experts given)."""
    X = decode(x)
    Wg, Wu, Wd = decode(w_gate), decode(w_up), decode(w_down)
    gate = np.einsum("ti,gri->tgr", X, Wg)
    up = np.einsum("ti,gri->tgr", X, Wu)
    h = gate / (1.0 + np.exp(-gate)) * up
    return np.einsum("tgr,gcr->tgc", h, Wd)


def np_moe_forward(x, w_r, bias, w_gate, w_up, w_down, k, n_shared=1, routed_scale=1.0,
                   logits=None):
    """Brute-force dense layer: out = shared + routed_scale * sum_e P[t,e] * y[t,e]."""
    E = np.asarray(w_r).shape[0]
    if logits is None:
        logits = np_logits(x, w_r)
    idx, gates, _ = np_select(logits, bias, k)
    G = np.zeros((logits.shape[0], E), np.float64)
    np.put_along_axis(G, idx.astype(np.int64), gates.astype(np.float64), axis=1)
    Y = np_swiglu_all(x, w_gate, w_up, w_down)
    out = routed_scale * np.einsum("te,tec->tc", G, Y[:, :E, :])
    if n_shared:
        out = out + Y[:, E, :]
    return out, idx, gates, logits

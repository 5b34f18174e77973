"""ctypes wrapper around the plain-C oracle (``moe_oracle.c``) -- test infrastructure only.

Arrays are NumPy; bf16 tensors are passed as their raw 16-bit patterns (``np.uint16``).
The wrapper only marshals arguments: every arithmetic step is in ``moe_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_moe.so")

F32 = 0
BF16 = 1

_lib = None


def build_oracle(force: bool = False) -> str:
    """Compile moe_oracle.c into liboracle_moe.so (gcc, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", _SRC, "-o", _LIB, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build_oracle()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_router_logits.argtypes = [P, P, I, I, I, I, P]
        lib.oracle_route.argtypes = [P, P, I, I, I, P, P]
        lib.oracle_gates.argtypes = [P, P, I, I, I, P]
        lib.oracle_permute.argtypes = [P, I, I, I, P, P, P, P]
        lib.oracle_expert_ffn.argtypes = [P, P, P, P, I, I, I, P]
        lib.oracle_moe_forward.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I,
                                           ctypes.c_double, P, I, P, P, P, P, P]
        lib.oracle_num_threads.restype = I
        lib.oracle_set_num_threads.argtypes = [I]
        lib.oracle_router_stats.argtypes = [P, P, I, I, I, I, P, P, P, P]
        lib.oracle_bias_update.argtypes = [P, I, I, ctypes.c_float, P]
        lib.oracle_expert_act_rms.argtypes = [P, P, P, I, I, I, I, I, I, P, I, P]
        lib.oracle_moe_backward.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I,
                                            ctypes.c_double, P, P, P, P, P, P, P]
        lib.oracle_expert_param_norms.argtypes = [P, P, P, I, I, I, I, P]
        lib.oracle_moe_backward_sampled.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I,
                                                    ctypes.c_double, P, P, I, P, P, I, P, P, P,
                                                    P, I, P, P]
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _as_input(a):
    """Contiguous fp32 or bf16-bits array and its dtype code."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return a, BF16
    if a.dtype == np.float32:
        return a, F32
    raise TypeError(f"oracle inputs are float32 or bf16 bits (uint16), got {a.dtype}")


def oracle_num_threads() -> int:
    return int(_load().oracle_num_threads())


def oracle_set_num_threads(n: int) -> None:
    """OpenMP threads for the following oracle calls (overrides OMP_NUM_THREADS)."""
    _load().oracle_set_num_threads(int(n))


def oracle_router_logits(x, w_r):
    x, dt = _as_input(x)
    w_r, dt2 = _as_input(w_r)
    assert dt == dt2
    T, d = x.shape
    E = w_r.shape[0]
    out = np.empty((T, E), np.float32)
    _load().oracle_router_logits(_ptr(x), _ptr(w_r), dt, T, d, E, _ptr(out))
    return out


def oracle_route(logits, bias, k):
    logits = np.ascontiguousarray(logits, np.float32)
    T, E = logits.shape
    bias = None if bias is None else np.ascontiguousarray(bias, np.float32)
    idx = np.empty((T, k), np.int32)
    gates = np.empty((T, k), np.float32)
    _load().oracle_route(_ptr(logits), _ptr(bias), T, E, k, _ptr(idx), _ptr(gates))
    return idx, gates


def oracle_gates(logits, idx):
    """Gates [T, k] of a given selection idx [T, k] from fp32 logits [T, E]: softmax over
    the selected unbiased logits (the same arithmetic oracle_route applies to its own)."""
    logits = np.ascontiguousarray(logits, np.float32)
    idx = np.ascontiguousarray(idx, np.int32)
    T, E = logits.shape
    k = idx.shape[1]
    assert idx.shape[0] == T and (idx >= 0).all() and (idx < E).all()
    gates = np.empty((T, k), np.float32)
    _load().oracle_gates(_ptr(logits), _ptr(idx), T, E, k, _ptr(gates))
    return gates


def oracle_permute(idx, E):
    idx = np.ascontiguousarray(idx, np.int32)
    T, k = idx.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(T * k, np.int32)
    slot_row = np.empty(T * k, np.int32)
    _load().oracle_permute(_ptr(idx), T, E, k, _ptr(counts), _ptr(offsets), _ptr(perm),
                           _ptr(slot_row))
    return counts, offsets, perm, slot_row.reshape(T, k)


def oracle_expert_ffn(x_row, wg, wu, wd):
    x_row, dt = _as_input(x_row)
    wg, _ = _as_input(wg)
    wu, _ = _as_input(wu)
    wd, _ = _as_input(wd)
    f, d = wg.shape
    y = np.empty(d, np.float64)
    _load().oracle_expert_ffn(_ptr(x_row), _ptr(wg), _ptr(wu), _ptr(wd), dt, d, f, _ptr(y))
    return y


def oracle_moe_forward(x, w_r, bias, w_gate, w_up, w_down, k, n_shared=1, routed_scale=1.0,
                       tokens=None, logits_in=None):
    """Layer output (float64) for `tokens` (default: all), plus idx, gates, logits."""
    x, dt = _as_input(x)
    w_r, _ = _as_input(w_r)
    w_gate, _ = _as_input(w_gate)
    w_up, _ = _as_input(w_up)
    w_down, _ = _as_input(w_down)
    T, d = x.shape
    E = w_r.shape[0]
    f = w_gate.shape[1]
    assert w_gate.shape[0] == E + n_shared
    if tokens is None:
        tokens = np.arange(T, dtype=np.int32)
    tokens = np.ascontiguousarray(tokens, np.int32)
    n = len(tokens)
    out = np.empty((n, d), np.float64)
    idx = np.empty((n, k), np.int32)
    gates = np.empty((n, k), np.float32)
    logits = np.empty((n, E), np.float32)
    if logits_in is not None:
        logits_in = np.ascontiguousarray(logits_in, np.float32)
        assert logits_in.shape == (n, E)
    bias = np.ascontiguousarray(bias, np.float32)
    _load().oracle_moe_forward(_ptr(x), _ptr(w_r), _ptr(bias), _ptr(w_gate), _ptr(w_up),
                               _ptr(w_down), dt, d, E, k, f, n_shared, float(routed_scale),
                               _ptr(tokens), n, _ptr(logits_in), _ptr(out), _ptr(idx),
                               _ptr(gates), _ptr(logits))
    return out, idx, gates, logits


def oracle_router_stats(logits, idx, n_groups):
    """p_mean [E], f_sel [E], L_EP, routing confidence (see moe_oracle.c)."""
    logits = np.ascontiguousarray(logits, np.float32)
    idx = np.ascontiguousarray(idx, np.int32)
    T, E = logits.shape
    k = idx.shape[1]
    p_mean = np.empty(E, np.float32)
    f_sel = np.empty(E, np.float32)
    l_ep = np.empty(1, np.float32)
    conf = np.empty(1, np.float32)
    _load().oracle_router_stats(_ptr(logits), _ptr(idx), T, E, k, int(n_groups), _ptr(p_mean),
                                _ptr(f_sel), _ptr(l_ep), _ptr(conf))
    return p_mean, f_sel, float(l_ep[0]), float(conf[0])


def oracle_bias_update(counts, Tk, gamma, bias):
    counts = np.ascontiguousarray(counts, np.int32)
    out = np.array(bias, np.float32, copy=True)
    _load().oracle_bias_update(_ptr(counts), len(counts), int(Tk), float(gamma), _ptr(out))
    return out


def oracle_expert_act_rms(x, w_gate, w_up, idx, n_experts, n_shared=1):
    """Per-expert RMS of the SwiGLU activation over the tokens routed to it [G] (float64)."""
    x, dt = _as_input(x)
    w_gate, _ = _as_input(w_gate)
    w_up, _ = _as_input(w_up)
    idx = np.ascontiguousarray(idx, np.int32)
    T, d = x.shape
    f = w_gate.shape[1]
    k = idx.shape[1]
    G = n_experts + n_shared
    out = np.empty(G, np.float64)
    _load().oracle_expert_act_rms(_ptr(x), _ptr(w_gate), _ptr(w_up), dt, T, d, f, n_experts,
                                  n_shared, _ptr(idx), k, _ptr(out))
    return out


def oracle_expert_param_norms(w_gate, w_up, w_down):
    """Frobenius norm of each expert's (W_gate, W_up, W_down) together [G] (float64)."""
    w_gate, dt = _as_input(w_gate)
    w_up, _ = _as_input(w_up)
    w_down, _ = _as_input(w_down)
    G, f, d = w_gate.shape
    out = np.empty(G, np.float64)
    _load().oracle_expert_param_norms(_ptr(w_gate), _ptr(w_up), _ptr(w_down), dt, d, f, G,
                                      _ptr(out))
    return out


def oracle_health_ratios(act_rms, param_norms, idx, n_experts):
    """Cross-expert ratios over the routed experts: median / max of the activation RMS of
    the experts some token chose, and min / median of the parameter norms (NumPy median:
    mean of the two middle values for an even count)."""
    chosen = np.unique(np.asarray(idx).ravel())
    a = np.asarray(act_rms, np.float64)[chosen]
    pn = np.asarray(param_norms, np.float64)[:n_experts]
    return float(np.median(a) / a.max()), float(pn.min() / np.median(pn))


def oracle_moe_backward(x, dout, w_r, w_gate, w_up, w_down, idx, gates, routed_scale=1.0,
                        n_shared=1):
    """Gradients of the layer output for the given selection: dict of float64 arrays dx
    [T,d], dw_router [E,d], dw_gate / dw_up [G,f,d], dw_down [G,d,f] (see moe_oracle.c)."""
    x, dt = _as_input(x)
    dout, dt2 = _as_input(dout)
    assert dt == dt2
    w_r, _ = _as_input(w_r)
    w_gate, _ = _as_input(w_gate)
    w_up, _ = _as_input(w_up)
    w_down, _ = _as_input(w_down)
    idx = np.ascontiguousarray(idx, np.int32)
    gates = np.ascontiguousarray(gates, np.float32)
    T, d = x.shape
    E = w_r.shape[0]
    G, f, _ = w_gate.shape
    k = idx.shape[1]
    out = dict(dx=np.empty((T, d)), dw_router=np.empty((E, d)), dw_gate=np.empty((G, f, d)),
               dw_up=np.empty((G, f, d)), dw_down=np.empty((G, d, f)))
    _load().oracle_moe_backward(_ptr(x), _ptr(dout), _ptr(w_r), _ptr(w_gate), _ptr(w_up),
                                _ptr(w_down), dt, T, d, E, k, f, n_shared, float(routed_scale),
                                _ptr(idx), _ptr(gates), _ptr(out["dx"]), _ptr(out["dw_router"]),
                                _ptr(out["dw_gate"]), _ptr(out["dw_up"]), _ptr(out["dw_down"]))
    return out


def oracle_moe_backward_sampled(x, dout, w_r, w_gate, w_up, w_down, idx, gates, toks, exps,
                                rexps, routed_scale=1.0, n_shared=1):
    """Selected parts of oracle_moe_backward's result, for sizes whose full weight gradients
    do not fit in memory: dict of float64 arrays dx [len(toks), d] (those tokens' rows),
    dw_gate / dw_up [len(exps), f, d], dw_down [len(exps), d, f] (those experts; the shared
    expert is index E), dw_router [len(rexps), d] (those routed experts)."""
    x, dt = _as_input(x)
    dout, dt2 = _as_input(dout)
    assert dt == dt2
    w_r, _ = _as_input(w_r)
    w_gate, _ = _as_input(w_gate)
    w_up, _ = _as_input(w_up)
    w_down, _ = _as_input(w_down)
    idx = np.ascontiguousarray(idx, np.int32)
    gates = np.ascontiguousarray(gates, np.float32)
    toks = np.ascontiguousarray(toks, np.int32)
    exps = np.ascontiguousarray(exps, np.int32)
    rexps = np.ascontiguousarray(rexps, np.int32)
    T, d = x.shape
    E = w_r.shape[0]
    G, f, _ = w_gate.shape
    k = idx.shape[1]
    ne = len(exps)
    out = dict(dx=np.empty((len(toks), d)), dw_gate=np.empty((ne, f, d)),
               dw_up=np.empty((ne, f, d)), dw_down=np.empty((ne, d, f)),
               dw_router=np.empty((len(rexps), d)))
    _load().oracle_moe_backward_sampled(
        _ptr(x), _ptr(dout), _ptr(w_r), _ptr(w_gate), _ptr(w_up), _ptr(w_down), dt, T, d, E,
        k, f, n_shared, float(routed_scale), _ptr(idx), _ptr(gates), len(toks), _ptr(toks),
        _ptr(out["dx"]), ne, _ptr(exps), _ptr(out["dw_gate"]), _ptr(out["dw_up"]),
        _ptr(out["dw_down"]), len(rexps), _ptr(rexps), _ptr(out["dw_router"]))
    return out

"""Thin ctypes binding of ``libmoe_layer.so`` (C ABI declared in ``include/moe_layer.h``).

Argument marshalling only: torch tensors supply device pointers and the current CUDA
stream; every step of the layer runs in the library's kernels.  There is no fallback: if
the shared library is missing or fails to load, importing the functions raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_layer.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_ALIGNMENT = 3
MOE_ERR_WORKSPACE = 4
MOE_ERR_CUDA = 5
MOE_ERR_DEVICE_TIMEOUT = 6

MOE_F32 = 0
MOE_BF16 = 1

# every entry point the header declares (checked by tests against the built library)
EXPORTS = ("moe_layer_init", "moe_layer_destroy", "moe_workspace_size", "moe_workspace_init",
           "moe_route", "moe_route_from_logits", "moe_forward", "moe_forward_profiled",
           "moe_device_status", "moe_status_string", "moe_router_logits_static",
           "moe_router_stats", "moe_update_router_bias", "moe_forward_launch_count",
           "moe_selftest_wait_timeout", "moe_expert_health", "moe_backward",
           "moe_backward_workspace_size", "moe_saved_size", "moe_forward_save",
           "moe_backward_saved", "moe_backward_ex", "moe_set_option", "moe_layer_init_ep",
           "moe_forward_partial", "moe_ep_plan", "moe_ep_pack", "moe_ep_combine",
           "moe_gemm_clock")
MOE_BACKWARD_OVERWRITE = 1
MOE_OPTION_H_HANDOVER = 1
MOE_OPTION_SHARED_SIDE_SMS = 2
MOE_OPTION_ROW_GATHER_IN_GEMM = 3
MOE_OPTION_GEMM_CLOCK = 4
MOE_PROFILE_STAGES = 7
PROFILE_STAGE_NAMES = ("router_logits", "topk_gates_hist", "permute_scatter", "row_gather",
                       "expert_up_swiglu", "expert_down", "combine")


class moe_config(ctypes.Structure):
    _fields_ = [("max_tokens", ctypes.c_int), ("d_model", ctypes.c_int),
                ("n_experts", ctypes.c_int), ("top_k", ctypes.c_int), ("d_ff", ctypes.c_int),
                ("n_shared", ctypes.c_int), ("dtype", ctypes.c_int),
                ("routed_scale", ctypes.c_float)]


class moe_weights(ctypes.Structure):
    _fields_ = [("w_router", ctypes.c_void_p), ("router_bias", ctypes.c_void_p),
                ("w_gate", ctypes.c_void_p), ("w_up", ctypes.c_void_p),
                ("w_down", ctypes.c_void_p)]


class MoEError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: status {status} ({status_string(status)})")
        self.status = status


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmoe_layer.so (raises OSError if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise OSError(f"{path} is missing: build it with `python -m "
                          "sparse_moe_layer_warp_b200.build`")
        lib = ctypes.CDLL(path)
        P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        lib.moe_layer_init.argtypes = [ctypes.POINTER(moe_config), ctypes.POINTER(moe_weights),
                                       ctypes.POINTER(P)]
        lib.moe_layer_destroy.argtypes = [P]
        lib.moe_workspace_size.argtypes = [P, I]
        lib.moe_workspace_size.restype = Z
        lib.moe_workspace_init.argtypes = [P, P, Z, P]
        lib.moe_route.argtypes = [P, P, I, P, P, P, P, P, P, P, P, Z, P]
        lib.moe_route_from_logits.argtypes = [P, P, I, P, P, P, P, P, P, P, Z, P]
        lib.moe_forward.argtypes = [P, P, I, P, P, Z, P]
        lib.moe_forward_profiled.argtypes = [P, P, I, P, P, Z, P, ctypes.POINTER(P), I]
        lib.moe_device_status.argtypes = [P, P, Z, P]
        lib.moe_gemm_clock.argtypes = [P, P, Z, ctypes.POINTER(ctypes.c_double), P]
        lib.moe_router_logits_static.argtypes = [P, P, I, P, P]
        lib.moe_router_stats.argtypes = [P, P, P, I, I, P, P, P, P, Z, P]
        lib.moe_update_router_bias.argtypes = [P, P, I, ctypes.c_float, P, P]
        lib.moe_selftest_wait_timeout.argtypes = [P, P, Z, I, P]
        lib.moe_expert_health.argtypes = [P, I, P, P, P, P, Z, P]
        lib.moe_backward.argtypes = [P, P, I, P, P, P, P, P, P, P, Z, P]
        lib.moe_backward_workspace_size.argtypes = [P, I]
        lib.moe_backward_workspace_size.restype = Z
        lib.moe_saved_size.argtypes = [P, I]
        lib.moe_saved_size.restype = Z
        lib.moe_forward_save.argtypes = [P, P, I, P, P, Z, P, Z, P]
        lib.moe_backward_saved.argtypes = [P, P, I, P, P, Z, P, P, P, P, P, P, Z, P]
        lib.moe_backward_ex.argtypes = [P, P, I, P, P, Z, ctypes.c_uint, P, P, P, P, P, P, Z, P]
        lib.moe_set_option.argtypes = [P, I, I]
        lib.moe_layer_init_ep.argtypes = [ctypes.POINTER(moe_config),
                                          ctypes.POINTER(moe_weights), I, I, ctypes.POINTER(P)]
        lib.moe_forward_partial.argtypes = [P, P, I, P, P, I, I, I, I, P, P, Z, P]
        lib.moe_ep_plan.argtypes = [P, P, I, I, P, P, P, P, P, Z, P]
        lib.moe_ep_pack.argtypes = [P, P, P, P, I, I, P, P, P, P, P, P]
        lib.moe_ep_combine.argtypes = [P, P, P, P, P, I, I, P, P]
        lib.moe_forward_launch_count.argtypes = [P, I]
        lib.moe_forward_launch_count.restype = I
        lib.moe_status_string.argtypes = [I]
        lib.moe_status_string.restype = ctypes.c_char_p
        for name in ("moe_layer_init", "moe_layer_destroy", "moe_workspace_init", "moe_route",
                     "moe_route_from_logits", "moe_forward", "moe_forward_profiled",
                     "moe_device_status", "moe_router_logits_static", "moe_router_stats",
                     "moe_update_router_bias", "moe_selftest_wait_timeout",
                     "moe_expert_health", "moe_backward", "moe_forward_save",
                     "moe_backward_saved", "moe_backward_ex", "moe_set_option", "moe_layer_init_ep",
                     "moe_forward_partial", "moe_ep_plan", "moe_ep_pack", "moe_ep_combine",
                     "moe_gemm_clock"):
            getattr(lib, name).restype = I
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load_library().moe_status_string(int(status)).decode()


def _check(fn: str, status: int) -> None:
    if status != MOE_OK:
        raise MoEError(fn, status)


def _addr(t) -> int:
    """Device address of a tensor handed to the C ABI.  The library reads and writes dense
    row-major device memory through raw pointers, so a strided view or a host tensor is
    refused here, before anything is launched."""
    if not t.is_contiguous():
        raise ValueError(f"the library takes contiguous (dense row-major) tensors; got shape "
                         f"{tuple(t.shape)} with strides {tuple(t.stride())}")
    if not t.is_cuda:
        raise ValueError(f"the library takes CUDA tensors; got one on {t.device}")
    return t.data_ptr()


def _p(t):
    return None if t is None else ctypes.c_void_p(_addr(t))


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


# ------------------------------------------------------------------ C-ABI mirrors
def moe_layer_init(cfg: moe_config, w_router, router_bias, w_gate, w_up, w_down):
    lib = load_library()
    w = moe_weights(_addr(w_router), None if router_bias is None else _addr(router_bias),
                    _addr(w_gate), _addr(w_up), _addr(w_down))
    h = ctypes.c_void_p()
    _check("moe_layer_init", lib.moe_layer_init(ctypes.byref(cfg), ctypes.byref(w),
                                                ctypes.byref(h)))
    return h


def moe_layer_init_ep(cfg: moe_config, expert_begin: int, expert_end: int, w_router,
                      router_bias, w_gate, w_up, w_down):
    """Handle over the routed experts [expert_begin, expert_end) of a bf16 layer (weights:
    those experts then the shared expert; the full router)."""
    lib = load_library()
    w = moe_weights(_addr(w_router), None if router_bias is None else _addr(router_bias),
                    _addr(w_gate), _addr(w_up), _addr(w_down))
    h = ctypes.c_void_p()
    _check("moe_layer_init_ep", lib.moe_layer_init_ep(ctypes.byref(cfg), ctypes.byref(w),
                                                      int(expert_begin), int(expert_end),
                                                      ctypes.byref(h)))
    return h


def moe_forward_partial(handle, x, n_tokens, topk_idx, topk_gate, expert_begin, expert_end,
                        shared_begin, shared_end, out, ws, stream=None) -> None:
    """fp32 partial output of an expert range (see include/moe_layer.h)."""
    _check("moe_forward_partial", load_library().moe_forward_partial(
        handle, _p(x), int(n_tokens), _p(topk_idx), _p(topk_gate), int(expert_begin),
        int(expert_end), int(shared_begin), int(shared_end), _p(out), _p(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def moe_ep_plan(handle, topk_idx, n_tokens, n_ranks, send_counts, send_offsets, send_perm,
                send_slot, ws, stream=None) -> None:
    _check("moe_ep_plan", load_library().moe_ep_plan(
        handle, _p(topk_idx), int(n_tokens), int(n_ranks), _p(send_counts), _p(send_offsets),
        _p(send_perm), _p(send_slot), _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def moe_ep_pack(handle, x, topk_idx, topk_gate, n_tokens, n_ranks, send_perm, send_offsets,
                x_send, idx_send, gate_send, stream=None) -> None:
    _check("moe_ep_pack", load_library().moe_ep_pack(
        handle, _p(x), _p(topk_idx), _p(topk_gate), int(n_tokens), int(n_ranks), _p(send_perm),
        _p(send_offsets), _p(x_send), _p(idx_send), _p(gate_send), _stream(stream)))


def moe_ep_combine(handle, back, send_slot, send_offsets, shared, n_tokens, n_ranks, out,
                   stream=None) -> None:
    _check("moe_ep_combine", load_library().moe_ep_combine(
        handle, _p(back), _p(send_slot), _p(send_offsets), _p(shared), int(n_tokens),
        int(n_ranks), _p(out), _stream(stream)))


def moe_layer_destroy(handle) -> None:
    _check("moe_layer_destroy", load_library().moe_layer_destroy(handle))


def moe_set_option(handle, option: int, value: int) -> None:
    """Launch-plan option of a handle (MOE_OPTION_H_HANDOVER; see include/moe_layer.h)."""
    _check("moe_set_option", load_library().moe_set_option(handle, int(option), int(value)))


def moe_workspace_size(handle, n_tokens: int) -> int:
    return int(load_library().moe_workspace_size(handle, int(n_tokens)))


def moe_workspace_init(handle, ws, stream=None) -> None:
    _check("moe_workspace_init", load_library().moe_workspace_init(
        handle, _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def moe_route(handle, x, n_tokens, logits_out, topk_idx, topk_gate, expert_counts,
              expert_offsets, perm, slot_row, ws, stream=None) -> None:
    _check("moe_route", load_library().moe_route(
        handle, _p(x), int(n_tokens), _p(logits_out), _p(topk_idx), _p(topk_gate),
        _p(expert_counts), _p(expert_offsets), _p(perm), _p(slot_row), _p(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def moe_route_from_logits(handle, logits, n_tokens, topk_idx, topk_gate, expert_counts,
                          expert_offsets, perm, slot_row, ws, stream=None) -> None:
    _check("moe_route_from_logits", load_library().moe_route_from_logits(
        handle, _p(logits), int(n_tokens), _p(topk_idx), _p(topk_gate), _p(expert_counts),
        _p(expert_offsets), _p(perm), _p(slot_row), _p(ws), ws.numel() * ws.element_size(),
        _stream(stream)))


def moe_forward(handle, x, n_tokens, out, ws, stream=None) -> None:
    _check("moe_forward", load_library().moe_forward(
        handle, _p(x), int(n_tokens), _p(out), _p(ws), ws.numel() * ws.element_size(),
        _stream(stream)))


def moe_backward_workspace_size(handle, n_tokens: int) -> int:
    return int(load_library().moe_backward_workspace_size(handle, int(n_tokens)))


def moe_backward(handle, x, n_tokens, dout, dx, dw_router, dw_gate, dw_up, dw_down, ws,
                 stream=None) -> None:
    """Gradients of <forward(x), dout> (see include/moe_layer.h); fp32 outputs."""
    _check("moe_backward", load_library().moe_backward(
        handle, _p(x), int(n_tokens), _p(dout), _p(dx), _p(dw_router), _p(dw_gate), _p(dw_up),
        _p(dw_down), _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def moe_saved_size(handle, n_tokens: int) -> int:
    return int(load_library().moe_saved_size(handle, int(n_tokens)))


def moe_forward_save(handle, x, n_tokens, out, saved, ws, stream=None) -> None:
    """moe_forward that also keeps the fp32 pre-activations for moe_backward_saved."""
    _check("moe_forward_save", load_library().moe_forward_save(
        handle, _p(x), int(n_tokens), _p(out), _p(saved), saved.numel() * saved.element_size(),
        _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def moe_backward_saved(handle, x, n_tokens, dout, saved, dx, dw_router, dw_gate, dw_up, dw_down,
                       ws, stream=None) -> None:
    """moe_backward reading the pre-activations kept by moe_forward_save."""
    _check("moe_backward_saved", load_library().moe_backward_saved(
        handle, _p(x), int(n_tokens), _p(dout), _p(saved), saved.numel() * saved.element_size(),
        _p(dx), _p(dw_router), _p(dw_gate), _p(dw_up), _p(dw_down), _p(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def moe_backward_ex(handle, x, n_tokens, dout, saved, flags, dx, dw_router, dw_gate, dw_up,
                    dw_down, ws, stream=None) -> None:
    """moe_backward with options: `saved` (or None) and flags (MOE_BACKWARD_OVERWRITE)."""
    nbytes = 0 if saved is None else saved.numel() * saved.element_size()
    _check("moe_backward_ex", load_library().moe_backward_ex(
        handle, _p(x), int(n_tokens), _p(dout), None if saved is None else _p(saved), nbytes,
        int(flags), _p(dx), _p(dw_router), _p(dw_gate), _p(dw_up), _p(dw_down), _p(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def moe_expert_health(handle, n_tokens, act_rms, param_norm, ratios, ws, stream=None) -> None:
    """Expert health signals of the last forward on `ws` (see include/moe_layer.h)."""
    _check("moe_expert_health", load_library().moe_expert_health(
        handle, int(n_tokens), _p(act_rms), _p(param_norm), _p(ratios), _p(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def moe_selftest_wait_timeout(handle, ws, limit_us: int, stream=None) -> None:
    """Launch the library's timeout self-test kernel (see include/moe_layer.h)."""
    _check("moe_selftest_wait_timeout", load_library().moe_selftest_wait_timeout(
        handle, _p(ws), ws.numel() * ws.element_size(), int(limit_us), _stream(stream)))


def moe_forward_launch_count(handle, n_tokens: int) -> int:
    """Kernel launches of one moe_forward of n_tokens tokens (-1: invalid arguments)."""
    return int(load_library().moe_forward_launch_count(handle, int(n_tokens)))


def moe_forward_profiled(handle, x, n_tokens, out, ws, events, stream=None) -> None:
    """`events`: MOE_PROFILE_STAGES + 1 torch.cuda.Event(enable_timing=True) objects."""
    for e in events:
        if e.cuda_event == 0:  # torch creates the CUDA event on its first record
            e.record()
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _check("moe_forward_profiled", load_library().moe_forward_profiled(
        handle, _p(x), int(n_tokens), _p(out), _p(ws), ws.numel() * ws.element_size(),
        _stream(stream), arr, len(events)))


def moe_router_logits_static(handle, x, n_tokens, logits_out, stream=None, *, d_model=None,
                             n_experts=None, dtype=None) -> None:
    """Router logits with the library's own static scratch (no workspace argument), for
    callers that cannot allocate device memory; see include/moe_layer.h for the limits.
    With d_model, n_experts and dtype given (MoELayer passes them), x and logits_out are
    checked to hold n_tokens rows before the library reads and writes them."""
    if d_model is not None:
        if x.dtype != dtype or x.numel() < int(n_tokens) * int(d_model):
            raise ValueError(f"x: expected at least {int(n_tokens)} x {int(d_model)} elements "
                             f"of {dtype}, got {tuple(x.shape)} of {x.dtype}")
        if (logits_out.dtype != torch.float32 or
                logits_out.numel() < int(n_tokens) * int(n_experts)):
            raise ValueError(f"logits_out: expected at least {int(n_tokens)} x {int(n_experts)}"
                             f" fp32 elements, got {tuple(logits_out.shape)} of "
                             f"{logits_out.dtype}")
    _check("moe_router_logits_static", load_library().moe_router_logits_static(
        handle, _p(x), int(n_tokens), _p(logits_out), _stream(stream)))


def moe_router_stats(handle, logits, topk_idx, n_tokens, n_groups, p_mean, f_sel, scalars, ws,
                     stream=None) -> None:
    _check("moe_router_stats", load_library().moe_router_stats(
        handle, _p(logits), _p(topk_idx), int(n_tokens), int(n_groups), _p(p_mean), _p(f_sel),
        _p(scalars), _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def moe_update_router_bias(handle, expert_counts, n_tokens, gamma, bias, stream=None) -> None:
    _check("moe_update_router_bias", load_library().moe_update_router_bias(
        handle, _p(expert_counts), int(n_tokens), float(gamma), _p(bias), _stream(stream)))


def moe_device_status(handle, ws, stream=None) -> int:
    return int(load_library().moe_device_status(handle, _p(ws), ws.numel() * ws.element_size(),
                                                 _stream(stream)))


def moe_gemm_clock(handle, ws, stream=None) -> tuple:
    """(up, down) effective SM clock in MHz of the expert GEMMs run with MOE_OPTION_GEMM_CLOCK
    since the last call (0.0 when none ran); clears the sums."""
    mhz = (ctypes.c_double * 2)()
    _check("moe_gemm_clock", load_library().moe_gemm_clock(
        handle, _p(ws), ws.numel() * ws.element_size(), mhz, _stream(stream)))
    return float(mhz[0]), float(mhz[1])


# ------------------------------------------------------------------ convenience wrapper
def _expect(t, shape, dtype, name):
    """The C ABI sees only pointers: a tensor of another shape or type would be read or
    written out of its bounds, so the class below checks every tensor it passes."""
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype:
        raise ValueError(f"{name}: expected shape {tuple(shape)} of {dtype}, got "
                         f"{tuple(t.shape)} of {t.dtype}")


class MoELayer:
    """Owns a handle and a workspace; holds references to the weight tensors."""

    def __init__(self, w_router, router_bias, w_gate, w_up, w_down, top_k: int,
                 max_tokens: int, n_shared: int = 1, routed_scale: float = 1.0):
        if w_router.dtype not in (torch.bfloat16, torch.float32) or w_router.dim() != 2:
            raise ValueError("w_router: expected a [E, d] bf16 or fp32 tensor")
        dt = MOE_BF16 if w_router.dtype == torch.bfloat16 else MOE_F32
        E, d = w_router.shape
        f = w_gate.shape[1]
        G = int(E) + int(n_shared)
        _expect(w_gate, (G, f, d), w_router.dtype, "w_gate")
        _expect(w_up, (G, f, d), w_router.dtype, "w_up")
        _expect(w_down, (G, d, f), w_router.dtype, "w_down")
        if router_bias is not None:
            _expect(router_bias, (E,), torch.float32, "router_bias")
        self.cfg = moe_config(int(max_tokens), int(d), int(E), int(top_k), int(f),
                              int(n_shared), dt, float(routed_scale))
        self.tensors = (w_router, router_bias, w_gate, w_up, w_down)
        self.handle = moe_layer_init(self.cfg, *self.tensors)
        self.device = w_router.device
        self.dtype = w_router.dtype
        self.ws = None
        self.bw_ws = None
        self.E, self.k, self.d = int(E), int(top_k), int(d)

    def _rows(self, x, name="x"):
        """Token count of a [T, d] activation of the layer's type."""
        if x.dim() != 2:
            raise ValueError(f"{name}: expected a [T, {self.d}] tensor, got {tuple(x.shape)}")
        _expect(x, (x.shape[0], self.d), self.dtype, name)
        return int(x.shape[0])

    def router_logits_static(self, x, logits_out=None, stream=None):
        """Router logits [T, E] fp32 through the workspace-free entry point."""
        T = self._rows(x)
        if logits_out is None:
            logits_out = torch.empty((T, self.E), dtype=torch.float32, device=self.device)
        _expect(logits_out, (T, self.E), torch.float32, "logits_out")
        moe_router_logits_static(self.handle, x, T, logits_out, stream, d_model=self.d,
                                 n_experts=self.E, dtype=self.dtype)
        return logits_out

    def set_option(self, option: int, value: int) -> None:
        moe_set_option(self.handle, option, value)

    def workspace(self, n_tokens: int):
        need = moe_workspace_size(self.handle, n_tokens)
        if self.ws is None or self.ws.numel() < need:
            self.ws = torch.empty(need, dtype=torch.uint8, device=self.device)
            moe_workspace_init(self.handle, self.ws)
        return self.ws

    def forward(self, x, out=None, stream=None):
        T = self._rows(x)
        out = torch.empty_like(x) if out is None else out
        _expect(out, x.shape, x.dtype, "out")
        moe_forward(self.handle, x, T, out, self.workspace(T), stream)
        return out

    def route(self, x=None, logits=None, want_logits=False, stream=None):
        if x is not None:
            T = self._rows(x)
        else:
            T = int(logits.shape[0])
            _expect(logits, (T, self.E), torch.float32, "logits")
        dev = self.device
        r = dict(
            idx=torch.empty((T, self.k), dtype=torch.int32, device=dev),
            gates=torch.empty((T, self.k), dtype=torch.float32, device=dev),
            counts=torch.empty((self.E,), dtype=torch.int32, device=dev),
            offsets=torch.empty((self.E + 1,), dtype=torch.int32, device=dev),
            perm=torch.empty((T * self.k,), dtype=torch.int32, device=dev),
            slot_row=torch.empty((T, self.k), dtype=torch.int32, device=dev))
        ws = self.workspace(T)
        if logits is not None:
            moe_route_from_logits(self.handle, logits, T, r["idx"], r["gates"], r["counts"],
                                  r["offsets"], r["perm"], r["slot_row"], ws, stream)
        else:
            lg = torch.empty((T, self.E), dtype=torch.float32, device=dev) if want_logits else None
            moe_route(self.handle, x, T, lg, r["idx"], r["gates"], r["counts"], r["offsets"],
                      r["perm"], r["slot_row"], ws, stream)
            if lg is not None:
                r["logits"] = lg
        return r

    def router_stats(self, logits, topk_idx, n_groups, stream=None):
        """p_mean [E], f_sel [E] and scalars [L_EP, routing confidence] (device tensors)."""
        T = int(logits.shape[0])
        _expect(logits, (T, self.E), torch.float32, "logits")
        _expect(topk_idx, (T, self.k), torch.int32, "topk_idx")
        p_mean = torch.empty(self.E, dtype=torch.float32, device=self.device)
        f_sel = torch.empty(self.E, dtype=torch.float32, device=self.device)
        scalars = torch.empty(2, dtype=torch.float32, device=self.device)
        moe_router_stats(self.handle, logits, topk_idx, T, n_groups, p_mean, f_sel, scalars,
                         self.workspace(T), stream)
        return p_mean, f_sel, scalars

    def forward_save(self, x, out=None, saved=None, stream=None):
        """Training forward (bf16): (out, saved) with `saved` the fp32 pre-activations that
        backward(..., saved=saved) reads instead of recomputing them."""
        T = self._rows(x)
        ws = self.workspace(T)
        if out is None:
            out = torch.empty_like(x)
        _expect(out, x.shape, x.dtype, "out")
        if saved is None:
            saved = torch.empty(moe_saved_size(self.handle, T) // 4, dtype=torch.float32,
                                device=self.device)
        moe_forward_save(self.handle, x, T, out, saved, ws, stream)
        return out, saved

    def backward(self, x, dout, stream=None, grads=None, saved=None, overwrite=False):
        """dict of fp32 gradients dx, dw_router, dw_gate, dw_up, dw_down (device tensors); the
        weight gradients are added to `grads`' tensors when given (new zeroed ones if not),
        or set when `overwrite`.  With `saved` (from forward_save of the same x) the
        pre-activations are not recomputed."""
        T = self._rows(x)
        _expect(dout, x.shape, x.dtype, "dout")
        need = moe_backward_workspace_size(self.handle, T)
        if self.bw_ws is None or self.bw_ws.numel() < need:
            self.bw_ws = torch.empty(need, dtype=torch.uint8, device=self.device)
            moe_workspace_init(self.handle, self.bw_ws)
        G = self.E + int(self.cfg.n_shared)
        f = int(self.cfg.d_ff)
        kw = dict(dtype=torch.float32, device=self.device)
        if grads is not None:
            g = dict(grads)
            g["dx"] = torch.empty((T, self.d), **kw)
        elif overwrite:  # every element is written
            g = dict(dx=torch.empty((T, self.d), **kw),
                     dw_router=torch.empty((self.E, self.d), **kw),
                     dw_gate=torch.empty((G, f, self.d), **kw),
                     dw_up=torch.empty((G, f, self.d), **kw),
                     dw_down=torch.empty((G, self.d, f), **kw))
        else:  # the weight gradients accumulate: start them at zero
            g = dict(dx=torch.empty((T, self.d), **kw),
                     dw_router=torch.zeros((self.E, self.d), **kw),
                     dw_gate=torch.zeros((G, f, self.d), **kw),
                     dw_up=torch.zeros((G, f, self.d), **kw),
                     dw_down=torch.zeros((G, self.d, f), **kw))
        for name, shape in (("dw_router", (self.E, self.d)), ("dw_gate", (G, f, self.d)),
                            ("dw_up", (G, f, self.d)), ("dw_down", (G, self.d, f))):
            _expect(g[name], shape, torch.float32, name)
        if overwrite:
            moe_backward_ex(self.handle, x, T, dout, saved, MOE_BACKWARD_OVERWRITE, g["dx"],
                            g["dw_router"], g["dw_gate"], g["dw_up"], g["dw_down"], self.bw_ws,
                            stream)
        elif saved is not None:
            moe_backward_saved(self.handle, x, T, dout, saved, g["dx"], g["dw_router"],
                               g["dw_gate"], g["dw_up"], g["dw_down"], self.bw_ws, stream)
        else:
            moe_backward(self.handle, x, T, dout, g["dx"], g["dw_router"], g["dw_gate"],
                         g["dw_up"], g["dw_down"], self.bw_ws, stream)
        return g

    def expert_health(self, n_tokens, stream=None):
        """act_rms [G], param_norm [G], ratios [2] of the last forward of n_tokens tokens."""
        G = self.E + int(self.cfg.n_shared)
        act = torch.empty(G, dtype=torch.float32, device=self.device)
        par = torch.empty(G, dtype=torch.float32, device=self.device)
        ratios = torch.empty(2, dtype=torch.float32, device=self.device)
        moe_expert_health(self.handle, n_tokens, act, par, ratios, self.workspace(n_tokens),
                          stream)
        return act, par, ratios

    def gemm_clock_mhz(self, stream=None) -> tuple:
        """(up, down) effective SM clock of the forward's expert GEMMs since the last call, for
        forwards run with MOE_OPTION_GEMM_CLOCK set (see moe_gemm_clock)."""
        return moe_gemm_clock(self.handle, self.ws, stream)

    def device_status(self, stream=None) -> int:
        """Device status of the forward's and the backward's workspaces (0: no bounded wait
        gave up in either)."""
        st = 0
        for ws in (self.ws, self.bw_ws):
            if ws is not None:
                st = st or moe_device_status(self.handle, ws, stream)
        return st

    def close(self):
        if self.handle is not None:
            moe_layer_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

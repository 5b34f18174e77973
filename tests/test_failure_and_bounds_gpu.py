"""Failure detection and out-of-bounds writes (GPU).

* A bounded device wait that runs out (the library's self-test kernel waits on an mbarrier and
  a flag that nothing signals) is reported by moe_device_status as MOE_ERR_DEVICE_TIMEOUT; the
  context stays usable and the next forward is unchanged.  Nothing faults or traps.
* Canaries: output, workspace and routing buffers are carved out of larger buffers whose
  margins hold a fill pattern; a forward and a routing call must leave every margin intact.
"""
import time

import pytest
import torch

from sparse_moe_layer_warp_b200 import (MoEError, moe_forward, moe_route,
                                        moe_selftest_wait_timeout, moe_workspace_init,
                                        moe_workspace_size, synth)
from tests.helpers import make_layer

pytestmark = pytest.mark.gpu

MOE_ERR_DEVICE_TIMEOUT = 6


def test_device_timeout_reported_and_context_survives(cuda_ok):
    w = synth.WORKLOADS["tiny_fp32"].replace(dtype="bf16", T=40, d=256, E=32, k=4, f=128)
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp)
    ref = layer.forward(inp.x).clone()
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    t0 = time.monotonic()
    moe_selftest_wait_timeout(layer.handle, layer.ws, 20000)  # two waits of 20 ms each
    assert layer.device_status() == MOE_ERR_DEVICE_TIMEOUT
    assert time.monotonic() - t0 < 5.0
    assert layer.device_status() == 0  # reading the word clears it
    out = layer.forward(inp.x)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    assert layer.device_status() == 0


def test_selftest_rejects_bad_limits(cuda_ok):
    w = synth.WORKLOADS["tiny_fp32"].replace(dtype="bf16", T=8, d=256, E=16, k=2, f=128)
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp)
    layer.workspace(w.T)
    for bad in (0, 2_000_001):
        with pytest.raises(MoEError):
            moe_selftest_wait_timeout(layer.handle, layer.ws, bad)


def _guarded(n, dtype, fill, margin=4096):
    """A tensor of n elements inside a buffer with `margin` elements of `fill` on each side."""
    big = torch.full((n + 2 * margin,), fill, dtype=dtype, device="cuda")
    return big, big[margin:margin + n]


def _margins_intact(big, n, fill, margin=4096):
    return bool((big[:margin] == fill).all()) and bool((big[margin + n:] == fill).all())


@pytest.mark.parametrize("kw", [
    {"dtype": "bf16", "T": 16, "d": 512, "E": 64, "k": 8, "f": 256},     # decode routing, gather4
    {"dtype": "bf16", "T": 300, "d": 512, "E": 32, "k": 8, "f": 256},    # row gather, 1-CTA GEMMs
    {"dtype": "bf16", "T": 700, "d": 768, "E": 8, "k": 4, "f": 512},     # CTA-pair GEMMs
    {"dtype": "bf16", "T": 1100, "d": 256, "E": 41, "k": 3, "f": 128},   # token-major router
    {"dtype": "f32", "T": 100},
])
def test_no_writes_outside_buffers(cuda_ok, kw):
    w = synth.WORKLOADS["tiny_fp32"].replace(**kw)
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp)
    T, d, E, k = w.T, w.d, w.E, w.k
    ref = layer.forward(inp.x).clone()
    torch.cuda.synchronize()

    # workspace: 256-byte aligned slice of a byte buffer filled with 0xA5
    need = moe_workspace_size(layer.handle, T)
    ws_big, ws = _guarded(need, torch.uint8, 0xA5)
    assert ws.data_ptr() % 256 == 0
    moe_workspace_init(layer.handle, ws)
    # output: bit pattern 0x7BAD (a finite bf16 / half of an fp32 word) around the rows
    odt = torch.int16 if w.dtype == "bf16" else torch.int32
    out_big, out_flat = _guarded(T * d, odt, 0x7BAD)
    out = out_flat.view(inp.x.dtype).view(T, d)
    moe_forward(layer.handle, inp.x, T, out, ws)
    torch.cuda.synchronize()
    assert _margins_intact(out_big, T * d, 0x7BAD)
    assert _margins_intact(ws_big, need, 0xA5)
    assert torch.equal(out, ref)

    # routing outputs
    bufs = {}
    shapes = {"logits": (T * E, torch.int32), "idx": (T * k, torch.int32),
              "gate": (T * k, torch.int32), "counts": (E, torch.int32),
              "offsets": (E + 1, torch.int32), "perm": (T * k, torch.int32),
              "slot_row": (T * k, torch.int32)}
    for name, (n, dt) in shapes.items():
        bufs[name] = _guarded(n, dt, 0x5EED)
    v = {name: b[1] for name, b in bufs.items()}
    moe_route(layer.handle, inp.x, T, v["logits"].view(torch.float32), v["idx"],
              v["gate"].view(torch.float32), v["counts"], v["offsets"], v["perm"],
              v["slot_row"], ws)
    torch.cuda.synchronize()
    for name, (n, _) in shapes.items():
        assert _margins_intact(bufs[name][0], n, 0x5EED), name
    assert _margins_intact(ws_big, need, 0xA5)
    assert int(v["offsets"][E]) == T * k
    assert layer.device_status() == 0


@pytest.mark.parametrize("kw", [
    {"dtype": "bf16", "T": 16, "d": 256, "E": 64, "k": 8, "f": 256},     # decode routing, 1-CTA
    {"dtype": "bf16", "T": 200, "d": 256, "E": 16, "k": 4, "f": 256,     # pair weight gradients
     "bias": "zipf"},
    {"dtype": "bf16", "T": 300, "d": 256, "E": 8, "k": 4, "f": 512},     # pair dgrad + fused tail
    {"dtype": "f32", "T": 40},
])
def test_backward_no_writes_outside_buffers(cuda_ok, kw):
    """moe_backward writes only inside dx, the four gradient buffers and its workspace; the
    gradient rows of experts no token chose keep their previous contents."""
    from sparse_moe_layer_warp_b200 import moe_backward, moe_backward_workspace_size
    w = synth.WORKLOADS["tiny_fp32"].replace(**kw)
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp)
    dout = synth.make_x(w, w.T, device="cuda", seed=5)
    ref = layer.backward(inp.x, dout)
    counts = layer.route(x=inp.x)["counts"]
    torch.cuda.synchronize()
    T, d, E, f = w.T, w.d, w.E, w.f
    G = E + w.n_shared
    need = moe_backward_workspace_size(layer.handle, T)
    ws_big, ws = _guarded(need, torch.uint8, 0xA5)
    moe_workspace_init(layer.handle, ws)
    sizes = {"dx": T * d, "dw_router": E * d, "dw_gate": G * f * d, "dw_up": G * f * d,
             "dw_down": G * d * f}
    fill = 0x3F800000  # 1.0f: the gradients accumulate onto ones
    bufs = {n: _guarded(m, torch.int32, fill) for n, m in sizes.items()}
    v = {n: b[1].view(torch.float32) for n, b in bufs.items()}
    moe_backward(layer.handle, inp.x, T, dout, v["dx"], v["dw_router"], v["dw_gate"], v["dw_up"],
                 v["dw_down"], ws)
    torch.cuda.synchronize()
    assert _margins_intact(ws_big, need, 0xA5)
    for n, m in sizes.items():
        assert _margins_intact(bufs[n][0], m, fill), n
    # dx is overwritten; the weight gradients are added to the ones
    assert torch.equal(v["dx"].view(T, d), ref["dx"])
    unchosen = torch.nonzero(counts == 0).flatten()
    for n in ("dw_router", "dw_gate", "dw_up", "dw_down"):
        got = v[n].view(ref[n].shape)
        # one fp32 addition onto 1.0: |(1 + r) - 1 - r| <= 2^-24 (1 + |r|)
        tol = 1.2e-7 * (1.0 + ref[n].abs().max().item())
        assert torch.allclose(got - 1.0, ref[n], rtol=0, atol=tol), n
        if len(unchosen):
            assert (got[unchosen] == 1.0).all(), n


def test_backward_rejects_bad_arguments(cuda_ok):
    from sparse_moe_layer_warp_b200 import moe_backward, moe_backward_workspace_size
    w = synth.WORKLOADS["tiny_fp32"].replace(dtype="bf16", T=16, d=256, E=16, k=2, f=128)
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp)
    T, d, E, f, G = w.T, w.d, w.E, w.f, w.E + 1
    ws = torch.zeros(moe_backward_workspace_size(layer.handle, T), dtype=torch.uint8,
                     device="cuda")
    moe_workspace_init(layer.handle, ws)
    dout = synth.make_x(w, T, device="cuda", seed=6)
    g = {"dx": torch.zeros(T, d, device="cuda"), "dwr": torch.zeros(E, d, device="cuda"),
         "dwg": torch.zeros(G, f, d, device="cuda"), "dwu": torch.zeros(G, f, d, device="cuda"),
         "dwd": torch.zeros(G, d, f, device="cuda")}

    def call(x=inp.x, n=T, dx=g["dx"], wsb=ws):
        moe_backward(layer.handle, x, n, dout, dx, g["dwr"], g["dwg"], g["dwu"], g["dwd"], wsb)

    with pytest.raises(MoEError):
        call(n=T + 1)                               # more tokens than max_tokens
    with pytest.raises(MoEError):
        call(wsb=ws[:-256])                          # workspace too small
    with pytest.raises(MoEError):
        call(wsb=ws[16:])                            # workspace not 256-byte aligned
    dx_big = torch.zeros(T * d + 4, device="cuda")
    with pytest.raises(MoEError):
        call(dx=dx_big[1:1 + T * d].view(T, d))      # dx not 16-byte aligned
    from sparse_moe_layer_warp_b200 import moe_backward_ex
    with pytest.raises(MoEError):                   # unknown flag bits
        moe_backward_ex(layer.handle, inp.x, T, dout, None, 2, g["dx"], g["dwr"], g["dwg"],
                        g["dwu"], g["dwd"], ws)
    call()                                          # the valid call still works
    torch.cuda.synchronize()
    assert layer.device_status() == 0


def test_training_pair_bounds_and_arguments(cuda_ok):
    """moe_forward_save writes inside `saved` only; short, misaligned or fp32-layer calls
    of the training pair are rejected before any launch."""
    from sparse_moe_layer_warp_b200 import (moe_backward_saved, moe_backward_workspace_size,
                                            moe_forward_save, moe_saved_size)
    w = synth.WORKLOADS["tiny_fp32"].replace(dtype="bf16", T=50, d=256, E=16, k=4, f=128)
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp)
    T, d = w.T, w.d
    n = moe_saved_size(layer.handle, T) // 4
    assert n == 2 * T * (w.k + w.n_shared) * w.f
    big, saved_i = _guarded(n, torch.int32, 0x5EED)
    saved = saved_i.view(torch.float32)
    out = torch.empty_like(inp.x)
    ws = layer.workspace(T)
    moe_forward_save(layer.handle, inp.x, T, out, saved, ws)
    torch.cuda.synchronize()
    assert _margins_intact(big, n, 0x5EED)
    assert torch.equal(out, layer.forward(inp.x))
    with pytest.raises(MoEError):
        moe_forward_save(layer.handle, inp.x, T, out, saved[:-4], ws)      # too short
    with pytest.raises(MoEError):
        moe_forward_save(layer.handle, inp.x, T, out, big.view(torch.float32)[1:1 + n], ws)
    bws = torch.empty(moe_backward_workspace_size(layer.handle, T), dtype=torch.uint8,
                      device="cuda")
    moe_workspace_init(layer.handle, bws)
    G = w.E + 1
    gr = [torch.zeros(T, d, device="cuda"), torch.zeros(w.E, d, device="cuda"),
          torch.zeros(G, w.f, d, device="cuda"), torch.zeros(G, w.f, d, device="cuda"),
          torch.zeros(G, d, w.f, device="cuda")]
    dout = synth.make_x(w, T, device="cuda", seed=9)
    with pytest.raises(MoEError):
        moe_backward_saved(layer.handle, inp.x, T, dout, saved[:-4], *gr, bws)
    moe_backward_saved(layer.handle, inp.x, T, dout, saved, *gr, bws)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    # the fp32 layer has no training pair
    w32 = synth.WORKLOADS["tiny_fp32"]
    inp32 = synth.make_inputs(w32, device="cuda")
    layer32 = make_layer(inp32)
    s32 = torch.empty(moe_saved_size(layer32.handle, w32.T) // 4, device="cuda")
    with pytest.raises(MoEError):
        moe_forward_save(layer32.handle, inp32.x, w32.T, torch.empty_like(inp32.x), s32,
                         layer32.workspace(w32.T))

"""The allocation-free router entry point (moe_router_logits_static).

Some callers cannot allocate device memory -- for example a plugin host that only hands
over input and output buffers -- so this
entry point keeps its scratch in the library's own static device buffer instead of a
caller workspace.  These tests call it through the C ABI and check it against the regular
workspace-based routing call, twice in a row (the shared buffer keeps the previous call's
contents).  The file is named to be collected last, and passes alone or after the others.
"""
import ctypes

import pytest
import torch

from sparse_moe_layer_warp_b200 import binding, synth
from tests.helpers import make_layer

pytestmark = pytest.mark.gpu


def _workspace_logits(layer, x):
    r = layer.route(x=x, want_logits=True)
    torch.cuda.synchronize()
    return r["logits"]


def _assert_same_logits(out, want, x, w_router):
    # both calls accumulate x . W_r in fp32, possibly in different orders (bf16 decode
    # batches route through the one-launch decode router): each is within d * 2^-24 *
    # sum_i |x_i w_i| of the exact value, so they are within twice that of each other
    bound = 2 * x.shape[1] * 2.0**-24 * (x.double().abs() @ w_router.double().abs().T)
    assert torch.isfinite(out).all()
    assert ((out.double() - want.double()).abs() <= bound).all()


@pytest.mark.parametrize("T,E,d,dtype", [(16, 288, 4096, "bf16"), (5, 40, 512, "bf16"),
                                         (64, 96, 1024, "bf16"), (9, 16, 256, "f32")])
def test_static_scratch_router_matches_workspace_router(cuda_ok, T, E, d, dtype):
    w = synth.Workload("noalloc", T=T, d=d, E=E, k=4, f=128, dtype=dtype, seed=T)
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp)
    ref = _workspace_logits(layer, inp.x)
    x2 = synth.make_x(w, T, device="cuda", seed=99)
    ref2 = _workspace_logits(layer, x2)
    for x, want in ((inp.x, ref), (x2, ref2), (inp.x, ref)):  # consecutive calls
        out = torch.full((T, E), float("nan"), device="cuda", dtype=torch.float32)
        binding.moe_router_logits_static(layer.handle, x, T, out)
        torch.cuda.synchronize()
        _assert_same_logits(out, want, x, inp.w_router)


def test_static_scratch_router_rejects_oversized_requests(cuda_ok):
    w = synth.Workload("noalloc", T=65, d=4096, E=288, k=8, f=128)
    inp = synth.make_inputs(w, device="cuda")
    layer = make_layer(inp)
    out = torch.empty((65, 288), device="cuda", dtype=torch.float32)
    lib = binding.load_library()
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.moe_router_logits_static(layer.handle, ctypes.c_void_p(inp.x.data_ptr()), 65,
                                      ctypes.c_void_p(out.data_ptr()), st)
    assert rc == binding.MOE_ERR_UNSUPPORTED  # more than 64 tokens
    big = synth.Workload("noalloc", T=64, d=4096, E=600, k=8, f=128)
    inp2 = synth.make_inputs(big, device="cuda")
    layer2 = make_layer(inp2)
    out2 = torch.empty((64, 600), device="cuda", dtype=torch.float32)
    rc = lib.moe_router_logits_static(layer2.handle, ctypes.c_void_p(inp2.x.data_ptr()), 64,
                                      ctypes.c_void_p(out2.data_ptr()), st)
    assert rc == binding.MOE_ERR_UNSUPPORTED  # 16 splits x 64 x 600 x 4 B > 2 MiB
    # a request that fits still works after the rejected ones
    rc = lib.moe_router_logits_static(layer2.handle, ctypes.c_void_p(inp2.x.data_ptr()), 8,
                                      ctypes.c_void_p(out2.data_ptr()), st)
    assert rc == binding.MOE_OK
    torch.cuda.synchronize()
    x8 = inp2.x[:8].contiguous()
    ref = _workspace_logits(layer2, x8)
    _assert_same_logits(out2[:8], ref, x8, inp2.w_router)

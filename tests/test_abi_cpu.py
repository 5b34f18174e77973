"""C-ABI checks that need no GPU: the library loads, exports every symbol the header
declares, and rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

from sparse_moe_layer_warp_b200 import binding
from sparse_moe_layer_warp_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return binding.load_library()


def _declared():
    text = open(os.path.join(ROOT, "include", "moe_layer.h")).read()
    return set(re.findall(r"^\S[^\n(]*?\b(moe_\w+)\s*\(", text, flags=re.M))


def test_header_and_binding_agree():
    assert _declared() == set(binding.EXPORTS)


def test_header_constants_match_binding():
    """Status codes, dtype codes, flags and the profile stage count are the header's values."""
    text = open(os.path.join(ROOT, "include", "moe_layer.h")).read()
    enums = dict((n, int(v)) for n, v in re.findall(r"\b(MOE_[A-Z0-9_]+)\s*=\s*(\d+)", text))
    defines = dict((n, int(v)) for n, v in
                   re.findall(r"^#define\s+(MOE_[A-Z0-9_]+)\s+(\d+)u?\s*$", text, flags=re.M))
    assert len(enums) == 9 and len(defines) == 6
    for name, value in {**enums, **defines}.items():
        assert getattr(binding, name) == value, name
    assert len(binding.PROFILE_STAGE_NAMES) == binding.MOE_PROFILE_STAGES


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for s in range(7):
        assert binding.status_string(s) not in ("", "unknown status")
    assert binding.status_string(99) == "unknown status"


def test_init_rejects_bad_config_without_device(lib):
    cfg = binding.moe_config(16, 4096, 288, 8, 1280, 1, binding.MOE_BF16, 1.0)
    w = binding.moe_weights(16, 0, 32, 48, 64)
    h = ctypes.c_void_p()
    assert lib.moe_layer_init(None, ctypes.byref(w), ctypes.byref(h)) == binding.MOE_ERR_INVALID_ARG
    bad = binding.moe_config(16, 4096, 288, 300, 1280, 1, binding.MOE_BF16, 1.0)  # k > E
    assert lib.moe_layer_init(ctypes.byref(bad), ctypes.byref(w), ctypes.byref(h)) == binding.MOE_ERR_INVALID_ARG
    bad = binding.moe_config(16, 4096, 288, 8, 1280, 2, binding.MOE_BF16, 1.0)  # n_shared 2
    assert lib.moe_layer_init(ctypes.byref(bad), ctypes.byref(w), ctypes.byref(h)) == binding.MOE_ERR_INVALID_ARG
    bad = binding.moe_config(16, 4000, 288, 8, 1280, 1, binding.MOE_BF16, 1.0)  # d % 128
    assert lib.moe_layer_init(ctypes.byref(bad), ctypes.byref(w), ctypes.byref(h)) == binding.MOE_ERR_UNSUPPORTED
    bad = binding.moe_config(16, 4096, 2048, 8, 1280, 1, binding.MOE_BF16, 1.0)  # E > 1024
    assert lib.moe_layer_init(ctypes.byref(bad), ctypes.byref(w), ctypes.byref(h)) == binding.MOE_ERR_UNSUPPORTED
    bad = binding.moe_config(16, 4096, 288, 40, 1280, 1, binding.MOE_BF16, 1.0)  # k > 32
    assert lib.moe_layer_init(ctypes.byref(bad), ctypes.byref(w), ctypes.byref(h)) == binding.MOE_ERR_UNSUPPORTED
    wmis = binding.moe_weights(16, 0, 33, 48, 64)  # misaligned w_gate
    assert lib.moe_layer_init(ctypes.byref(cfg), ctypes.byref(wmis), ctypes.byref(h)) == binding.MOE_ERR_ALIGNMENT
    wnull = binding.moe_weights(16, 0, 0, 48, 64)
    assert lib.moe_layer_init(ctypes.byref(cfg), ctypes.byref(wnull), ctypes.byref(h)) == binding.MOE_ERR_INVALID_ARG


def test_null_handle_calls_rejected(lib):
    assert lib.moe_workspace_size(None, 16) == 0
    assert lib.moe_forward(None, None, 16, None, None, 0, None) == binding.MOE_ERR_INVALID_ARG
    assert lib.moe_layer_destroy(None) == binding.MOE_ERR_INVALID_ARG
    assert lib.moe_route(None, None, 1, None, None, None, None, None, None, None, None, 0, None) == binding.MOE_ERR_INVALID_ARG
    # backward and training-pair entry points
    assert lib.moe_backward_workspace_size(None, 16) == 0
    assert lib.moe_saved_size(None, 16) == 0
    assert lib.moe_backward(None, None, 1, None, None, None, None, None, None, None, 0,
                            None) == binding.MOE_ERR_INVALID_ARG
    assert lib.moe_backward_saved(None, None, 1, None, None, 0, None, None, None, None, None,
                                  None, 0, None) == binding.MOE_ERR_INVALID_ARG
    assert lib.moe_backward_ex(None, None, 1, None, None, 0, 0, None, None, None, None, None,
                               None, 0, None) == binding.MOE_ERR_INVALID_ARG
    assert lib.moe_forward_save(None, None, 1, None, None, 0, None, 0,
                                None) == binding.MOE_ERR_INVALID_ARG
    assert lib.moe_expert_health(None, 1, None, None, None, None, 0,
                                 None) == binding.MOE_ERR_INVALID_ARG
    assert lib.moe_set_option(None, binding.MOE_OPTION_H_HANDOVER,
                              0) == binding.MOE_ERR_INVALID_ARG


def test_binding_refuses_strided_and_host_tensors(lib):
    """The binding hands raw pointers to a library that reads dense device memory: a strided
    view or a host tensor is refused in Python, before any library call or launch."""
    import torch

    strided = torch.zeros(8, 4).t()
    with pytest.raises(ValueError, match="contiguous"):
        binding._p(strided)
    with pytest.raises(ValueError, match="CUDA tensors"):
        binding._p(torch.zeros(8))
    assert binding._p(None) is None
    # the weights of a layer go through the same check
    cfg = binding.moe_config(16, 256, 16, 2, 128, 1, binding.MOE_F32, 1.0)
    w = [torch.zeros(16, 256), None, torch.zeros(17, 128, 256), torch.zeros(17, 128, 256),
         torch.zeros(17, 256, 128)]
    with pytest.raises(ValueError, match="CUDA tensors"):
        binding.moe_layer_init(cfg, *w)


def test_layer_class_checks_shapes_and_types(lib):
    """MoELayer passes only pointers to the library, so it checks every weight's shape and
    type against the configuration first (a mismatch would be read out of bounds)."""
    import torch

    E, d, f = 16, 256, 128
    good = dict(w_router=torch.zeros(E, d), router_bias=torch.zeros(E),
                w_gate=torch.zeros(E + 1, f, d), w_up=torch.zeros(E + 1, f, d),
                w_down=torch.zeros(E + 1, d, f))
    bad_cases = [
        dict(w_gate=torch.zeros(E, f, d)),                    # no room for the shared expert
        dict(w_up=torch.zeros(E + 1, f, d + 8)),              # wrong d
        dict(w_down=torch.zeros(E + 1, f, d)),                # transposed down projection
        dict(router_bias=torch.zeros(E, dtype=torch.float64)),
        dict(w_up=torch.zeros(E + 1, f, d, dtype=torch.bfloat16)),  # mixed types
        dict(w_router=torch.zeros(E, d, dtype=torch.float16)),
    ]
    for change in bad_cases:
        kw = dict(good, **change)
        with pytest.raises(ValueError):
            binding.MoELayer(kw["w_router"], kw["router_bias"], kw["w_gate"], kw["w_up"],
                             kw["w_down"], top_k=2, max_tokens=8)
    # consistent shapes pass the Python checks and reach the pointer check (host tensors)
    with pytest.raises(ValueError, match="CUDA tensors"):
        binding.MoELayer(good["w_router"], good["router_bias"], good["w_gate"], good["w_up"],
                         good["w_down"], top_k=2, max_tokens=8)


def test_expert_parallel_and_option_calls_rejected_on_the_host(lib):
    """The expert-parallel entry points and moe_set_option check their arguments before any
    CUDA call: a null handle, an empty or out-of-range expert slice, a non-bf16 slice."""
    cfg = binding.moe_config(16, 4096, 288, 8, 1280, 1, binding.MOE_BF16, 1.0)
    w = binding.moe_weights(16, 0, 32, 48, 64)
    h = ctypes.c_void_p()
    ep = lib.moe_layer_init_ep
    assert ep(None, ctypes.byref(w), 0, 36, ctypes.byref(h)) == binding.MOE_ERR_INVALID_ARG
    for e0, e1 in ((36, 36), (40, 36), (-1, 36), (0, 289)):
        assert ep(ctypes.byref(cfg), ctypes.byref(w), e0, e1,
                  ctypes.byref(h)) == binding.MOE_ERR_INVALID_ARG, (e0, e1)
    f32 = binding.moe_config(16, 4096, 288, 8, 1280, 1, binding.MOE_F32, 1.0)
    assert ep(ctypes.byref(f32), ctypes.byref(w), 0, 36,
              ctypes.byref(h)) == binding.MOE_ERR_UNSUPPORTED
    assert lib.moe_forward_partial(None, None, 1, None, None, 0, 1, 0, 0, None, None, 0,
                                   None) == binding.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_plan(None, None, 1, 2, None, None, None, None, None, 0,
                           None) == binding.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_pack(None, None, None, None, 1, 2, None, None, None, None, None,
                           None) == binding.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_combine(None, None, None, None, None, 1, 2, None,
                              None) == binding.MOE_ERR_INVALID_ARG
    assert lib.moe_set_option(None, binding.MOE_OPTION_SHARED_SIDE_SMS,
                              32) == binding.MOE_ERR_INVALID_ARG
    mhz = (ctypes.c_double * 2)()
    assert lib.moe_gemm_clock(None, None, 0, mhz, None) == binding.MOE_ERR_INVALID_ARG


def test_expert_range_partition():
    from sparse_moe_layer_warp_b200.expert_parallel import expert_range

    parts = [expert_range(288, q, 8) for q in range(8)]
    assert parts[0] == (0, 36) and parts[-1] == (252, 288)
    assert all(parts[q][1] == parts[q + 1][0] for q in range(7))
    with pytest.raises(ValueError):
        expert_range(288, 0, 7)

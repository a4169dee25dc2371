"""The C-ABI library loads and exports every entry point include/arl2.h declares.

CPU only: no call here reaches the GPU (argument checks return before any
CUDA call).
"""
import ctypes
import os
import re

import pytest

import hybrid_softmax_gated_b200 as arl2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "arl2.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(arl2_[a-z_]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_boundary_calls():
    names = declared_functions()
    for required in ("arl2_create", "arl2_frame_forward", "arl2_state_reset", "arl2_state_get",
                     "arl2_state_set", "arl2_destroy", "arl2_status_string"):
        assert required in names


@pytest.mark.parametrize("name", declared_functions())
def test_library_exports_declared_symbol(name):
    lib = ctypes.CDLL(arl2.library_path())
    assert hasattr(lib, name), name


def test_binding_covers_every_export():
    assert sorted(arl2.EXPORTED) == declared_functions()


def test_version_and_status_strings():
    assert arl2.version() == 10300
    for code in range(0, -8, -1):
        s = arl2._lib.arl2_status_string(code).decode()
        assert s and s != "unknown status"
    assert arl2._lib.arl2_status_string(-99).decode() == "unknown status"


def test_null_arguments_are_rejected_before_any_cuda_call():
    lib = arl2._lib
    h = ctypes.c_void_p()
    assert lib.arl2_create(None, None, ctypes.byref(h)) == -1
    cfg = arl2.Arl2Config(1, 1, 16, 16, 1, None, None, None, 0.0, 0, 0, 0)
    assert lib.arl2_create(ctypes.byref(cfg), None, None) == -1
    assert lib.arl2_create(ctypes.byref(cfg), None, ctypes.byref(h)) == -1  # null weights
    assert lib.arl2_frame_forward(None, None, None, None, None, None, 0, None, None) == -1
    assert lib.arl2_state_reset(None, None) == -1
    assert lib.arl2_state_get(None, None, None) == -1
    assert lib.arl2_state_set(None, None, None) == -1
    assert lib.arl2_phi_apply(None, 0, None, None, None) == -1
    assert lib.arl2_device_status(None, None) == -1
    assert lib.arl2_selftest_wait_timeout(None, 1000, None) == -1
    assert lib.arl2_device_bytes(None) == 0
    assert lib.arl2_kernel_launches(None) == 0
    lib.arl2_destroy(None)


def test_shape_and_alignment_checks_come_before_cuda():
    lib = arl2._lib
    h = ctypes.c_void_p()
    fake = 0x1000  # never dereferenced: validation fails first
    for bad in [(0, 1, 16, 16), (1, 0, 16, 16), (1, 1, 0, 16), (1, 1, 129, 16), (1, 1, 16, 0)]:
        cfg = arl2.Arl2Config(*bad, 1, fake, fake, fake, 0.0, 0, 0, 0)
        assert lib.arl2_create(ctypes.byref(cfg), None, ctypes.byref(h)) == -2
    cfg = arl2.Arl2Config(1, 1, 16, 16, 1, fake + 4, fake, fake, 0.0, 0, 0, 0)
    assert lib.arl2_create(ctypes.byref(cfg), None, ctypes.byref(h)) == -3
    cfg = arl2.Arl2Config(1, 1, 64, 16, 0, fake, fake, fake, 0.0, 0, 0, 0)  # bf16 tensor cores need d=128
    assert lib.arl2_create(ctypes.byref(cfg), None, ctypes.byref(h)) == -7
    cfg = arl2.Arl2Config(1, 1, 16, 16, 7, fake, fake, fake, 0.0, 0, 0, 0)  # bad dtype
    assert lib.arl2_create(ctypes.byref(cfg), None, ctypes.byref(h)) == -1
    cfg = arl2.Arl2Config(1, 1, 16, 16, 1, fake, fake, fake, -1.0, 0, 0)  # bad scale
    assert lib.arl2_create(ctypes.byref(cfg), None, ctypes.byref(h)) == -1


def test_gating_mode_is_validated_before_cuda():
    lib = arl2._lib
    h = ctypes.c_void_p()
    fake = 0x1000
    cfg = arl2.Arl2Config(1, 1, 16, 16, 1, fake, fake, fake, 0.0, 0, 0, 0, 5)  # no such gating
    assert lib.arl2_create(ctypes.byref(cfg), None, ctypes.byref(h)) == -1
    cfg = arl2.Arl2Config(1, 1, 16, 16, 1, fake, fake, fake, 0.0, 0, 0, -1, arl2.ARL2_GATE_ELEMENTWISE)
    assert lib.arl2_create(ctypes.byref(cfg), None, ctypes.byref(h)) == -1  # (max_ctas < 0)


def test_teacher_layer_arguments_are_validated_before_cuda():
    lib = arl2._lib
    h = ctypes.c_void_p()
    K = arl2.Arl2KvConfig
    assert lib.arl2_kv_create(None, None, ctypes.byref(h)) == -1
    cfg = K(1, 1, 16, 16, 4, arl2.ARL2_FP32, 0.0, 0, 0, 0)
    assert lib.arl2_kv_create(ctypes.byref(cfg), None, None) == -1
    for bad in [(0, 1, 16, 16, 4), (1, 0, 16, 16, 4), (1, 1, 0, 16, 4), (1, 1, 129, 16, 4),
                (1, 1, 16, 0, 4), (1, 1, 16, 16, 0), (1, 1, 16, 1 << 20, 1 << 7)]:
        cfg = K(*bad, arl2.ARL2_FP32, 0.0, 0, 0, 0)
        assert lib.arl2_kv_create(ctypes.byref(cfg), None, ctypes.byref(h)) == -2, bad
    cfg = K(1, 1, 64, 16, 4, arl2.ARL2_BF16, 0.0, 0, 0, 0)  # tensor cores need d = 128
    assert lib.arl2_kv_create(ctypes.byref(cfg), None, ctypes.byref(h)) == -7
    cfg = K(1, 1, 16, 16, 4, 9, 0.0, 0, 0, 0)  # no such dtype
    assert lib.arl2_kv_create(ctypes.byref(cfg), None, ctypes.byref(h)) == -1
    cfg = K(1, 1, 16, 16, 4, arl2.ARL2_FP32, -0.5, 0, 0, 0)  # bad scale
    assert lib.arl2_kv_create(ctypes.byref(cfg), None, ctypes.byref(h)) == -1
    cfg = K(1, 1, 16, 16, 4, arl2.ARL2_FP32, 0.0, 0, 3, 0)  # no such impl
    assert lib.arl2_kv_create(ctypes.byref(cfg), None, ctypes.byref(h)) == -1
    assert lib.arl2_kv_frame_forward(None, None, None, None, 0, None, None) == -1
    assert lib.arl2_kv_frame_forward_host(None, None, None, None, 0, None, None) == -1
    assert lib.arl2_kv_reset(None) == -1
    assert lib.arl2_kv_frames(None) == -1
    assert lib.arl2_kv_cache_get(None, None, None, None) == -1
    assert lib.arl2_kv_cache_set(None, None, None, 0, None) == -1
    assert lib.arl2_kv_device_status(None, None) == -1
    assert lib.arl2_kv_device_bytes(None) == 0
    assert lib.arl2_kv_cache_bytes(None) == 0
    assert lib.arl2_kv_kernel_launches(None) == 0
    lib.arl2_kv_destroy(None)


def test_gate_projection_config_is_validated_before_cuda():
    lib = arl2._lib
    h = ctypes.c_void_p()
    fake = 0x1000

    def cfg(hidden, w_gate, b_gate, gating=arl2.ARL2_GATE_HEADWISE, heads=2):
        return arl2.Arl2Config(1, heads, 16, 16, arl2.ARL2_FP32, fake, fake, fake, 0.0, 0, 0, 0, gating,
                               arl2.ARL2_ACCESS_FRAME, hidden, w_gate, b_gate)

    assert lib.arl2_create(ctypes.byref(cfg(32, fake, None)), None, ctypes.byref(h)) == -1  # no bias
    for hidden in (0, 7, 12):
        assert lib.arl2_create(ctypes.byref(cfg(hidden, fake, fake)), None, ctypes.byref(h)) == -2
    assert lib.arl2_create(ctypes.byref(cfg(32, fake, fake, heads=49)), None, ctypes.byref(h)) == -2
    assert lib.arl2_create(ctypes.byref(cfg(32, fake + 8, fake)), None, ctypes.byref(h)) == -3
    assert lib.arl2_create(ctypes.byref(cfg(32, fake, fake + 4)), None, ctypes.byref(h)) == -3
    assert lib.arl2_create(ctypes.byref(cfg(32, fake, fake, gating=arl2.ARL2_GATE_ELEMENTWISE)), None,
                           ctypes.byref(h)) == -7
    assert lib.arl2_gates_apply(None, None, None, None, None) == -1
    assert lib.arl2_frame_forward_hidden(None, None, None, None, None, 1, None, None) == -1
    assert lib.arl2_frame_forward_hidden_host(None, None, None, None, None, 1, None, None) == -1


def test_noalloc_update_arguments_are_validated_before_cuda():
    lib = arl2._lib
    fake = ctypes.c_void_p(0x1000)  # never dereferenced: validation fails first
    f = lambda *dims, dt=arl2.ARL2_FP32, ptr=fake: lib.arl2_state_update_noalloc(
        *dims, dt, ptr, ptr, ptr, ptr, ptr, ptr, ptr, None)
    assert f(1, 1, 16, 16, ptr=None) == -1
    assert f(1, 1, 16, 16, dt=9) == -1
    for bad in [(0, 1, 16, 16), (1, 0, 16, 16), (1, 1, 0, 16), (1, 1, 129, 16), (1, 1, 16, 0),
                (1, 70000, 1, 1), (70000, 1, 1, 1), (1, 1025, 1, 1)]:
        assert f(*bad) == -2, bad
    tokens = arl2.NOALLOC_MAX_ELEMENTS // (12 * 128) + 1
    assert f(1, 12, 128, tokens) == -2
    assert f(1, 1, 16, 16, ptr=ctypes.c_void_p(0x1004)) == -3

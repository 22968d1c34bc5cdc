"""The C ABI without a GPU: the library loads, exports every symbol that
include/moe.h declares, and rejects bad arguments on the host with the
documented status codes before touching the device."""
import ctypes
import os
import re

import pytest

import sparse_mixture_experts_08_b200 as moe
from sparse_mixture_experts_08_b200.moe import MoEAtomicConfig, MoEConfig

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    with open(os.path.join(ROOT, "include", "moe.h")) as fh:
        text = fh.read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert _declared() == sorted(moe.moe.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = moe.moe.lib()
    for name in _declared():
        assert hasattr(lib, name), name


def test_struct_layouts_match_header():
    assert ctypes.sizeof(MoEConfig) == 40
    assert ctypes.sizeof(MoEAtomicConfig) == 28
    assert moe.moe.LIS_BYTES == 16


def test_status_strings():
    lib = moe.moe.lib()
    for code in range(7):
        assert moe.moe_status_string(code)
    assert moe.moe_status_string(99) == "unknown status"


def _ws_size(**kw):
    base = dict(T=64, d=128, f=256, m=8, k=2, n_shared=0, f_shared=0, dtype=moe.F32, act=moe.SWIGLU, renormalize=0)
    base.update(kw)
    c = MoEConfig(**base)
    n = ctypes.c_size_t(0)
    return moe.moe.lib().moe_workspace_size(ctypes.byref(c), ctypes.byref(n)), n.value


@pytest.mark.parametrize("kw,code", [
    (dict(T=0), moe.ERR_INVALID_ARG),        # LIS undefined for an empty batch
    (dict(k=9), moe.ERR_INVALID_ARG),        # k > m
    (dict(k=0), moe.ERR_INVALID_ARG),
    (dict(dtype=7), moe.ERR_INVALID_ARG),
    (dict(act=5), moe.ERR_INVALID_ARG),
    (dict(renormalize=2), moe.ERR_INVALID_ARG),
    (dict(d=100), moe.ERR_UNSUPPORTED),      # d % 8
    (dict(f=12), moe.ERR_UNSUPPORTED),
    (dict(m=2048, k=2), moe.ERR_UNSUPPORTED),
    (dict(m=64, k=33), moe.ERR_UNSUPPORTED),
    (dict(n_shared=1, f_shared=0), moe.ERR_INVALID_ARG),
    (dict(n_shared=9, f_shared=64), moe.ERR_UNSUPPORTED),
])
def test_config_validation(kw, code):
    rc, _ = _ws_size(**kw)
    assert rc == code


def test_workspace_size_grows_with_tokens():
    rc1, a = _ws_size(T=64)
    rc2, b = _ws_size(T=640)
    assert rc1 == rc2 == moe.OK and b > a > 0
    assert moe.moe.lib().moe_workspace_size(None, None) == moe.ERR_INVALID_ARG


def _fake(addr):
    return ctypes.c_void_p(addr)


def test_calls_reject_bad_pointers_and_small_workspace_before_launch():
    lib = moe.moe.lib()
    c = MoEConfig(64, 128, 256, 8, 2, 0, 0, moe.BF16, moe.SWIGLU, 0)
    ok_ws = _fake(1 << 20)
    a = _fake(1 << 24)
    # missing outputs
    assert lib.moe_route(ctypes.byref(c), a, a, None, None, None, None, None, ok_ws, 1 << 30, None) == \
        moe.ERR_INVALID_ARG
    # misaligned pointer
    assert lib.moe_route(ctypes.byref(c), _fake((1 << 24) + 4), a, None, None, None, a, a, ok_ws, 1 << 30, None) == \
        moe.ERR_INVALID_ARG
    # workspace too small / misaligned
    assert lib.moe_route(ctypes.byref(c), a, a, None, None, None, a, a, ok_ws, 16, None) == moe.ERR_WORKSPACE
    assert lib.moe_layer_forward(ctypes.byref(c), a, a, None, a, a, a, None, None, None, a, None, None, None, None,
                                 None, None, None, None, None, _fake((1 << 20) + 16), 1 << 30, None) == \
        moe.ERR_INVALID_ARG
    assert lib.moe_layer_forward(ctypes.byref(c), a, a, None, a, a, a, None, None, None, a, None, None, None, None,
                                 None, None, None, None, None, ok_ws, 1024, None) == moe.ERR_WORKSPACE
    # a misaligned inspection output (the permutation copies) is rejected too
    assert lib.moe_layer_forward(ctypes.byref(c), a, a, None, a, a, a, None, None, None, a, None, None, None, None,
                                 None, None, _fake((1 << 24) + 8), None, None, ok_ws, 1 << 30, None) == \
        moe.ERR_INVALID_ARG
    # SwiGLU needs w_up
    assert lib.moe_grouped_ffn(ctypes.byref(c), a, a, a, None, a, None, None, a, ok_ws, 1 << 30, None) == \
        moe.ERR_INVALID_ARG
    # task weights need perm
    assert lib.moe_grouped_ffn(ctypes.byref(c), a, a, a, a, a, a, None, a, ok_ws, 1 << 30, None) == \
        moe.ERR_INVALID_ARG
    assert lib.moe_permute(ctypes.byref(c), a, a, None, a, a, a, ok_ws, 1 << 30, None) == moe.ERR_INVALID_ARG
    assert lib.moe_combine(ctypes.byref(c), a, None, None, a, None) == moe.ERR_INVALID_ARG
    assert lib.moe_read_device_status(None, None, None) == moe.ERR_INVALID_ARG


@pytest.mark.parametrize("kw,code", [
    (dict(K=4097), moe.ERR_UNSUPPORTED),
    (dict(Nr=64, Nc=64, K=4097), moe.ERR_INVALID_ARG),   # more than the grid holds
    (dict(K=65), moe.OK),
    (dict(K=4096), moe.OK),
    (dict(Nr=32), moe.ERR_UNSUPPORTED),
    (dict(Nc=2048), moe.ERR_UNSUPPORTED),
    (dict(dtype=moe.F32), moe.ERR_UNSUPPORTED),
    (dict(act=3), moe.ERR_INVALID_ARG),
    (dict(T=0), moe.ERR_INVALID_ARG),
])
def test_atomic_config_validation(kw, code):
    base = dict(T=16, d=4096, Nr=512, Nc=512, K=64, act=moe.ATOMIC_SILU, dtype=moe.BF16)
    base.update(kw)
    c = MoEAtomicConfig(**base)
    n = ctypes.c_size_t(0)
    assert moe.moe.lib().moe_atomic_workspace_size(ctypes.byref(c), ctypes.byref(n)) == code


def test_atomic_workspace_size_ok():
    c = MoEAtomicConfig(16, 4096, 512, 512, 64, moe.ATOMIC_SILU, moe.BF16)
    assert moe.moe_atomic_workspace_size(c) > 0


def test_debug_wait_limit_hook():
    lib = moe.moe.lib()
    assert lib.moe_debug_set_wait_limit_ns(5) == moe.OK
    assert lib.moe_debug_set_wait_limit_ns(0) == moe.OK
    assert moe.moe_launch_count() >= 0


def test_replica_entry_points_validate_on_the_host():
    lib = moe.moe.lib()
    a = _fake(1 << 24)
    ws = _fake(1 << 20)
    c = MoEConfig(64, 128, 256, 8, 2, 0, 0, moe.BF16, moe.SWIGLU, 0)
    # missing inputs
    assert lib.moe_replica_split(ctypes.byref(c), a, None, a, a, a, None, None, ws, 1 << 30, None) == \
        moe.ERR_INVALID_ARG
    # the replica would be expert 1024
    big = MoEConfig(64, 128, 256, 1024, 2, 0, 0, moe.BF16, moe.SWIGLU, 0)
    assert lib.moe_replica_split(ctypes.byref(big), a, a, a, a, a, None, None, ws, 1 << 30, None) == \
        moe.ERR_UNSUPPORTED
    assert lib.moe_layer_forward_replicated(ctypes.byref(big), a, a, None, a, a, a, None, None, None, a, None, None,
                                            None, None, None, None, None, ws, 1 << 30, None) == moe.ERR_UNSUPPORTED
    # bf16 only
    f32 = MoEConfig(64, 128, 256, 8, 2, 0, 0, moe.F32, moe.SWIGLU, 0)
    assert lib.moe_layer_forward_replicated(ctypes.byref(f32), a, a, None, a, a, a, None, None, None, a, None, None,
                                            None, None, None, None, None, ws, 1 << 30, None) == moe.ERR_UNSUPPORTED
    # the workspace must fit the config with m + 1 experts
    c1 = MoEConfig(64, 128, 256, 9, 2, 0, 0, moe.BF16, moe.SWIGLU, 0)
    n0, n1 = ctypes.c_size_t(0), ctypes.c_size_t(0)
    assert lib.moe_workspace_size(ctypes.byref(c), ctypes.byref(n0)) == moe.OK
    assert lib.moe_workspace_size(ctypes.byref(c1), ctypes.byref(n1)) == moe.OK
    assert n1.value > n0.value
    assert lib.moe_layer_forward_replicated(ctypes.byref(c), a, a, None, a, a, a, None, None, None, a, None, None,
                                            None, None, None, None, None, ws, n0.value, None) == moe.ERR_WORKSPACE


def test_floe_entry_points_validate_on_the_host():
    lib = moe.moe.lib()
    a = _fake(1 << 24)
    ok = MoEConfig(16, 256, 320, 4, 2, 0, 0, moe.BF16, moe.SWIGLU, 0)
    n = ctypes.c_size_t(0)
    assert lib.moe_floe_workspace_size(ctypes.byref(ok), ctypes.byref(n)) == moe.OK and n.value > 0
    for bad in (MoEConfig(16, 256, 320, 4, 2, 0, 0, moe.F32, moe.SWIGLU, 0),   # bf16 only
                MoEConfig(16, 256, 320, 4, 2, 0, 0, moe.BF16, moe.RELU, 0),    # SwiGLU only
                MoEConfig(16, 256, 320, 4, 2, 1, 64, moe.BF16, moe.SWIGLU, 0)):  # no shared experts
        assert lib.moe_floe_workspace_size(ctypes.byref(bad), ctypes.byref(n)) == moe.ERR_UNSUPPORTED
    assert lib.moe_floe_calibrate(ctypes.byref(ok), a, 8, a, ctypes.c_double(1.5), a, a, a, 1 << 30, None) == \
        moe.ERR_INVALID_ARG  # sparsity outside [0, 1]
    assert lib.moe_floe_calibrate(ctypes.byref(ok), a, 0, a, ctypes.c_double(0.9), a, a, a, 1 << 30, None) == \
        moe.ERR_INVALID_ARG  # no calibration tokens
    assert lib.moe_layer_forward_floe(ctypes.byref(ok), a, a, None, a, a, a, None, a, None, None, None, None, None,
                                      a, 1 << 30, None) == moe.ERR_INVALID_ARG  # thresholds missing
    assert lib.moe_layer_forward_floe(ctypes.byref(ok), a, a, None, a, a, a, a, a, None, None, None, None, None,
                                      a, n.value - 256, None) == moe.ERR_WORKSPACE


def test_fp8_entry_points_validate_on_the_host():
    lib = moe.moe.lib()
    a = _fake(1 << 24)
    ok = MoEConfig(16, 256, 320, 4, 2, 1, 64, moe.BF16, moe.SWIGLU, 0)
    n = ctypes.c_size_t(0)
    base = ctypes.c_size_t(0)
    assert lib.moe_fp8_workspace_size(ctypes.byref(ok), ctypes.byref(n)) == moe.OK
    assert lib.moe_workspace_size(ctypes.byref(ok), ctypes.byref(base)) == moe.OK
    # the bf16 workspace plus codes of x and h (bytes) and their row scales
    assert n.value >= base.value + 16 * 2 * (256 + 320 + 8) + 16 * (256 + 64 + 4)
    for bad in (MoEConfig(16, 256, 320, 4, 2, 0, 0, moe.F32, moe.SWIGLU, 0),    # bf16 layers only
                MoEConfig(16, 264, 320, 4, 2, 0, 0, moe.BF16, moe.SWIGLU, 0),   # d % 16
                MoEConfig(16, 256, 328, 4, 2, 0, 0, moe.BF16, moe.SWIGLU, 0),   # f % 16
                MoEConfig(16, 256, 320, 4, 2, 1, 72, moe.BF16, moe.SWIGLU, 0)):  # f_shared % 16
        assert lib.moe_fp8_workspace_size(ctypes.byref(bad), ctypes.byref(n)) == moe.ERR_UNSUPPORTED
    assert lib.moe_fp8_workspace_size(ctypes.byref(ok), ctypes.byref(n)) == moe.OK
    # quantizer: rows of 16-byte multiples only, aligned pointers
    assert lib.moe_quantize_e4m3(4, 24, a, a, a, None) == moe.ERR_UNSUPPORTED
    assert lib.moe_quantize_e4m3(-1, 32, a, a, a, None) == moe.ERR_INVALID_ARG
    assert lib.moe_quantize_e4m3(4, 32, _fake((1 << 24) + 8), a, a, None) == moe.ERR_INVALID_ARG
    assert lib.moe_quantize_e4m3(0, 32, None, None, None, None) == moe.OK
    full = {f: 1 << 24 for f, _ in moe.moe.MoEFp8Experts._fields_}
    wq = moe.moe.MoEFp8Experts(**full)
    call = lambda cfg, w, ws_bytes: lib.moe_layer_forward_fp8(ctypes.byref(cfg), a, a, None, ctypes.byref(w), a, None,
                                                              None, None, None, None, None, None, None, a, ws_bytes,
                                                              None)
    assert call(ok, wq, n.value - 256) == moe.ERR_WORKSPACE
    for missing in ("up_scale", "down", "sh_up"):
        w = moe.moe.MoEFp8Experts(**dict(full, **{missing: None}))
        assert call(ok, w, 1 << 30) == moe.ERR_INVALID_ARG, missing
    relu = MoEConfig(16, 256, 320, 4, 2, 0, 0, moe.BF16, moe.RELU, 0)
    w = moe.moe.MoEFp8Experts(**dict(full, up=None, up_scale=None, sh_gate=None, sh_gate_scale=None, sh_up=None,
                                     sh_up_scale=None, sh_down=None, sh_down_scale=None))
    assert lib.moe_fp8_workspace_size(ctypes.byref(relu), ctypes.byref(n)) == moe.OK
    assert call(relu, w, n.value - 256) == moe.ERR_WORKSPACE   # the pointer set itself is complete for ReLU
    w = moe.moe.MoEFp8Experts(**dict(full, gate=(1 << 24) + 4))
    assert call(ok, w, 1 << 30) == moe.ERR_INVALID_ARG         # codes must be 16-byte aligned


def test_atomic_workspace_holds_the_expert_sort_at_prefill_budgets():
    """From 16384 (token, slot) tasks on, the workspace adds the counting sort of the
    tasks by expert: one int32 run end per expert and one int32 per task."""
    lib = moe.moe.lib()
    n = ctypes.c_size_t(0)

    def size(T, K):
        c = MoEAtomicConfig(T=T, d=4096, Nr=512, Nc=512, K=K, act=moe.ATOMIC_SILU, dtype=moe.BF16)
        assert lib.moe_atomic_workspace_size(ctypes.byref(c), ctypes.byref(n)) == moe.OK
        return n.value

    small = size(16, 64)        # 1024 tasks: the single cooperative launch, no sort
    wide = size(4096, 512)      # 2M tasks
    per_task_no_sort = 3 * 4    # idx, g, coef
    assert wide - small >= (4096 * 512 - 16 * 64) * (per_task_no_sort + 4) + 512 * 512 * 4

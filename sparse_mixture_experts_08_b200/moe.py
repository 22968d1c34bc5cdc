"""Python binding of libmoe.so (the C ABI declared in include/moe.h).

Argument marshalling only: every function has the C entry point's name, takes
torch tensors (device memory) or None for nullable pointers, passes their data
pointers and the CUDA stream through ctypes, and raises MoEError on a non-OK
status. No step of the layer runs here. The library must be built
(``python -m sparse_mixture_experts_08_b200.build``); importing this module
without it fails loudly - there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT, ERR_DEVICE_INDEX = range(7)
F32, BF16 = 0, 1
SWIGLU, RELU = 0, 1
ATOMIC_SILU, ATOMIC_SIGMOID = 0, 1

STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
                4: "MOE_ERR_CUDA", 5: "MOE_ERR_TIMEOUT", 6: "MOE_ERR_DEVICE_INDEX"}

# every symbol include/moe.h declares
EXPORTS = ["moe_workspace_size", "moe_atomic_workspace_size", "moe_route", "moe_histogram_lis", "moe_permute",
           "moe_grouped_ffn", "moe_shared_ffn", "moe_combine", "moe_layer_forward", "moe_atomic_route",
           "moe_atomic_experts", "moe_atomic_forward", "moe_lis_from_counts", "moe_read_device_status", "moe_status_string",
           "moe_debug_set_wait_limit_ns", "moe_debug_set_barrier_extra", "moe_set_stage_events", "moe_launch_count", "moe_route_static",
           "moe_replica_split", "moe_layer_forward_replicated", "moe_floe_pack_down", "moe_floe_calibrate",
           "moe_floe_workspace_size", "moe_layer_forward_floe", "moe_quantize_e4m3", "moe_fp8_workspace_size",
           "moe_layer_forward_fp8"]


class MoEConfig(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("f", ctypes.c_int32), ("m", ctypes.c_int32),
                ("k", ctypes.c_int32), ("n_shared", ctypes.c_int32), ("f_shared", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("act", ctypes.c_int32), ("renormalize", ctypes.c_int32)]


class MoEAtomicConfig(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("Nr", ctypes.c_int32), ("Nc", ctypes.c_int32),
                ("K", ctypes.c_int32), ("act", ctypes.c_int32), ("dtype", ctypes.c_int32)]


LIS_BYTES = 16  # moe_lis_t: int32 max_count, int32 argmax_expert, double lis


class MoEFp8Experts(ctypes.Structure):
    """moe_fp8_experts_t: device pointers to E4M3 codes (uint8) and fp32 row scales."""
    _fields_ = [(name, ctypes.c_void_p) for name in (
        "gate", "gate_scale", "up", "up_scale", "down", "down_scale", "sh_gate", "sh_gate_scale", "sh_up",
        "sh_up_scale", "sh_down", "sh_down_scale")]


class MoEError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} returned {STATUS_NAMES.get(status, status)}")


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m sparse_mixture_experts_08_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, S = ctypes.c_void_p, ctypes.c_size_t
        sig = {
            "moe_workspace_size": [P, P],
            "moe_atomic_workspace_size": [P, P],
            "moe_route": [P, P, P, P, P, P, P, P, P, S, P],
            "moe_histogram_lis": [P, P, P, P, P, P, S, P],
            "moe_permute": [P, P, P, P, P, P, P, P, S, P],
            "moe_lis_from_counts": [ctypes.c_int32, ctypes.c_int64, P, P, P],
            "moe_grouped_ffn": [P, P, P, P, P, P, P, P, P, P, S, P],
            "moe_shared_ffn": [P, P, P, P, P, P, P, S, P],
            "moe_combine": [P, P, P, P, P, P],
            "moe_layer_forward": [P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, S, P],
            "moe_replica_split": [P, P, P, P, P, P, P, P, P, S, P],
            "moe_floe_pack_down": [P, P, P, P],
            "moe_floe_calibrate": [P, P, ctypes.c_int32, P, ctypes.c_double, P, P, P, S, P],
            "moe_floe_workspace_size": [P, P],
            "moe_layer_forward_floe": [P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, S, P],
            "moe_layer_forward_replicated": [P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, S, P],
            "moe_atomic_route": [P, P, P, P, P, P, P, P, P, S, P],
            "moe_atomic_experts": [P, P, P, P, P, P, P, P, S, P],
            "moe_atomic_forward": [P, P, P, P, P, P, P, P, P, P, S, P],
            "moe_read_device_status": [P, P, P],
            "moe_debug_set_wait_limit_ns": [ctypes.c_uint64],
            "moe_debug_set_barrier_extra": [ctypes.c_uint32],
            "moe_set_stage_events": [P, ctypes.c_int],
            "moe_route_static": [P, P, P, P, P, P, P, P, P, P],
            "moe_quantize_e4m3": [ctypes.c_int64, ctypes.c_int64, P, P, P, P],
            "moe_fp8_workspace_size": [P, P],
            "moe_layer_forward_fp8": [P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, S, P],
        }
        for name, args in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.moe_status_string.argtypes = [ctypes.c_int]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_launch_count.argtypes = []
        L.moe_launch_count.restype = ctypes.c_uint64
        _lib = L
    return _lib


# ------------------------------------------------------------------ marshalling helpers

def _p(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, rc: int):
    if rc != OK:
        raise MoEError(fn, rc)


def make_config(T, d, f, m, k, n_shared=0, f_shared=0, dtype=BF16, act=SWIGLU, renormalize=False) -> MoEConfig:
    return MoEConfig(T, d, f, m, k, n_shared, f_shared, dtype, act, int(bool(renormalize)))


def make_atomic_config(T, d, Nr, Nc, K, act=ATOMIC_SILU, dtype=BF16) -> MoEAtomicConfig:
    return MoEAtomicConfig(T, d, Nr, Nc, K, act, dtype)


# ------------------------------------------------------------------ entry points (same names as the C ABI)

def moe_workspace_size(cfg: MoEConfig) -> int:
    n = ctypes.c_size_t(0)
    _check("moe_workspace_size", lib().moe_workspace_size(ctypes.byref(cfg), ctypes.byref(n)))
    return n.value


def moe_atomic_workspace_size(cfg: MoEAtomicConfig) -> int:
    n = ctypes.c_size_t(0)
    _check("moe_atomic_workspace_size", lib().moe_atomic_workspace_size(ctypes.byref(cfg), ctypes.byref(n)))
    return n.value


def moe_route(cfg, x, w_router, bias, logits_in, logits_out, topk_idx, topk_w, ws, stream=None):
    _check("moe_route", lib().moe_route(ctypes.byref(cfg), _p(x), _p(w_router), _p(bias), _p(logits_in),
                                        _p(logits_out), _p(topk_idx), _p(topk_w), _p(ws), ws.numel(),
                                        _stream(stream)))


def moe_route_static(cfg, x, w_router, bias, logits_in, logits_out, topk_idx, topk_w, device_status_out=None,
                     stream=None):
    """moe_route without a workspace (scratch compiled into the library; see include/moe.h)."""
    _check("moe_route_static", lib().moe_route_static(ctypes.byref(cfg), _p(x), _p(w_router), _p(bias),
                                                      _p(logits_in), _p(logits_out), _p(topk_idx), _p(topk_w),
                                                      _p(device_status_out), _stream(stream)))


def moe_histogram_lis(cfg, topk_idx, counts, offsets, lis, ws, stream=None):
    _check("moe_histogram_lis", lib().moe_histogram_lis(ctypes.byref(cfg), _p(topk_idx), _p(counts), _p(offsets),
                                                        _p(lis), _p(ws), ws.numel(), _stream(stream)))


def moe_lis_from_counts(m, tasks, counts, lis, stream=None):
    _check("moe_lis_from_counts", lib().moe_lis_from_counts(int(m), int(tasks), _p(counts), _p(lis),
                                                            _stream(stream)))


def moe_permute(cfg, x, topk_idx, offsets, x_perm, perm, inv_perm, ws, stream=None):
    _check("moe_permute", lib().moe_permute(ctypes.byref(cfg), _p(x), _p(topk_idx), _p(offsets), _p(x_perm),
                                            _p(perm), _p(inv_perm), _p(ws), ws.numel(), _stream(stream)))


def moe_grouped_ffn(cfg, x_perm, offsets, w_gate, w_up, w_down, task_w, perm, y_perm, ws, stream=None):
    _check("moe_grouped_ffn", lib().moe_grouped_ffn(ctypes.byref(cfg), _p(x_perm), _p(offsets), _p(w_gate),
                                                    _p(w_up), _p(w_down), _p(task_w), _p(perm), _p(y_perm),
                                                    _p(ws), ws.numel(), _stream(stream)))


def moe_shared_ffn(cfg, x, ws_gate, ws_up, ws_down, y_shared, ws, stream=None):
    _check("moe_shared_ffn", lib().moe_shared_ffn(ctypes.byref(cfg), _p(x), _p(ws_gate), _p(ws_up), _p(ws_down),
                                                  _p(y_shared), _p(ws), ws.numel(), _stream(stream)))


def moe_combine(cfg, y_perm, inv_perm, y_shared, out, stream=None):
    _check("moe_combine", lib().moe_combine(ctypes.byref(cfg), _p(y_perm), _p(inv_perm), _p(y_shared), _p(out),
                                            _stream(stream)))


def moe_layer_forward(cfg, x, w_router, bias, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, out, ws,
                      logits_out=None, topk_idx_out=None, topk_w_out=None, counts_out=None, lis_out=None,
                      offsets_out=None, perm_out=None, inv_perm_out=None, x_perm_out=None, stream=None):
    _check("moe_layer_forward", lib().moe_layer_forward(
        ctypes.byref(cfg), _p(x), _p(w_router), _p(bias), _p(w_gate), _p(w_up), _p(w_down), _p(ws_gate),
        _p(ws_up), _p(ws_down), _p(out), _p(logits_out), _p(topk_idx_out), _p(topk_w_out), _p(counts_out),
        _p(lis_out), _p(offsets_out), _p(perm_out), _p(inv_perm_out), _p(x_perm_out), _p(ws), ws.numel(),
        _stream(stream)))


def moe_replica_split(cfg, topk_idx, offsets, inv_perm, lis, idx_out, ws, counts_out=None, lis_out=None,
                      stream=None):
    _check("moe_replica_split", lib().moe_replica_split(ctypes.byref(cfg), _p(topk_idx), _p(offsets), _p(inv_perm),
                                                        _p(lis), _p(idx_out), _p(counts_out), _p(lis_out), _p(ws),
                                                        ws.numel(), _stream(stream)))


def moe_layer_forward_replicated(cfg, x, w_router, bias, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, out, ws,
                                 logits_out=None, topk_idx_out=None, topk_w_out=None, dispatch_idx_out=None,
                                 counts_out=None, lis_before_out=None, lis_after_out=None, stream=None):
    """ws: a workspace for the same config with m + 1 experts (replica_workspace)."""
    _check("moe_layer_forward_replicated", lib().moe_layer_forward_replicated(
        ctypes.byref(cfg), _p(x), _p(w_router), _p(bias), _p(w_gate), _p(w_up), _p(w_down), _p(ws_gate),
        _p(ws_up), _p(ws_down), _p(out), _p(logits_out), _p(topk_idx_out), _p(topk_w_out), _p(dispatch_idx_out),
        _p(counts_out), _p(lis_before_out), _p(lis_after_out), _p(ws), ws.numel(), _stream(stream)))


def moe_floe_pack_down(cfg, w_down, w_down_t, stream=None):
    _check("moe_floe_pack_down", lib().moe_floe_pack_down(ctypes.byref(cfg), _p(w_down), _p(w_down_t),
                                                          _stream(stream)))


def moe_floe_calibrate(cfg, x_calib, w_up, sparsity, u_scratch, thresholds_out, ws, stream=None):
    _check("moe_floe_calibrate", lib().moe_floe_calibrate(ctypes.byref(cfg), _p(x_calib), int(x_calib.shape[0]),
                                                          _p(w_up), float(sparsity), _p(u_scratch),
                                                          _p(thresholds_out), _p(ws), ws.numel(), _stream(stream)))


def moe_floe_workspace_size(cfg) -> int:
    n = ctypes.c_size_t(0)
    _check("moe_floe_workspace_size", lib().moe_floe_workspace_size(ctypes.byref(cfg), ctypes.byref(n)))
    return n.value


def moe_layer_forward_floe(cfg, x, w_router, bias, w_gate, w_up, w_down_t, thresholds, out, ws, topk_idx_out=None,
                           topk_w_out=None, kept_out=None, u_out=None, perm_out=None, stream=None):
    _check("moe_layer_forward_floe", lib().moe_layer_forward_floe(
        ctypes.byref(cfg), _p(x), _p(w_router), _p(bias), _p(w_gate), _p(w_up), _p(w_down_t), _p(thresholds),
        _p(out), _p(topk_idx_out), _p(topk_w_out), _p(kept_out), _p(u_out), _p(perm_out), _p(ws), ws.numel(),
        _stream(stream)))


def moe_quantize_e4m3(src, codes, scales, stream=None):
    """Per-row E4M3 codes [rows, cols] (uint8) and fp32 scales [rows] of a bf16 matrix."""
    rows = src.numel() // src.shape[-1]
    _check("moe_quantize_e4m3", lib().moe_quantize_e4m3(rows, int(src.shape[-1]), _p(src), _p(codes), _p(scales),
                                                        _stream(stream)))


def moe_fp8_workspace_size(cfg) -> int:
    n = ctypes.c_size_t(0)
    _check("moe_fp8_workspace_size", lib().moe_fp8_workspace_size(ctypes.byref(cfg), ctypes.byref(n)))
    return n.value


def moe_layer_forward_fp8(cfg, x, w_router, bias, wq, out, ws, logits_out=None, topk_idx_out=None, topk_w_out=None,
                          counts_out=None, lis_out=None, h_out=None, h_shared_out=None, perm_out=None, stream=None):
    """wq: a dict of device tensors as quantize_experts returns (kept alive by the caller)."""
    st = MoEFp8Experts(**{k: _p(wq.get(k)) for k, _ in MoEFp8Experts._fields_})
    _check("moe_layer_forward_fp8", lib().moe_layer_forward_fp8(
        ctypes.byref(cfg), _p(x), _p(w_router), _p(bias), ctypes.byref(st), _p(out), _p(logits_out),
        _p(topk_idx_out), _p(topk_w_out), _p(counts_out), _p(lis_out), _p(h_out), _p(h_shared_out), _p(perm_out),
        _p(ws), ws.numel(), _stream(stream)))


def quantize_experts(w_gate, w_up, w_down, ws_gate=None, ws_up=None, ws_down=None, stream=None) -> dict:
    """E4M3 codes + per-output-channel scales of every expert weight (device bf16
    tensors in, device tensors out), keyed as moe_fp8_experts_t's fields."""
    out = {}
    for key, w in (("gate", w_gate), ("up", w_up), ("down", w_down), ("sh_gate", ws_gate), ("sh_up", ws_up),
                   ("sh_down", ws_down)):
        if w is None:
            continue
        codes = torch.empty(w.shape, dtype=torch.uint8, device=w.device)
        scales = torch.empty(w.shape[:-1], dtype=torch.float32, device=w.device)
        moe_quantize_e4m3(w, codes, scales, stream=stream)
        out[key], out[key + "_scale"] = codes, scales
    return out


def fp8_workspace(cfg, device="cuda") -> torch.Tensor:
    return torch.zeros(max(moe_fp8_workspace_size(cfg), 256), dtype=torch.uint8, device=device)


def floe_workspace(cfg, device="cuda") -> torch.Tensor:
    return torch.zeros(max(moe_floe_workspace_size(cfg), 256), dtype=torch.uint8, device=device)


def moe_atomic_route(cfg, x, w_row, w_col, row_logp_out, col_logp_out, idx_out, g_out, ws, stream=None):
    _check("moe_atomic_route", lib().moe_atomic_route(ctypes.byref(cfg), _p(x), _p(w_row), _p(w_col),
                                                      _p(row_logp_out), _p(col_logp_out), _p(idx_out), _p(g_out),
                                                      _p(ws), ws.numel(), _stream(stream)))


def moe_atomic_experts(cfg, x, w_in, w_out, idx, g, out, ws, stream=None):
    _check("moe_atomic_experts", lib().moe_atomic_experts(ctypes.byref(cfg), _p(x), _p(w_in), _p(w_out), _p(idx),
                                                          _p(g), _p(out), _p(ws), ws.numel(), _stream(stream)))


def moe_atomic_forward(cfg, x, w_row, w_col, w_in, w_out, out, ws, idx_out=None, g_out=None, stream=None):
    _check("moe_atomic_forward", lib().moe_atomic_forward(ctypes.byref(cfg), _p(x), _p(w_row), _p(w_col), _p(w_in),
                                                          _p(w_out), _p(out), _p(idx_out), _p(g_out), _p(ws),
                                                          ws.numel(), _stream(stream)))


def moe_read_device_status(ws, stream=None) -> int:
    out = ctypes.c_int(0)
    _check("moe_read_device_status", lib().moe_read_device_status(_p(ws), _stream(stream), ctypes.byref(out)))
    return out.value


def moe_status_string(status: int) -> str:
    return lib().moe_status_string(status).decode()


def moe_debug_set_wait_limit_ns(ns: int):
    _check("moe_debug_set_wait_limit_ns", lib().moe_debug_set_wait_limit_ns(ns))


def moe_debug_set_barrier_extra(n: int):
    _check("moe_debug_set_barrier_extra", lib().moe_debug_set_barrier_extra(n))


def moe_set_stage_events(events):
    """events: list of torch.cuda.Event (enable_timing=True, already recorded once so
    that the CUDA event exists) or None entries (boundary not recorded); [] switches
    the hook off."""
    handles = [0 if e is None else e.cuda_event for e in events]
    if any(e is not None and not h for e, h in zip(events, handles)):
        raise ValueError("moe_set_stage_events: record each torch.cuda.Event once before passing it")
    arr = (ctypes.c_void_p * max(1, len(handles)))(*handles)
    _check("moe_set_stage_events", lib().moe_set_stage_events(arr if handles else None, len(handles)))


def moe_launch_count() -> int:
    return int(lib().moe_launch_count())


# ------------------------------------------------------------------ allocation helpers (torch memory)

def replica_workspace(cfg, device="cuda") -> torch.Tensor:
    """A zeroed workspace for moe_layer_forward_replicated: the same config with m + 1 experts."""
    c1 = MoEConfig.from_buffer_copy(cfg)
    c1.m = cfg.m + 1
    return workspace(c1, device=device)


def workspace(cfg, device="cuda") -> torch.Tensor:
    """A zeroed workspace of the size the config needs (uint8, 256-byte aligned)."""
    n = moe_atomic_workspace_size(cfg) if isinstance(cfg, MoEAtomicConfig) else moe_workspace_size(cfg)
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=device)


def lis_buffer(device="cuda") -> torch.Tensor:
    return torch.zeros(LIS_BYTES, dtype=torch.uint8, device=device)


def unpack_lis(buf: torch.Tensor):
    """(max_count, argmax_expert, lis) from a 16-byte moe_lis_t buffer."""
    b = buf.detach().cpu().contiguous()
    ints = b[:8].view(torch.int32)
    return int(ints[0]), int(ints[1]), float(b[8:16].view(torch.float64)[0])

"""CPU oracle for the sparse-MoE layer forward (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package. It wraps ``liboracle.so`` (plain C, fp64, one token at
a time; see ``moe_oracle.c`` for the definitions and the passages they follow)
with numpy in/out. It shares no code with the CUDA path; both draw their inputs
from ``workloads``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

F32, BF16 = 0, 1
SWIGLU, RELU = 0, 1
ACT_SILU, ACT_SIGMOID = 0, 1


class OracleCfg(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("f", ctypes.c_int32),
                ("m", ctypes.c_int32), ("k", ctypes.c_int32), ("act", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("n_shared", ctypes.c_int32), ("f_shared", ctypes.c_int32),
                ("renorm", ctypes.c_int32)]


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (plain -O2, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fPIC", "-shared", "-std=c99",
                               "-o", _LIB_PATH, _SRC, "-lm", "-lpthread"])
    return _LIB_PATH


_lib = None
_P = ctypes.c_void_p


def _L():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        i = ctypes.c_int
        sig = {
            "oracle_router_logits": [i, i, i, i, _P, _P, _P, _P],
            "oracle_topk_softmax": [i, i, i, i, _P, _P, _P],
            "oracle_histogram_lis": [i, i, i, _P, _P, _P, _P, _P, _P],
            "oracle_permutation": [i, i, i, _P, _P, _P, _P],
            "oracle_replica_split": [i, i, i, _P, _P, _P],
            "oracle_expert_ffn": [i, i, i, i, _P, _P, _P, _P, _P],
            "oracle_moe_output": [_P, _P, i, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, i],
            "oracle_layer_forward": [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                     _P, _P, _P, _P, _P, i],
            "oracle_dense_masked": [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P],
            "oracle_atomic_logprobs": [i, i, i, i, i, _P, _P, _P, _P, _P],
            "oracle_atomic_select": [i, i, i, i, _P, _P, _P, _P],
            "oracle_atomic_output": [i, i, i, i, i, _P, _P, _P, _P, _P, _P, i, _P],
        }
        for name, args in sig.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"{what} failed with code {rc}")


def _np_dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError(f"unsupported array dtype {a.dtype}")


def _cfg(c, T=None) -> OracleCfg:
    return OracleCfg(T if T is not None else c.T, c.d, c.f, c.m, c.k, c.act, c.dtype,
                     getattr(c, "n_shared", 0), getattr(c, "f_shared", 0), int(bool(c.renorm)))


def _default_threads() -> int:
    return max(1, os.cpu_count() or 1)


# ------------------------------------------------------------------------- routing

def router_logits(x: np.ndarray, w_r: np.ndarray, bias: Optional[np.ndarray]) -> np.ndarray:
    T, d = x.shape
    m = w_r.shape[0]
    dt = _np_dtype_code(x)
    out = np.empty((T, m), dtype=np.float32)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    _check(_L().oracle_router_logits(T, d, m, dt, _ptr(x), _ptr(w_r), _ptr(b), _ptr(out)), "router_logits")
    return out


def topk_softmax(logits: np.ndarray, k: int, renorm: bool):
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, m = logits.shape
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    _check(_L().oracle_topk_softmax(T, m, k, int(renorm), _ptr(logits), _ptr(idx), _ptr(w)), "topk_softmax")
    return idx, w


def histogram_lis(idx: np.ndarray, m: int):
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    counts = np.empty(m, dtype=np.int32)
    offsets = np.empty(m + 1, dtype=np.int32)
    mx = np.zeros(1, np.int32)
    am = np.zeros(1, np.int32)
    lis = np.zeros(1, np.float64)
    _check(_L().oracle_histogram_lis(T, k, m, _ptr(idx), _ptr(counts), _ptr(offsets), _ptr(mx), _ptr(am),
                                     _ptr(lis)), "histogram_lis")
    return {"counts": counts, "offsets": offsets, "max_count": int(mx[0]), "argmax": int(am[0]),
            "lis": float(lis[0])}


def permutation(idx: np.ndarray, m: int, offsets: np.ndarray):
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    perm = np.empty(T * k, dtype=np.int32)
    inv = np.empty(T * k, dtype=np.int32)
    _check(_L().oracle_permutation(T, k, m, _ptr(idx), _ptr(np.ascontiguousarray(offsets, np.int32)),
                                   _ptr(perm), _ptr(inv)), "permutation")
    return perm, inv


def replica_split(idx: np.ndarray, m: int):
    """R&Q replica dispatch: (routing over m + 1 experts, heavy-hitter h). Every
    second task of h, in task order, goes to the replica expert m."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    out = np.empty_like(idx)
    h = np.zeros(1, np.int32)
    _check(_L().oracle_replica_split(T, k, m, _ptr(idx), _ptr(out), _ptr(h)), "replica_split")
    return out, int(h[0])


def replica_inputs(inp: Dict[str, np.ndarray], heavy: int) -> Dict[str, np.ndarray]:
    """The layer's inputs with expert m appended as a copy of the heavy-hitter's
    weights (R&Q Algorithm 3 appends quant(layer[h]); unquantised here)."""
    out = dict(inp)
    for key in ("w_gate", "w_up", "w_down"):
        if inp.get(key) is not None:
            out[key] = np.ascontiguousarray(np.concatenate([inp[key], inp[key][heavy:heavy + 1]], axis=0))
    return out


# ------------------------------------------------------------------------- experts

def expert_ffn(x_row: np.ndarray, wg: np.ndarray, wu: Optional[np.ndarray], wd: np.ndarray, act: int):
    d = x_row.shape[-1]
    f = wg.shape[0]
    y = np.empty(d, dtype=np.float64)
    _check(_L().oracle_expert_ffn(d, f, act, _np_dtype_code(x_row), _ptr(x_row), _ptr(wg), _ptr(wu), _ptr(wd),
                                  _ptr(y)), "expert_ffn")
    return y


def moe_output(cfg, inp: Dict[str, np.ndarray], idx: np.ndarray, w: np.ndarray, tokens=None,
               nthreads: Optional[int] = None) -> np.ndarray:
    """Layer output (float64) for `tokens` (all tokens when None) given the routing."""
    c = _cfg(cfg, T=inp["x"].shape[0])
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
    ntok = c.T if tok is None else len(tok)
    out = np.empty((ntok, c.d), dtype=np.float64)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float64)
    _check(_L().oracle_moe_output(ctypes.byref(c), _ptr(tok), ntok, _ptr(inp["x"]), _ptr(inp["w_gate"]),
                                  _ptr(inp.get("w_up")), _ptr(inp["w_down"]), _ptr(inp.get("ws_gate")),
                                  _ptr(inp.get("ws_up")), _ptr(inp.get("ws_down")), _ptr(idx), _ptr(w),
                                  _ptr(out), nthreads or _default_threads()), "moe_output")
    return out


def layer_forward(cfg, inp: Dict[str, np.ndarray], logits_in: Optional[np.ndarray] = None,
                  nthreads: Optional[int] = None) -> Dict[str, object]:
    """Every step of the layer forward on all tokens of `inp` (T = rows of x)."""
    x = inp["x"]
    c = _cfg(cfg, T=x.shape[0])
    T, m, k, d = c.T, c.m, c.k, c.d
    logits = np.empty((T, m), np.float32)
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    counts = np.empty(m, np.int32)
    offsets = np.empty(m + 1, np.int32)
    perm = np.empty(T * k, np.int32)
    inv = np.empty(T * k, np.int32)
    mx = np.zeros(1, np.int32)
    am = np.zeros(1, np.int32)
    lis = np.zeros(1, np.float64)
    out = np.empty((T, d), np.float64)
    li = None if logits_in is None else np.ascontiguousarray(logits_in, dtype=np.float32)
    bias = inp.get("bias")
    _check(_L().oracle_layer_forward(ctypes.byref(c), _ptr(x), _ptr(inp["w_router"]), _ptr(bias), _ptr(li),
                                     _ptr(inp["w_gate"]), _ptr(inp.get("w_up")), _ptr(inp["w_down"]),
                                     _ptr(inp.get("ws_gate")), _ptr(inp.get("ws_up")), _ptr(inp.get("ws_down")),
                                     _ptr(logits), _ptr(idx), _ptr(w), _ptr(counts), _ptr(offsets), _ptr(perm),
                                     _ptr(inv), _ptr(mx), _ptr(am), _ptr(lis), _ptr(out),
                                     nthreads or _default_threads()), "layer_forward")
    return {"logits": logits, "idx": idx, "w": w, "counts": counts, "offsets": offsets, "perm": perm,
            "inv_perm": inv, "max_count": int(mx[0]), "argmax": int(am[0]), "lis": float(lis[0]), "out": out}


def dense_masked(cfg, inp: Dict[str, np.ndarray], idx: np.ndarray, w: np.ndarray) -> np.ndarray:
    c = _cfg(cfg, T=inp["x"].shape[0])
    out = np.empty((c.T, c.d), np.float64)
    _check(_L().oracle_dense_masked(ctypes.byref(c), _ptr(inp["x"]), _ptr(inp["w_gate"]), _ptr(inp.get("w_up")),
                                    _ptr(inp["w_down"]), _ptr(inp.get("ws_gate")), _ptr(inp.get("ws_up")),
                                    _ptr(inp.get("ws_down")), _ptr(np.ascontiguousarray(idx, np.int32)),
                                    _ptr(np.ascontiguousarray(w, np.float64)), _ptr(out)), "dense_masked")
    return out


# ------------------------------------------------------- FloE contextual sparsity

def floe_threshold(u_abs: np.ndarray, sparsity: float) -> np.float32:
    """FloE Eq. 6: the threshold from the empirical CDF of |up-projection
    activations| at target sparsity s: the ceil(s n)-th smallest of the n values
    (1-based; at least the 1st), so a fraction s of the sample lies at or below it."""
    v = np.sort(np.asarray(u_abs, dtype=np.float32).ravel())
    r = max(1, int(np.ceil(sparsity * v.size)))
    return np.float32(v[min(r, v.size) - 1])


def floe_expert(x_row: np.ndarray, wg: np.ndarray, wu: np.ndarray, wd: np.ndarray, thr: float, dtype: int,
                u_mask: Optional[np.ndarray] = None):
    """One expert on one token with FloE contextual sparsity (FloE "Core claim",
    Sec. 3.2): u = x W_up^T; channel j is kept when |u_j| >= thr; for kept channels
    g_j = x . W_gate[j] and h_j = g_j sigma(g_j) u_j, others contribute nothing;
    y = sum over kept j of h_j W_down[:, j]. fp64. `u_mask`, when given, is the
    up-projection output whose magnitudes decide the mask (so both sides of a
    comparison decide from the same numbers); the arithmetic uses the fp64 u.
    Returns (y, kept mask)."""
    as64 = lambda a: np.asarray(_values(a, dtype), dtype=np.float64)
    x = as64(x_row)
    u = as64(wu) @ x
    keep = np.abs(np.asarray(u_mask, np.float32) if u_mask is not None else u) >= thr
    g = as64(wg)[keep] @ x
    h = g / (1.0 + np.exp(-g)) * u[keep]
    y = as64(wd)[:, keep] @ h
    return y, keep


def _values(a, dtype):
    """bf16 bit patterns (uint16) or fp32 -> fp32 values (input decoding only)."""
    if dtype == BF16 or a.dtype == np.uint16:
        return (np.asarray(a, np.uint16).astype(np.uint32) << 16).view(np.float32)
    return np.asarray(a, np.float32)


# -------------------------------------------------------------------- atomic experts

def atomic_logprobs(x: np.ndarray, w_row: np.ndarray, w_col: np.ndarray):
    T, d = x.shape
    Nr, Nc = w_row.shape[0], w_col.shape[0]
    lr = np.empty((T, Nr), np.float32)
    lc = np.empty((T, Nc), np.float32)
    _check(_L().oracle_atomic_logprobs(T, d, Nr, Nc, _np_dtype_code(x), _ptr(x), _ptr(w_row), _ptr(w_col),
                                       _ptr(lr), _ptr(lc)), "atomic_logprobs")
    return lr, lc


def atomic_select(lr: np.ndarray, lc: np.ndarray, K: int):
    lr = np.ascontiguousarray(lr, np.float32)
    lc = np.ascontiguousarray(lc, np.float32)
    T, Nr = lr.shape
    Nc = lc.shape[1]
    idx = np.empty((T, K), np.int32)
    g = np.empty((T, K), np.float64)
    _check(_L().oracle_atomic_select(T, Nr, Nc, K, _ptr(lr), _ptr(lc), _ptr(idx), _ptr(g)), "atomic_select")
    return idx, g


def atomic_output(x: np.ndarray, w_in: np.ndarray, w_out: np.ndarray, idx: np.ndarray, g: np.ndarray, act: int,
                  tokens=None) -> np.ndarray:
    T, d = x.shape
    K = idx.shape[1]
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
    ntok = T if tok is None else len(tok)
    out = np.empty((ntok, d), np.float64)
    _check(_L().oracle_atomic_output(T, d, K, act, _np_dtype_code(x), _ptr(x), _ptr(w_in), _ptr(w_out),
                                     _ptr(np.ascontiguousarray(idx, np.int32)),
                                     _ptr(np.ascontiguousarray(g, np.float64)), _ptr(tok), ntok, _ptr(out)),
           "atomic_output")
    return out

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


# ----------------------------------------------------- 8-bit expert weights (e4m3)
#
# R&Q ("Free parameters": quantization precision) stores quantized expert copies
# in 8 bits and names no format or scaling. Reading taken here: OCP E4M3 (1 sign
# bit, 4 exponent bits with bias 7, 3 mantissa bits, no infinities, largest finite
# magnitude 448), one fp32 scale per row (per output channel of a weight matrix,
# per task row of an activation), scale = row max |v| / 448, code = the E4M3 value
# nearest to v / scale (ties to the even code, saturating at +-448). Both GEMM
# operands of an 8-bit tensor-core product are 8-bit, so the activations entering
# each projection are quantized the same way, per row; the hidden activation h is
# stored in bf16 (round to nearest even) before it is quantized.

E4M3_MAX = 448.0


def e4m3_round(v) -> np.ndarray:
    """float32 values -> E4M3 codes (uint8): round to nearest, ties to even,
    saturating at +-448; the sign bit follows the sign of v (so -0 -> 0x80).

    A magnitude a in the binade [2^e, 2^(e+1)), e >= -6, is a multiple of the
    quantum 2^(e-3); below 2^-6 the quantum is 2^-9 (subnormals). With n = a /
    quantum rounded half to even, the non-negative codes count the representable
    magnitudes in increasing order, 8 per binade from 2^-6 up and 8 subnormal ones
    (0 .. 7 * 2^-9) below, so the code is 8 (e + 6) + n for e >= -6 and n below
    2^-6. n = 16 (a rounded up to 2^(e+1)) lands on the first code of the next
    binade by the same formula."""
    v = np.asarray(v, dtype=np.float32)
    a = np.minimum(np.abs(v).astype(np.float64), E4M3_MAX)
    _, ex = np.frexp(a)                             # a = mant * 2^ex, mant in [0.5, 1)
    e = np.where(a >= 2.0 ** -6, ex - 1, -6)        # binade exponent; the subnormal range (and 0) uses -6
    n = np.rint(np.ldexp(a, 3 - e))                 # exact scaling by a power of two; rint: half to even
    code = (8 * (e + 6) + n).astype(np.int64)
    code |= np.signbit(v).astype(np.int64) << 7
    return code.astype(np.uint8)


def _e4m3_table() -> np.ndarray:
    """Values of the 256 codes from the bit fields: sign, exponent E (bias 7,
    E = 0 subnormal), mantissa M; S.1111.111 is NaN."""
    c = np.arange(256, dtype=np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    E = (c >> 3) & 0xF
    M = c & 0x7
    mag = np.where(E == 0, M * 2.0 ** -9, (1.0 + M / 8.0) * np.ldexp(1.0, E - 7))
    mag = np.where((E == 0xF) & (M == 0x7), np.nan, mag)
    return s * mag


_E4M3_VALUES = _e4m3_table()


def e4m3_value(codes) -> np.ndarray:
    """E4M3 codes -> float64 values (NaN for the two NaN codes)."""
    return _E4M3_VALUES[np.asarray(codes, dtype=np.uint8)]


def quantize_rows(a) -> tuple:
    """Per-row E4M3 quantization of a 2-D float32 array: (codes uint8, scales
    float32). scale = fl32(max |row| / 448) (1 for an all-zero row); code =
    e4m3_round(fl32(v / scale)). Both divisions are IEEE fp32."""
    a = np.asarray(a, dtype=np.float32)
    amax = np.max(np.abs(a), axis=1) if a.shape[1] else np.zeros(a.shape[0], np.float32)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    codes = np.empty(a.shape, np.uint8)
    for r0 in range(0, a.shape[0], 256):            # row blocks: bounded temporaries
        r1 = min(a.shape[0], r0 + 256)
        codes[r0:r1] = e4m3_round((a[r0:r1] / scale[r0:r1, None]).astype(np.float32))
    return codes, scale


def round_bf16(v) -> np.ndarray:
    """float64 -> float32 (nearest) -> bf16 (nearest, ties to even), returned as float32."""
    f = np.asarray(v, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16 << 16
    return u.astype(np.uint32).view(np.float32)


def quantize_experts(cfg, inp: Dict[str, np.ndarray]) -> Dict[str, np.ndarray]:
    """Every expert weight matrix of `inp` quantized per output channel: for key
    K in (w_gate, w_up, w_down, ws_gate, ws_up, ws_down), K -> codes with the
    same shape and K + "_scale" -> one scale per row of the last axis."""
    out = {}
    for key in ("w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down"):
        w = inp.get(key)
        if w is None:
            continue
        vals = _values(w, cfg.dtype)
        codes, sc = quantize_rows(vals.reshape(-1, vals.shape[-1]))
        out[key] = codes.reshape(vals.shape)
        out[key + "_scale"] = sc.reshape(vals.shape[:-1])
    return out


def fp8_expert_up(xq, sx, gq, gs, uq, us, act) -> np.ndarray:
    """First half of an 8-bit expert on quantized token rows (fp64 arithmetic on
    the dequantized values): a = x . w_gate [, b = x . w_up]; h = silu(a) b
    (SwiGLU) or relu(a). Returns h in fp64, one row per task."""
    X = e4m3_value(xq) * sx[:, None].astype(np.float64)
    a = X @ (e4m3_value(gq) * gs[:, None].astype(np.float64)).T
    if act == SWIGLU:
        b = X @ (e4m3_value(uq) * us[:, None].astype(np.float64)).T
        return a / (1.0 + np.exp(-a)) * b
    return np.maximum(a, 0.0)


def fp8_expert_down(h_stored, dq, ds) -> np.ndarray:
    """Second half: the stored (bf16-valued, as float32) h rows are quantized per
    row and multiplied by the quantized W_down: y = h_q . w_down (fp64)."""
    hq, hs = quantize_rows(h_stored)
    H = e4m3_value(hq) * hs[:, None].astype(np.float64)
    return H @ (e4m3_value(dq) * ds[:, None].astype(np.float64)).T


def _ffn_fp8(xq, sx, gq, gs, uq, us, dq, ds, act):
    """An 8-bit expert: h is stored in bf16 between the two halves."""
    return fp8_expert_down(round_bf16(fp8_expert_up(xq, sx, gq, gs, uq, us, act)), dq, ds)


class QuantizedExperts:
    """quantize_experts computed on first use, one expert matrix at a time:
    q["w_gate"][e] -> codes, q["w_gate_scale"][e] -> scales (same values)."""

    def __init__(self, cfg, inp):
        self.cfg, self.inp, self.cache = cfg, inp, {}

    def _get(self, key, e):
        if (key, e) not in self.cache:
            vals = _values(self.inp[key][e], self.cfg.dtype)
            self.cache[(key, e)] = quantize_rows(vals.reshape(-1, vals.shape[-1]))
        return self.cache[(key, e)]

    def __getitem__(self, name):
        key, part = (name[:-6], 1) if name.endswith("_scale") else (name, 0)
        outer = self

        class _Rows:
            def __getitem__(self, e):
                return outer._get(key, int(e))[part]
        return _Rows()


def layer_forward_fp8(cfg, inp: Dict[str, np.ndarray], qw: Optional[Dict[str, np.ndarray]] = None,
                      tokens=None, logits_in: Optional[np.ndarray] = None) -> Dict[str, object]:
    """The layer forward with 8-bit expert weights: the router as in the bf16
    layer (bf16 operands, fp32 logits, top-k softmax); each token row of x is
    quantized once (its k tasks share codes and scale); every routed task and
    every shared expert runs _ffn_fp8; out_t = sum_s w[t,s] y_{t,s} + sum of the
    shared experts' y. Returns out (float64) for `tokens` (all when None), the
    routing, and the quantized x. With logits_in the top-k is taken on those logits."""
    x = inp["x"]
    T = x.shape[0]
    if qw is None:  # quantize only the experts the tokens reach (per output channel, as quantize_experts)
        qw = QuantizedExperts(cfg, inp)
    logits = router_logits(x, inp["w_router"], inp.get("bias")) if logits_in is None else logits_in
    idx, w = topk_softmax(logits, cfg.k, bool(cfg.renorm))
    xq, sx = quantize_rows(_values(x, cfg.dtype))
    tok = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    out = np.zeros((len(tok), cfg.d), np.float64)
    swiglu = cfg.act == SWIGLU
    for e in np.unique(idx[tok]):
        rows, slots = np.nonzero(idx[tok] == e)
        t = tok[rows]
        y = _ffn_fp8(xq[t], sx[t], qw["w_gate"][e], qw["w_gate_scale"][e],
                     qw["w_up"][e] if swiglu else None, qw["w_up_scale"][e] if swiglu else None,
                     qw["w_down"][e], qw["w_down_scale"][e], cfg.act)
        np.add.at(out, rows, w[t, slots][:, None] * y)
    for sh in range(cfg.n_shared):
        out += _ffn_fp8(xq[tok], sx[tok], qw["ws_gate"][sh], qw["ws_gate_scale"][sh],
                        qw["ws_up"][sh] if swiglu else None, qw["ws_up_scale"][sh] if swiglu else None,
                        qw["ws_down"][sh], qw["ws_down_scale"][sh], cfg.act)
    return {"out": out, "idx": idx, "w": w, "logits": logits, "xq": xq, "sx": sx}

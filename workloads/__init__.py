"""Seeded synthetic workloads for the sparse-MoE layer forward.

This module only generates inputs; it holds none of the method's arithmetic.
Both the CPU oracle (in tests) and the GPU path take their operands from here,
so the two sides see bit-identical values.

Shapes follow the model families the reviewed pages evaluate (Switch Transformer,
Mixtral-8x7B, DeepSeek-V2-Lite, OmniMoE atomic experts); the values are synthetic
because no checkpoint or dataset is used:

* x ~ N(0, 1); every weight matrix ~ N(0, std = 1/sqrt(fan_in)) with fan_in the
  contraction length (d for router/gate/up/row/col/in projections, f for down).
  Atomic-expert output vectors scale a single scalar, so their fan_in is 1.
* A per-expert router bias of Zipf shape, bias[pi(r)] = -alpha * s * ln(r) for
  rank r = 1..m, with pi a seeded permutation of the expert ids (so no expert
  index is special). alpha is 1 except where a config names a target LIS; there
  it is calibrated once against the oracle and frozen in ``zipf_alpha.json``.
* Everything is rounded to the config's dtype (fp32, or bf16 via fp32, both
  round-to-nearest-even). bf16 arrays are carried as uint16 bit patterns.
* seed = 20260000 + 100 * config_index + replicate.
"""
from __future__ import annotations

import ctypes
import json
import math
import os
import subprocess
from dataclasses import dataclass, field, replace
from typing import Dict, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libmoegen.so")

# Stream ids: one independent counter stream per tensor.
STREAM = {
    "x": 1, "w_router": 2, "w_gate": 3, "w_up": 4, "w_down": 5,
    "ws_gate": 6, "ws_up": 7, "ws_down": 8, "bias_perm": 9,
    "w_row": 10, "w_col": 11, "w_in": 12, "w_out": 13,
}

F32, BF16 = 0, 1
SWIGLU, RELU = 0, 1
ACT_SILU, ACT_SIGMOID = 0, 1


@dataclass(frozen=True)
class MoEWorkload:
    """One coarse-expert MoE layer configuration (token-choice top-k routing)."""
    name: str
    index: int          # 1-based config number; enters the seed
    T: int              # tokens in the batch (the pages' n)
    d: int              # d_model
    f: int              # d_ff of one routed expert
    m: int              # routed experts
    k: int              # experts per token
    act: int            # SWIGLU or RELU
    dtype: int          # F32 or BF16
    zipf_s: float       # Zipf exponent of the router bias (0 = no bias)
    renorm: bool        # renormalise the k gate weights to sum to 1
    n_shared: int = 0   # always-on shared experts
    f_shared: int = 0   # d_ff of one shared expert
    lis_target: Optional[float] = None  # when set, alpha is calibrated to this LIS
    note: str = ""

    @property
    def tasks(self) -> int:
        return self.T * self.k

    def seed(self, replicate: int = 0) -> int:
        return 20260000 + 100 * self.index + replicate


@dataclass(frozen=True)
class AtomicWorkload:
    """Atomic-expert layer with a Cartesian-product router (Nr x Nc grid)."""
    name: str
    index: int
    T: int
    d: int
    Nr: int
    Nc: int
    K: int
    act: int            # ACT_SILU or ACT_SIGMOID
    dtype: int = BF16
    note: str = ""

    @property
    def N(self) -> int:
        return self.Nr * self.Nc

    def seed(self, replicate: int = 0) -> int:
        return 20260000 + 100 * self.index + replicate


CONFIGS: Dict[str, object] = {
    "tiny": MoEWorkload("tiny", 1, T=64, d=128, f=256, m=8, k=2, act=SWIGLU, dtype=F32,
                        zipf_s=1.2, renorm=False,
                        note="64 tokens, d_model 128, d_ff 256, 8 experts, top-2, fp32"),
    "switch": MoEWorkload("switch", 2, T=8192, d=768, f=3072, m=128, k=1, act=RELU, dtype=BF16,
                          zipf_s=1.0, renorm=False, lis_target=3.0,
                          note="Switch-style: 8192 tokens, d_model 768, d_ff 3072 ReLU, 128 experts, top-1"),
    "mixtral": MoEWorkload("mixtral", 3, T=4096, d=4096, f=14336, m=8, k=2, act=SWIGLU, dtype=BF16,
                           zipf_s=0.8, renorm=True,
                           note="Mixtral-8x7B-shaped prefill: 4096 tokens, d_model 4096, d_ff 14336, 8 experts, top-2 renormalised"),
    "dsv2lite": MoEWorkload("dsv2lite", 4, T=2048, d=2048, f=1408, m=64, k=6, act=SWIGLU, dtype=BF16,
                            zipf_s=1.1, renorm=False, n_shared=2, f_shared=1408, lis_target=4.0,
                            note="DeepSeek-V2-Lite-shaped: 2048 tokens, d_model 2048, 64 routed experts d_ff 1408 + 2 shared, top-6"),
    "decode": MoEWorkload("decode", 5, T=16, d=4096, f=14336, m=8, k=2, act=SWIGLU, dtype=BF16,
                          zipf_s=0.0, renorm=False,
                          note="decode regime: 16 tokens, d_model 4096, d_ff 14336, 8 experts, top-2"),
    "atomic": AtomicWorkload("atomic", 6, T=16, d=4096, Nr=512, Nc=512, K=64, act=ACT_SILU,
                             note="atomic experts: 16 tokens, d_model 4096, 512x512 Cartesian router, top-64 of 262144"),
    "atomic_prefill": AtomicWorkload("atomic_prefill", 7, T=4096, d=4096, Nr=512, Nc=512, K=512, act=ACT_SILU,
                                     note="atomic experts at prefill scale: 4096 tokens, d_model 4096, 512x512 "
                                          "Cartesian router, top-512 of 262144"),
}

_ALPHA_FILE = os.path.join(_HERE, "zipf_alpha.json")


def zipf_alpha(name: str) -> float:
    """alpha of the Zipf bias for a config (1.0 unless calibrated to a LIS target)."""
    cfg = CONFIGS[name]
    if getattr(cfg, "lis_target", None) is None:
        return 1.0
    with open(_ALPHA_FILE) as fh:
        return float(json.load(fh)[name]["alpha"])


# ----------------------------------------------------------------------------- C generator

def build_generator(force: bool = False) -> str:
    src = os.path.join(_HERE, "gen.c")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c99", "-o", _LIB_PATH, src,
                               "-lm", "-lpthread"])
    return _LIB_PATH


_lib = None


def _gen():
    global _lib
    if _lib is None:
        build_generator()
        lib = ctypes.CDLL(_LIB_PATH)
        lib.gen_normal.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_double, ctypes.c_int,
                                   ctypes.c_void_p, ctypes.c_int64, ctypes.c_int]
        lib.gen_normal.restype = ctypes.c_int
        lib.gen_permutation.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int32, ctypes.c_void_p]
        lib.gen_permutation.restype = ctypes.c_int
        lib.gen_u64.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        lib.gen_u64.restype = ctypes.c_uint64
        lib.gen_stream_key.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        lib.gen_stream_key.restype = ctypes.c_uint64
        _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def normal(seed: int, stream: int, shape, std: float, dtype: int, nthreads: Optional[int] = None,
           out: Optional[np.ndarray] = None) -> np.ndarray:
    """std * N(0,1) array of `shape`; float32 for F32, uint16 bf16 bits for BF16."""
    n = int(np.prod(shape)) if len(shape) else 1
    np_dt = np.float32 if dtype == F32 else np.uint16
    if out is None:
        out = np.empty(shape, dtype=np_dt)
    assert out.dtype == np_dt and out.flags["C_CONTIGUOUS"] and out.size == n
    rc = _gen().gen_normal(seed, stream, float(std), dtype, out.ctypes.data, n,
                           nthreads or default_threads())
    if rc != 0:
        raise RuntimeError("gen_normal failed")
    return out


def permutation(seed: int, stream: int, m: int) -> np.ndarray:
    out = np.empty(m, dtype=np.int32)
    if _gen().gen_permutation(seed, stream, m, out.ctypes.data) != 0:
        raise RuntimeError("gen_permutation failed")
    return out


def zipf_bias(m: int, s: float, alpha: float, seed: int) -> np.ndarray:
    """bias[pi(r-1)] = -alpha*s*ln(r), r = 1..m, rounded to fp32 (zeros when s == 0)."""
    bias = np.zeros(m, dtype=np.float32)
    if s == 0.0:
        return bias
    pi = permutation(seed, STREAM["bias_perm"], m)
    for r in range(1, m + 1):
        bias[pi[r - 1]] = np.float32(-alpha * s * math.log(r))
    return bias


def bf16_to_f32(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float32."""
    return (a.astype(np.uint32) << 16).view(np.float32)


def as_f32(a: np.ndarray, dtype: int) -> np.ndarray:
    return a if dtype == F32 else bf16_to_f32(a)


def make_moe_inputs(cfg: MoEWorkload, replicate: int = 0, alpha: Optional[float] = None,
                    nthreads: Optional[int] = None, weights: bool = True) -> Dict[str, np.ndarray]:
    """All inputs of one MoE-layer forward, as host arrays.

    Layouts (row-major, nn.Linear [out, in]): x [T,d]; w_router [m,d]; bias [m] fp32;
    w_gate, w_up [m,f,d]; w_down [m,d,f]; ws_gate, ws_up [n_shared,f_shared,d];
    ws_down [n_shared,d,f_shared]. ReLU experts use w_gate as W1 and have no w_up.
    """
    seed = cfg.seed(replicate)
    if alpha is None:
        alpha = zipf_alpha(cfg.name) if cfg.name in CONFIGS else 1.0
    T, d, f, m = cfg.T, cfg.d, cfg.f, cfg.m
    g = lambda key, shape, std: normal(seed, STREAM[key], shape, std, cfg.dtype, nthreads)
    out = {
        "x": g("x", (T, d), 1.0),
        "w_router": g("w_router", (m, d), 1.0 / math.sqrt(d)),
        "bias": zipf_bias(m, cfg.zipf_s, alpha, seed),
    }
    if weights:
        out["w_gate"] = g("w_gate", (m, f, d), 1.0 / math.sqrt(d))
        if cfg.act == SWIGLU:
            out["w_up"] = g("w_up", (m, f, d), 1.0 / math.sqrt(d))
        out["w_down"] = g("w_down", (m, d, f), 1.0 / math.sqrt(f))
        if cfg.n_shared:
            fs = cfg.f_shared
            out["ws_gate"] = g("ws_gate", (cfg.n_shared, fs, d), 1.0 / math.sqrt(d))
            if cfg.act == SWIGLU:
                out["ws_up"] = g("ws_up", (cfg.n_shared, fs, d), 1.0 / math.sqrt(d))
            out["ws_down"] = g("ws_down", (cfg.n_shared, d, fs), 1.0 / math.sqrt(fs))
    return out


def make_atomic_inputs(cfg: AtomicWorkload, replicate: int = 0, nthreads: Optional[int] = None,
                       experts: bool = True) -> Dict[str, np.ndarray]:
    """Inputs of the atomic-expert layer: x [T,d]; w_row [Nr,d]; w_col [Nc,d];
    w_in [N,d] (std 1/sqrt(d)); w_out [N,d] (std 1). No router bias."""
    seed = cfg.seed(replicate)
    g = lambda key, shape, std: normal(seed, STREAM[key], shape, std, cfg.dtype, nthreads)
    out = {
        "x": g("x", (cfg.T, cfg.d), 1.0),
        "w_row": g("w_row", (cfg.Nr, cfg.d), 1.0 / math.sqrt(cfg.d)),
        "w_col": g("w_col", (cfg.Nc, cfg.d), 1.0 / math.sqrt(cfg.d)),
    }
    if experts:
        out["w_in"] = g("w_in", (cfg.N, cfg.d), 1.0 / math.sqrt(cfg.d))
        out["w_out"] = g("w_out", (cfg.N, cfg.d), 1.0)
    return out


def small_moe(T, d, f, m, k, act=SWIGLU, dtype=BF16, zipf_s=1.0, renorm=False,
              n_shared=0, f_shared=0, index=90, name="small") -> MoEWorkload:
    """An ad-hoc small workload (tests): same recipe, its own seed index."""
    return MoEWorkload(name, index, T=T, d=d, f=f, m=m, k=k, act=act, dtype=dtype, zipf_s=zipf_s,
                       renorm=renorm, n_shared=n_shared, f_shared=f_shared)


def with_tokens(cfg: MoEWorkload, T: int) -> MoEWorkload:
    return replace(cfg, T=T)

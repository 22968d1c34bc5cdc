"""Helpers for the GPU parity tests: move generator arrays to the device, run the
C-ABI calls, and compare with the oracle under the stated tolerances."""
from __future__ import annotations

import numpy as np
import torch

import sparse_mixture_experts_08_b200 as moe
import workloads as W

# Float tolerances (per-token infinity-norm relative error, max over tokens):
# 2e-2 for bf16 operands with fp32 accumulation, 1e-5 for fp32.
TOL = {W.BF16: 2e-2, W.F32: 1e-5}
# Gate weights: fp32 softmax against the oracle's fp64 softmax of the same fp32 logits.
GATE_RTOL = 1e-6


def require_gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device (B200)"
    major, minor = torch.cuda.get_device_capability(0)
    assert (major, minor) == (10, 0), f"GPU tests need sm_100, found sm_{major}{minor}"


def dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    """Host array (float32, uint16 bf16 bits, int32, float64) -> device tensor with the same bits."""
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)
    return t.detach().cpu().numpy()


def out_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def torch_dtype(dt: int):
    return torch.float32 if dt == W.F32 else torch.bfloat16


def config_of(cfg: W.MoEWorkload) -> moe.MoEConfig:
    return moe.make_config(cfg.T, cfg.d, cfg.f, cfg.m, cfg.k, cfg.n_shared, cfg.f_shared, cfg.dtype, cfg.act,
                           cfg.renorm)


def token_rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    num = np.abs(got - ref).max(axis=1)
    den = np.abs(ref).max(axis=1)
    return float((num / np.maximum(den, 1e-300)).max())


def elem_rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    """Elementwise companion figure (reported, not asserted): max |got - ref| /
    (|ref| + 1e-3 rms(ref)) over all elements."""
    rms = float(np.sqrt(np.mean(np.square(ref)))) if ref.size else 0.0
    return float((np.abs(got - ref) / (np.abs(ref) + 1e-3 * rms + 1e-300)).max()) if ref.size else 0.0


def err_report(got: np.ndarray, ref: np.ndarray) -> str:
    return (f"max per-token relative error {token_rel_err(got, ref):.3e}, "
            f"elementwise max |d|/(|ref| + 1e-3 rms) {elem_rel_err(got, ref):.3e}")


def tile_cover_tokens(perm: np.ndarray, offsets: np.ndarray, k: int, step: int = 16) -> np.ndarray:
    """Tokens whose tasks sit at every `step`-th row of every expert segment (counted
    from the segment start), and at its last row. The grouped GEMM cuts a segment into
    token tiles whose height is a multiple of 16, so every tile of either projection
    starts at a segment row that is a multiple of 16 and holds a checked task, whatever
    tile height the library picked."""
    pick = set()
    for e in range(len(offsets) - 1):
        a, b = int(offsets[e]), int(offsets[e + 1])
        for r0 in range(a, b, step):
            pick.add(int(perm[r0]) // k)
        if b > a:
            pick.add(int(perm[b - 1]) // k)
    return np.array(sorted(pick), dtype=np.int32)


def covered_tiles(tokens: np.ndarray, perm: np.ndarray, offsets: np.ndarray, k: int, tile: int) -> bool:
    """True when every `tile`-row tile of every segment holds a task of `tokens`."""
    chosen = np.zeros(len(perm), bool)
    chosen[np.isin(perm // k, tokens)] = True
    for e in range(len(offsets) - 1):
        a, b = int(offsets[e]), int(offsets[e + 1])
        for r0 in range(a, b, tile):
            if not chosen[r0:min(b, r0 + tile)].any():
                return False
    return True


def device_inputs(inp):
    return {k: dev(v) for k, v in inp.items()}


def layer_forward(cfg: W.MoEWorkload, d_in, ws=None, stream=None):
    """Run moe_layer_forward; returns dict of device outputs."""
    c = config_of(cfg)
    if ws is None:
        ws = moe.workspace(c)
    T, m, k = cfg.T, cfg.m, cfg.k
    out = torch.empty((T, cfg.d), dtype=torch_dtype(cfg.dtype), device="cuda")
    logits = torch.empty((T, m), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    counts = torch.empty((m,), dtype=torch.int32, device="cuda")
    lis = moe.lis_buffer()
    offsets = torch.full((m + 1,), -7, dtype=torch.int32, device="cuda")
    perm = torch.full((T * k,), -7, dtype=torch.int32, device="cuda")
    inv_perm = torch.full((T * k,), -7, dtype=torch.int32, device="cuda")
    x_perm = torch.empty((T * k, cfg.d), dtype=torch_dtype(cfg.dtype), device="cuda")
    moe.moe_layer_forward(c, d_in["x"], d_in["w_router"], d_in["bias"], d_in["w_gate"], d_in.get("w_up"),
                          d_in["w_down"], d_in.get("ws_gate"), d_in.get("ws_up"), d_in.get("ws_down"), out, ws,
                          logits_out=logits, topk_idx_out=idx, topk_w_out=w, counts_out=counts, lis_out=lis,
                          offsets_out=offsets, perm_out=perm, inv_perm_out=inv_perm, x_perm_out=x_perm,
                          stream=stream)
    return {"out": out, "logits": logits, "idx": idx, "w": w, "counts": counts, "lis": lis, "ws": ws,
            "offsets": offsets, "perm": perm, "inv_perm": inv_perm, "x_perm": x_perm}


def sample_tokens(idx: np.ndarray, counts: np.ndarray, T: int, n: int, seed: int = 0) -> np.ndarray:
    """A token sample that always includes the first and last token, tokens of the
    most loaded expert and of the least loaded non-empty expert, and random others."""
    rng = np.random.default_rng(seed)
    pick = {0, T - 1}
    hot = int(np.argmax(counts))
    nz = np.nonzero(counts)[0]
    cold = int(nz[np.argmin(counts[nz])])
    for e in (hot, cold):
        toks = np.nonzero((idx == e).any(axis=1))[0]
        pick.update(toks[:2].tolist())
        pick.update(toks[-2:].tolist())
    while len(pick) < min(n, T):
        pick.add(int(rng.integers(0, T)))
    return np.array(sorted(pick), dtype=np.int32)

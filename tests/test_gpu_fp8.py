"""8-bit (E4M3) expert weights on the GPU against the oracle.

- Codes and scales: bit-exact. Both sides take max |row| / 448 and v / scale as
  IEEE fp32 divisions and round to nearest even.
- Routing: as the bf16 layer. Top-k ids, counts and LIS are decided on the GPU's
  own fp32 logits and compared bit-exactly.
- Stored h: within the bf16 layer tolerance of the oracle's h computed from the
  same quantized x and weights.
- Output, with h's codes decided on the GPU's stored h (same precision on both
  sides): within FP8_DECIDED_TOL. What is left is fp32 accumulation and the
  bf16 rounding of out.
- Output end to end, the oracle using its own h: within FP8_TOL. A bf16 rounding
  of a row's largest |h| that falls the other way moves that row's scale by one
  bf16 step and shifts up to ~1.5 % of the task's output.
"""
import numpy as np
import pytest
import torch

import oracle as O
import sparse_mixture_experts_08_b200 as moe
import workloads as W
from gpu_helpers import GATE_RTOL, TOL, config_of, dev, device_inputs, host, out_f64, require_gpu, token_rel_err

pytestmark = pytest.mark.gpu

FP8_DECIDED_TOL = 1e-2
FP8_TOL = 3e-2


@pytest.fixture(autouse=True, scope="module")
def _gpu():
    require_gpu()


def _bf16_bits(a32):
    return (np.ascontiguousarray(a32, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _quantize_gpu(bits):
    t = dev(bits)
    codes = torch.empty(t.shape, dtype=torch.uint8, device="cuda")
    scales = torch.empty(t.shape[:-1], dtype=torch.float32, device="cuda")
    moe.moe_quantize_e4m3(t, codes, scales)
    return host(codes), host(scales)


@pytest.mark.parametrize("shape", [(37, 256), (5, 14336), (300, 16), (64, 1408)])
def test_quantizer_is_bit_exact(shape):
    rng = np.random.default_rng(shape[0] * 7 + shape[1])
    rows, cols = shape
    a = rng.standard_normal(shape) * np.exp2(rng.integers(-30, 30, (rows, 1)))
    a[0] = 0.0                                           # all-zero row: scale 1, codes 0
    a[1, :] = -0.0
    a[2] = rng.integers(-3, 4, cols) * 2.0 ** -120       # tiny values (scale far below 2^-126)
    a[3] = np.where(rng.random(cols) < 0.5, 448.0, -3.5)  # values on codes and their negatives
    bits = _bf16_bits(a.astype(np.float32))
    codes, scales = _quantize_gpu(bits)
    ref_codes, ref_scales = O.quantize_rows(W.bf16_to_f32(bits))
    np.testing.assert_array_equal(scales.view(np.uint32), ref_scales.view(np.uint32))
    np.testing.assert_array_equal(codes, ref_codes)


def test_quantizer_on_generated_weights():
    cfg = W.small_moe(T=4, d=256, f=384, m=3, k=1, dtype=W.BF16, index=120)
    inp = W.make_moe_inputs(cfg)
    for key in ("w_gate", "w_up", "w_down"):
        codes, scales = _quantize_gpu(inp[key])
        ref = O.quantize_experts(cfg, inp)
        np.testing.assert_array_equal(codes, ref[key])
        np.testing.assert_array_equal(scales, ref[key + "_scale"])


def _fp8_layer(cfg, inp):
    c = config_of(cfg)
    d_in = device_inputs(inp)
    wq = moe.quantize_experts(d_in["w_gate"], d_in.get("w_up"), d_in["w_down"], d_in.get("ws_gate"),
                              d_in.get("ws_up"), d_in.get("ws_down"))
    ws = moe.fp8_workspace(c)
    T, k = cfg.T, cfg.k
    r = {"out": torch.empty((T, cfg.d), dtype=torch.bfloat16, device="cuda"),
         "logits": torch.empty((T, cfg.m), dtype=torch.float32, device="cuda"),
         "idx": torch.empty((T, k), dtype=torch.int32, device="cuda"),
         "w": torch.empty((T, k), dtype=torch.float32, device="cuda"),
         "counts": torch.empty((cfg.m,), dtype=torch.int32, device="cuda"),
         "lis": moe.lis_buffer(),
         "h": torch.empty((T * k, cfg.f), dtype=torch.bfloat16, device="cuda"),
         "h_sh": torch.empty((max(cfg.n_shared, 1) * T, max(cfg.f_shared, 16)), dtype=torch.bfloat16, device="cuda"),
         "perm": torch.empty((T * k,), dtype=torch.int32, device="cuda")}
    moe.moe_layer_forward_fp8(c, d_in["x"], d_in["w_router"], d_in["bias"], wq, r["out"], ws,
                              logits_out=r["logits"], topk_idx_out=r["idx"], topk_w_out=r["w"],
                              counts_out=r["counts"], lis_out=r["lis"], h_out=r["h"],
                              h_shared_out=r["h_sh"] if cfg.n_shared else None, perm_out=r["perm"])
    assert moe.moe_read_device_status(ws) == moe.OK
    return r


def _check_fp8(cfg, inp, tokens=None):
    r = _fp8_layer(cfg, inp)
    lg, idx, w = host(r["logits"]), host(r["idx"]), host(r["w"])
    oidx, ow = O.topk_softmax(lg, cfg.k, cfg.renorm)
    np.testing.assert_array_equal(idx, oidx)
    np.testing.assert_allclose(w, ow, rtol=GATE_RTOL, atol=1e-12)
    ref = O.histogram_lis(oidx, cfg.m)
    np.testing.assert_array_equal(host(r["counts"]), ref["counts"])
    assert moe.unpack_lis(r["lis"]) == (ref["max_count"], ref["argmax"], ref["lis"])
    toks = np.arange(cfg.T) if tokens is None else np.asarray(tokens)
    got = out_f64(r["out"])
    assert np.all(np.isfinite(got))
    # -- the permutation it ran on (bit-exact), then the stored h of every task of the
    # checked tokens, and the output from it
    perm = host(r["perm"])
    np.testing.assert_array_equal(perm, O.permutation(oidx, cfg.m, ref["offsets"])[0])
    row_of_task = np.empty(cfg.T * cfg.k, np.int64)
    row_of_task[perm] = np.arange(cfg.T * cfg.k)
    h_gpu = W.bf16_to_f32(host(r["h"]))
    xq, sx = O.quantize_rows(W.bf16_to_f32(inp["x"]))
    q = O.QuantizedExperts(cfg, inp)
    swiglu = cfg.act == W.SWIGLU
    decided = np.zeros((len(toks), cfg.d))
    h_err = 0.0
    for e in np.unique(oidx[toks]):  # one expert at a time, all its checked tasks together
        rows, slots = np.nonzero(oidx[toks] == e)
        t = toks[rows]
        h_ref = O.fp8_expert_up(xq[t], sx[t], q["w_gate"][e], q["w_gate_scale"][e],
                                q["w_up"][e] if swiglu else None, q["w_up_scale"][e] if swiglu else None, cfg.act)
        hg = h_gpu[row_of_task[t * cfg.k + slots]]
        h_err = max(h_err, token_rel_err(hg.astype(np.float64), h_ref))
        y = O.fp8_expert_down(hg, q["w_down"][e], q["w_down_scale"][e])
        np.add.at(decided, rows, ow[t, slots][:, None] * y)
    h_sh = W.bf16_to_f32(host(r["h_sh"])) if cfg.n_shared else None
    for sh in range(cfg.n_shared):
        decided += O.fp8_expert_down(h_sh[sh * cfg.T + toks], q["ws_down"][sh], q["ws_down_scale"][sh])
    assert h_err <= TOL[W.BF16], f"stored h: max relative error {h_err:.3e}"
    err_decided = token_rel_err(got[toks], decided)
    assert err_decided <= FP8_DECIDED_TOL, f"output (h decided on the GPU's h): {err_decided:.3e}"
    # -- end to end against the oracle's own h
    full = O.layer_forward_fp8(cfg, inp, qw=q, tokens=toks, logits_in=lg)["out"]
    err = token_rel_err(got[toks], full)
    assert err <= FP8_TOL, f"output end to end: {err:.3e}"
    return ref, err_decided, err


CASES = {
    # top-1 ReLU, K split of the down projection re-cut into 128-element blocks
    "relu_k1_split": dict(T=300, d=256, f=512, m=8, k=1, act=W.RELU, zipf_s=1.0),
    # 8192 tokens: fused router, one K range, top-1 combine fused into the down epilogue
    "relu_k1_fused": dict(T=8192, d=768, f=256, m=128, k=1, act=W.RELU, zipf_s=1.0),
    "swiglu_k2_renorm": dict(T=200, d=256, f=384, m=6, k=2, act=W.SWIGLU, zipf_s=0.8, renorm=True),
    "shared_k6": dict(T=96, d=256, f=128, m=16, k=6, act=W.SWIGLU, zipf_s=1.1, n_shared=2, f_shared=128),
    "decode_shape": dict(T=4, d=512, f=1024, m=8, k=2, act=W.SWIGLU, zipf_s=0.0),
    "empty_experts": dict(T=8, d=128, f=128, m=32, k=1, act=W.SWIGLU, zipf_s=0.0),
    "ragged_tail": dict(T=77, d=144, f=208, m=12, k=3, act=W.SWIGLU, zipf_s=1.5, n_shared=1, f_shared=80),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_fp8_layer(case):
    kw = dict(CASES[case])
    cfg = W.small_moe(dtype=W.BF16, index=121 + sorted(CASES).index(case), **kw)
    inp = W.make_moe_inputs(cfg)
    tokens = None if cfg.T <= 400 else np.r_[0:24, cfg.T - 24:cfg.T]
    _check_fp8(cfg, inp, tokens)


def test_fp8_decode_full_size():
    cfg = W.CONFIGS["decode"]
    _check_fp8(cfg, W.make_moe_inputs(cfg))


def test_fp8_output_stays_close_to_bf16_layer():
    """The quantization error itself (not a parity bar): the 8-bit layer stays within
    a few per cent of the bf16 layer, as the oracle's own comparison shows."""
    cfg = W.small_moe(T=64, d=512, f=768, m=8, k=2, dtype=W.BF16, zipf_s=0.5, index=130)
    inp = W.make_moe_inputs(cfg)
    r = _fp8_layer(cfg, inp)
    ref = O.layer_forward(cfg, inp, logits_in=host(r["logits"]))["out"]
    rel = np.linalg.norm(out_f64(r["out"]) - ref) / np.linalg.norm(ref)
    assert 5e-3 < rel < 0.15, rel

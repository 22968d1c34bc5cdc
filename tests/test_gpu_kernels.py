"""Kernel-by-kernel parity of the CUDA path (through the C ABI) against the oracle.

Integer work (top-k ids, counts, offsets, LIS, permutation) must match bit for
bit; the oracle takes the GPU's own fp32 logits for it, so both sides decide
from identical numbers. Float outputs must stay within the per-token relative
tolerance (2e-2 bf16, 1e-5 fp32); gate weights within 1e-6 relative.
"""
import numpy as np
import pytest
import torch

import oracle as O
import sparse_mixture_experts_08_b200 as moe
import workloads as W
from gpu_helpers import (GATE_RTOL, TOL, config_of, dev, device_inputs, host, out_f64, require_gpu,
                         token_rel_err, torch_dtype)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _gpu():
    require_gpu()


def _route(cfg, d_in, logits_in=None):
    c = config_of(cfg)
    ws = moe.workspace(c)
    lg = torch.empty((cfg.T, cfg.m), dtype=torch.float32, device="cuda")
    idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    w = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device="cuda")
    moe.moe_route(c, d_in.get("x"), d_in.get("w_router"), d_in.get("bias"), logits_in, lg, idx, w, ws)
    assert moe.moe_read_device_status(ws) == moe.OK
    return host(lg), host(idx), host(w)


ROUTE_CASES = [
    W.small_moe(T=64, d=128, f=256, m=8, k=2, dtype=W.F32, zipf_s=1.2, name="tiny_like"),
    W.small_moe(T=300, d=200, f=64, m=128, k=1, dtype=W.BF16, zipf_s=1.0, index=81),
    W.small_moe(T=257, d=512, f=64, m=64, k=6, dtype=W.BF16, zipf_s=1.1, index=82),
    W.small_moe(T=33, d=64, f=64, m=8, k=2, dtype=W.BF16, zipf_s=0.8, renorm=True, index=83),
    W.small_moe(T=5, d=72, f=64, m=200, k=7, dtype=W.BF16, zipf_s=1.0, index=84),
    W.small_moe(T=1, d=4096, f=64, m=8, k=2, dtype=W.BF16, zipf_s=0.0, index=85),
    W.small_moe(T=8269, d=72, f=64, m=200, k=8, dtype=W.BF16, zipf_s=0.7, renorm=True, index=89),
    W.small_moe(T=8192, d=64, f=64, m=256, k=2, dtype=W.BF16, zipf_s=1.0, index=90),
    # few experts (m <= 16): logits, top-k and gate weights in one CUDA-core launch;
    # ragged last block (T not a multiple of the tokens per block), m not a power of two
    W.small_moe(T=4099, d=4096, f=64, m=8, k=2, dtype=W.BF16, zipf_s=0.8, renorm=True, index=96),
    W.small_moe(T=777, d=264, f=64, m=12, k=3, dtype=W.BF16, zipf_s=1.0, index=97),
    W.small_moe(T=130, d=2048, f=64, m=16, k=16, dtype=W.BF16, zipf_s=0.5, index=98),
    W.small_moe(T=3, d=8, f=64, m=1, k=1, dtype=W.BF16, zipf_s=0.0, index=99),
    # 17 to 64 experts: the logits GEMM then the warp top-k (one and two logits per lane)
    W.small_moe(T=300, d=256, f=64, m=24, k=3, dtype=W.BF16, zipf_s=1.0, renorm=True, index=100),
    W.small_moe(T=2053, d=2048, f=64, m=64, k=6, dtype=W.BF16, zipf_s=1.0, index=101),
]


@pytest.mark.parametrize("cfg", ROUTE_CASES, ids=lambda c: f"T{c.T}_d{c.d}_m{c.m}_k{c.k}_{c.dtype}")
def test_route_topk_bit_exact_on_gpu_logits(cfg):
    inp = W.make_moe_inputs(cfg, weights=False)
    lg, idx, w = _route(cfg, device_inputs(inp))
    ref_lg = O.router_logits(inp["x"], inp["w_router"], inp["bias"])
    # fp32 accumulation of exact bf16/fp32 products vs the fp64 sum rounded once
    np.testing.assert_allclose(lg, ref_lg, rtol=0, atol=2e-5 * np.sqrt(cfg.d) * np.abs(ref_lg).max())
    oidx, ow = O.topk_softmax(lg, cfg.k, cfg.renorm)  # oracle decides on the GPU's own logits
    np.testing.assert_array_equal(idx, oidx)
    np.testing.assert_allclose(w, ow, rtol=GATE_RTOL, atol=1e-12)


def test_route_without_logits_output_selects_the_same():
    # the fused tensor-core router (8192+ tokens) writes logits only when asked; the
    # selection must not change
    cfg = W.small_moe(T=8269, d=72, f=64, m=200, k=8, dtype=W.BF16, zipf_s=0.7, renorm=True, index=89)
    d_in = device_inputs(W.make_moe_inputs(cfg, weights=False))
    _, idx, w = _route(cfg, d_in)
    c = config_of(cfg)
    ws = moe.workspace(c)
    idx2 = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    w2 = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device="cuda")
    moe.moe_route(c, d_in["x"], d_in["w_router"], d_in["bias"], None, None, idx2, w2, ws)
    assert moe.moe_read_device_status(ws) == moe.OK
    np.testing.assert_array_equal(host(idx2), idx)
    np.testing.assert_array_equal(host(w2), w)


def test_route_logits_in_verbatim_with_ties():
    cfg = W.small_moe(T=40, d=64, f=64, m=16, k=4, dtype=W.BF16)
    rng = np.random.default_rng(7)
    lg_in = (rng.integers(-2, 3, size=(cfg.T, cfg.m)) * 0.5).astype(np.float32)
    lg_in[0] = 0.0  # all equal -> experts 0..k-1
    lg, idx, w = _route(cfg, {}, logits_in=dev(lg_in))
    np.testing.assert_array_equal(lg, lg_in)
    oidx, ow = O.topk_softmax(lg_in, cfg.k, False)
    np.testing.assert_array_equal(idx, oidx)
    assert idx[0].tolist() == [0, 1, 2, 3]
    np.testing.assert_allclose(w, ow, rtol=GATE_RTOL)


@pytest.mark.parametrize("m,k", [(64, 6), (300, 17), (1024, 32)])
def test_route_logits_in_wide_rows_ties_signed_zeros_and_infinities(m, k):
    # the top-k kernel's register layouts (2, 8 and 32 logits per lane), heavy ties,
    # -0 against +0 (equal: the lower expert first), -inf logits and whole rows of them
    T = 67
    cfg = W.small_moe(T=T, d=64, f=64, m=m, k=k, dtype=W.BF16)
    rng = np.random.default_rng(m + k)
    lg_in = (rng.integers(-3, 4, size=(T, m)) * 0.25).astype(np.float32)
    lg_in[rng.random((T, m)) < 0.2] = -np.inf
    zeros = rng.random((T, m)) < 0.3
    lg_in[zeros] = np.where(rng.random(int(zeros.sum())) < 0.5, -0.0, 0.0).astype(np.float32)
    lg_in[1] = -0.0
    lg_in[2, : m // 2] = 0.0
    lg_in[2, m // 2:] = -0.0
    lg_in[3] = -np.inf
    lg_in[3, m - 1] = 1.0
    lg, idx, w = _route(cfg, {}, logits_in=dev(lg_in))
    np.testing.assert_array_equal(lg.view(np.uint32), lg_in.view(np.uint32))
    oidx, ow = O.topk_softmax(lg_in, k, False)
    np.testing.assert_array_equal(idx, oidx)
    assert idx[1].tolist() == list(range(k)) and idx[2].tolist() == list(range(k))
    assert idx[3, 0] == m - 1 and idx[3, 1:].tolist() == list(range(k - 1))
    np.testing.assert_allclose(w, ow, rtol=GATE_RTOL, atol=1e-12)


def _hist(cfg, idx_np):
    c = config_of(cfg)
    ws = moe.workspace(c)
    counts = torch.full((cfg.m,), -7, dtype=torch.int32, device="cuda")
    offsets = torch.full((cfg.m + 1,), -7, dtype=torch.int32, device="cuda")
    lis = moe.lis_buffer()
    moe.moe_histogram_lis(c, dev(idx_np), counts, offsets, lis, ws)
    st = moe.moe_read_device_status(ws)
    return st, host(counts), host(offsets), moe.unpack_lis(lis)


HIST_CASES = [(64, 8, 2), (8192, 128, 1), (2048, 64, 6), (1, 8, 2), (1000, 1024, 8), (3, 5, 5), (4096, 8, 2)]


@pytest.mark.parametrize("T,m,k", HIST_CASES)
@pytest.mark.parametrize("pattern", ["random", "one_expert", "balanced", "skewed"])
def test_histogram_lis_bit_exact(T, m, k, pattern):
    cfg = W.small_moe(T=T, d=64, f=64, m=m, k=k)
    rng = np.random.default_rng(T * 7 + m)
    if pattern == "random":
        idx = np.stack([rng.choice(m, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    elif pattern == "one_expert":
        idx = np.tile(np.arange(m - k, m, dtype=np.int32), (T, 1))
    elif pattern == "balanced":
        idx = ((np.arange(T)[:, None] * k + np.arange(k)[None, :]) % m).astype(np.int32)
        if k > 1 and m < k * 2:
            idx = np.stack([np.roll(np.arange(m), -t)[:k] for t in range(T)]).astype(np.int32)
    else:
        p = 1.0 / np.arange(1, m + 1) ** 1.5
        idx = np.stack([rng.choice(m, size=k, replace=False, p=p / p.sum()) for _ in range(T)]).astype(np.int32)
    st, counts, offsets, (mx, am, lis) = _hist(cfg, idx)
    assert st == moe.OK
    ref = O.histogram_lis(idx, m)
    np.testing.assert_array_equal(counts, ref["counts"])
    np.testing.assert_array_equal(offsets, ref["offsets"])
    assert (mx, am) == (ref["max_count"], ref["argmax"])
    assert lis == ref["lis"]  # one correctly rounded fp64 division on both sides


def test_lis_from_counts_of_two_batches_is_the_whole_batch_lis():
    """The job-wide LIS (bench --global-lis): two batches' histograms from the GPU,
    summed as the all-reduce across ranks sums them, then moe_lis_from_counts; equal
    to the oracle's max, argmax and LIS of the two routings taken together."""
    m, k = 64, 6
    rng = np.random.default_rng(12)
    p = 1.0 / np.arange(1, m + 1) ** 1.2
    batches = [np.stack([rng.choice(m, size=k, replace=False, p=p / p.sum()) for _ in range(T)]).astype(np.int32)
               for T in (300, 517)]
    total = torch.zeros(m, dtype=torch.int32, device="cuda")
    for idx in batches:
        cfg = W.small_moe(T=idx.shape[0], d=64, f=64, m=m, k=k)
        st, counts, _, _ = _hist(cfg, idx)
        assert st == moe.OK
        total += dev(counts)
    lis = moe.lis_buffer()
    moe.moe_lis_from_counts(m, sum(b.shape[0] for b in batches) * k, total, lis)
    ref = O.histogram_lis(np.concatenate(batches), m)
    assert moe.unpack_lis(lis) == (ref["max_count"], ref["argmax"], ref["lis"])
    # equal maxima: the lowest expert index, as in moe_histogram_lis
    tied = torch.zeros(m, dtype=torch.int32, device="cuda")
    tied[[5, 40, 63]] = 9
    moe.moe_lis_from_counts(m, 27, tied, lis)
    assert moe.unpack_lis(lis) == (9, 5, m * 9 / 27)


def test_histogram_rejects_bad_expert_id_without_writing():
    cfg = W.small_moe(T=10, d=64, f=64, m=8, k=2)
    idx = np.tile(np.array([1, 2], np.int32), (10, 1))
    idx[7, 1] = 8  # == m
    st, counts, offsets, _ = _hist(cfg, idx)
    assert st == moe.ERR_DEVICE_INDEX
    assert np.all(counts == -7) and np.all(offsets == -7)
    idx[7, 1] = -1
    st, counts, _, _ = _hist(cfg, idx)
    assert st == moe.ERR_DEVICE_INDEX and np.all(counts == -7)


@pytest.mark.parametrize("T,m,k,d,dtype", [(64, 8, 2, 128, W.F32), (8192, 128, 1, 768, W.BF16),
                                           (2048, 64, 6, 2048, W.BF16), (1, 8, 2, 4096, W.BF16),
                                           (999, 1024, 8, 64, W.BF16)])
def test_permute_bit_exact(T, m, k, d, dtype):
    cfg = W.small_moe(T=T, d=d, f=64, m=m, k=k, dtype=dtype, zipf_s=1.0, index=86)
    inp = W.make_moe_inputs(cfg, weights=False)
    rng = np.random.default_rng(3)
    p = 1.0 / np.arange(1, m + 1) ** 1.1
    idx = np.stack([rng.choice(m, size=k, replace=False, p=p / p.sum()) for _ in range(T)]).astype(np.int32)
    ref = O.histogram_lis(idx, m)
    rperm, rinv = O.permutation(idx, m, ref["offsets"])
    c = config_of(cfg)
    ws = moe.workspace(c)
    x = dev(inp["x"])
    x_perm = torch.empty((T * k, d), dtype=x.dtype, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * k, dtype=torch.int32, device="cuda")
    moe.moe_permute(c, x, dev(idx), dev(ref["offsets"]), x_perm, perm, inv, ws)
    assert moe.moe_read_device_status(ws) == moe.OK
    np.testing.assert_array_equal(host(perm), rperm)
    np.testing.assert_array_equal(host(inv), rinv)
    np.testing.assert_array_equal(host(x_perm), inp["x"][rperm // k])


FFN_CASES = [
    # (T, d, f, m, k, act, dtype, zipf_s) - tile edges: d, f not multiples of 64/128; ragged segments
    (64, 128, 256, 8, 2, W.SWIGLU, W.F32, 1.2),
    (64, 128, 256, 8, 2, W.SWIGLU, W.BF16, 1.2),
    (200, 200, 136, 6, 2, W.SWIGLU, W.BF16, 1.0),
    (300, 256, 384, 16, 1, W.RELU, W.BF16, 1.0),
    (37, 72, 520, 5, 3, W.SWIGLU, W.BF16, 2.0),
    (1, 512, 1024, 8, 2, W.SWIGLU, W.BF16, 0.0),
    (700, 64, 64, 4, 1, W.RELU, W.BF16, 3.0),
    (130, 96, 160, 3, 2, W.RELU, W.F32, 0.5),
    # 256+ rows per expert on average: two-CTA pair tiles (256 weight rows over two SMs,
    # up to 256 token rows); f and K not multiples of the tile, ragged and skewed segments
    (1000, 256, 384, 4, 2, W.SWIGLU, W.BF16, 1.0),
    (2048, 136, 200, 4, 1, W.RELU, W.BF16, 2.0),
    (600, 512, 256, 2, 1, W.SWIGLU, W.BF16, 0.0),
    (1300, 64, 520, 3, 2, W.SWIGLU, W.BF16, 3.0),
]


@pytest.mark.parametrize("T,d,f,m,k,act,dtype,s", FFN_CASES)
def test_grouped_ffn_vs_oracle(T, d, f, m, k, act, dtype, s):
    cfg = W.small_moe(T=T, d=d, f=f, m=m, k=k, act=act, dtype=dtype, zipf_s=s, index=87)
    inp = W.make_moe_inputs(cfg)
    logits = O.router_logits(inp["x"], inp["w_router"], inp["bias"])
    idx, wgt = O.topk_softmax(logits, k, False)
    ref = O.histogram_lis(idx, m)
    perm, inv = O.permutation(idx, m, ref["offsets"])
    x_perm = inp["x"][perm // k]
    task_w = wgt.astype(np.float32).ravel()
    c = config_of(cfg)
    ws = moe.workspace(c)
    d_in = device_inputs(inp)
    y = torch.full((T * k, d), float("nan"), dtype=torch.float32, device="cuda")
    moe.moe_grouped_ffn(c, dev(np.ascontiguousarray(x_perm)), dev(ref["offsets"]), d_in["w_gate"], d_in.get("w_up"),
                        d_in["w_down"], dev(task_w), dev(perm), y, ws)
    assert moe.moe_read_device_status(ws) == moe.OK
    got = out_f64(y)
    exp = np.empty_like(got)
    for pos in range(T * k):
        q = perm[pos]
        e = idx[q // k, q % k]
        yy = O.expert_ffn(inp["x"][q // k], inp["w_gate"][e], inp["w_up"][e] if act == W.SWIGLU else None,
                          inp["w_down"][e], act)
        exp[pos] = float(task_w[q]) * yy
    assert token_rel_err(got, exp) <= TOL[dtype]


@pytest.mark.parametrize("dtype", [W.F32, W.BF16])
def test_shared_ffn_and_combine(dtype):
    cfg = W.small_moe(T=50, d=96, f=64, m=6, k=2, act=W.SWIGLU, dtype=dtype, n_shared=2, f_shared=80, index=88)
    inp = W.make_moe_inputs(cfg)
    c = config_of(cfg)
    ws = moe.workspace(c)
    d_in = device_inputs(inp)
    ysh = torch.empty((2, cfg.T, cfg.d), dtype=torch.float32, device="cuda")
    moe.moe_shared_ffn(c, d_in["x"], d_in["ws_gate"], d_in["ws_up"], d_in["ws_down"], ysh, ws)
    assert moe.moe_read_device_status(ws) == moe.OK
    for s in range(2):
        exp = np.stack([O.expert_ffn(inp["x"][t], inp["ws_gate"][s], inp["ws_up"][s], inp["ws_down"][s], W.SWIGLU)
                        for t in range(cfg.T)])
        assert token_rel_err(out_f64(ysh[s]), exp) <= TOL[dtype]
    # combine: out[t] = sum_s y_perm[inv[t k + s]] + sum_sh ysh[sh, t]
    rng = np.random.default_rng(9)
    y_perm = rng.standard_normal((cfg.T * 2, cfg.d)).astype(np.float32)
    inv = rng.permutation(cfg.T * 2).astype(np.int32)
    out = torch.empty((cfg.T, cfg.d), dtype=torch_dtype(dtype), device="cuda")
    moe.moe_combine(c, dev(y_perm), dev(inv), ysh, out)
    torch.cuda.synchronize()
    ref = y_perm[inv.reshape(cfg.T, 2)].astype(np.float64).sum(1) + out_f64(ysh).sum(0)
    assert token_rel_err(out_f64(out), ref) <= (TOL[dtype] if dtype == W.BF16 else 1e-6)

"""End-to-end parity of moe_layer_forward (the call the benchmark times) on every
workload at full size, plus the atomic-expert variant.

All tokens: top-k ids, counts, max/argmax, LIS, segment offsets, perm and
inv_perm bit-exact against the oracle deciding on the GPU's own fp32 logits, and
every permuted token row a bit copy of its token's row. Outputs: every token for
the small workloads; for the large ones a sample the oracle can evaluate token by
token that reaches every 128-row token tile of every expert segment (plus the
first and last token and tokens of the most and least loaded experts), within the
per-token relative tolerance; the elementwise figure is reported beside it.
"""
import numpy as np
import pytest
import torch

import oracle as O
import sparse_mixture_experts_08_b200 as moe
import workloads as W
from gpu_helpers import (GATE_RTOL, TOL, covered_tiles, device_inputs, err_report, host, layer_forward, out_f64,
                         require_gpu, sample_tokens, tile_cover_tokens, token_rel_err)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _gpu():
    require_gpu()


def _check_layer(cfg, inp, n_sample):
    d_in = device_inputs(inp)
    r = layer_forward(cfg, d_in)
    assert moe.moe_read_device_status(r["ws"]) == moe.OK
    lg, idx, w, counts = host(r["logits"]), host(r["idx"]), host(r["w"]), host(r["counts"])
    # integer parity on the GPU's logits (whole batch)
    oidx, ow = O.topk_softmax(lg, cfg.k, cfg.renorm)
    np.testing.assert_array_equal(idx, oidx)
    np.testing.assert_allclose(w, ow, rtol=GATE_RTOL, atol=1e-12)
    ref = O.histogram_lis(oidx, cfg.m)
    np.testing.assert_array_equal(counts, ref["counts"])
    mx, am, lis = moe.unpack_lis(r["lis"])
    assert (mx, am, lis) == (ref["max_count"], ref["argmax"], ref["lis"])
    # the expert-centric permutation (OmniMoE Fig. 3), whichever routing path ran
    np.testing.assert_array_equal(host(r["offsets"]), ref["offsets"])
    operm, oinv = O.permutation(oidx, cfg.m, ref["offsets"])
    perm = host(r["perm"])
    np.testing.assert_array_equal(perm, operm)
    np.testing.assert_array_equal(host(r["inv_perm"]), oinv)
    x_perm = host(r["x_perm"])
    assert np.array_equal(x_perm.view(np.uint32 if x_perm.dtype == np.float32 else np.uint16),
                          inp["x"][operm // cfg.k].view(np.uint32 if x_perm.dtype == np.float32 else np.uint16))
    # float parity
    if n_sample >= cfg.T:
        toks = np.arange(cfg.T, dtype=np.int32)
    else:
        toks = np.union1d(sample_tokens(oidx, ref["counts"], cfg.T, n_sample),
                          tile_cover_tokens(operm, ref["offsets"], cfg.k)).astype(np.int32)
        assert covered_tiles(toks, operm, ref["offsets"], cfg.k, 16)
    exp = O.moe_output(cfg, inp, oidx, ow, tokens=toks)
    got = out_f64(r["out"])[toks]
    err = token_rel_err(got, exp)
    assert err <= TOL[cfg.dtype], err_report(got, exp)
    assert np.all(np.isfinite(out_f64(r["out"])))
    return ref, err


def test_tiny_fp32_all_tokens():
    cfg = W.CONFIGS["tiny"]
    _check_layer(cfg, W.make_moe_inputs(cfg), n_sample=cfg.T)


def test_tiny_fp32_renormalised_and_shared():
    cfg = W.small_moe(T=64, d=128, f=256, m=8, k=2, dtype=W.F32, zipf_s=1.2, renorm=True, n_shared=1, f_shared=64,
                      index=71)
    _check_layer(cfg, W.make_moe_inputs(cfg), n_sample=cfg.T)


def test_switch_full_size():
    cfg = W.CONFIGS["switch"]
    ref, _ = _check_layer(cfg, W.make_moe_inputs(cfg), n_sample=48)
    assert 2.0 <= ref["lis"] <= 4.0


def test_mixtral_full_size():
    cfg = W.CONFIGS["mixtral"]
    _check_layer(cfg, W.make_moe_inputs(cfg), n_sample=12)


def test_dsv2lite_full_size():
    cfg = W.CONFIGS["dsv2lite"]
    ref, _ = _check_layer(cfg, W.make_moe_inputs(cfg), n_sample=24)
    assert 3.5 <= ref["lis"] <= 4.5


def test_decode_all_tokens():
    cfg = W.CONFIGS["decode"]
    _check_layer(cfg, W.make_moe_inputs(cfg), n_sample=cfg.T)


@pytest.mark.parametrize("case", ["one_hot", "one_hot_fused", "T1", "ragged_small", "relu_many_experts",
                                  "max_experts_max_k", "routed_k8_m200", "pair_shared", "pair_empty_and_single",
                                  "pair_relu_top1", "pair_dual_shared"])
def test_layer_edge_cases(case):
    if case in ("one_hot", "one_hot_fused"):  # every token's top-1 is the same expert (huge bias)
        T = 300 if case == "one_hot" else 8192  # 8192: the fused router and scatter
        cfg = W.small_moe(T=T, d=256, f=192, m=16, k=2, dtype=W.BF16, zipf_s=0.0, index=72)
        inp = W.make_moe_inputs(cfg)
        inp["bias"][:] = 0.0
        inp["bias"][11] = 1000.0
    elif case == "T1":
        cfg = W.small_moe(T=1, d=1024, f=512, m=8, k=2, dtype=W.BF16, zipf_s=0.8, renorm=True, index=73)
        inp = W.make_moe_inputs(cfg)
    elif case == "ragged_small":
        cfg = W.small_moe(T=77, d=136, f=200, m=12, k=3, dtype=W.BF16, zipf_s=1.5, n_shared=1, f_shared=72,
                          index=74)
        inp = W.make_moe_inputs(cfg)
    elif case == "relu_many_experts":
        cfg = W.small_moe(T=1500, d=128, f=320, m=256, k=2, act=W.RELU, dtype=W.BF16, zipf_s=1.0, index=75)
        inp = W.make_moe_inputs(cfg)
    elif case == "routed_k8_m200":  # fused router (8192+ tokens): largest k, m not a power of two, ragged tile
        cfg = W.small_moe(T=8269, d=64, f=64, m=200, k=8, dtype=W.BF16, zipf_s=0.7, renorm=True, index=78)
        inp = W.make_moe_inputs(cfg)
    elif case == "pair_shared":  # pair tiles (256+ rows per expert) with a shared expert as a second class
        cfg = W.small_moe(T=1024, d=256, f=256, m=4, k=1, dtype=W.BF16, zipf_s=1.0, n_shared=1, f_shared=136,
                          index=79)
        inp = W.make_moe_inputs(cfg)
    elif case == "pair_empty_and_single":  # pair tiles; one expert gets no task, one exactly one
        cfg = W.small_moe(T=1200, d=192, f=320, m=4, k=1, dtype=W.BF16, zipf_s=0.0, index=80)
        inp = W.make_moe_inputs(cfg)
        inp["bias"][:] = 0.0
        inp["bias"][2] = -1000.0                          # expert 2: no task
        inp["bias"][3] = -100.0                           # expert 3: only token 0, through input column 5
        inp["x"][:, 5] = 0
        inp["x"][0, 5] = 0x4180                           # bf16 16.0
        inp["w_router"][3, :] = 0
        inp["w_router"][3, 5] = 0x4280                    # bf16 64.0: logit 1024 - 100 for token 0, -100 for the rest
    elif case == "pair_relu_top1":  # pair tiles, top-1 ReLU: the down epilogue writes the layer output;
        # d = 640: the down projection's two 256-row feature blocks, the second one ragged
        cfg = W.small_moe(T=2048, d=640, f=512, m=4, k=1, act=W.RELU, dtype=W.BF16, zipf_s=1.5, index=81)
        inp = W.make_moe_inputs(cfg)
    elif case == "pair_dual_shared":  # two feature blocks per down tile (d = 768) beside a shared expert
        cfg = W.small_moe(T=1024, d=768, f=256, m=4, k=2, dtype=W.BF16, zipf_s=1.0, n_shared=1, f_shared=128,
                          index=82)
        inp = W.make_moe_inputs(cfg)
    else:  # the largest expert count and top-k the library accepts (m = 1024, k = 32)
        cfg = W.small_moe(T=700, d=64, f=64, m=1024, k=32, dtype=W.BF16, zipf_s=0.5, index=77)
        inp = W.make_moe_inputs(cfg)
    ref, _ = _check_layer(cfg, inp, n_sample=min(cfg.T, 64))
    if case.startswith("one_hot"):  # expert 11 holds every token: LIS reaches its maximum m / k
        assert ref["counts"][11] == cfg.T and ref["lis"] == cfg.m / cfg.k
    if case == "pair_empty_and_single":
        assert ref["counts"][2] == 0 and ref["counts"][3] == 1


def test_workspace_reuse_is_stable():
    cfg = W.small_moe(T=257, d=256, f=384, m=8, k=2, dtype=W.BF16, zipf_s=1.0, index=76)
    d_in = device_inputs(W.make_moe_inputs(cfg))
    r1 = layer_forward(cfg, d_in)
    r2 = layer_forward(cfg, d_in, ws=r1["ws"])
    torch.cuda.synchronize()
    assert torch.equal(r1["out"], r2["out"])  # deterministic: no atomics on float data


# ------------------------------------------------------------------ atomic experts

def _atomic(cfg, inp):
    c = moe.make_atomic_config(cfg.T, cfg.d, cfg.Nr, cfg.Nc, cfg.K, cfg.act)
    ws = moe.workspace(c)
    d_in = device_inputs(inp)
    lr = torch.empty((cfg.T, cfg.Nr), dtype=torch.float32, device="cuda")
    lc = torch.empty((cfg.T, cfg.Nc), dtype=torch.float32, device="cuda")
    idx = torch.empty((cfg.T, cfg.K), dtype=torch.int32, device="cuda")
    g = torch.empty((cfg.T, cfg.K), dtype=torch.float32, device="cuda")
    moe.moe_atomic_route(c, d_in["x"], d_in["w_row"], d_in["w_col"], lr, lc, idx, g, ws)
    out = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device="cuda")
    moe.moe_atomic_experts(c, d_in["x"], d_in["w_in"], d_in["w_out"], idx, g, out, ws)
    out2 = torch.empty_like(out)
    moe.moe_atomic_forward(c, d_in["x"], d_in["w_row"], d_in["w_col"], d_in["w_in"], d_in["w_out"], out2, ws)
    assert moe.moe_read_device_status(ws) == moe.OK
    return host(lr), host(lc), host(idx), host(g), out, out2


@pytest.mark.parametrize("case", ["small", "full", "wide_k"])
def test_atomic_layer(case):
    if case == "full":
        cfg = W.CONFIGS["atomic"]
    elif case == "wide_k":  # a prefill budget: K = 512 (the radix selection), every slot through the experts
        cfg = W.AtomicWorkload("atomic_wide", 95, T=6, d=256, Nr=64, Nc=128, K=512, act=W.ACT_SILU)
    else:
        cfg = W.AtomicWorkload("atomic_small", 92, T=5, d=256, Nr=64, Nc=128, K=16, act=W.ACT_SIGMOID)
    inp = W.make_atomic_inputs(cfg)
    lr, lc, idx, g, out, out2 = _atomic(cfg, inp)
    olr, olc = O.atomic_logprobs(inp["x"], inp["w_row"], inp["w_col"])
    np.testing.assert_allclose(lr, olr, rtol=0, atol=2e-4)
    np.testing.assert_allclose(lc, olc, rtol=0, atol=2e-4)
    oidx, og = O.atomic_select(lr, lc, cfg.K)  # oracle selects on the GPU's own log-probabilities
    np.testing.assert_array_equal(idx, oidx)
    np.testing.assert_allclose(g, og, rtol=GATE_RTOL * 4, atol=1e-9)
    exp = O.atomic_output(inp["x"], inp["w_in"], inp["w_out"], oidx, og, cfg.act)
    assert token_rel_err(out_f64(out), exp) <= TOL[W.BF16]
    torch.cuda.synchronize()
    assert torch.equal(out, out2)


def test_atomic_select_ties_and_rounding_collapse():
    # Row/column weights built so many grid scores tie exactly: x = e_0 and integer-valued
    # logits; the exact top-K must follow (S desc, flat id asc).
    cfg = W.AtomicWorkload("atomic_ties", 93, T=2, d=64, Nr=64, Nc=64, K=64, act=W.ACT_SILU)
    inp = W.make_atomic_inputs(cfg)
    x = np.zeros((2, 64), np.uint16)
    x[:, 0] = 0x3F80  # bf16 1.0
    inp["x"] = x
    rng = np.random.default_rng(5)
    for key in ("w_row", "w_col"):
        vals = rng.integers(0, 3, size=64).astype(np.float32)  # 0, 1, 2 -> heavy ties
        wr = np.zeros((64, 64), np.uint16)
        wr[:, 0] = (vals.view(np.uint32) >> 16).astype(np.uint16)
        inp[key] = wr
    lr, lc, idx, g, out, _ = _atomic(cfg, inp)
    oidx, og = O.atomic_select(lr, lc, cfg.K)
    np.testing.assert_array_equal(idx, oidx)


def _route_only(cfg, inp):
    c = moe.make_atomic_config(cfg.T, cfg.d, cfg.Nr, cfg.Nc, cfg.K, cfg.act)
    ws = moe.workspace(c)
    d_in = device_inputs(inp)
    lr = torch.empty((cfg.T, cfg.Nr), dtype=torch.float32, device="cuda")
    lc = torch.empty((cfg.T, cfg.Nc), dtype=torch.float32, device="cuda")
    idx = torch.empty((cfg.T, cfg.K), dtype=torch.int32, device="cuda")
    g = torch.empty((cfg.T, cfg.K), dtype=torch.float32, device="cuda")
    moe.moe_atomic_route(c, d_in["x"], d_in["w_row"], d_in["w_col"], lr, lc, idx, g, ws)
    assert moe.moe_read_device_status(ws) == moe.OK
    return host(lr), host(lc), host(idx), host(g)


def _level_weights(rows, d, levels, seed):
    """bf16 weights whose only non-zero column is 0, holding integers in [0, levels)."""
    vals = np.random.default_rng(seed).integers(0, levels, size=rows).astype(np.float32)
    w = np.zeros((rows, d), np.uint16)
    w[:, 0] = (vals.view(np.uint32) >> 16).astype(np.uint16)
    return w


@pytest.mark.parametrize("Nr,Nc,K,kind", [
    (64, 1024, 7, "random"),      # rectangular grid, K below the row count
    (1024, 64, 1, "random"),      # K = 1
    (1024, 1024, 64, "random"),   # largest grid, largest K
    (1024, 1024, 64, "equal"),    # every pair ties: the K lowest flat ids
    (128, 128, 64, "levels"),     # few distinct scores: long tied runs per row
    (1024, 512, 33, "levels"),
    # K > 64: the radix selection over the whole grid
    (128, 128, 65, "random"),
    (64, 64, 4096, "random"),      # K = N: the whole grid in order
    (512, 512, 512, "random"),
    (1024, 1024, 4096, "random"),  # largest grid, largest K
    (512, 512, 1000, "levels"),    # ties at the threshold: lowest flat ids among them
    (1024, 64, 2000, "levels"),
    (256, 256, 4096, "equal"),     # every pair ties
])
def test_atomic_select_grid_shapes(Nr, Nc, K, kind):
    cfg = W.AtomicWorkload("atomic_grid", 94, T=3, d=64, Nr=Nr, Nc=Nc, K=K, act=W.ACT_SILU)
    inp = W.make_atomic_inputs(cfg, experts=False)
    if kind != "random":
        x = np.zeros((cfg.T, cfg.d), np.uint16)
        x[:, 0] = 0x3F80  # bf16 1.0: the logits are column 0 of the weights
        inp["x"] = x
        levels = 1 if kind == "equal" else 3
        inp["w_row"] = _level_weights(Nr, cfg.d, levels, 6)
        inp["w_col"] = _level_weights(Nc, cfg.d, levels, 7)
    lr, lc, idx, g = _route_only(cfg, inp)
    oidx, og = O.atomic_select(lr, lc, cfg.K)
    np.testing.assert_array_equal(idx, oidx)
    np.testing.assert_allclose(g, og, rtol=GATE_RTOL * 4, atol=1e-9)
    if kind == "equal":
        np.testing.assert_array_equal(idx, np.tile(np.arange(K, dtype=np.int32), (cfg.T, 1)))


def test_atomic_prefill_full_size():
    """4096 tokens, K = 512 of a 512 x 512 grid: routing of every token bit-exact on the
    GPU's log-probabilities; the output of a token sample within the bf16 tolerance."""
    cfg = W.CONFIGS["atomic_prefill"]
    inp = W.make_atomic_inputs(cfg)
    lr, lc, idx, g, out, out2 = _atomic(cfg, inp)
    olr, olc = O.atomic_logprobs(inp["x"][:8], inp["w_row"], inp["w_col"])
    np.testing.assert_allclose(lr[:8], olr, rtol=0, atol=2e-4)
    np.testing.assert_allclose(lc[:8], olc, rtol=0, atol=2e-4)
    toks = np.r_[0:6, 2047, cfg.T - 6:cfg.T]
    oidx, og = O.atomic_select(lr[toks], lc[toks], cfg.K)
    np.testing.assert_array_equal(idx[toks], oidx)
    np.testing.assert_allclose(g[toks], og, rtol=GATE_RTOL * 4, atol=1e-9)
    assert np.all((idx >= 0) & (idx < cfg.N))
    assert np.all(np.sort(idx, axis=1)[:, 1:] != np.sort(idx, axis=1)[:, :-1])  # K distinct experts per token
    idx_s = np.zeros((cfg.T, cfg.K), np.int32)  # the oracle's routing at the sampled tokens
    g_s = np.zeros((cfg.T, cfg.K), np.float64)
    idx_s[toks], g_s[toks] = oidx, og
    exp = O.atomic_output(inp["x"], inp["w_in"], inp["w_out"], idx_s, g_s, cfg.act, tokens=toks)
    assert token_rel_err(out_f64(out)[toks], exp) <= TOL[W.BF16]
    torch.cuda.synchronize()
    assert torch.equal(out, out2)

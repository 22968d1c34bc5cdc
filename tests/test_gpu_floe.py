"""FloE contextual sparsity on the GPU against the oracle. The keep decision is a
comparison of floats, so the oracle takes it on the GPU's own up-projection
values (returned by the layer), as the router's integer parity uses the GPU's
logits; everything else it computes in fp64."""
import numpy as np
import pytest
import torch

import oracle as O
import sparse_mixture_experts_08_b200 as moe
import workloads as W
from gpu_helpers import TOL, config_of, dev, device_inputs, host, layer_forward, out_f64, require_gpu, token_rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _gpu():
    require_gpu()


def test_pack_down_is_the_per_expert_transpose():
    cfg = W.small_moe(T=4, d=72, f=104, m=3, k=1, dtype=W.BF16, index=110)
    inp = W.make_moe_inputs(cfg)
    c = config_of(cfg)
    wt = torch.empty((cfg.m, cfg.f, cfg.d), dtype=torch.bfloat16, device="cuda")
    moe.moe_floe_pack_down(c, dev(inp["w_down"]), wt)
    np.testing.assert_array_equal(host(wt), np.ascontiguousarray(inp["w_down"].transpose(0, 2, 1)))


def _calibrate(cfg, inp_w, s, Tc=24):
    c = config_of(cfg)
    xc = W.make_moe_inputs(W.with_tokens(cfg, Tc), replicate=1, weights=False)["x"]  # a different batch
    u = torch.empty((Tc, cfg.m * cfg.f), dtype=torch.float32, device="cuda")
    thr = torch.empty(cfg.m, dtype=torch.float32, device="cuda")
    ws = moe.workspace(c)
    moe.moe_floe_calibrate(c, dev(xc), dev(inp_w["w_up"]), s, u, thr, ws)
    assert moe.moe_read_device_status(ws) == moe.OK
    return xc, host(u), host(thr)


@pytest.mark.parametrize("s", [0.0, 0.5, 0.9, 0.99])
def test_calibrated_thresholds_are_the_order_statistic(s):
    cfg = W.small_moe(T=16, d=256, f=320, m=4, k=2, dtype=W.BF16, index=111)
    inp = W.make_moe_inputs(cfg)
    xc, u, thr = _calibrate(cfg, inp, s)
    for e in range(cfg.m):
        assert thr[e] == O.floe_threshold(np.abs(u[:, e * cfg.f:(e + 1) * cfg.f]), s)
    # the calibration activations themselves: fp32 accumulation of bf16 products
    x64 = np.asarray(W.as_f32(xc, W.BF16), np.float64)
    ref = x64 @ np.asarray(W.as_f32(inp["w_up"], W.BF16), np.float64).reshape(cfg.m * cfg.f, cfg.d).T
    np.testing.assert_allclose(u, ref, rtol=0, atol=2e-5 * np.sqrt(cfg.d) * np.abs(ref).max())


def _floe_layer(cfg, inp, thr):
    c = config_of(cfg)
    d_in = device_inputs(inp)
    wt = torch.empty((cfg.m, cfg.f, cfg.d), dtype=torch.bfloat16, device="cuda")
    moe.moe_floe_pack_down(c, d_in["w_down"], wt)
    ws = moe.floe_workspace(c)
    Tk = cfg.T * cfg.k
    out = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    w = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device="cuda")
    kept = torch.empty(cfg.m, dtype=torch.int32, device="cuda")
    u = torch.empty((Tk, cfg.f), dtype=torch.float32, device="cuda")
    perm = torch.empty(Tk, dtype=torch.int32, device="cuda")
    moe.moe_layer_forward_floe(c, d_in["x"], d_in["w_router"], d_in["bias"], d_in["w_gate"], d_in["w_up"], wt,
                               dev(np.asarray(thr, np.float32)), out, ws, topk_idx_out=idx, topk_w_out=w,
                               kept_out=kept, u_out=u, perm_out=perm)
    assert moe.moe_read_device_status(ws) == moe.OK
    return d_in, {"out": out, "idx": host(idx), "w": host(w), "kept": host(kept), "u": host(u), "perm": host(perm)}


CASES = [
    (W.small_moe(T=16, d=256, f=320, m=4, k=2, dtype=W.BF16, zipf_s=0.5, index=112, name="small"), 0.8),
    (W.CONFIGS["decode"], 0.9),
    # d > 4096: four 16-byte column chunks per thread, two channels per stage, a
    # ragged last column slice; ~27 rows per expert = several 4-row passes (sparsity
    # high enough that the union over an expert's rows still skips channels)
    (W.small_moe(T=40, d=4352, f=200, m=3, k=2, dtype=W.BF16, zipf_s=0.3, index=114, name="wide"), 0.97),
    # 3 keep-list chunks (the last ragged) and a hot expert with many passes
    (W.small_moe(T=300, d=512, f=2056, m=6, k=2, dtype=W.BF16, zipf_s=1.2, index=115, name="chunks"), 0.995),
    # f = 16 caps the channel ranges per expert, so its blocks also split the passes
    (W.small_moe(T=300, d=256, f=16, m=2, k=1, dtype=W.BF16, zipf_s=0.0, index=116, name="row_split"), 0.995),
    # more experts than blocks to share out, most of them without tokens
    (W.small_moe(T=64, d=64, f=48, m=160, k=2, dtype=W.BF16, zipf_s=0.8, index=117, name="many_experts"), 0.5),
    # the tensor-core variants: 4 and 8 column units per warp (d = 2048 without column
    # checks), and token rows staged in shared memory with a ragged last unit (d = 3000)
    # and without (d = 4096), several 8-row passes each
    (W.small_moe(T=48, d=768, f=264, m=4, k=2, dtype=W.BF16, zipf_s=0.4, index=118, name="d768"), 0.95),
    (W.small_moe(T=40, d=2048, f=200, m=4, k=2, dtype=W.BF16, zipf_s=0.4, index=119, name="d2048"), 0.95),
    (W.small_moe(T=40, d=3000, f=136, m=3, k=2, dtype=W.BF16, zipf_s=0.4, index=120, name="d3000"), 0.97),
    (W.small_moe(T=64, d=4096, f=256, m=4, k=2, dtype=W.BF16, zipf_s=0.4, index=121, name="d4096_passes"), 0.97),
]


@pytest.mark.parametrize("cfg,s", CASES, ids=lambda v: getattr(v, "name", str(v)))
def test_floe_layer_vs_oracle(cfg, s):
    inp = W.make_moe_inputs(cfg)
    _, _, thr = _calibrate(cfg, inp, s)
    _, r = _floe_layer(cfg, inp, thr)
    k, f = cfg.k, cfg.f
    exp = np.zeros((cfg.T, cfg.d))
    kept = np.zeros((cfg.m, f), bool)
    for row, q in enumerate(r["perm"]):
        t, sl = divmod(int(q), k)
        e = int(r["idx"][t, sl])
        y, keep = O.floe_expert(inp["x"][t], inp["w_gate"][e], inp["w_up"][e], inp["w_down"][e], float(thr[e]),
                                W.BF16, u_mask=r["u"][row])
        exp[t] += float(r["w"][t, sl]) * y
        kept[e] |= keep
    np.testing.assert_array_equal(r["kept"], kept.sum(axis=1))
    assert token_rel_err(out_f64(r["out"]), exp) <= TOL[W.BF16]
    frac = r["kept"][r["kept"] > 0].mean() / f
    assert frac < 1.0  # channels were skipped


def test_floe_with_zero_thresholds_is_the_dense_layer():
    cfg = W.small_moe(T=16, d=256, f=320, m=4, k=2, dtype=W.BF16, zipf_s=0.5, index=113)
    inp = W.make_moe_inputs(cfg)
    d_in, r = _floe_layer(cfg, inp, np.zeros(cfg.m, np.float32))
    active = np.unique(r["idx"])
    assert (r["kept"][active] == cfg.f).all()
    plain = layer_forward(cfg, d_in)
    assert token_rel_err(out_f64(r["out"]), out_f64(plain["out"])) <= TOL[W.BF16]

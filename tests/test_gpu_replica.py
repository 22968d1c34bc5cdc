"""R&Q replica dispatch on the GPU against the oracle (bit-exact ids, counts and
LIS; the layer output within the bf16 tolerance, and equal to the layer without
the replica up to rounding order, since the replica computes with the
heavy-hitter's own weights)."""
import numpy as np
import pytest
import torch

import oracle as O
import sparse_mixture_experts_08_b200 as moe
import workloads as W
from gpu_helpers import (GATE_RTOL, TOL, config_of, dev, device_inputs, host, layer_forward, out_f64, require_gpu,
                         sample_tokens, token_rel_err)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _gpu():
    require_gpu()


def _zipf_routing(T, m, k, a, seed):
    rng = np.random.default_rng(seed)
    p = 1.0 / np.arange(1, m + 1) ** a
    p = p[rng.permutation(m)]
    p /= p.sum()
    return np.stack([rng.choice(m, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)


@pytest.mark.parametrize("T,m,k,a", [(1000, 8, 2, 1.2), (4096, 128, 1, 1.0), (777, 64, 6, 0.8), (33, 1023, 3, 2.0)])
def test_replica_split_bit_exact(T, m, k, a):
    idx = _zipf_routing(T, m, k, a, seed=T + m)
    cfg = W.small_moe(T=T, d=64, f=64, m=m, k=k, dtype=W.BF16)
    c = config_of(cfg)
    ws = moe.workspace(c)
    counts = torch.empty(m, dtype=torch.int32, device="cuda")
    offsets = torch.empty(m + 1, dtype=torch.int32, device="cuda")
    lis = moe.lis_buffer()
    d_idx = dev(idx)
    moe.moe_histogram_lis(c, d_idx, counts, offsets, lis, ws)
    x = torch.zeros((T, 64), dtype=torch.bfloat16, device="cuda")
    x_perm = torch.empty((T * k, 64), dtype=torch.bfloat16, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * k, dtype=torch.int32, device="cuda")
    moe.moe_permute(c, x, d_idx, offsets, x_perm, perm, inv, ws)
    idx2 = torch.empty_like(d_idx)
    counts2 = torch.empty(m + 1, dtype=torch.int32, device="cuda")
    lis2 = moe.lis_buffer()
    moe.moe_replica_split(c, d_idx, offsets, inv, lis, idx2, ws, counts_out=counts2, lis_out=lis2)
    assert moe.moe_read_device_status(ws) == moe.OK
    ref_idx, h = O.replica_split(idx, m)
    np.testing.assert_array_equal(host(idx2), ref_idx)
    ref = O.histogram_lis(ref_idx, m + 1)
    np.testing.assert_array_equal(host(counts2), ref["counts"])
    assert moe.unpack_lis(lis2) == (ref["max_count"], ref["argmax"], ref["lis"])
    assert moe.unpack_lis(lis)[1] == h


def _replicated(cfg, inp):
    d_in = device_inputs(inp)
    c = config_of(cfg)
    ws = moe.replica_workspace(c)
    T, m, k = cfg.T, cfg.m, cfg.k
    out = torch.empty((T, cfg.d), dtype=torch.bfloat16, device="cuda")
    lg = torch.empty((T, m), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    idx2 = torch.empty((T, k), dtype=torch.int32, device="cuda")
    counts = torch.empty(m + 1, dtype=torch.int32, device="cuda")
    lis0, lis1 = moe.lis_buffer(), moe.lis_buffer()
    moe.moe_layer_forward_replicated(c, d_in["x"], d_in["w_router"], d_in["bias"], d_in["w_gate"], d_in.get("w_up"),
                                     d_in["w_down"], d_in.get("ws_gate"), d_in.get("ws_up"), d_in.get("ws_down"),
                                     out, ws, logits_out=lg, topk_idx_out=idx, topk_w_out=w, dispatch_idx_out=idx2,
                                     counts_out=counts, lis_before_out=lis0, lis_after_out=lis1)
    assert moe.moe_read_device_status(ws) == moe.OK
    return d_in, {"out": out, "logits": host(lg), "idx": host(idx), "w": host(w), "idx2": host(idx2),
                  "counts": host(counts), "lis0": moe.unpack_lis(lis0), "lis1": moe.unpack_lis(lis1)}


CASES = [
    W.small_moe(T=700, d=256, f=192, m=16, k=1, act=W.RELU, dtype=W.BF16, zipf_s=1.4, index=96, name="top1"),
    W.small_moe(T=300, d=128, f=160, m=8, k=2, dtype=W.BF16, zipf_s=1.2, renorm=True, n_shared=1, f_shared=96,
                index=97, name="k2_shared"),
    W.CONFIGS["switch"],
]


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_layer_forward_replicated(cfg):
    inp = W.make_moe_inputs(cfg)
    d_in, r = _replicated(cfg, inp)
    # routing on the GPU's own logits, then the split, against the oracle
    oidx, ow = O.topk_softmax(r["logits"], cfg.k, cfg.renorm)
    np.testing.assert_array_equal(r["idx"], oidx)
    np.testing.assert_allclose(r["w"], ow, rtol=GATE_RTOL, atol=1e-12)
    ref0 = O.histogram_lis(oidx, cfg.m)
    assert r["lis0"] == (ref0["max_count"], ref0["argmax"], ref0["lis"])
    idx2, h = O.replica_split(oidx, cfg.m)
    np.testing.assert_array_equal(r["idx2"], idx2)
    ref1 = O.histogram_lis(idx2, cfg.m + 1)
    np.testing.assert_array_equal(r["counts"], ref1["counts"])
    assert r["lis1"] == (ref1["max_count"], ref1["argmax"], ref1["lis"])
    assert ref1["max_count"] <= ref0["max_count"]  # no expert gains load; the heavy-hitter's is halved
    # the output: the layer over m + 1 experts with the replica's weights = the heavy-hitter's
    cfg1 = W.small_moe(T=cfg.T, d=cfg.d, f=cfg.f, m=cfg.m + 1, k=cfg.k, act=cfg.act, dtype=cfg.dtype,
                       renorm=cfg.renorm, n_shared=cfg.n_shared, f_shared=cfg.f_shared)
    toks = sample_tokens(idx2, ref1["counts"], cfg.T, 48)
    exp = O.moe_output(cfg1, O.replica_inputs(inp, h), idx2, ow, tokens=toks)
    assert token_rel_err(out_f64(r["out"])[toks], exp) <= TOL[W.BF16]
    plain = layer_forward(cfg, d_in)
    assert token_rel_err(out_f64(r["out"]), out_f64(plain["out"])) <= TOL[W.BF16]

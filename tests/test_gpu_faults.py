"""Device-side failure handling, exercised without faulting the GPU.

* Bounded waits: the test hook shrinks every mbarrier wait limit of the
  tensor-core kernels to 1 ns, so the first wait that does not succeed at once
  gives up. The kernel must record MOE_ERR_TIMEOUT in the status word, drain its
  copies and MMAs, free TMEM and return; the context stays usable and the next
  call (default limit) is correct again.
* Corrupted routing tables: expert ids outside [0, m) and inconsistent segment
  offsets become MOE_ERR_DEVICE_INDEX with no out-of-range write.
* The atomic-expert kernel's grid barrier: a test hook makes it wait for one
  arrival more than the grid has, so it ends only at its (1 ms) limit; the kernel
  records MOE_ERR_TIMEOUT and its blocks return.
"""
import numpy as np
import pytest
import torch

import oracle as O
import sparse_mixture_experts_08_b200 as moe
import workloads as W
from gpu_helpers import TOL, config_of, dev, device_inputs, host, out_f64, require_gpu, token_rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _gpu():
    require_gpu()


def _ffn_case():
    cfg = W.small_moe(T=96, d=256, f=384, m=4, k=2, dtype=W.BF16, zipf_s=1.0, index=51)
    inp = W.make_moe_inputs(cfg)
    logits = O.router_logits(inp["x"], inp["w_router"], inp["bias"])
    idx, wgt = O.topk_softmax(logits, cfg.k, False)
    ref = O.histogram_lis(idx, cfg.m)
    perm, _ = O.permutation(idx, cfg.m, ref["offsets"])
    return cfg, inp, idx, wgt, ref["offsets"], perm


def _run_ffn(cfg, inp, offsets, perm, wgt, ws):
    c = config_of(cfg)
    d = device_inputs(inp)
    x_perm = np.ascontiguousarray(inp["x"][perm // cfg.k])
    y = torch.full((cfg.T * cfg.k, cfg.d), 7.0, dtype=torch.float32, device="cuda")
    moe.moe_grouped_ffn(c, dev(x_perm), dev(offsets), d["w_gate"], d["w_up"], d["w_down"],
                        dev(wgt.astype(np.float32).ravel()), dev(perm), y, ws)
    return y


def test_bounded_wait_times_out_and_context_recovers():
    cfg, inp, idx, wgt, offsets, perm = _ffn_case()
    ws = moe.workspace(config_of(cfg))
    try:
        moe.moe_debug_set_wait_limit_ns(1)
        _run_ffn(cfg, inp, offsets, perm, wgt, ws)
        st = moe.moe_read_device_status(ws)  # synchronises: the kernels returned
    finally:
        moe.moe_debug_set_wait_limit_ns(0)
    assert st == moe.ERR_TIMEOUT
    assert moe.moe_read_device_status(ws) == moe.OK  # cleared by the read
    y = _run_ffn(cfg, inp, offsets, perm, wgt, ws)
    assert moe.moe_read_device_status(ws) == moe.OK
    got = out_f64(y)
    exp = np.stack([float(wgt.ravel()[q]) * O.expert_ffn(inp["x"][q // cfg.k], inp["w_gate"][idx.ravel()[q]],
                                                          inp["w_up"][idx.ravel()[q]], inp["w_down"][idx.ravel()[q]],
                                                          W.SWIGLU) for q in perm])
    assert token_rel_err(got, exp) <= TOL[W.BF16]


def test_inconsistent_offsets_are_rejected_on_device():
    cfg, inp, idx, wgt, offsets, perm = _ffn_case()
    ws = moe.workspace(config_of(cfg))
    bad = offsets.copy()
    bad[2] = bad[3] + 5  # segment 1 ends after segment 2 starts: negative length
    y = _run_ffn(cfg, inp, bad, perm, wgt, ws)
    assert moe.moe_read_device_status(ws) == moe.ERR_DEVICE_INDEX
    bad = offsets.copy()
    bad[-1] = cfg.T * cfg.k + 64  # last segment runs past the rows that exist
    y = _run_ffn(cfg, inp, bad, perm, wgt, ws)
    assert moe.moe_read_device_status(ws) == moe.ERR_DEVICE_INDEX
    assert torch.isfinite(y).all()


def test_permute_rejects_bad_expert_id_without_writing():
    cfg = W.small_moe(T=40, d=64, f=64, m=8, k=2, dtype=W.BF16, index=52)
    inp = W.make_moe_inputs(cfg, weights=False)
    idx = np.tile(np.array([1, 5], np.int32), (cfg.T, 1))
    ref = O.histogram_lis(idx, cfg.m)
    idx[13, 0] = 9  # outside [0, m)
    c = config_of(cfg)
    ws = moe.workspace(c)
    x_perm = torch.zeros((cfg.T * cfg.k, cfg.d), dtype=torch.bfloat16, device="cuda")
    perm = torch.full((cfg.T * cfg.k,), -5, dtype=torch.int32, device="cuda")
    inv = torch.full((cfg.T * cfg.k,), -5, dtype=torch.int32, device="cuda")
    moe.moe_permute(c, dev(inp["x"]), dev(idx), dev(ref["offsets"]), x_perm, perm, inv, ws)
    assert moe.moe_read_device_status(ws) == moe.ERR_DEVICE_INDEX
    assert torch.all(perm == -5) and torch.all(x_perm == 0) and torch.all(inv == -1)


def test_layer_forward_after_errors_is_exact_again():
    # a layer call whose tensor-core waits run out (1 ns limit) records TIMEOUT; the
    # next call on the same workspace, with the default limit, is exact again
    cfg = W.small_moe(T=64, d=128, f=256, m=8, k=2, dtype=W.BF16, zipf_s=1.2, index=53)
    inp = W.make_moe_inputs(cfg)
    d = device_inputs(inp)
    c = config_of(cfg)
    ws = moe.workspace(c)
    out = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device="cuda")
    lg = torch.empty((cfg.T, cfg.m), dtype=torch.float32, device="cuda")
    try:
        moe.moe_debug_set_wait_limit_ns(1)
        moe.moe_layer_forward(c, d["x"], d["w_router"], d["bias"], d["w_gate"], d["w_up"], d["w_down"], None, None,
                              None, out, ws, logits_out=lg)
        st = moe.moe_read_device_status(ws)
    finally:
        moe.moe_debug_set_wait_limit_ns(0)
    assert st == moe.ERR_TIMEOUT
    out.fill_(float("nan"))
    moe.moe_layer_forward(c, d["x"], d["w_router"], d["bias"], d["w_gate"], d["w_up"], d["w_down"], None, None, None,
                          out, ws, logits_out=lg)
    assert moe.moe_read_device_status(ws) == moe.OK
    r = O.layer_forward(cfg, inp, logits_in=host(lg))
    assert token_rel_err(out_f64(out), r["out"]) <= TOL[W.BF16]


def test_atomic_grid_barrier_times_out_and_recovers():
    # the atomic-expert FFN is one cooperative launch with a grid-wide barrier. The
    # test hook makes the barrier wait for one arrival more than the grid has, so it
    # can only end at its time limit (1 ms here): the kernel must record
    # MOE_ERR_TIMEOUT and return, and the next call with the normal barrier is exact.
    cfg = W.AtomicWorkload("atomic_fault", 93, T=4, d=256, Nr=64, Nc=64, K=16, act=W.ACT_SILU)
    inp = W.make_atomic_inputs(cfg)
    c = moe.make_atomic_config(cfg.T, cfg.d, cfg.Nr, cfg.Nc, cfg.K, cfg.act)
    ws = moe.workspace(c)
    d = device_inputs(inp)
    idx = torch.empty((cfg.T, cfg.K), dtype=torch.int32, device="cuda")
    g = torch.empty((cfg.T, cfg.K), dtype=torch.float32, device="cuda")
    moe.moe_atomic_route(c, d["x"], d["w_row"], d["w_col"], None, None, idx, g, ws)
    assert moe.moe_read_device_status(ws) == moe.OK
    out = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device="cuda")
    for forward in (False, True):  # the experts call alone, and the whole layer (select zeroes the barrier)
        try:
            moe.moe_debug_set_wait_limit_ns(1_000_000)
            moe.moe_debug_set_barrier_extra(1)
            if forward:
                moe.moe_atomic_forward(c, d["x"], d["w_row"], d["w_col"], d["w_in"], d["w_out"], out, ws)
            else:
                moe.moe_atomic_experts(c, d["x"], d["w_in"], d["w_out"], idx, g, out, ws)
            st = moe.moe_read_device_status(ws)
        finally:
            moe.moe_debug_set_barrier_extra(0)
            moe.moe_debug_set_wait_limit_ns(0)
        assert st == moe.ERR_TIMEOUT
    moe.moe_atomic_experts(c, d["x"], d["w_in"], d["w_out"], idx, g, out, ws)
    assert moe.moe_read_device_status(ws) == moe.OK
    ref = O.atomic_output(inp["x"], inp["w_in"], inp["w_out"], host(idx), host(g), cfg.act)
    assert token_rel_err(out_f64(out), ref) <= TOL[W.BF16]
    out2 = torch.empty_like(out)
    moe.moe_atomic_forward(c, d["x"], d["w_row"], d["w_col"], d["w_in"], d["w_out"], out2, ws)
    assert moe.moe_read_device_status(ws) == moe.OK
    torch.cuda.synchronize()
    assert torch.equal(out, out2)

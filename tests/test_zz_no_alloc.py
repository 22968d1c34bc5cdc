"""moe_route_static: the router for callers that cannot allocate device memory.

Some callers cannot give the library a workspace: plugins that only see the
tensors a host framework passes in (the framework owns the allocator), and
request paths that must not allocate (an allocation can block or fail under
memory pressure). This entry point keeps its scratch (the status word and, when
the caller does not ask for them, the router logits) in a fixed array compiled
into the library. These tests call it through the C ABI twice in a row and check
it against moe_route, which uses a caller-provided workspace (the top-k ids must
match exactly and the gate weights within the 1e-6 relative tolerance used for
gate weights elsewhere), and against the oracle: its logits within the router's
fp32 tolerance, its top-k and gate weights decided by the oracle on the same
fp32 logits. This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import sparse_mixture_experts_08_b200 as moe
import workloads as W
from gpu_helpers import GATE_RTOL, config_of, device_inputs, host, require_gpu

pytestmark = pytest.mark.gpu

CASES = [
    W.small_moe(T=8192, d=768, f=64, m=128, k=1, dtype=W.BF16, zipf_s=1.0, index=61, name="switch_router"),
    W.small_moe(T=300, d=512, f=64, m=64, k=6, dtype=W.BF16, zipf_s=1.1, index=62, name="k6_router"),
    W.small_moe(T=16, d=4096, f=64, m=8, k=2, dtype=W.BF16, zipf_s=0.0, renorm=True, index=63, name="decode_router"),
    W.small_moe(T=64, d=128, f=64, m=8, k=2, dtype=W.F32, zipf_s=1.2, index=64, name="fp32_router"),
]


@pytest.fixture(autouse=True, scope="module")
def _gpu():
    require_gpu()


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_static_router_matches_workspace_router_twice(cfg):
    inp = W.make_moe_inputs(cfg, weights=False)
    d = device_inputs(inp)
    c = config_of(cfg)
    ws = moe.workspace(c)
    ref_idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    ref_w = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device="cuda")
    moe.moe_route(c, d["x"], d["w_router"], d["bias"], None, None, ref_idx, ref_w, ws)
    assert moe.moe_read_device_status(ws) == moe.OK
    # the oracle's decision on the logits this router computes (the same kernels write
    # them to a caller buffer here), and those logits against the oracle's own
    lg = torch.empty((cfg.T, cfg.m), dtype=torch.float32, device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    w = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device="cuda")
    moe.moe_route_static(c, d["x"], d["w_router"], d["bias"], None, lg, idx, w, device_status_out=status)
    torch.cuda.synchronize()
    assert int(status.item()) == moe.OK
    ref_lg = O.router_logits(inp["x"], inp["w_router"], inp["bias"])
    np.testing.assert_allclose(host(lg), ref_lg, rtol=0, atol=2e-5 * np.sqrt(cfg.d) * np.abs(ref_lg).max())
    oidx, ow = O.topk_softmax(host(lg), cfg.k, cfg.renorm)
    np.testing.assert_array_equal(host(idx), oidx)
    np.testing.assert_allclose(host(w), ow, rtol=GATE_RTOL, atol=1e-12)
    for _ in range(2):  # logits in the array; the second call reuses what the first one left behind
        idx = torch.full((cfg.T, cfg.k), -1, dtype=torch.int32, device="cuda")
        w = torch.full((cfg.T, cfg.k), float("nan"), dtype=torch.float32, device="cuda")
        status.fill_(-1)
        moe.moe_route_static(c, d["x"], d["w_router"], d["bias"], None, None, idx, w, device_status_out=status)
        torch.cuda.synchronize()
        assert int(status.item()) == moe.OK
        np.testing.assert_array_equal(host(idx), host(ref_idx))
        np.testing.assert_allclose(host(w), host(ref_w), rtol=GATE_RTOL, atol=1e-12)
        np.testing.assert_array_equal(host(idx), oidx)
        np.testing.assert_allclose(host(w), ow, rtol=GATE_RTOL, atol=1e-12)


def test_static_router_rejects_sizes_beyond_its_array():
    # T * m logits must fit the 8 MiB array (minus the status word) when the caller
    # asks for no logits output; the call is refused before any launch. Every pointer
    # is a real allocation of the stated shape, so a check that came too late would
    # give a wrong answer here, never a stray access.
    T, d, m = 32768, 64, 128
    c = moe.make_config(T=T, d=d, f=64, m=m, k=1, dtype=moe.BF16)
    x = torch.zeros((T, d), dtype=torch.bfloat16, device="cuda")
    wr = torch.zeros((m, d), dtype=torch.bfloat16, device="cuda")
    idx = torch.full((T, 1), -3, dtype=torch.int32, device="cuda")
    wt = torch.full((T, 1), -3.0, dtype=torch.float32, device="cuda")
    lib = moe.moe.lib()
    rc = lib.moe_route_static(ctypes.byref(c), x.data_ptr(), wr.data_ptr(), None, None, None, idx.data_ptr(),
                              wt.data_ptr(), None, None)
    assert rc == moe.ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(idx == -3) and torch.all(wt == -3.0)  # nothing ran
    # with a caller-provided logits buffer the array only holds the status word
    x = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    c2 = moe.make_config(T=64, d=64, f=64, m=8, k=1, dtype=moe.BF16)
    wr = torch.zeros((8, 64), dtype=torch.bfloat16, device="cuda")
    lg = torch.empty((64, 8), dtype=torch.float32, device="cuda")
    idx = torch.empty((64, 1), dtype=torch.int32, device="cuda")
    wt = torch.empty((64, 1), dtype=torch.float32, device="cuda")
    moe.moe_route_static(c2, x, wr, None, None, lg, idx, wt)
    torch.cuda.synchronize()
    assert host(idx).ravel().tolist() == [0] * 64  # all-zero logits: lowest index wins

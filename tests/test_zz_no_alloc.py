"""moe_route_static: the router for callers that cannot allocate device memory.

Callers such as code running under CUDA-graph capture (where cudaMalloc is not
allowed), plugins that only see the tensors a host framework passes in, or request
paths that must not allocate cannot give the library a workspace. This entry point
keeps its scratch (the status word and, when the caller does not ask for them, the
router logits) in a fixed array compiled into the library. These tests call it
through the C ABI twice in a row and check it against moe_route, which uses a
caller-provided workspace: the top-k ids must match exactly and the gate weights
within the 1e-6 relative tolerance used for gate weights elsewhere. This file is
collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

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
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for _ in range(2):  # the second call reuses the array the first one left behind
        idx = torch.full((cfg.T, cfg.k), -1, dtype=torch.int32, device="cuda")
        w = torch.full((cfg.T, cfg.k), float("nan"), dtype=torch.float32, device="cuda")
        moe.moe_route_static(c, d["x"], d["w_router"], d["bias"], None, None, idx, w, device_status_out=status)
        torch.cuda.synchronize()
        assert int(status.item()) == moe.OK
        np.testing.assert_array_equal(host(idx), host(ref_idx))
        np.testing.assert_allclose(host(w), host(ref_w), rtol=GATE_RTOL, atol=1e-12)


def test_static_router_rejects_sizes_beyond_its_array():
    # T * m logits must fit the 8 MiB array (minus the status word) when the caller
    # asks for no logits output; the call is refused before any launch.
    lib = moe.moe.lib()
    c = moe.make_config(T=32768, d=64, f=64, m=128, k=1, dtype=moe.BF16)
    dummy = ctypes.c_void_p(1 << 24)
    rc = lib.moe_route_static(ctypes.byref(c), dummy, dummy, None, None, None, dummy, dummy, None, None)
    assert rc == moe.ERR_WORKSPACE
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

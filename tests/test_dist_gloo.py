"""The multi-rank (data-parallel) path on CPU: world size 2 over gloo.

bench.py runs one process per GPU; every rank holds the same weights and its own
token batch, and the step time is the maximum over ranks. These tests check that
host-side logic with two CPU ranks: identical weights, distinct batches, the MAX
reduction, and that splitting tokens across ranks leaves every token's layer output
unchanged (the layer is dropless, so a token's output does not depend on the rest
of its batch) - the property that makes token sharding need no data-path exchange.
"""
import hashlib
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys

    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import oracle as O
        import workloads as W

        cfg = W.small_moe(T=24, d=64, f=96, m=6, k=2, dtype=W.BF16, zipf_s=1.0, index=41, name="dp_small")
        inp = bench.rank_inputs(cfg, rank)
        wh = hashlib.sha256(b"".join(inp[k].tobytes() for k in sorted(inp) if k != "x")).hexdigest()
        xh = hashlib.sha256(inp["x"].tobytes()).hexdigest()
        hashes = [None] * world
        dist.all_gather_object(hashes, (wh, xh))
        out = O.layer_forward(cfg, inp)["out"]
        out8 = O.layer_forward_fp8(cfg, inp)["out"]  # the 8-bit layer: per-row scales, so also per token
        outs = [None] * world
        dist.all_gather_object(outs, (inp["x"], out, out8))
        mx = bench.max_over_ranks([float(rank + 1), 10.0 - rank], dist)
        # the whole job's histogram (bench --global-lis): each rank's counts summed
        routed = O.layer_forward(cfg, inp)
        summed = bench.global_histogram(torch.from_numpy(routed["counts"].copy()), dist).numpy()
        q.put((rank, hashes, outs, mx, summed))
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(res, key=lambda r: r[0])


def test_ranks_share_weights_and_own_their_batch(two_ranks):
    hashes = two_ranks[0][1]
    assert hashes[0][0] == hashes[1][0]  # same expert / router weights
    assert hashes[0][1] != hashes[1][1]  # different token batches


def test_max_over_ranks(two_ranks):
    for _, _, _, mx, _ in two_ranks:
        assert mx == [2.0, 10.0]


def test_token_sharding_leaves_outputs_unchanged(two_ranks):
    import sys

    sys.path.insert(0, ROOT)
    import oracle as O
    import workloads as W

    cfg = W.small_moe(T=48, d=64, f=96, m=6, k=2, dtype=W.BF16, zipf_s=1.0, index=41, name="dp_small")
    outs = two_ranks[0][2]
    inp = W.make_moe_inputs(cfg, replicate=0)
    inp["x"] = np.concatenate([outs[0][0], outs[1][0]])
    whole = O.layer_forward(cfg, inp)["out"]
    np.testing.assert_array_equal(whole, np.concatenate([outs[0][1], outs[1][1]]))


def test_token_sharding_leaves_8bit_outputs_unchanged(two_ranks):
    """x and h are quantized per row (token, task), never across the batch, so the 8-bit
    layer shards by tokens with no exchange either."""
    import sys

    sys.path.insert(0, ROOT)
    import oracle as O
    import workloads as W

    cfg = W.small_moe(T=48, d=64, f=96, m=6, k=2, dtype=W.BF16, zipf_s=1.0, index=41, name="dp_small")
    outs = two_ranks[0][2]
    inp = W.make_moe_inputs(cfg, replicate=0)
    inp["x"] = np.concatenate([outs[0][0], outs[1][0]])
    whole = O.layer_forward_fp8(cfg, inp)["out"]
    np.testing.assert_allclose(whole, np.concatenate([outs[0][2], outs[1][2]]), rtol=1e-12, atol=0)


def test_global_histogram_is_the_whole_batch_histogram(two_ranks):
    """R&Q Definition 1 over the whole job's batch: the per-expert counts summed over
    the two ranks equal the oracle's histogram of the two batches together, and the
    LIS of that histogram (what moe_lis_from_counts computes from it on the GPU) is
    the oracle's LIS of the concatenated routing."""
    import sys

    sys.path.insert(0, ROOT)
    import oracle as O
    import workloads as W

    cfg = W.small_moe(T=48, d=64, f=96, m=6, k=2, dtype=W.BF16, zipf_s=1.0, index=41, name="dp_small")
    outs = two_ranks[0][2]
    inp = W.make_moe_inputs(cfg, replicate=0)
    inp["x"] = np.concatenate([outs[0][0], outs[1][0]])
    whole = O.layer_forward(cfg, inp)
    for r in range(2):
        np.testing.assert_array_equal(two_ranks[r][4], whole["counts"])
    c = two_ranks[0][4]
    assert whole["max_count"] == int(c.max()) and whole["argmax"] == int(np.argmax(c))
    assert whole["lis"] == cfg.m * int(c.max()) / (cfg.T * cfg.k)

"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test checks the oracle against something the reviewed pages or mathematics
fix: hand-worked values (tests/golden), closed forms of the Load Imbalance Score
(R&Q Definition 1), library routines computing the same thing by another route
(numpy lexsort / stable argsort / bincount, scipy softmax, torch fp64 matmuls),
invariants, and a brute-force dense-masked evaluation. A plausible slip in the
oracle (dropped bias, wrong tie-break, missing renormalisation, unstable
permutation, transposed weight, missing SiLU or up factor, shared branch lost,
wrong LIS formula) fails at least one of them; test_oracle_mutations.py plants
such slips in a copy of the oracle and checks exactly that.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import torch

import oracle as O
import workloads as W

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


def _golden(path):
    rows = []
    with open(path) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            rows.append([c.strip() for c in line.split("|")])
    return rows


def _t64(a, dtype):
    return torch.from_numpy(np.asarray(W.as_f32(a, dtype), dtype=np.float64))


# ------------------------------------------------------------------------- LIS

def test_lis_golden_cases(golden_dir):
    for name, m, k, routing, counts, mx, am, lis in _golden(os.path.join(golden_dir, "lis_cases.txt")):
        m, k = int(m), int(k)
        idx = np.array([[int(e) for e in tok.split(",")] for tok in routing.split(";")], dtype=np.int32)
        assert idx.shape[1] == k, name
        r = O.histogram_lis(idx, m)
        assert r["counts"].tolist() == [int(c) for c in counts.split(",")], name
        assert r["max_count"] == int(mx) and r["argmax"] == int(am), name
        assert r["lis"] == float(Fraction(lis)), name


def _favouring_logits(T, m, k, pick):
    """Logits where token t's slot s clearly prefers expert pick(t, s)."""
    lg = np.zeros((T, m), dtype=np.float32)
    for t in range(T):
        for s in range(k):
            lg[t, pick(t, s)] = np.float32(10.0 - s)
    return lg


def test_lis_balanced_construction_is_one():
    # (t*k + s) mod m with T*k divisible by m gives every expert T*k/m tasks -> LIS = 1
    T, m, k = 64, 8, 2
    idx, _ = O.topk_softmax(_favouring_logits(T, m, k, lambda t, s: (t * k + s) % m), k, False)
    r = O.histogram_lis(idx, m)
    assert set(r["counts"].tolist()) == {T * k // m}
    assert r["lis"] == 1.0


def test_lis_all_tokens_same_experts_is_maximum():
    T, m, k = 50, 16, 4
    idx, _ = O.topk_softmax(_favouring_logits(T, m, k, lambda t, s: 3 + s), k, False)
    r = O.histogram_lis(idx, m)
    assert r["lis"] == m / k  # the largest value: n_j <= T
    assert r["argmax"] == 3


@pytest.mark.parametrize("c", [1, 7, 33, 64])
def test_lis_constructed_max_count(c):
    T, m, k = 64, 8, 1
    # the first c tokens go to expert 5, the rest spread round-robin over the other 7
    others = [e for e in range(m) if e != 5]
    pick = lambda t, s: 5 if t < c else others[t % len(others)]
    idx, _ = O.topk_softmax(_favouring_logits(T, m, k, pick), k, False)
    counts = np.bincount(idx.ravel(), minlength=m)
    r = O.histogram_lis(idx, m)
    assert r["lis"] == m * counts.max() / (T * k)
    if c > (T - c) / 7 + 1:
        assert r["argmax"] == 5 and r["max_count"] == c


def test_lis_bounds_and_counts_random():
    rng = np.random.default_rng(0)
    for _ in range(20):
        T, m = int(rng.integers(1, 300)), int(rng.integers(2, 40))
        k = int(rng.integers(1, m + 1))
        lg = rng.standard_normal((T, m)).astype(np.float32)
        idx, _ = O.topk_softmax(lg, k, False)
        r = O.histogram_lis(idx, m)
        np.testing.assert_array_equal(r["counts"], np.bincount(idx.ravel(), minlength=m))
        np.testing.assert_array_equal(r["offsets"], np.concatenate([[0], np.cumsum(r["counts"])]))
        assert r["counts"].sum() == T * k
        assert 1.0 - 1e-12 <= r["lis"] <= m / k + 1e-12


def test_histogram_rejects_out_of_range_ids():
    with pytest.raises(ValueError):
        O.histogram_lis(np.array([[0], [4]], dtype=np.int32), 4)
    with pytest.raises(ValueError):
        O.histogram_lis(np.array([[-1], [1]], dtype=np.int32), 4)


# --------------------------------------------------------------- top-k, softmax

def _parse_logit(s):
    return np.float32(math.log(float(s[3:]))) if s.startswith("ln:") else np.float32(float(s))


def test_topk_golden(golden_dir):
    for name, k, rn, logits, idx, wts in _golden(os.path.join(golden_dir, "topk_cases.txt")):
        lg = np.array([[_parse_logit(v) for v in logits.split(",")]], dtype=np.float32)
        i, w = O.topk_softmax(lg, int(k), bool(int(rn)))
        assert i[0].tolist() == [int(v) for v in idx.split(",")], name
        np.testing.assert_allclose(w[0], [float(Fraction(v)) for v in wts.split(",")], rtol=1e-6, err_msg=name)


def test_topk_matches_lexsort_with_many_ties():
    rng = np.random.default_rng(1)
    for m in (2, 7, 8, 64, 128):
        T = 200
        lg = (rng.integers(-3, 4, size=(T, m)) * 0.5).astype(np.float32)  # heavy ties
        for k in sorted({1, 2, min(6, m), m}):
            idx, _ = O.topk_softmax(lg, k, False)
            for t in range(T):
                order = np.lexsort((np.arange(m), -lg[t].astype(np.float64)))
                assert idx[t].tolist() == order[:k].tolist()


def test_constant_logits_pick_first_k():
    idx, w = O.topk_softmax(np.zeros((3, 9), np.float32), 4, False)
    assert idx.tolist() == [[0, 1, 2, 3]] * 3
    np.testing.assert_allclose(w, 1.0 / 9.0, rtol=1e-15)


@pytest.mark.parametrize("renorm", [False, True])
def test_gate_weights_vs_scipy_softmax(renorm):
    rng = np.random.default_rng(2)
    lg = (rng.standard_normal((300, 64)) * 3).astype(np.float32)
    idx, w = O.topk_softmax(lg, 6, renorm)
    p = scipy.special.softmax(lg.astype(np.float64), axis=1)
    sel = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    if renorm:
        sel = sel / sel.sum(axis=1, keepdims=True)
        np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(w, sel, rtol=1e-12)


def test_top1_weight_closed_form():
    rng = np.random.default_rng(3)
    lg = rng.standard_normal((100, 16)).astype(np.float32)
    idx, w = O.topk_softmax(lg, 1, False)
    for t in range(100):
        e = idx[t, 0]
        others = np.delete(lg[t].astype(np.float64), e)
        assert w[t, 0] == pytest.approx(1.0 / (1.0 + np.exp(others - lg[t, e]).sum()), rel=1e-13)


# -------------------------------------------------------------------- router

@pytest.mark.parametrize("dtype", [W.F32, W.BF16])
def test_router_logits_vs_torch_fp64(dtype):
    cfg = W.small_moe(T=33, d=96, f=32, m=12, k=2, dtype=dtype, zipf_s=1.0)
    inp = W.make_moe_inputs(cfg, weights=False)
    got = O.router_logits(inp["x"], inp["w_router"], inp["bias"])
    ref = (_t64(inp["x"], dtype) @ _t64(inp["w_router"], dtype).T + torch.from_numpy(
        inp["bias"].astype(np.float64))).float().numpy()
    # both are fp64 sums rounded once to fp32; summation order may move a tie by one ulp
    np.testing.assert_array_max_ulp(got, ref, maxulp=1)
    assert (got == ref).mean() > 0.99
    assert np.any(inp["bias"] != 0)


def test_zipf_bias_shape():
    b = W.zipf_bias(16, 1.1, 0.5, seed=123)
    r = np.sort(-b)  # ranks 1..m in increasing -bias order
    np.testing.assert_allclose(r, [0.5 * 1.1 * math.log(i) for i in range(1, 17)], rtol=1e-6)
    assert len(set(np.argsort(-b).tolist())) == 16


# --------------------------------------------------------------- permutation

def test_permutation_is_stable_argsort_by_expert():
    rng = np.random.default_rng(4)
    for m, k in ((8, 2), (128, 1), (64, 6), (3, 3)):
        T = 257
        lg = rng.standard_normal((T, m)).astype(np.float32)
        idx, _ = O.topk_softmax(lg, k, False)
        r = O.histogram_lis(idx, m)
        perm, inv = O.permutation(idx, m, r["offsets"])
        np.testing.assert_array_equal(perm, np.argsort(idx.ravel(), kind="stable"))
        np.testing.assert_array_equal(perm[inv], np.arange(T * k))
        np.testing.assert_array_equal(inv[perm], np.arange(T * k))
        flat = idx.ravel()
        for e in range(m):
            seg = perm[r["offsets"][e]:r["offsets"][e + 1]]
            assert np.all(flat[seg] == e)
            assert np.all(np.diff(seg) > 0)


# ----------------------------------------------------------------- expert FFN

def _torch_ffn(x, wg, wu, wd, act):
    a = x @ wg.T
    h = torch.nn.functional.silu(a) * (x @ wu.T) if act == W.SWIGLU else torch.relu(a)
    return h @ wd.T


@pytest.mark.parametrize("act", [W.SWIGLU, W.RELU])
@pytest.mark.parametrize("dtype", [W.F32, W.BF16])
def test_single_expert_is_textbook_ffn(act, dtype):
    # m = 1, k = 1: the layer is one dense FFN with weight 1
    cfg = W.small_moe(T=9, d=64, f=80, m=1, k=1, act=act, dtype=dtype, zipf_s=0.0)
    inp = W.make_moe_inputs(cfg)
    r = O.layer_forward(cfg, inp)
    assert np.all(r["idx"] == 0) and np.allclose(r["w"], 1.0)
    t = lambda key: _t64(inp[key], dtype)
    ref = _torch_ffn(t("x"), t("w_gate")[0], t("w_up")[0] if act == W.SWIGLU else None, t("w_down")[0], act)
    np.testing.assert_allclose(r["out"], ref.numpy(), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("shared", [0, 2])
@pytest.mark.parametrize("act", [W.SWIGLU, W.RELU])
def test_dense_masked_equals_sparse(shared, act):
    cfg = W.small_moe(T=12, d=32, f=48, m=6, k=2, act=act, dtype=W.BF16, zipf_s=1.0, n_shared=shared,
                      f_shared=40 if shared else 0)
    inp = W.make_moe_inputs(cfg)
    r = O.layer_forward(cfg, inp)
    np.testing.assert_allclose(O.dense_masked(cfg, inp, r["idx"], r["w"]), r["out"], rtol=1e-12, atol=1e-14)


def test_full_mixture_when_k_equals_m():
    cfg = W.small_moe(T=7, d=48, f=40, m=4, k=4, act=W.SWIGLU, dtype=W.BF16, zipf_s=1.0, renorm=True)
    inp = W.make_moe_inputs(cfg)
    r = O.layer_forward(cfg, inp)
    t = lambda key: _t64(inp[key], W.BF16)
    p = torch.softmax(torch.from_numpy(r["logits"].astype(np.float64)), dim=1)
    ref = sum(p[:, e:e + 1] * _torch_ffn(t("x"), t("w_gate")[e], t("w_up")[e], t("w_down")[e], W.SWIGLU)
              for e in range(4))
    np.testing.assert_allclose(r["out"], ref.numpy(), rtol=1e-10, atol=1e-12)


def test_identical_experts_with_renorm_ignore_routing():
    cfg = W.small_moe(T=10, d=32, f=24, m=5, k=3, act=W.SWIGLU, dtype=W.F32, zipf_s=1.0, renorm=True)
    inp = W.make_moe_inputs(cfg)
    for key in ("w_gate", "w_up", "w_down"):
        inp[key][:] = inp[key][0:1]
    r = O.layer_forward(cfg, inp)
    t = lambda key: _t64(inp[key], W.F32)
    ref = _torch_ffn(t("x"), t("w_gate")[0], t("w_up")[0], t("w_down")[0], W.SWIGLU)
    np.testing.assert_allclose(r["out"], ref.numpy(), rtol=1e-10, atol=1e-12)


def test_shared_experts_add_plain_ffns():
    cfg = W.small_moe(T=6, d=32, f=24, m=4, k=2, act=W.SWIGLU, dtype=W.BF16, zipf_s=1.0, n_shared=2,
                      f_shared=16)
    inp = W.make_moe_inputs(cfg)
    with_sh = O.layer_forward(cfg, inp)
    cfg0 = W.small_moe(T=6, d=32, f=24, m=4, k=2, act=W.SWIGLU, dtype=W.BF16, zipf_s=1.0)
    no_sh = O.layer_forward(cfg0, {k: v for k, v in inp.items() if not k.startswith("ws_")})
    t = lambda key: _t64(inp[key], W.BF16)
    shared = sum(_torch_ffn(t("x"), t("ws_gate")[s], t("ws_up")[s], t("ws_down")[s], W.SWIGLU) for s in range(2))
    np.testing.assert_allclose(with_sh["out"] - no_sh["out"], shared.numpy(), rtol=1e-9, atol=1e-11)


def test_sampled_tokens_match_full_output():
    cfg = W.small_moe(T=20, d=32, f=24, m=4, k=2, act=W.RELU, dtype=W.BF16)
    inp = W.make_moe_inputs(cfg)
    r = O.layer_forward(cfg, inp)
    tok = np.array([19, 0, 7, 7], np.int32)
    np.testing.assert_array_equal(O.moe_output(cfg, inp, r["idx"], r["w"], tokens=tok), r["out"][tok])


# -------------------------------------------------------------- atomic experts

def _small_atomic(T=3, d=64, Nr=16, Nc=12, K=8, act=W.ACT_SILU):
    return W.AtomicWorkload("atomic_small", 91, T=T, d=d, Nr=Nr, Nc=Nc, K=K, act=act)


def test_atomic_logprobs_vs_torch():
    cfg = _small_atomic()
    inp = W.make_atomic_inputs(cfg)
    lr, lc = O.atomic_logprobs(inp["x"], inp["w_row"], inp["w_col"])
    x = _t64(inp["x"], W.BF16)
    rr = torch.log_softmax(x @ _t64(inp["w_row"], W.BF16).T, dim=1).float().numpy()
    rc = torch.log_softmax(x @ _t64(inp["w_col"], W.BF16).T, dim=1).float().numpy()
    np.testing.assert_array_max_ulp(lr, rr, maxulp=1)
    np.testing.assert_array_max_ulp(lc, rc, maxulp=1)


def _lexsort_topk(lr, lc, K):
    S = (lr[:, None] + lc[None, :]).astype(np.float32).ravel()  # fp32 sums, row-major flat id
    order = np.lexsort((np.arange(S.size), -S.astype(np.float64)))
    return order[:K], S


def test_atomic_select_vs_lexsort():
    rng = np.random.default_rng(5)
    for trial in range(6):
        Nr, Nc, K = 9, 13, 10
        lr = (rng.integers(-4, 1, size=(2, Nr)) * 0.25).astype(np.float32)  # many ties
        lc = (rng.integers(-4, 1, size=(2, Nc)) * 0.25).astype(np.float32)
        if trial % 2:
            lr += rng.standard_normal((2, Nr)).astype(np.float32)
        idx, g = O.atomic_select(lr, lc, K)
        for t in range(2):
            order, S = _lexsort_topk(lr[t], lc[t], K)
            assert idx[t].tolist() == order.tolist()
            np.testing.assert_allclose(g[t], scipy.special.softmax(S[order].astype(np.float64)), rtol=1e-12)


def test_atomic_gates_are_renormalised_product_of_factors():
    # OmniMoE Eq. 8: p(i,j|x) ~ p_r(i|x) p_c(j|x); softmax over the selected
    # S = log p_r + log p_c is the product renormalised over the selection.
    cfg = _small_atomic(T=2, Nr=32, Nc=32, K=16)
    inp = W.make_atomic_inputs(cfg, experts=False)
    lr, lc = O.atomic_logprobs(inp["x"], inp["w_row"], inp["w_col"])
    idx, g = O.atomic_select(lr, lc, cfg.K)
    for t in range(2):
        pr, pc = np.exp(lr[t].astype(np.float64)), np.exp(lc[t].astype(np.float64))
        prod = pr[idx[t] // cfg.Nc] * pc[idx[t] % cfg.Nc]
        np.testing.assert_allclose(g[t], prod / prod.sum(), rtol=2e-6)  # S is rounded to fp32
        assert np.all(np.diff(g[t]) <= 0)


@pytest.mark.parametrize("act", [W.ACT_SILU, W.ACT_SIGMOID])
def test_atomic_output_vs_torch(act):
    cfg = _small_atomic(act=act)
    inp = W.make_atomic_inputs(cfg)
    lr, lc = O.atomic_logprobs(inp["x"], inp["w_row"], inp["w_col"])
    idx, g = O.atomic_select(lr, lc, cfg.K)
    out = O.atomic_output(inp["x"], inp["w_in"], inp["w_out"], idx, g, act)
    x = _t64(inp["x"], W.BF16)
    wi, wo = _t64(inp["w_in"], W.BF16), _t64(inp["w_out"], W.BF16)
    z = (x[:, None, :] * wi[torch.from_numpy(idx.astype(np.int64))]).sum(-1)
    a = torch.nn.functional.silu(z) if act == W.ACT_SILU else torch.sigmoid(z)
    ref = ((torch.from_numpy(g) * a)[:, :, None] * wo[torch.from_numpy(idx.astype(np.int64))]).sum(1)
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-10, atol=1e-12)


# ---------------------------------------- exactness of the grid top-K candidate method

def grid_topk_threshold_method(lr, lc, K):
    """The selection method the GPU kernel uses (restated here in plain Python):
    candidates = top-K rows x top-K cols (each by value desc, index asc); tau =
    the K-th best candidate score; every pair scoring above tau lies inside the
    candidate block, so the answer is those plus the first (in flat-id order)
    pairs of the whole grid that score exactly tau."""
    Nr, Nc = len(lr), len(lc)
    rows = sorted(range(Nr), key=lambda i: (-float(lr[i]), i))[:min(K, Nr)]
    cols = sorted(range(Nc), key=lambda j: (-float(lc[j]), j))[:min(K, Nc)]
    cand = sorted(((np.float32(lr[i]) + np.float32(lc[j]), i * Nc + j) for i in rows for j in cols),
                  key=lambda p: (-float(p[0]), p[1]))
    tau = cand[K - 1][0]
    above = [p for p in cand if p[0] > tau]
    need, tied = K - len(above), []
    for q in range(Nr * Nc):
        if len(tied) == need:
            break
        s = np.float32(lr[q // Nc]) + np.float32(lc[q % Nc])
        if s == tau:
            tied.append((s, q))
    return [q for _, q in sorted(above + tied, key=lambda p: (-float(p[0]), p[1]))]


def _collapse_case():
    # rows 1 and 2 beat row 0 by less than half an ulp of the sum, so all three
    # sums with column 0 round to the same fp32 value; flat id then decides.
    lr = np.array([-1.0, np.nextafter(np.float32(-1.0), np.float32(0)),
                   np.nextafter(np.float32(-1.0), np.float32(0)), -50.0], np.float32)
    lc = np.array([-8.0, -100.0, -100.0, -100.0], np.float32)
    return lr, lc


def test_grid_topk_method_exact_on_adversarial_grids():
    rng = np.random.default_rng(6)
    cases = [_collapse_case(), (np.zeros(8, np.float32), np.zeros(8, np.float32))]
    for _ in range(40):
        Nr, Nc = int(rng.integers(1, 12)), int(rng.integers(1, 12))
        q = rng.choice([0.25, 1e-7, 0.0])
        lr = (rng.integers(-3, 1, Nr) * q + rng.standard_normal(Nr) * (q == 1e-7) * 1e-7 - 5).astype(np.float32)
        lc = (rng.integers(-3, 1, Nc) * q - 7).astype(np.float32)
        cases.append((lr, lc))
    for lr, lc in cases:
        for K in sorted({1, 2, min(5, lr.size * lc.size), lr.size * lc.size}):
            idx, _ = O.atomic_select(lr[None], lc[None], K)
            assert grid_topk_threshold_method(lr, lc, K) == idx[0].tolist()


def grid_topk_staircase_method(lr, lc, K):
    """The prefill-budget selection method (K > 64) of the GPU kernel, restated in plain
    Python: with rows and columns sorted by (value desc, index asc), the candidates are
    the staircase pairs (a, b) with (a+1)(b+1) <= K; tau = the K-th best candidate score.
    If every staircase row's first pair past the staircase, and the first row left out,
    score below tau, the answer is the first K of the staircase pairs scoring >= tau in
    (score desc, id asc) order; otherwise the pairs above tau plus the lowest-id pairs of
    the whole grid scoring exactly tau. Returns (flat ids, whether the bound held)."""
    Nr, Nc = len(lr), len(lc)
    rows = sorted(range(Nr), key=lambda i: (-float(lr[i]), i))
    cols = sorted(range(Nc), key=lambda j: (-float(lc[j]), j))
    S = lambda i, j: np.float32(np.float32(lr[i]) + np.float32(lc[j]))
    kr = min(Nr, K)
    stair = [(S(rows[a], cols[b]), rows[a] * Nc + cols[b]) for a in range(kr) for b in range(min(Nc, K // (a + 1)))]
    tau = sorted((p[0] for p in stair), key=lambda v: -float(v))[K - 1]
    outside = any(min(Nc, K // (a + 1)) < Nc and S(rows[a], cols[min(Nc, K // (a + 1))]) >= tau for a in range(kr))
    outside = outside or (kr < Nr and S(rows[kr], cols[0]) >= tau)
    if not outside:
        win = sorted((p for p in stair if p[0] >= tau), key=lambda p: (-float(p[0]), p[1]))[:K]
        return [q for _, q in win], True
    above = [p for p in stair if p[0] > tau]
    need = K - len(above)
    tied = [(S(q // Nc, q % Nc), q) for q in range(Nr * Nc) if S(q // Nc, q % Nc) == tau][:need]
    return [q for _, q in sorted(above + tied, key=lambda p: (-float(p[0]), p[1]))], False


def test_grid_topk_staircase_method_exact():
    """Both branches of the prefill-budget method against the oracle's brute-force sort:
    random grids (the bound holds), level grids and all-equal grids (ties reach past
    the staircase), and the rounding-collapse case, for K up to the whole grid."""
    rng = np.random.default_rng(12)
    cases = [_collapse_case(), (np.zeros(9, np.float32), np.zeros(7, np.float32))]
    for _ in range(12):
        Nr, Nc = int(rng.integers(2, 40)), int(rng.integers(2, 40))
        cases.append(((rng.standard_normal(Nr) - 6).astype(np.float32), (rng.standard_normal(Nc) - 6).astype(np.float32)))
        cases.append(((rng.integers(0, 3, Nr) - 5).astype(np.float32), (rng.integers(0, 3, Nc) - 5).astype(np.float32)))
    branches = set()
    for lr, lc in cases:
        N = lr.size * lc.size
        for K in sorted({1, 2, min(65, N), min(100, N), N // 2 or 1, N}):
            idx, _ = O.atomic_select(lr[None], lc[None], K)
            got, fast = grid_topk_staircase_method(lr, lc, K)
            assert got == idx[0].tolist(), (lr.size, lc.size, K)
            branches.add(fast)
    assert branches == {True, False}  # both branches were exercised


def test_plain_candidate_block_is_not_always_exact():
    # Selecting only inside top-K rows x top-K cols misses (0, 0) here: the
    # rounding of the fp32 sums ties it with rows 1 and 2, and it has the lowest id.
    lr, lc = _collapse_case()
    K = 2
    idx, _ = O.atomic_select(lr[None], lc[None], K)
    assert idx[0].tolist() == [0, 4]
    rows = sorted(range(4), key=lambda i: (-float(lr[i]), i))[:K]
    assert 0 not in rows


# ------------------------------------------------------------------ R&Q replica dispatch

def _routing(text):
    return np.array([[int(e) for e in tok.split(",")] for tok in text.split(";")], dtype=np.int32)


def test_replica_split_golden(golden_dir):
    for name, m, k, before, heavy, after, counts, lis0, lis1 in _golden(os.path.join(golden_dir, "replica_cases.txt")):
        m, k = int(m), int(k)
        idx, idx2 = _routing(before), _routing(after)
        got, h = O.replica_split(idx, m)
        assert h == int(heavy), name
        np.testing.assert_array_equal(got, idx2, err_msg=name)
        assert O.histogram_lis(idx, m)["lis"] == float(Fraction(lis0)), name
        r = O.histogram_lis(got, m + 1)
        assert r["counts"].tolist() == [int(c) for c in counts.split(",")], name
        assert r["lis"] == float(Fraction(lis1)), name


@pytest.mark.parametrize("seed,T,m,k", [(0, 200, 8, 2), (1, 333, 16, 1), (2, 64, 4, 4), (3, 1000, 64, 6)])
def test_replica_split_closed_form(seed, T, m, k):
    # counts after: the heavy-hitter keeps ceil(n_h / 2), the replica gets floor(n_h / 2),
    # every other expert and every task of another expert is untouched, and in task
    # order the heavy-hitter's tasks alternate original, replica, original, ...
    rng = np.random.default_rng(seed)
    p = rng.dirichlet(np.full(m, 0.3))
    idx = np.stack([rng.choice(m, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    counts = np.bincount(idx.ravel(), minlength=m)
    h_ref = int(np.flatnonzero(counts == counts.max())[0])
    got, h = O.replica_split(idx, m)
    assert h == h_ref
    c2 = np.bincount(got.ravel(), minlength=m + 1)
    assert c2[h] == -(-counts[h] // 2) and c2[m] == counts[h] // 2
    keep = np.ones(m + 1, bool)
    keep[[h, m]] = False
    np.testing.assert_array_equal(c2[keep], counts[np.arange(m) != h])
    flat, flat2 = idx.ravel(), got.ravel()
    np.testing.assert_array_equal(flat2[flat != h], flat[flat != h])
    seq = flat2[flat == h]
    np.testing.assert_array_equal(seq, np.where(np.arange(len(seq)) % 2 == 0, h, m))
    assert O.histogram_lis(got, m + 1)["lis"] == (m + 1) * c2.max() / (T * k)


@pytest.mark.parametrize("dtype,act", [(W.F32, W.SWIGLU), (W.BF16, W.RELU)])
def test_replica_leaves_layer_output_unchanged(dtype, act):
    # the replica carries the heavy-hitter's own weights, so every task computes the
    # same expert function: the layer output is identical in fp64
    cfg = W.small_moe(T=24, d=32, f=24, m=5, k=2, act=act, dtype=dtype, zipf_s=1.5, index=95)
    inp = W.make_moe_inputs(cfg)
    r = O.layer_forward(cfg, inp)
    idx2, h = O.replica_split(r["idx"], cfg.m)
    assert (idx2 == cfg.m).any()
    cfg2 = W.small_moe(T=24, d=32, f=24, m=6, k=2, act=act, dtype=dtype, zipf_s=1.5, index=95)
    out2 = O.moe_output(cfg2, O.replica_inputs(inp, h), idx2, r["w"])
    np.testing.assert_array_equal(out2, r["out"])


# ------------------------------------------------------------------ FloE contextual sparsity

@pytest.mark.parametrize("s,expect", [(0.0, 0.1), (0.25, 0.1), (0.5, 0.2), (0.75, 0.3), (0.9, 0.5), (1.0, 0.5)])
def test_floe_threshold_hand_cases(s, expect):
    # n = 4 values; the ceil(s n)-th smallest (at least the first)
    assert O.floe_threshold(np.array([0.5, 0.1, 0.3, 0.2], np.float32), s) == np.float32(expect)


@pytest.mark.parametrize("s", [0.5, 0.8, 0.9, 0.97])
def test_floe_threshold_is_the_cdf_quantile(s):
    # a fraction >= s of the sample lies at or below t, and < s strictly below it
    v = np.abs(np.random.default_rng(int(100 * s)).standard_normal(5003)).astype(np.float32)
    t = O.floe_threshold(v, s)
    assert (v <= t).mean() >= s and (v < t).mean() < s


def _expert_case(act_seed=0):
    cfg = W.small_moe(T=3, d=48, f=40, m=2, k=1, dtype=W.BF16, zipf_s=0.0, index=98 + act_seed)
    return cfg, W.make_moe_inputs(cfg)


def test_floe_expert_threshold_zero_is_the_dense_expert():
    cfg, inp = _expert_case()
    for t in range(cfg.T):
        y, keep = O.floe_expert(inp["x"][t], inp["w_gate"][1], inp["w_up"][1], inp["w_down"][1], 0.0, W.BF16)
        assert keep.all()
        ref = O.expert_ffn(inp["x"][t], inp["w_gate"][1], inp["w_up"][1], inp["w_down"][1], W.SWIGLU)
        np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-14)


def test_floe_expert_infinite_threshold_is_zero():
    cfg, inp = _expert_case()
    y, keep = O.floe_expert(inp["x"][0], inp["w_gate"][0], inp["w_up"][0], inp["w_down"][0], np.inf, W.BF16)
    assert not keep.any() and not y.any()


def test_floe_expert_is_the_dense_expert_with_pruned_channels_zeroed():
    cfg, inp = _expert_case(1)
    t64 = lambda a: torch.from_numpy(np.asarray(W.as_f32(a, W.BF16), np.float64))
    x, wg, wu, wd = t64(inp["x"][2]), t64(inp["w_gate"][0]), t64(inp["w_up"][0]), t64(inp["w_down"][0])
    u = wu @ x
    thr = float(np.quantile(np.abs(u.numpy()), 0.7))
    y, keep = O.floe_expert(inp["x"][2], inp["w_gate"][0], inp["w_up"][0], inp["w_down"][0], thr, W.BF16)
    h = torch.nn.functional.silu(wg @ x) * u
    h[torch.from_numpy(~keep)] = 0.0
    assert 0 < keep.sum() < keep.size
    np.testing.assert_allclose(y, (wd @ h).numpy(), rtol=1e-12, atol=1e-14)


def test_floe_mask_keeps_the_threshold_itself():
    # Eq. 6 prunes activations strictly below t; one exactly at t is kept
    cfg, inp = _expert_case(1)
    u = np.asarray(W.as_f32(inp["w_up"][0], W.BF16), np.float64) @ np.asarray(W.as_f32(inp["x"][1], W.BF16),
                                                                                 np.float64)
    j = int(np.argsort(np.abs(u))[len(u) // 2])
    u32 = u.astype(np.float32)  # the mask compares these; the threshold is one of them exactly
    thr = float(abs(u32[j]))
    _, keep = O.floe_expert(inp["x"][1], inp["w_gate"][0], inp["w_up"][0], inp["w_down"][0], thr, W.BF16,
                            u_mask=u32)
    assert keep[j] and keep.sum() == (np.abs(u32) >= np.float32(thr)).sum()


# ---------------------------------------------------------- 8-bit expert weights
# Facts of the OCP E4M3 format: bias 7, 3 mantissa bits, no infinities, one NaN
# pattern per sign (S.1111.111), largest finite 0x7E = 1.75 * 2^8 = 448, smallest
# subnormal 0x01 = 2^-9, smallest normal 0x08 = 2^-6, 0x38 = 1.

E4M3_FACTS = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0, 0x39: 1.125,
              0x40: 2.0, 0x7E: 448.0, 0x80: -0.0, 0xB8: -1.0, 0xFE: -448.0}


def test_e4m3_decode_format_facts():
    for code, val in E4M3_FACTS.items():
        got = O.e4m3_value(np.uint8(code))
        assert got == val and np.signbit(got) == np.signbit(val), hex(code)
    assert np.isnan(O.e4m3_value(np.uint8(0x7F))) and np.isnan(O.e4m3_value(np.uint8(0xFF)))


def test_e4m3_decode_matches_torch_float8():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    got = O.e4m3_value(codes)
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], got[ok])


def _e4m3_brute(v):
    """Nearest finite E4M3 value by exhaustive search over the 127 non-negative
    finite codes; a tie goes to the code with an even mantissa (lowest bit 0);
    magnitudes past 448 saturate. Sign copied from v."""
    pos = np.arange(0x7F, dtype=np.uint8)
    vals = O.e4m3_value(pos)
    out = []
    for x in np.asarray(v, np.float32):
        a = min(abs(float(x)), 448.0)
        dist = np.abs(vals - a)
        best = np.flatnonzero(dist == dist.min())
        code = int(best[0]) if len(best) == 1 else int([b for b in best if b % 2 == 0][0])
        out.append(code | (0x80 if np.signbit(x) else 0))
    return np.array(out, np.uint8)


def _e4m3_probe_values(rng):
    vals = O.e4m3_value(np.arange(0x7F, dtype=np.uint8))
    mids = (vals[:-1] + vals[1:]) / 2                 # every tie between neighbouring codes
    rnd = rng.standard_normal(3000) * np.exp2(rng.integers(-14, 10, 3000))
    edge = np.array([447.9, 448, 455.9, 464.0, 470.0, 1e6, 1e30, 2.0 ** -10, 2.0 ** -12, 0.0, -0.0])
    v = np.concatenate([vals, mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9), rnd, edge]).astype(np.float32)
    return np.concatenate([v, -v])


def test_e4m3_round_is_nearest_even_by_exhaustive_search():
    v = _e4m3_probe_values(np.random.default_rng(7))
    np.testing.assert_array_equal(O.e4m3_round(v), _e4m3_brute(v))


def test_e4m3_round_matches_torch_cast_in_range():
    v = _e4m3_probe_values(np.random.default_rng(8))
    v = v[np.abs(v) < 464]                             # torch's cast gives NaN, not 448, past the last tie
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(O.e4m3_round(v), ref)


def test_quantize_rows_invariants():
    rng = np.random.default_rng(9)
    a = (rng.standard_normal((40, 96)) * np.exp2(rng.integers(-20, 20, (40, 1)))).astype(np.float32)
    a[3] = 0.0
    a[5, :] = 0.0
    a[5, 17] = -3.0
    codes, sc = O.quantize_rows(a)
    assert sc[3] == 1.0 and not codes[3].any()
    for r in range(40):
        if r == 3:
            continue
        j = int(np.argmax(np.abs(a[r])))
        assert codes[r, j] & 0x7F == 0x7E                # the row maximum lands on 448
        assert sc[r] == np.float32(np.abs(a[r]).max() / np.float32(448))
        dq = O.e4m3_value(codes[r]) * np.float64(sc[r])
        err = np.abs(dq - a[r])
        # half a quantum: 2^-4 relative in the normal range, 2^-10 * scale below it
        bound = np.maximum(np.abs(a[r]).astype(np.float64) * 2.0 ** -4, 2.0 ** -10 * np.float64(sc[r])) * (1 + 1e-6)
        assert np.all(err <= bound), r


def _pow2_bf16(rng, shape, lo, hi, p_zero=0.2):
    """bf16 bit patterns of +-2^e (e uniform in [lo, hi]) with some exact zeros."""
    e = rng.integers(lo, hi + 1, shape)
    bits = ((e + 127) << 7) | (rng.integers(0, 2, shape) << 15)
    bits = np.where(rng.random(shape) < p_zero, 0, bits)
    return bits.astype(np.uint16)


def test_fp8_layer_is_lossless_on_power_of_two_inputs():
    """With one-hot token rows and weights that are signed powers of two, every
    product, every ReLU output and every quantized row is exactly representable
    (up to the fp32 rounding of the scales), so the 8-bit layer equals the bf16
    layer to ~1e-6: each scale (x, weight rows, h) must be applied exactly once."""
    cfg = W.small_moe(T=24, d=32, f=16, m=4, k=2, act=W.RELU, dtype=W.BF16, zipf_s=0.5, n_shared=1,
                      f_shared=16, index=93)
    inp = W.make_moe_inputs(cfg)
    rng = np.random.default_rng(10)
    x = np.zeros((cfg.T, cfg.d), np.uint16)
    x[np.arange(cfg.T), rng.integers(0, cfg.d, cfg.T)] = _pow2_bf16(rng, cfg.T, 0, 2, p_zero=0.0)
    inp["x"] = x
    for key in ("w_gate", "w_down", "ws_gate", "ws_down"):
        inp[key] = _pow2_bf16(rng, inp[key].shape, -3, 0)
    ref = O.layer_forward(cfg, inp)["out"]
    got = O.layer_forward_fp8(cfg, inp)["out"]
    assert np.abs(ref).max() > 0.1
    np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-6 * np.abs(ref).max())


def _swiglu_pow2_case(seed):
    """A SwiGLU layer whose 8-bit run is exact: one-hot token rows of +-2^9 or 2^10,
    gate and down weights +-2^-3 .. 2^0, up weights +-2^-6 .. 2^-3 (some zero). Every
    gate pre-activation is then 0 or +-2^6 .. 2^10: at +2^6 and above the logistic
    function is 1 in fp64 (exp(-64) is below half an ulp of 1), so SiLU(g) = g and
    h = g u is a power of two; at -2^6 and below h is ~1e-26 u. A row's non-negligible
    h values (2^9 .. 2^17) span at most 2^8, so each lands on an E4M3 code after its row scale;
    the negligible ones quantize to 0."""
    cfg = W.small_moe(T=20, d=32, f=16, m=4, k=2, act=W.SWIGLU, dtype=W.BF16, zipf_s=0.5, n_shared=1,
                      f_shared=16, index=96)
    inp = W.make_moe_inputs(cfg)
    rng = np.random.default_rng(seed)
    x = np.zeros((cfg.T, cfg.d), np.uint16)
    x[np.arange(cfg.T), rng.integers(0, cfg.d, cfg.T)] = _pow2_bf16(rng, cfg.T, 9, 10, p_zero=0.0)
    inp["x"] = x
    for key in ("w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down"):
        lo, hi = (-6, -3) if key.endswith("up") else (-3, 0)  # up rows on another scale than gate rows
        inp[key] = _pow2_bf16(rng, inp[key].shape, lo, hi)
    return cfg, inp


def test_fp8_swiglu_layer_is_lossless_on_power_of_two_inputs():
    """The SwiGLU branch of the 8-bit oracle (gate and up scales, SiLU, h's row
    scale) against the bf16 oracle on inputs where every quantization is exact:
    equal up to the fp32 rounding of the scales. A swapped scale, a dropped SiLU or
    a dropped up factor changes the output by a power of two or more."""
    cfg, inp = _swiglu_pow2_case(12)
    ref = O.layer_forward(cfg, inp)["out"]
    got = O.layer_forward_fp8(cfg, inp)["out"]
    assert np.abs(ref).max() > 1.0
    np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-6 * np.abs(ref).max())


# --------------------------------------------- bf16 rounding of stored activations
# bf16 keeps 8 significand bits (7 stored): next to 1 its spacing is 2^-7. A value
# exactly half way between two bf16 numbers goes to the one with an even last
# significand bit (IEEE 754 round to nearest, ties to even); the oracle rounds
# float64 to float32 first, then float32 to bf16.
BF16_CASES = [
    (1.0 + 2.0 ** -8, 1.0),                       # tie between 1 (even) and 1 + 2^-7 (odd): down
    (1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -6),       # tie between 1 + 2^-7 (odd) and 1 + 2^-6 (even): up
    (1.0 + 2.0 ** -8 + 2.0 ** -20, 1.0 + 2.0 ** -7),  # just above the tie: up
    (1.0 + 2.0 ** -8 - 2.0 ** -20, 1.0),          # just below: down
    (-(1.0 + 2.0 ** -8), -1.0),                   # the sign does not change the tie rule
    (-(1.0 + 3 * 2.0 ** -8), -(1.0 + 2.0 ** -6)),
    (1.0 + 2.0 ** -8 + 2.0 ** -30, 1.0),          # 2^-30 is lost in the float32 step; then a tie
    (255.5, 256.0),                               # 255 and 256 are neighbours near 2^8: the tie goes to 256
    (3.0, 3.0),                                   # representable values are unchanged
    (2.0 ** -133, 2.0 ** -133),                   # a float32 subnormal that bf16 holds exactly
    (0.0, 0.0),
]


def test_round_bf16_hand_worked_ties_to_even():
    v = np.array([a for a, _ in BF16_CASES], np.float64)
    got = O.round_bf16(v)
    assert got.dtype == np.float32
    assert got.tolist() == [b for _, b in BF16_CASES]
    assert np.signbit(O.round_bf16(np.array([-0.0])))[0]
    big = O.round_bf16(np.array([np.finfo(np.float32).max], np.float64))  # past the largest bf16: infinity
    assert np.isinf(big[0])


def test_round_bf16_matches_torch_bfloat16_cast():
    rng = np.random.default_rng(31)
    bits = rng.integers(0, 2 ** 32, 200000, dtype=np.uint64).astype(np.uint32)
    bits = bits[(bits & 0x7F800000) != 0x7F800000]   # no inf / NaN patterns
    ties = ((rng.integers(0, 2 ** 16, 20000, dtype=np.uint64) << 16) | 0x8000).astype(np.uint32)
    ties = ties[(ties & 0x7F800000) != 0x7F800000]   # exact ties, both parities of the kept part
    f = np.concatenate([bits, ties]).view(np.float32)
    ref = torch.from_numpy(f.copy()).to(torch.bfloat16).float().numpy()
    got = O.round_bf16(f.astype(np.float64))
    np.testing.assert_array_equal(got.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("act", [W.SWIGLU, W.RELU])
def test_fp8_layer_is_close_to_bf16_layer(act):
    """On random bf16 inputs the 8-bit layer differs from the bf16 layer by the
    quantization error only. Each of the three rounding steps (x, weights, h) has a
    relative error uniform in +-2^-4, about 3.6 % rms, so the normwise error is a few
    per cent: never zero, never the size of the output."""
    cfg = W.small_moe(T=40, d=64, f=48, m=4, k=2, act=act, dtype=W.BF16, zipf_s=0.5, n_shared=1, f_shared=32,
                      index=94)
    inp = W.make_moe_inputs(cfg)
    ref = O.layer_forward(cfg, inp)["out"]
    got = O.layer_forward_fp8(cfg, inp)["out"]
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert 5e-3 < rel < 0.15, rel


def test_fp8_sampled_tokens_match_full_output():
    cfg = W.small_moe(T=30, d=32, f=32, m=5, k=2, act=W.SWIGLU, dtype=W.BF16, zipf_s=1.0, index=95)
    inp = W.make_moe_inputs(cfg)
    full = O.layer_forward_fp8(cfg, inp)["out"]
    tok = [29, 3, 3, 17]
    np.testing.assert_allclose(O.layer_forward_fp8(cfg, inp, tokens=tok)["out"], full[tok], rtol=1e-12, atol=0)

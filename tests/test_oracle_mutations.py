"""Plant plausible mistakes in a COPY of the oracle and check the pins catch them.

Each mutation edits the C source text of the oracle, compiles it into a temporary
library, loads the oracle's Python wrapper against that library and runs the
independent checks (hand-worked fixtures, library routines, closed forms). Every
mutant must fail at least one check; the unmodified oracle must pass all of them.
The shipped oracle is never modified.
"""
import importlib.util
import math
import os
import shutil
from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import torch

import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.c")

MUTATIONS = {
    "bias_dropped": ("if (bias) s += (double)bias[e];", ""),
    "tie_break_highest_index": ("lg[e] > lg[best]) best = e;", "lg[e] >= lg[best]) best = e;"),
    "renorm_ignored": ("if (renorm)\n", "if (0)\n"),
    "gate_weight_wrong_index": ("w[s] = exp((double)lg[idx[s]] - mx) / z;", "w[s] = exp((double)lg[s] - mx) / z;"),
    "lis_missing_k": ("/ (double)((int64_t)T * k);", "/ (double)T;"),
    "argmax_last_tie": ("if (counts[e] > counts[best]) best = e;", "if (counts[e] >= counts[best]) best = e;"),
    "permutation_reversed_in_segment": ("int32_t pos = offsets[e] + cursor[e]++;",
                                        "int32_t pos = offsets[e + 1] - 1 - cursor[e]++;"),
    "silu_dropped": ("h[j] = g * logistic(g) * u;", "h[j] = g * u;"),
    "up_dropped": ("h[j] = g * logistic(g) * u;", "h[j] = g * logistic(g);"),
    "relu_sign": ("h[j] = g > 0.0 ? g : 0.0;", "h[j] = g < 0.0 ? -g : 0.0;"),
    "down_transposed": ("val(wd, dtype, (int64_t)o * f + j)", "val(wd, dtype, (int64_t)j * d + o)"),
    "shared_dropped": ("for (int sh = 0; sh < c->n_shared; ++sh) {\n    const size_t mat",
                       "for (int sh = 0; sh < 0; ++sh) {\n    const size_t mat"),
    "atomic_activation_sigmoid": ("double a = act == O_SILU ? z * logistic(z) : logistic(z);",
                                  "double a = logistic(z);"),
    "atomic_tie_id_descending": ("return (p->id > q->id) - (p->id < q->id);",
                                 "return (p->id < q->id) - (p->id > q->id);"),
    "atomic_logprob_unnormalised": ("out[(int64_t)t * n + i] = (float)(z[i] - lse);",
                                    "out[(int64_t)t * n + i] = (float)(z[i] - mx);"),
    "replica_even_ranks": ("idx_out[q] = (r % 2 == 1) ? m : h;", "idx_out[q] = (r % 2 == 0) ? m : h;"),
    "replica_heavy_last_tie": ("if (counts[e] > counts[h]) h = e;", "if (counts[e] >= counts[h]) h = e;"),
}


# mistakes planted in the Python part of the oracle (oracle/__init__.py)
PY_MUTATIONS = {
    "floe_mask_strict": ("if u_mask is not None else u) >= thr", "if u_mask is not None else u) > thr"),
    "floe_gate_from_up": ("g = as64(wg)[keep] @ x", "g = as64(wu)[keep] @ x"),
    "floe_threshold_off_by_one": ("return np.float32(v[min(r, v.size) - 1])", "return np.float32(v[min(r, v.size - 1)])"),
    "e4m3_ties_away": ("n = np.rint(np.ldexp(a, 3 - e))", "n = np.floor(np.ldexp(a, 3 - e) + 0.5)"),
    "e4m3_no_saturation": ("a = np.minimum(np.abs(v).astype(np.float64), E4M3_MAX)", "a = np.abs(v).astype(np.float64)"),
    "e4m3_bias_8": ("np.ldexp(1.0, E - 7)", "np.ldexp(1.0, E - 8)"),
    "fp8_scale_240": ("amax / np.float32(E4M3_MAX)", "amax / np.float32(240.0)"),
    "fp8_h_scale_dropped": ("H = e4m3_value(hq) * hs[:, None].astype(np.float64)", "H = e4m3_value(hq)"),
    "fp8_x_scale_dropped": ("X = e4m3_value(xq) * sx[:, None].astype(np.float64)", "X = e4m3_value(xq)"),
    "fp8_column_scales": ("amax = np.max(np.abs(a), axis=1) if", "amax = np.max(np.abs(a), axis=0)[:a.shape[0]] if"),
    "fp8_up_scale_from_gate": ("b = X @ (e4m3_value(uq) * us[:, None].astype(np.float64)).T",
                               "b = X @ (e4m3_value(uq) * gs[:, None].astype(np.float64)).T"),
    "fp8_silu_dropped": ("return a / (1.0 + np.exp(-a)) * b", "return a * b"),
    "bf16_truncates": ("u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16 << 16", "u = u >> 16 << 16"),
    "bf16_ties_away": ("u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16 << 16", "u = (u + 0x8000) >> 16 << 16"),
}


def _load_oracle(tmpdir, src_text, py_text=None):
    c_path = os.path.join(tmpdir, "moe_oracle.c")
    with open(c_path, "w") as fh:
        fh.write(src_text)
    py_path = os.path.join(ROOT, "oracle", "__init__.py")
    if py_text is not None:
        py_path = os.path.join(tmpdir, "oracle_init.py")
        with open(py_path, "w") as fh:
            fh.write(py_text)
    spec = importlib.util.spec_from_file_location(f"oracle_copy_{abs(hash((src_text, py_text)))}", py_path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod._SRC = c_path
    mod._LIB_PATH = os.path.join(tmpdir, "liboracle.so")
    mod._lib = None
    mod.build(force=True)
    return mod


def _t64(a, dtype):
    return torch.from_numpy(np.asarray(W.as_f32(a, dtype), dtype=np.float64))


def _golden_rows(name):
    rows = []
    with open(os.path.join(ROOT, "tests", "golden", name)) as fh:
        for line in fh:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([c.strip() for c in line.split("|")])
    return rows


# ------------------------------------------------------------------ checks
def check_lis_golden(O):
    for name, m, k, routing, counts, mx, am, lis in _golden_rows("lis_cases.txt"):
        idx = np.array([[int(e) for e in tok.split(",")] for tok in routing.split(";")], dtype=np.int32)
        r = O.histogram_lis(idx, int(m))
        assert r["counts"].tolist() == [int(c) for c in counts.split(",")]
        assert r["argmax"] == int(am) and r["lis"] == float(Fraction(lis))


def check_topk(O):
    for name, k, rn, logits, idx, wts in _golden_rows("topk_cases.txt"):
        lg = np.array([[np.float32(math.log(float(v[3:]))) if v.startswith("ln:") else np.float32(float(v))
                        for v in logits.split(",")]], np.float32)
        i, w = O.topk_softmax(lg, int(k), bool(int(rn)))
        assert i[0].tolist() == [int(v) for v in idx.split(",")]
        np.testing.assert_allclose(w[0], [float(Fraction(v)) for v in wts.split(",")], rtol=1e-6)
    rng = np.random.default_rng(1)
    lg = (rng.integers(-3, 4, size=(50, 8)) * 0.5).astype(np.float32)
    idx, w = O.topk_softmax(lg, 2, True)
    for t in range(50):
        assert idx[t].tolist() == np.lexsort((np.arange(8), -lg[t].astype(np.float64)))[:2].tolist()
    p = scipy.special.softmax(lg.astype(np.float64), axis=1)
    sel = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    np.testing.assert_allclose(w, sel / sel.sum(1, keepdims=True), rtol=1e-12)


def check_router(O):
    cfg = W.small_moe(T=9, d=40, f=8, m=6, k=1, dtype=W.BF16, zipf_s=1.0)
    inp = W.make_moe_inputs(cfg, weights=False)
    got = O.router_logits(inp["x"], inp["w_router"], inp["bias"])
    ref = (_t64(inp["x"], W.BF16) @ _t64(inp["w_router"], W.BF16).T
           + torch.from_numpy(inp["bias"].astype(np.float64))).float().numpy()
    np.testing.assert_array_max_ulp(got, ref, maxulp=1)


def check_permutation(O):
    rng = np.random.default_rng(4)
    lg = rng.standard_normal((60, 8)).astype(np.float32)
    idx, _ = O.topk_softmax(lg, 2, False)
    r = O.histogram_lis(idx, 8)
    perm, inv = O.permutation(idx, 8, r["offsets"])
    np.testing.assert_array_equal(perm, np.argsort(idx.ravel(), kind="stable"))
    np.testing.assert_array_equal(inv[perm], np.arange(120))


def _torch_ffn(x, wg, wu, wd, act):
    a = x @ wg.T
    h = torch.nn.functional.silu(a) * (x @ wu.T) if act == W.SWIGLU else torch.relu(a)
    return h @ wd.T


def check_ffn(O):
    for act in (W.SWIGLU, W.RELU):
        cfg = W.small_moe(T=5, d=24, f=16, m=1, k=1, act=act, dtype=W.BF16, zipf_s=0.0)
        inp = W.make_moe_inputs(cfg)
        r = O.layer_forward(cfg, inp)
        t = lambda key: _t64(inp[key], W.BF16)
        ref = _torch_ffn(t("x"), t("w_gate")[0], t("w_up")[0] if act == W.SWIGLU else None, t("w_down")[0], act)
        np.testing.assert_allclose(r["out"], ref.numpy(), rtol=1e-10, atol=1e-12)


def check_shared(O):
    cfg = W.small_moe(T=4, d=24, f=16, m=3, k=1, act=W.SWIGLU, dtype=W.BF16, zipf_s=1.0, n_shared=1, f_shared=8)
    inp = W.make_moe_inputs(cfg)
    r = O.layer_forward(cfg, inp)
    t = lambda key: _t64(inp[key], W.BF16)
    x = t("x")
    ref = _torch_ffn(x, t("ws_gate")[0], t("ws_up")[0], t("ws_down")[0], W.SWIGLU)
    for tok in range(4):
        e = int(r["idx"][tok, 0])
        ref[tok] += float(r["w"][tok, 0]) * _torch_ffn(x[tok:tok + 1], t("w_gate")[e], t("w_up")[e],
                                                        t("w_down")[e], W.SWIGLU)[0]
    np.testing.assert_allclose(r["out"], ref.numpy(), rtol=1e-10, atol=1e-12)


def check_atomic(O):
    cfg = W.AtomicWorkload("atomic_small", 91, T=2, d=32, Nr=8, Nc=6, K=5, act=W.ACT_SILU)
    inp = W.make_atomic_inputs(cfg)
    lr, lc = O.atomic_logprobs(inp["x"], inp["w_row"], inp["w_col"])
    x = _t64(inp["x"], W.BF16)
    np.testing.assert_array_max_ulp(lr, torch.log_softmax(x @ _t64(inp["w_row"], W.BF16).T, 1).float().numpy(), 1)
    tl = np.zeros((1, 4), np.float32)
    idx, _ = O.atomic_select(tl, tl, 3)
    assert idx[0].tolist() == [0, 1, 2]
    idx, g = O.atomic_select(lr, lc, cfg.K)
    out = O.atomic_output(inp["x"], inp["w_in"], inp["w_out"], idx, g, W.ACT_SILU)
    wi, wo = _t64(inp["w_in"], W.BF16), _t64(inp["w_out"], W.BF16)
    ii = torch.from_numpy(idx.astype(np.int64))
    z = (x[:, None, :] * wi[ii]).sum(-1)
    ref = ((torch.from_numpy(g) * torch.nn.functional.silu(z))[:, :, None] * wo[ii]).sum(1)
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-10, atol=1e-12)


def check_replica(O):
    for name, m, k, before, heavy, after, counts, lis0, lis1 in _golden_rows("replica_cases.txt"):
        idx = np.array([[int(e) for e in tok.split(",")] for tok in before.split(";")], dtype=np.int32)
        got, h = O.replica_split(idx, int(m))
        assert h == int(heavy)
        assert got.ravel().tolist() == [int(e) for tok in after.split(";") for e in tok.split(",")]


def check_floe(O):
    v = np.array([0.5, 0.1, 0.3, 0.2], np.float32)
    assert [O.floe_threshold(v, s) for s in (0.0, 0.5, 0.75, 0.9)] == [np.float32(a) for a in (0.1, 0.2, 0.3, 0.5)]
    cfg = W.small_moe(T=2, d=32, f=24, m=1, k=1, dtype=W.BF16, zipf_s=0.0, index=99)
    inp = W.make_moe_inputs(cfg)
    y, _ = O.floe_expert(inp["x"][0], inp["w_gate"][0], inp["w_up"][0], inp["w_down"][0], 0.0, W.BF16)
    t = lambda key: _t64(inp[key], W.BF16)
    ref = _torch_ffn(t("x")[0:1], t("w_gate")[0], t("w_up")[0], t("w_down")[0], W.SWIGLU)[0]
    np.testing.assert_allclose(y, ref.numpy(), rtol=1e-10, atol=1e-12)
    u32 = (t("w_up")[0] @ t("x")[1]).numpy().astype(np.float32)
    j = int(np.argsort(np.abs(u32))[12])
    _, keep = O.floe_expert(inp["x"][1], inp["w_gate"][0], inp["w_up"][0], inp["w_down"][0], float(abs(u32[j])),
                            W.BF16, u_mask=u32)
    assert keep[j]


def check_fp8(O):
    for code, val in ((0x01, 2.0 ** -9), (0x08, 2.0 ** -6), (0x38, 1.0), (0x7E, 448.0), (0xFE, -448.0)):
        assert O.e4m3_value(np.uint8(code)) == val
    v = np.array([1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -11, 460.0, 1e6, -5.5, 0.3], np.float32)
    assert O.e4m3_round(v).tolist() == [0x38, 0x3A, 0x00, 0x01, 0x7E, 0x7E, 0xCB, 0x2A]
    rng = np.random.default_rng(11)
    a = rng.standard_normal((6, 40)).astype(np.float32)
    codes, sc = O.quantize_rows(a)
    assert all(codes[r, int(np.argmax(np.abs(a[r])))] & 0x7F == 0x7E for r in range(6))
    cfg = W.small_moe(T=16, d=32, f=16, m=3, k=2, act=W.RELU, dtype=W.BF16, zipf_s=0.5, n_shared=1,
                      f_shared=16, index=93)
    inp = W.make_moe_inputs(cfg)
    x = np.zeros((cfg.T, cfg.d), np.uint16)
    pw = lambda shape, lo, hi: (((rng.integers(lo, hi + 1, shape) + 127) << 7)
                                | (rng.integers(0, 2, shape) << 15)).astype(np.uint16)
    x[np.arange(cfg.T), rng.integers(0, cfg.d, cfg.T)] = pw(cfg.T, 0, 2)
    inp["x"] = x
    for key in ("w_gate", "w_down", "ws_gate", "ws_down"):
        inp[key] = pw(inp[key].shape, -3, 0)
    ref = O.layer_forward(cfg, inp)["out"]
    np.testing.assert_allclose(O.layer_forward_fp8(cfg, inp)["out"], ref, rtol=1e-5, atol=1e-6 * np.abs(ref).max())
    # SwiGLU on exact inputs: one-hot rows of 2^9..2^10 make every gate pre-activation
    # 0 or at least 2^6 in size, where SiLU(g) = g (or ~0); see test_oracle_pins
    cfg = W.small_moe(T=20, d=32, f=16, m=4, k=2, act=W.SWIGLU, dtype=W.BF16, zipf_s=0.5, n_shared=1,
                      f_shared=16, index=96)
    inp = W.make_moe_inputs(cfg)
    x = np.zeros((cfg.T, cfg.d), np.uint16)
    x[np.arange(cfg.T), rng.integers(0, cfg.d, cfg.T)] = (((rng.integers(9, 11, cfg.T) + 127) << 7)
                                                          | (rng.integers(0, 2, cfg.T) << 15)).astype(np.uint16)
    inp["x"] = x
    for key in ("w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down"):
        inp[key] = pw(inp[key].shape, -6, -3) if key.endswith("up") else pw(inp[key].shape, -3, 0)
    ref = O.layer_forward(cfg, inp)["out"]
    np.testing.assert_allclose(O.layer_forward_fp8(cfg, inp)["out"], ref, rtol=1e-5, atol=1e-6 * np.abs(ref).max())


def check_round_bf16(O):
    # hand-worked ties (bf16 spacing 2^-7 next to 1): 1 + 2^-8 -> 1, 1 + 3 2^-8 -> 1 + 2^-6
    v = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, 1 + 2.0 ** -8 + 2.0 ** -20, -(1 + 3 * 2.0 ** -8), 255.5])
    assert O.round_bf16(v).tolist() == [1.0, 1 + 2.0 ** -6, 1 + 2.0 ** -7, -(1 + 2.0 ** -6), 256.0]
    f = np.random.default_rng(3).standard_normal(5000).astype(np.float32)
    ref = torch.from_numpy(f).to(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(O.round_bf16(f.astype(np.float64)), ref)


CHECKS = [check_lis_golden, check_topk, check_router, check_permutation, check_ffn, check_shared, check_atomic,
          check_replica, check_floe, check_fp8, check_round_bf16]


def _failures(O):
    failed = []
    for chk in CHECKS:
        try:
            chk(O)
        except (AssertionError, ValueError):
            failed.append(chk.__name__)
    return failed


@pytest.fixture(scope="module")
def source():
    with open(SRC) as fh:
        return fh.read()


def test_unmodified_oracle_passes_every_check(tmp_path, source):
    assert _failures(_load_oracle(str(tmp_path), source)) == []


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutant_is_caught(tmp_path, source, name):
    old, new = MUTATIONS[name]
    assert source.count(old) >= 1, f"mutation anchor for {name} not found"
    mutated = source.replace(old, new, 1)
    failed = _failures(_load_oracle(str(tmp_path), mutated))
    assert failed, f"mutation {name} was not caught by any check"


@pytest.fixture(scope="module")
def py_source():
    with open(os.path.join(ROOT, "oracle", "__init__.py")) as fh:
        return fh.read()


@pytest.mark.parametrize("name", sorted(PY_MUTATIONS))
def test_python_mutant_is_caught(tmp_path, source, py_source, name):
    old, new = PY_MUTATIONS[name]
    assert py_source.count(old) == 1, f"mutation anchor for {name} not found"
    failed = _failures(_load_oracle(str(tmp_path), source, py_source.replace(old, new, 1)))
    assert failed, f"mutation {name} was not caught by any check"

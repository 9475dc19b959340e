"""Pins for the fp64 CPU oracle against what the pages and mathematics fix.

Each test ties one oracle function to something other than itself: values the
pages print (``tests/golden``), closed forms, invariants, an independent
formulation of the same rule, a library routine that the page itself names as
the definition, or central finite differences.  A plausible slip in the oracle
(dropped max-subtraction, wrong tie order, an off-by-one capacity, a wrong
normalisation of f, a sign or index error in the backward) fails at least one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests.conftest import GOLDEN


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# capacity
# --------------------------------------------------------------------------
def test_capacity_closed_form_and_workloads():
    # ceil(cf * T * k / E) at the five workload shapes (all exact integers).
    assert O.capacity(512, 2, 8, 1.25) == 160
    assert O.capacity(32768, 1, 64, 1.0) == 512
    assert O.capacity(16384, 8, 256, 1.25) == 640
    assert O.capacity(8192, 2, 64, 1.0) == 256
    # non-integer quotient rounds up; floor of one for tiny factors
    assert O.capacity(10, 1, 3, 1.0) == 4
    assert O.capacity(1, 1, 64, 1e-9) == 1
    for bad in (0.0, -1.0, float("nan"), float("inf")):
        with pytest.raises(ValueError):
            O.capacity(8, 2, 4, bad)
    with pytest.raises(ValueError):
        O.capacity(8, 5, 4, 1.0)  # k > E


# --------------------------------------------------------------------------
# router page: three worked examples, exact
# --------------------------------------------------------------------------
@pytest.mark.parametrize("i", [0, 1, 2])
def test_router_page_examples(i):
    g = _golden("router_load_statistics_examples.json")
    ex = g["examples"][i]
    tol = 0.5 * 10 ** -g["print_decimals"]
    x = np.array(ex["x"], float)
    w = np.array(ex["w_router"], float)
    k = ex["k"]
    s = O.router_logits(x, w)
    probs, sel, gates, counts, psum = O.route(s, k)
    T, E = s.shape
    assert sel.tolist() == ex["selected_experts"]
    np.testing.assert_allclose(gates, ex["selected_weights"], rtol=0, atol=1e-15)
    f, P, _ = O.aux(counts, psum, T, k)
    np.testing.assert_allclose(f, ex["token_fraction"], rtol=0, atol=0)
    np.testing.assert_allclose(P, ex["probability_mass"], rtol=0, atol=tol)
    kept = np.ones_like(sel, dtype=bool)
    y = O.combine_precomputed(np.array(ex["expert_outputs"], float), sel, kept, gates,
                              base=np.array(ex["shared_output"], float))
    np.testing.assert_allclose(y, ex["output"], rtol=0, atol=1e-12)


def test_router_page_example1_closed_form():
    # token scores are [1,0,1] and [0,1,1]: m = ((e+1)/(2(2e+1)), same, e/(2e+1))
    g = _golden("router_load_statistics_examples.json")["examples"][0]
    s = O.router_logits(np.array(g["x"], float), np.array(g["w_router"], float))
    _, _, _, counts, psum = O.route(s, 2)
    e = math.e
    m = [(e + 1) / (2 * (2 * e + 1)), (e + 1) / (2 * (2 * e + 1)), e / (2 * e + 1)]
    np.testing.assert_allclose(psum / 2, m, rtol=1e-15, atol=0)
    # example 2: softmax of [2, 1] = [sigma(1), sigma(-1)]
    g2 = _golden("router_load_statistics_examples.json")["examples"][1]
    s2 = O.router_logits(np.array(g2["x"], float), np.array(g2["w_router"], float))
    _, _, _, _, ps2 = O.route(s2, 1)
    np.testing.assert_allclose(ps2, [1 / (1 + math.exp(-1)), 1 / (1 + math.exp(1))], rtol=1e-15)


# --------------------------------------------------------------------------
# module-7 notebook pins
# --------------------------------------------------------------------------
def test_module7_capacity_fifo_case():
    g = _golden("module7_capacity_fifo.json")
    s = np.array(g["logits"])
    T, E = s.shape
    k = g["top_k"]
    _, sel, _, counts, _ = O.route(s, k)
    assert counts.tolist() == g["before_counts"]
    C = O.capacity(T, k, E, g["capacity_factor"])
    assert C == g["capacity_per_expert"]
    d = O.dispatch(sel, E, C)
    assert d["used"].tolist() == g["after_counts"]
    assert int((~d["kept"]).sum()) == g["dropped_assignments"]
    assert np.flatnonzero(d["drops"] == k).tolist() == g["fully_dropped_tokens"]
    assert (d["overflow"] == counts - d["used"]).all()


def test_module7_all_same_case():
    g = _golden("module7_capacity_fifo.json")["all_same_case"]
    s = np.array(g["logits"])
    T, E = s.shape
    _, sel, _, _, _ = O.route(s, g["top_k"])
    C = O.capacity(T, g["top_k"], E, g["capacity_factor"])
    assert C == 1
    d = O.dispatch(sel, E, C)
    assert d["kept"][:, 0].tolist() == g["accepted"]
    assert np.flatnonzero(d["drops"] == g["top_k"]).tolist() == g["fully_dropped_tokens"]


def test_module7_tie_and_extreme_logits():
    g = _golden("module7_router_checks.json")
    _, sel, _, _, _ = O.route(np.array([g["tie_case"]["logits"]]), g["tie_case"]["top_k"])
    assert sel[0].tolist() == g["tie_case"]["selected"]
    ex = g["extreme_case"]
    probs, sel, gates, _, _ = O.route(np.array([ex["logits"]]), ex["top_k"])
    assert sel[0].tolist() == ex["selected"]
    assert np.isfinite(probs).all() and np.isfinite(gates).all()
    # a two-way softmax of logits that differ by 1 is [sigma(1), sigma(-1)]
    np.testing.assert_allclose(gates[0], [1 / (1 + math.exp(-1)), 1 / (1 + math.exp(1))],
                               rtol=1e-15)


def test_module7_losses():
    g = _golden("module7_losses.json")
    s = np.array(g["aux_logits"])
    T, E = s.shape
    _, _, _, counts, psum = O.route(s, g["top_k"])
    _, _, aux = O.aux(counts, psum, T, g["top_k"], normalize_by_k=True)
    assert math.isclose(aux, g["switch_aux"], rel_tol=1e-12)
    assert math.isclose(O.z_loss(s), g["z_loss"], rel_tol=1e-12)
    z = np.array(g["z_square_before_mean_case"]["logits"])
    ln2 = math.log(2)
    assert math.isclose(O.z_loss(z), (ln2 ** 2 + (2 + ln2) ** 2) / 2, rel_tol=1e-12)


# --------------------------------------------------------------------------
# aux normalisation: uniform routing gives exactly 1 (numpy-layer page, section 3)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("E,k", [(8, 1), (8, 2), (16, 4)])
def test_aux_uniform_is_one(E, k):
    ver = _golden("numpy_layer_verification.json")
    T = E
    s = np.zeros((T, E))
    for t in range(T):
        for j in range(k):
            s[t, (t + j) % E] = 3.0  # each token prefers k experts; cyclic symmetry
    _, sel, _, counts, psum = O.route(s, k)
    assert (counts == k).all()
    f, P, aux = O.aux(counts, psum, T, k, normalize_by_k=True)
    assert abs(aux - ver["aux_uniform"]) < 1e-12
    assert math.isclose(f.sum(), k, rel_tol=1e-15)
    assert math.isclose(P.sum(), 1.0, rel_tol=1e-14)
    # the un-normalised (llm-atlas) form is k times larger
    _, _, aux5 = O.aux(counts, psum, T, k, normalize_by_k=False)
    assert math.isclose(aux5, k * aux, rel_tol=1e-14)


# --------------------------------------------------------------------------
# brute force against independent statements of the rules
# --------------------------------------------------------------------------
def _stable_rank(row, k):
    # the stable-sort statement: sort by (-score, index)
    return sorted(range(len(row)), key=lambda e: (-row[e], e))[:k]


@pytest.mark.parametrize("seed", range(6))
def test_topk_and_gates_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    T, E = 40, int(rng.integers(2, 9))
    k = int(rng.integers(1, E + 1))
    s = rng.integers(-3, 4, size=(T, E)).astype(float)  # many exact ties
    probs, sel, gates, counts, psum = O.route(s, k)
    for t in range(T):
        assert sel[t].tolist() == _stable_rank(s[t], k)
    # gate = p_sel / sum p_sel (the numpy-layer and llm-atlas form)
    psel = np.take_along_axis(probs, sel, axis=1)
    np.testing.assert_allclose(gates, psel / psel.sum(1, keepdims=True), rtol=1e-14, atol=0)
    np.testing.assert_allclose(gates.sum(1), 1.0, rtol=1e-15)
    np.testing.assert_allclose(probs.sum(1), 1.0, rtol=1e-15)
    assert counts.tolist() == np.bincount(sel.ravel(), minlength=E).tolist()
    np.testing.assert_allclose(psum, probs.sum(0), rtol=1e-15)
    # softmax values are invariant to a constant shift of a token's scores
    probs2, _, gates2, _, _ = O.route(s + 1000.0, k)
    np.testing.assert_allclose(probs2, probs, rtol=1e-12)
    np.testing.assert_allclose(gates2, gates, rtol=1e-12)


@pytest.mark.parametrize("seed", range(8))
def test_dispatch_equals_exclusive_cumsum(seed):
    # the dispatch/combine page computes a slot as the exclusive running count of
    # same-expert assignments; over the (t asc, j asc) stream it must equal the
    # greedy loop.
    rng = np.random.default_rng(200 + seed)
    T, E = int(rng.integers(1, 64)), int(rng.integers(1, 9))
    k = int(rng.integers(1, E + 1))
    sel = np.stack([rng.permutation(E)[:k] for _ in range(T)])
    C = int(rng.integers(0, 2 * T * k // E + 2))
    d = O.dispatch(sel, E, C)
    flat = sel.reshape(-1)
    onehot = np.eye(E, dtype=np.int64)[flat]
    pos = ((np.cumsum(onehot, axis=0) - onehot) * onehot).sum(1)
    keep = pos < C
    assert (d["kept"].reshape(-1) == keep).all()
    assert (d["slot"].reshape(-1) == np.where(keep, pos, -1)).all()
    cnt = np.bincount(flat, minlength=E)
    assert (d["used"] == np.minimum(cnt, C)).all()
    assert (d["overflow"] == cnt - np.minimum(cnt, C)).all()
    assert (d["drops"] == (~d["kept"]).sum(1)).all()
    # token_of_slot is the inverse map; each (e, c) holds at most one token
    tos = d["token_of_slot"]
    for e in range(E):
        for c in range(C):
            if c < d["used"][e]:
                t = tos[e, c]
                assert t >= 0 and any(sel[t, j] == e and d["slot"][t, j] == c for j in range(k))
            else:
                assert tos[e, c] == -1


def test_dispatch_duplicates_and_bad_index():
    # a repeated expert inside a token takes two slots in order; an index outside
    # [0, E) is reported and not placed
    d = O.dispatch(np.array([[0, 0], [0, 1]]), 2, 4)
    assert d["slot"].tolist() == [[0, 1], [2, 0]]
    d = O.dispatch(np.array([[0, 5], [-1, 1]]), 2, 4)
    assert d["bad_index"]
    assert d["kept"].tolist() == [[True, False], [False, True]]


# --------------------------------------------------------------------------
# sparse == dense (T,E,C) formulation; edge cases (numpy-layer page, section 3)
# --------------------------------------------------------------------------
def _tiny_linear_case(seed, T=12, D=5, E=4, k=2, cf=0.75, residual=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, D))
    s = rng.standard_normal((T, E))
    W = rng.standard_normal((E, D, D)) * 0.3
    C = O.capacity(T, k, E, cf)
    return x, s, W, C


@pytest.mark.parametrize("seed", range(4))
def test_sparse_equals_dense_tensors(seed):
    x, s, W, C = _tiny_linear_case(300 + seed)
    T, E = s.shape
    k = 2
    out = O.forward("linear", x, s, k, C, {"w1": W}, base_kind="input")
    y_dense, mask, comb = O.dense_linear(x, out["selected"], out["slot"], out["kept"],
                                         out["gates"], W, C, use_residual=True)
    np.testing.assert_allclose(out["y"], y_dense, rtol=1e-13, atol=1e-13)
    # dispatch is one-hot per kept assignment; each (e, c) holds at most one token
    assert mask.sum() == out["kept"].sum()
    assert (mask.sum(0) <= 1).all()
    # dispatch/combine are zero on dropped assignments
    for t in range(T):
        for j in range(k):
            e = out["selected"][t, j]
            if not out["kept"][t, j]:
                assert comb[t, e].sum() == 0 and mask[t, e].sum() == 0
            else:
                assert comb[t, e, out["slot"][t, j]] == out["gates"][t, j]
    # fully dropped tokens pass through the residual unmodified
    full = np.flatnonzero(out["drops"] == k)
    np.testing.assert_array_equal(out["y"][full], x[full])


def test_edge_cases():
    x, s, W, _ = _tiny_linear_case(400, T=10, D=4, E=4)
    # capacity 0: everything dropped, output exactly x
    out = O.forward("linear", x, s, 2, 0, {"w1": W}, base_kind="input")
    assert not out["kept"].any()
    np.testing.assert_array_equal(out["y"], x)
    # k == E: every expert selected once per token, gates = full softmax
    out = O.forward("linear", x, s, 4, 10, {"w1": W}, base_kind="input")
    np.testing.assert_allclose(np.sort(out["selected"], 1), np.tile(np.arange(4), (10, 1)))
    np.testing.assert_allclose(out["gates"], np.take_along_axis(out["probs"], out["selected"], 1),
                               rtol=1e-14)
    # single expert, k=1: gate 1, output = x + x @ W0 for every token
    out = O.forward("linear", x, s[:, :1], 1, 10, {"w1": W[:1]}, base_kind="input")
    np.testing.assert_allclose(out["y"], x + x @ W[0], rtol=1e-13, atol=1e-13)
    # single token
    out = O.forward("linear", x[:1], s[:1], 2, 1, {"w1": W}, base_kind="input")
    assert out["kept"].all()
    # no residual: zero base, dropped rows are all zero
    out = O.forward("linear", x, s, 2, 2, {"w1": W}, base_kind="zero")
    full = np.flatnonzero(out["drops"] == 2)
    assert len(full) > 0
    assert (out["y"][full] == 0).all()


# --------------------------------------------------------------------------
# expert functions against the libraries the pages define them with
# --------------------------------------------------------------------------
def test_gelu_mlp_expert_matches_torch_modules():
    # the llm-atlas expert is fc2(gelu(fc1(x))) with nn.Linear layers and exact GELU
    rng = np.random.default_rng(7)
    E, D, F, N, T = 3, 6, 10, 6, 9
    x = rng.standard_normal((T, D))
    W1 = rng.standard_normal((E, D, F)) * 0.5
    b1 = rng.standard_normal((E, F)) * 0.5
    W2 = rng.standard_normal((E, F, N)) * 0.5
    b2 = rng.standard_normal((E, N)) * 0.5
    experts = rng.integers(0, E, T)
    got = O.expert_rows("gelu_mlp", x, np.arange(T), experts, dict(w1=W1, b1=b1, w2=W2, b2=b2))
    xt = torch.tensor(x)
    for i in range(T):
        e = experts[i]
        h = torch.nn.functional.gelu(torch.nn.functional.linear(
            xt[i], torch.tensor(W1[e]).T, torch.tensor(b1[e])))
        ref = torch.nn.functional.linear(h, torch.tensor(W2[e]).T, torch.tensor(b2[e]))
        np.testing.assert_allclose(got[i], ref.numpy(), rtol=1e-13, atol=1e-14)


def test_swiglu_expert_closed_form_and_torch():
    # 1-d case: x=1, gate weight a=ln 3 (sigmoid(ln 3) = 3/4), up b, down c
    a, b, c = math.log(3.0), 1.5, -2.0
    out = O.expert_rows("swiglu", np.array([[1.0]]), [0], [0],
                        dict(w1=np.array([[[a]]]), w3=np.array([[[b]]]), w2=np.array([[[c]]])))
    assert math.isclose(out[0, 0], a * 0.75 * b * c, rel_tol=1e-15)
    # larger case against torch's SiLU
    rng = np.random.default_rng(8)
    E, D, F, T = 2, 7, 5, 6
    x = rng.standard_normal((T, D))
    Wg, Wu = rng.standard_normal((E, D, F)), rng.standard_normal((E, D, F))
    Wd = rng.standard_normal((E, F, D))
    experts = rng.integers(0, E, T)
    got = O.expert_rows("swiglu", x, np.arange(T), experts, dict(w1=Wg, w3=Wu, w2=Wd))
    for i in range(T):
        e = experts[i]
        xt = torch.tensor(x[i])
        h = torch.nn.functional.silu(xt @ torch.tensor(Wg[e])) * (xt @ torch.tensor(Wu[e]))
        np.testing.assert_allclose(got[i], (h @ torch.tensor(Wd[e])).numpy(), rtol=1e-13,
                                   atol=1e-13)


def test_linear_expert_and_router_match_matmul():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((5, 4))
    W = rng.standard_normal((3, 4, 6))
    got = O.expert_rows("linear", x, np.arange(5), [0, 1, 2, 1, 0], dict(w1=W))
    for i, e in enumerate([0, 1, 2, 1, 0]):
        np.testing.assert_allclose(got[i], np.matmul(x[i], W[e]), rtol=1e-14, atol=1e-14)
    wr = rng.standard_normal((4, 3))
    b = rng.standard_normal(3)
    np.testing.assert_allclose(O.router_logits(x, wr, b), np.matmul(x, wr) + b, rtol=1e-14,
                               atol=1e-14)


# --------------------------------------------------------------------------
# backward: central finite differences (numpy-layer page, section 3)
# --------------------------------------------------------------------------
def _loss(x, s, W, dy, sel0, kept, k, aux_coef, counts0, residual):
    probs, sel, gates, _, psum = O.route(s, k)
    assert (sel == sel0).all(), "perturbation changed the top-k decision"
    y = O.layer_rows("linear", x, sel, kept, gates, {"w1": W},
                     base_kind="input" if residual else "zero")
    T = x.shape[0]
    _, _, aux = O.aux(counts0, psum, T, k, normalize_by_k=True)
    return float((dy * y).sum() + aux_coef * aux)


@pytest.mark.parametrize("aux_coef,residual", [(0.0, True), (0.37, True), (0.0, False)])
def test_backward_finite_differences(aux_coef, residual):
    ver = _golden("numpy_layer_verification.json")
    rng = np.random.default_rng(11)
    T, D, E, k = 7, 4, 4, 2
    x = rng.standard_normal((T, D))
    s = rng.standard_normal((T, E))
    W = rng.standard_normal((E, D, D)) * 0.5
    dy = rng.standard_normal((T, D))
    C = 3  # forces drops
    out = O.forward("linear", x, s, k, C, {"w1": W}, base_kind="input" if residual else "zero")
    sel, kept, counts = out["selected"], out["kept"], out["counts"]
    assert (~kept).any()
    dx, dW, dl, dg = O.backward_linear(dy, x, s, sel, kept, out["gates"], W,
                                       use_residual=residual, aux_coef=aux_coef,
                                       normalize_by_k=True, counts=counts)
    h = 1e-6

    def fd(arr, name):
        g = np.zeros_like(arr)
        it = np.nditer(arr, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            a0 = arr[i]
            arr[i] = a0 + h
            lp = _loss(x, s, W, dy, sel, kept, k, aux_coef, counts, residual)
            arr[i] = a0 - h
            lm = _loss(x, s, W, dy, sel, kept, k, aux_coef, counts, residual)
            arr[i] = a0
            g[i] = (lp - lm) / (2 * h)
        return g

    bound = 10 * max(ver["backward_vs_finite_difference_max_err"].values())
    assert np.abs(fd(x, "x") - dx).max() < bound
    assert np.abs(fd(s, "s") - dl).max() < bound
    assert np.abs(fd(W, "W") - dW).max() < bound
    # dgate equals dy . expert output on kept assignments, 0 on dropped
    assert (dg[~kept] == 0).all()
    # a dropped-but-selected expert still receives a gradient through the
    # renormalisation denominator
    t, j = np.argwhere(~kept)[0]
    if kept[t].any():
        assert dl[t, sel[t, j]] != 0.0


def test_backward_top1_logit_gradient_is_zero():
    # k = 1: the renormalised gate is identically 1, so the logits get no gradient
    rng = np.random.default_rng(12)
    T, D, E = 6, 3, 4
    x, s = rng.standard_normal((T, D)), rng.standard_normal((T, E))
    W, dy = rng.standard_normal((E, D, D)), rng.standard_normal((T, D))
    out = O.forward("linear", x, s, 1, 6, {"w1": W}, base_kind="input")
    _, _, dl, _ = O.backward_linear(dy, x, s, out["selected"], out["kept"], out["gates"], W)
    assert np.abs(dl).max() < 1e-12


def _loss_swiglu(x, s, w, dy, sel0, kept, k, aux_coef, counts0, residual):
    probs, sel, gates, _, psum = O.route(s, k)
    assert (sel == sel0).all(), "perturbation changed the top-k decision"
    y = O.layer_rows("swiglu", x, sel, kept, gates, w, base_kind="input" if residual else "zero")
    _, _, aux = O.aux(counts0, psum, x.shape[0], k, normalize_by_k=True)
    return float((dy * y).sum() + aux_coef * aux)


@pytest.mark.parametrize("aux_coef,residual", [(0.0, False), (0.29, True)])
def test_backward_swiglu_finite_differences(aux_coef, residual):
    # The module-7 SwiGLU expert under the numpy-layer page's backward rules:
    # every analytic gradient against central differences of y . dy (+ aux).
    ver = _golden("numpy_layer_verification.json")
    rng = np.random.default_rng(21)
    T, D, F, E, k = 7, 4, 3, 4, 2
    x = rng.standard_normal((T, D))
    s = rng.standard_normal((T, E))
    w = {"w1": rng.standard_normal((E, D, F)) * 0.7, "w3": rng.standard_normal((E, D, F)) * 0.7,
         "w2": rng.standard_normal((E, F, D)) * 0.7}
    dy = rng.standard_normal((T, D))
    C = 3  # forces drops
    out = O.forward("swiglu", x, s, k, C, w, base_kind="input" if residual else "zero")
    sel, kept, counts = out["selected"], out["kept"], out["counts"]
    assert (~kept).any()
    dx, dWg, dWu, dWd, dl, dg = O.backward_swiglu(dy, x, s, sel, kept, out["gates"], w["w1"], w["w3"], w["w2"],
                                                  use_residual=residual, aux_coef=aux_coef, counts=counts)
    h = 1e-6

    def fd(arr):
        g = np.zeros_like(arr)
        it = np.nditer(arr, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            a0 = arr[i]
            arr[i] = a0 + h
            lp = _loss_swiglu(x, s, w, dy, sel, kept, k, aux_coef, counts, residual)
            arr[i] = a0 - h
            lm = _loss_swiglu(x, s, w, dy, sel, kept, k, aux_coef, counts, residual)
            arr[i] = a0
            g[i] = (lp - lm) / (2 * h)
        return g

    bound = 10 * max(ver["backward_vs_finite_difference_max_err"].values())
    assert np.abs(fd(x) - dx).max() < bound
    assert np.abs(fd(s) - dl).max() < bound
    assert np.abs(fd(w["w1"]) - dWg).max() < bound
    assert np.abs(fd(w["w3"]) - dWu).max() < bound
    assert np.abs(fd(w["w2"]) - dWd).max() < bound
    assert (dg[~kept] == 0).all()
    # dgate is dy . (ungated expert output) on kept assignments
    t, j = np.argwhere(kept)[0]
    o = O.expert_rows("swiglu", x, [t], [sel[t, j]], w)[0]
    assert math.isclose(dg[t, j], float(dy[t] @ o), rel_tol=1e-12)


def _loss_gelu(x, s, w, dy, sel0, kept, k, aux_coef, counts0, residual):
    probs, sel, gates, _, psum = O.route(s, k)
    assert (sel == sel0).all(), "perturbation changed the top-k decision"
    y = O.layer_rows("gelu_mlp", x, sel, kept, gates, w, base_kind="input" if residual else "zero")
    _, _, aux = O.aux(counts0, psum, x.shape[0], k, normalize_by_k=True)
    return float((dy * y).sum() + aux_coef * aux)


@pytest.mark.parametrize("aux_coef,residual", [(0.0, True), (0.41, False)])
def test_backward_gelu_finite_differences(aux_coef, residual):
    # The GELU-MLP expert (fc2(gelu(fc1 x)), biases on both layers) under the
    # numpy-layer page's backward rules, against central differences of y . dy (+ aux).
    ver = _golden("numpy_layer_verification.json")
    rng = np.random.default_rng(31)
    T, D, F, E, k = 7, 4, 5, 4, 2
    x = rng.standard_normal((T, D))
    s = rng.standard_normal((T, E))
    w = {"w1": rng.standard_normal((E, D, F)) * 0.8, "b1": rng.standard_normal((E, F)) * 0.5,
         "w2": rng.standard_normal((E, F, D)) * 0.8, "b2": rng.standard_normal((E, D)) * 0.5}
    dy = rng.standard_normal((T, D))
    C = 3  # forces drops
    out = O.forward("gelu_mlp", x, s, k, C, w, base_kind="input" if residual else "zero")
    sel, kept, counts = out["selected"], out["kept"], out["counts"]
    assert (~kept).any()
    dx, dW1, db1, dW2, db2, dl, dg = O.backward_gelu(dy, x, s, sel, kept, out["gates"], w["w1"], w["b1"],
                                                     w["w2"], w["b2"], use_residual=residual,
                                                     aux_coef=aux_coef, counts=counts)
    h = 1e-6

    def fd(arr):
        g = np.zeros_like(arr)
        it = np.nditer(arr, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            a0 = arr[i]
            arr[i] = a0 + h
            lp = _loss_gelu(x, s, w, dy, sel, kept, k, aux_coef, counts, residual)
            arr[i] = a0 - h
            lm = _loss_gelu(x, s, w, dy, sel, kept, k, aux_coef, counts, residual)
            arr[i] = a0
            g[i] = (lp - lm) / (2 * h)
        return g

    bound = 10 * max(ver["backward_vs_finite_difference_max_err"].values())
    assert np.abs(fd(x) - dx).max() < bound
    assert np.abs(fd(s) - dl).max() < bound
    assert np.abs(fd(w["w1"]) - dW1).max() < bound
    assert np.abs(fd(w["b1"]) - db1).max() < bound
    assert np.abs(fd(w["w2"]) - dW2).max() < bound
    assert np.abs(fd(w["b2"]) - db2).max() < bound
    assert (dg[~kept] == 0).all()
    t, j = np.argwhere(kept)[0]
    o = O.expert_rows("gelu_mlp", x, [t], [sel[t, j]], w)[0]
    assert math.isclose(dg[t, j], float(dy[t] @ o), rel_tol=1e-12)


def test_backward_gelu_bias_gradients_closed_form():
    # One expert, top-1, D = F = N = 1, x = 0: z = b1, so
    #   db2 = sum_t dy_t,  db1 = W2 * gelu'(b1) * sum_t dy_t,  dW1 = 0,
    # with gelu'(z) = Phi(z) + z phi(z) from scipy's normal distribution.
    from scipy.stats import norm
    T = 5
    x = np.zeros((T, 1))
    s = np.zeros((T, 1))
    dy = np.arange(1.0, T + 1.0).reshape(T, 1)
    b1v, w2v = 0.7, -1.3
    w = {"w1": np.full((1, 1, 1), 2.0), "b1": np.full((1, 1), b1v), "w2": np.full((1, 1, 1), w2v),
         "b2": np.full((1, 1), 0.25)}
    out = O.forward("gelu_mlp", x, s, 1, T, w)
    dx, dW1, db1, dW2, db2, dl, dg = O.backward_gelu(dy, x, s, out["selected"], out["kept"], out["gates"],
                                                     w["w1"], w["b1"], w["w2"], w["b2"])
    S = float(dy.sum())
    gprime = norm.cdf(b1v) + b1v * norm.pdf(b1v)
    assert math.isclose(float(db2[0, 0]), S, rel_tol=1e-14)
    assert math.isclose(float(db1[0, 0]), w2v * gprime * S, rel_tol=1e-13)
    assert float(dW1[0, 0, 0]) == 0.0
    # dW2 = gelu(b1) * sum dy with gelu(z) = z Phi(z)
    assert math.isclose(float(dW2[0, 0, 0]), b1v * norm.cdf(b1v) * S, rel_tol=1e-13)
    # dx_t = dy_t * W2 * gelu'(b1) * W1
    np.testing.assert_allclose(dx[:, 0], dy[:, 0] * w2v * gprime * 2.0, rtol=1e-13)
    assert np.abs(dl).max() == 0.0


def test_backward_swiglu_down_gradient_closed_form_and_top1():
    # With one hidden unit (F = 1) the down-projection gradient has a closed
    # form: dWd_e = sum over kept tokens of e of g * silu(a) * b * dy, with
    # a = x . wg_e and b = x . wu_e, written out here by hand.
    rng = np.random.default_rng(22)
    T, D, E, k = 5, 3, 2, 1
    x = rng.standard_normal((T, D))
    s = rng.standard_normal((T, E))
    w = {"w1": rng.standard_normal((E, D, 1)), "w3": rng.standard_normal((E, D, 1)),
         "w2": rng.standard_normal((E, 1, D))}
    dy = rng.standard_normal((T, D))
    out = O.forward("swiglu", x, s, k, T, w)
    sel, kept, gates = out["selected"], out["kept"], out["gates"]
    _, _, _, dWd, dl, _ = O.backward_swiglu(dy, x, s, sel, kept, gates, w["w1"], w["w3"], w["w2"])
    want = np.zeros((E, 1, D))
    for t in range(T):
        e = sel[t, 0]
        a = x[t] @ w["w1"][e][:, 0]
        b = x[t] @ w["w3"][e][:, 0]
        hval = a / (1 + math.exp(-a)) * b
        want[e, 0] += gates[t, 0] * hval * dy[t]
    np.testing.assert_allclose(dWd, want, rtol=1e-12, atol=1e-14)
    # k = 1: the renormalised gate is identically 1, so the logits get no gradient
    assert np.abs(dl).max() < 1e-12


def test_router_and_expert_backward_compose_to_the_full_gradient():
    # Module 7's layer end to end: s = x W_r + b, SwiGLU experts, y = x + sum gate * out.
    # With the routing decisions fixed, dL/dx = expert path + residual + dlogits W_r^T,
    # dL/dW_r = x^T dlogits, dL/db = sum_t dlogits; checked by central differences.
    ver = _golden("numpy_layer_verification.json")
    rng = np.random.default_rng(23)
    T, D, F, E, k = 6, 4, 3, 4, 2
    x = rng.standard_normal((T, D))
    wr = rng.standard_normal((D, E))
    b = rng.standard_normal(E) * 0.3
    w = {"w1": rng.standard_normal((E, D, F)) * 0.7, "w3": rng.standard_normal((E, D, F)) * 0.7,
         "w2": rng.standard_normal((E, F, D)) * 0.7}
    dy = rng.standard_normal((T, D))
    C = 3
    s0 = O.router_logits(x, wr, b)
    out = O.forward("swiglu", x, s0, k, C, w, base_kind="input")
    sel0, kept = out["selected"], out["kept"]

    def loss():
        s = O.router_logits(x, wr, b)
        _, sel, gates, _, _ = O.route(s, k)
        assert (sel == sel0).all()
        y = O.layer_rows("swiglu", x, sel, kept, gates, w, base_kind="input")
        return float((dy * y).sum())

    dxe, _, _, _, dl, _ = O.backward_swiglu(dy, x, s0, sel0, kept, out["gates"], w["w1"], w["w3"], w["w2"],
                                            use_residual=True)
    dxr, dwr, dbr = O.router_backward(x, wr, dl)
    h = 1e-6

    def fd(arr):
        g = np.zeros_like(arr)
        it = np.nditer(arr, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            a0 = arr[i]
            arr[i] = a0 + h
            lp = loss()
            arr[i] = a0 - h
            lm = loss()
            arr[i] = a0
            g[i] = (lp - lm) / (2 * h)
        return g

    bound = 10 * max(ver["backward_vs_finite_difference_max_err"].values())
    assert np.abs(fd(x) - (dxe + dxr)).max() < bound
    assert np.abs(fd(wr) - dwr).max() < bound
    assert np.abs(fd(b) - dbr).max() < bound


# --------------------------------------------------------------------------
# negative cases (module-7 negative tests)
# --------------------------------------------------------------------------
def test_rejects_invalid_inputs():
    with pytest.raises(ValueError):
        O.route(np.array([[1.0, 2.0]]), 3)
    with pytest.raises(ValueError):
        O.route(np.array([[1.0, np.nan]]), 1)
    with pytest.raises(ValueError):
        O.capacity(8, 2, 4, 0.0)


def test_golden_files_cite_their_source():
    for name in os.listdir(GOLDEN):
        if name.endswith(".json"):
            assert "source" in _golden(name), name


# --------------------------------------------------------------------------
# module-7 router variants: sigmoid scoring, selection-only bias, survivor renormalisation
# --------------------------------------------------------------------------
def test_module7_sigmoid_router_pins():
    g = _golden("module7_router_variants.json")
    tol = g["check_tolerance"]
    s = np.array([g["logits"]])
    clean, sel, gates, counts = O.route_variant(s, g["top_k"], "sigmoid")
    np.testing.assert_allclose(clean[0], g["scores"], rtol=0, atol=1e-15)
    assert sel[0].tolist() == g["selected"]
    np.testing.assert_allclose(gates[0], g["gates"], rtol=0, atol=tol)
    _, selb, gatesb, _ = O.route_variant(s, g["top_k"], "sigmoid", selection_bias=g["bias"])
    assert selb[0].tolist() == g["selected_with_bias"]
    np.testing.assert_allclose(gatesb[0], g["gates_with_bias"], rtol=0, atol=tol)
    # the bias moves the selection only: gates are the selected clean sigmoids, renormalised
    sig = np.array(g["scores"])[selb[0]]
    np.testing.assert_allclose(gatesb[0], sig / sig.sum(), rtol=1e-14)


def test_module7_sigmoid_extreme_logits_and_softmax_variant():
    # sigmoid gates stay finite where every sigmoid underflows; two logits 1 apart -> [sigma(1), sigma(-1)]
    _, sel, gates, _ = O.route_variant(np.array([[-1002.0, -1000.0, -1001.0]]), 2, "sigmoid")
    assert sel[0].tolist() == [1, 2]
    np.testing.assert_allclose(gates[0], [1 / (1 + math.exp(-1)), 1 / (1 + math.exp(1))], rtol=1e-12)
    # softmax scoring without a bias is the plain router
    rng = np.random.default_rng(21)
    s = rng.integers(-3, 4, size=(30, 6)).astype(float)
    clean, sel, gates, counts = O.route_variant(s, 3, "softmax")
    probs, sel0, gates0, counts0, _ = O.route(s, 3)
    np.testing.assert_array_equal(sel, sel0)
    np.testing.assert_allclose(gates, gates0, rtol=1e-15)
    np.testing.assert_allclose(clean, probs, rtol=1e-15)
    assert (counts == counts0).all()
    # softmax scoring with a selection bias ranks p + b, gates still come from the logits
    b = np.linspace(0.0, 0.5, 6)
    _, selb, gatesb, _ = O.route_variant(s, 3, "softmax", selection_bias=b)
    for t in range(30):
        key = probs[t] + b
        assert selb[t].tolist() == sorted(range(6), key=lambda e: (-key[e], e))[:3]
        z = s[t, selb[t]]
        np.testing.assert_allclose(gatesb[t], np.exp(z - z.max()) / np.exp(z - z.max()).sum(), rtol=1e-14)


def test_module7_survivor_renormalisation():
    g = _golden("module7_capacity_fifo.json")
    s = np.array(g["logits"])
    T, E = s.shape
    _, sel, gates, _, _ = O.route(s, g["top_k"])
    d = O.dispatch(sel, E, O.capacity(T, g["top_k"], E, g["capacity_factor"]))
    r = O.renormalize_kept(gates, d["kept"])
    # the capacity cell checks that the surviving weights of every token sum to one
    np.testing.assert_allclose(r.sum(1), 1.0, rtol=1e-15)
    assert (r[~d["kept"]] == 0).all()
    # all-same case: fully dropped tokens keep all-zero weights, no division by zero
    a = _golden("module7_capacity_fifo.json")["all_same_case"]
    s2 = np.array(a["logits"])
    _, sel2, gates2, _, _ = O.route(s2, a["top_k"])
    d2 = O.dispatch(sel2, 2, O.capacity(4, a["top_k"], 2, a["capacity_factor"]))
    r2 = O.renormalize_kept(gates2, d2["kept"])
    assert (r2[1:] == 0).all() and r2[0, 0] == 1.0


# --------------------------------------------------------------------------
# expert-major combine against the Dispatch page's one-hot contraction (step 6),
# and the Module 7 single-expert / shared-expert invariants of EducationalMoE
# --------------------------------------------------------------------------
def _one_hot_tec(selected, slot, kept, E, C):
    """The Dispatch page's (T, E, C) address tensor: 1 where token t sits in expert e at slot c."""
    T, k = selected.shape
    disp = np.zeros((T, E, C))
    for t in range(T):
        for j in range(k):
            if kept[t, j]:
                disp[t, selected[t, j], slot[t, j]] = 1.0
    return disp


@pytest.mark.parametrize("seed", range(3))
@pytest.mark.parametrize("base", ["zero", "input", "tensor"])
def test_combine_slots_equals_dispatch_page_einsum(seed, base):
    rng = np.random.default_rng(900 + seed)
    T, E, k, N = 23, 5, 2, 6
    C = O.capacity(T, k, E, 0.7)  # tight capacity: drops occur
    x = rng.standard_normal((T, N))
    s = rng.standard_normal((T, E))
    _, sel, gates, _, _ = O.route(s, k)
    d = O.dispatch(sel, E, C)
    assert (~d["kept"]).any() and d["kept"].any()
    disp = _one_hot_tec(sel, d["slot"], d["kept"], E, C)
    # the page's gather: expert_inputs = einsum("tec,td->ecd", dispatch, x) equals the rows that
    # the inverse map names; empty slots are all zero
    xbuf = np.einsum("tec,td->ecd", disp, x)
    for e in range(E):
        for c in range(C):
            t = d["token_of_slot"][e, c]
            np.testing.assert_array_equal(xbuf[e, c], x[t] if t >= 0 else np.zeros(N))
    # expert outputs, with the empty slots holding values that must never be read
    ybuf = rng.standard_normal((E, C, N))
    ybuf[d["token_of_slot"] < 0] = 1e6
    comb = disp * np.einsum("tj,tje->tje", gates, np.eye(E)[sel]).sum(1)[:, :, None]
    want = np.einsum("tec,ecd->td", comb, ybuf)
    base_t = {"zero": None, "input": x, "tensor": rng.standard_normal((T, N))}[base]
    if base_t is not None:
        want = want + base_t
    got = O.combine_slots(ybuf, sel, d["slot"], d["kept"], gates, base=base_t)
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-13)
    # dropped-everywhere tokens get exactly the base row (the page: all-zero dispatch row)
    full = np.flatnonzero(d["drops"] == k)
    for t in full:
        np.testing.assert_array_equal(got[t], np.zeros(N) if base_t is None else base_t[t])


def test_combine_slots_hand_worked_two_tokens():
    # T=2, E=2, k=2, C=1. Token 0 ranks [0, 1] and takes slot 0 of both experts; token 1 ranks
    # [1, 0] and finds both experts full, so it keeps only its base row.
    s = np.array([[1.0, 0.0], [0.0, 1.0]])
    _, sel, gates, _, _ = O.route(s, 2)
    d = O.dispatch(sel, 2, 1)
    assert sel.tolist() == [[0, 1], [1, 0]]
    assert d["kept"].tolist() == [[True, True], [False, False]]
    ybuf = np.array([[[2.0, -1.0]], [[4.0, 3.0]]])  # (E=2, C=1, N=2)
    base = np.array([[0.5, 0.25], [-7.0, 9.0]])
    g0 = math.e / (1.0 + math.e)  # softmax([1, 0])[0]
    want0 = base[0] + g0 * np.array([2.0, -1.0]) + (1.0 - g0) * np.array([4.0, 3.0])
    got = O.combine_slots(ybuf, sel, d["slot"], d["kept"], gates, base=base)
    np.testing.assert_allclose(got[0], want0, rtol=1e-15)
    np.testing.assert_array_equal(got[1], base[1])


def test_combine_slots_identity_expert_equals_layer():
    # with the identity as every expert, expert-major combine of the dispatched rows equals the
    # token-major layer sum  base + sum_kept gate * x_t
    rng = np.random.default_rng(31)
    T, E, k, D = 17, 4, 2, 5
    x = rng.standard_normal((T, D))
    _, sel, gates, _, _ = O.route(rng.standard_normal((T, E)), k)
    C = O.capacity(T, k, E, 0.8)
    d = O.dispatch(sel, E, C)
    xbuf = np.zeros((E, C, D))
    for e in range(E):
        for c in range(C):
            if d["token_of_slot"][e, c] >= 0:
                xbuf[e, c] = x[d["token_of_slot"][e, c]]
    eye = np.tile(np.eye(D), (E, 1, 1))
    want = O.layer_rows("linear", x, sel, d["kept"], gates, {"w1": eye}, base_kind="input")
    got = O.combine_slots(xbuf, sel, d["slot"], d["kept"], gates, base=x)
    np.testing.assert_allclose(got, want, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(want, x * (1.0 + (gates * d["kept"]).sum(1))[:, None], rtol=1e-14)


def _swiglu_np(x, g, u, dn):
    """Module 7 swiglu_expert written out: (a * sigmoid(a) * b) @ down with a = x@g, b = x@u."""
    a, b = x @ g, x @ u
    return (a / (1.0 + np.exp(-a)) * b) @ dn


def test_module7_single_expert_and_shared_expert_invariants():
    # The invariant cell after EducationalMoE: one routed expert with k=1 is the dense SwiGLU
    # expert (atol 1e-12 as on the page); an always-on shared expert adds its own output.
    rng = np.random.default_rng(60)
    H, I, T = 8, 12, 16
    x = rng.standard_normal((T, H))
    router_w = rng.standard_normal((H, 1)) / math.sqrt(H)
    gate = rng.standard_normal((1, H, I)) / math.sqrt(H)
    up = rng.standard_normal((1, H, I)) / math.sqrt(H)
    down = rng.standard_normal((1, I, H)) / math.sqrt(I)
    w = {"w1": gate, "w3": up, "w2": down}
    s = O.router_logits(x, router_w)
    out = O.forward("swiglu", x, s, 1, T, w, base_kind="zero")
    dense = _swiglu_np(x, gate[0], up[0], down[0])
    np.testing.assert_allclose(out["y"], dense, rtol=0, atol=1e-12)
    sg = rng.standard_normal((1, H, I)) / math.sqrt(H)
    su = rng.standard_normal((1, H, I)) / math.sqrt(H)
    sd = rng.standard_normal((1, I, H)) / math.sqrt(I)
    shared = _swiglu_np(x, sg[0], su[0], sd[0])
    y = O.layer_rows("swiglu", x, out["selected"], out["kept"], out["gates"], w, base_kind="tensor",
                     base=shared)
    np.testing.assert_allclose(y, dense + shared, rtol=0, atol=1e-12)
    # a subset of tokens in scrambled order reads each token's own base row
    toks = rng.permutation(T)[:7]
    ys = O.layer_rows("swiglu", x, out["selected"], out["kept"], out["gates"], w, base_kind="tensor",
                      base=shared, tokens=toks)
    np.testing.assert_allclose(ys, (dense + shared)[toks], rtol=0, atol=1e-12)
    # the shared expert computed by the oracle's own expert path is the same function
    sh = O.expert_rows("swiglu", x, np.arange(T), np.zeros(T, np.int64), {"w1": sg, "w3": su, "w2": sd})
    np.testing.assert_allclose(sh, shared, rtol=0, atol=1e-12)
    # with drops (capacity 5 of 16 tokens), dropped tokens keep exactly the shared row
    d = O.dispatch(out["selected"], 1, 5)
    yd = O.layer_rows("swiglu", x, out["selected"], d["kept"], out["gates"], w, base_kind="tensor",
                      base=shared)
    dropped = np.flatnonzero(~d["kept"][:, 0])
    assert len(dropped) == T - 5
    np.testing.assert_array_equal(yd[dropped], shared[dropped])
    np.testing.assert_allclose(yd[:5], (dense + shared)[:5], rtol=0, atol=1e-12)

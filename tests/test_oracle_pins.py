"""Pins of the fp64 CPU oracle against facts other than itself.

Every stage of the oracle is checked here against closed forms, library
special cases, invariants or brute force on tiny inputs, chosen so that a
plausible mistake (a dropped term, a wrong sign or index, a transposed
operand, a missing rounding point) fails at least one test. No GPU needed.
"""
import math

import numpy as np
import pytest
from scipy.special import expit, softmax

import oracle
import synth

RNG = np.random.default_rng(12345)


def bf(bits):
    return synth.bf16_bits_to_f32(np.asarray(bits, dtype=np.uint16)).astype(np.float64)


def to_bits(v):
    return synth.f32_to_bf16_bits(np.asarray(v, dtype=np.float32))


def rand_bf16(shape, scale=1.0):
    return to_bits(RNG.standard_normal(shape) * scale)


# ---- bf16 rounding ----------------------------------------------------------------

def test_bf16_round_ties_to_even():
    # 1 + 2^-8 is the midpoint between 1 and 1 + 2^-7: ties go to the even 1.0.
    assert oracle.bf16_round(1.0 + 2.0 ** -8) == 1.0
    # 1 + 3*2^-8 is the midpoint between 1 + 2^-7 (odd) and 1 + 2^-6 (even).
    assert oracle.bf16_round(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6
    assert oracle.bf16_round(-(1.0 + 2.0 ** -8)) == -1.0
    # just above the midpoint rounds up
    assert oracle.bf16_round(1.0 + 2.0 ** -8 + 2.0 ** -30) == 1.0 + 2.0 ** -7
    assert oracle.bf16_round(0.0) == 0.0
    assert math.isinf(oracle.bf16_round(3.5e38))


def test_bf16_round_matches_integer_rne_on_fp32_values():
    # For fp32-representable inputs the fp64 rounding must agree with the
    # classic integer round-to-nearest-even on the fp32 bit pattern.
    v = (RNG.standard_normal(20000) * np.exp(RNG.uniform(-20, 20, 20000))).astype(np.float32)
    ref = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(v))
    got = np.array([oracle.bf16_round(float(t)) for t in v])
    assert np.array_equal(got, ref.astype(np.float64))


def test_bf16_round_is_nearest():
    for t in RNG.standard_normal(2000) * 10:
        r = oracle.bf16_round(float(t))
        b = int(to_bits(np.array([r]))[0])
        assert synth.bf16_bits_to_f32(np.array([b], np.uint16))[0] == r  # r is a bf16 value
        up = float(synth.bf16_bits_to_f32(np.array([b + 1], np.uint16))[0])
        dn = float(synth.bf16_bits_to_f32(np.array([b - 1], np.uint16))[0])
        assert abs(t - r) <= abs(t - up) and abs(t - r) <= abs(t - dn)


# ---- top-k --------------------------------------------------------------------------

@pytest.mark.parametrize("E,k", [(1, 1), (5, 2), (16, 4), (64, 4), (64, 64), (200, 16)])
def test_topk_matches_full_stable_sort(E, k):
    for trial in range(30):
        if trial % 2 == 0:
            v = RNG.integers(-3, 4, E).astype(np.float64)   # many planted ties
        else:
            v = RNG.standard_normal(E)
        brute = sorted(range(E), key=lambda e: (-v[e], e))[:k]
        assert list(oracle.topk(v, k)) == brute


def test_topk_all_equal_picks_lowest_indices():
    assert list(oracle.topk(np.zeros(10), 3)) == [0, 1, 2]


def test_topk_rejects_nonfinite():
    v = np.zeros(8)
    v[3] = np.nan
    with pytest.raises(ValueError):
        oracle.topk(v, 2)


# ---- softmax renormalisation --------------------------------------------------------------

def test_softmax_selected_sums_to_one_and_orders():
    for _ in range(20):
        lg = RNG.standard_normal(50) * 3
        idx = oracle.topk(lg, 7)
        w = oracle.softmax_selected(lg, idx)
        assert abs(w.sum() - 1.0) < 1e-12
        assert np.all(np.diff(w) <= 0)


def test_softmax_selected_k_equals_E_is_full_softmax():
    lg = RNG.standard_normal(30) * 2
    idx = oracle.topk(lg, 30)
    w = oracle.softmax_selected(lg, idx)
    np.testing.assert_allclose(w, softmax(lg)[idx], rtol=1e-13, atol=0)


def test_softmax_selected_two_experts_is_logistic():
    lg = np.array([0.3, 2.0, -1.0, 1.25])
    idx = oracle.topk(lg, 2)                      # experts 1 and 3
    w = oracle.softmax_selected(lg, idx)
    np.testing.assert_allclose(w[0], expit(2.0 - 1.25), rtol=1e-14)
    np.testing.assert_allclose(w[1], expit(1.25 - 2.0), rtol=1e-14)


def test_softmax_is_renormalised_full_softmax():
    # Renormalising the full softmax over the selected set gives the same weights.
    lg = RNG.standard_normal(40)
    idx = oracle.topk(lg, 5)
    full = softmax(lg)
    np.testing.assert_allclose(oracle.softmax_selected(lg, idx), full[idx] / full[idx].sum(),
                               rtol=1e-13)


# ---- RMSNorm --------------------------------------------------------------------------------

def test_rmsnorm_constant_vector():
    H = 64
    for eps in (1e-6, 0.25, 4.0):
        for c in (0.5, 1.0, 3.0, -2.0):
            x = to_bits(np.full(H, c))
            g = to_bits(np.ones(H))
            n = oracle.rmsnorm(x, g, eps)
            cf = bf(x)[0]
            want = oracle.bf16_round(cf / math.sqrt(cf * cf + eps))
            assert np.all(n == want)


def test_rmsnorm_one_hot_gives_sqrt_H_gamma():
    H, eps = 256, 1e-6
    gamma = to_bits(1.0 + RNG.standard_normal(H) * 0.1)
    for i in (0, 17, 255):
        x = np.zeros(H, np.float32)
        x[i] = 2.0
        n = oracle.rmsnorm(to_bits(x), gamma, eps)
        want = oracle.bf16_round(2.0 / math.sqrt(4.0 / H + eps) * bf(gamma)[i])
        assert n[i] == want
        assert np.count_nonzero(n) == 1


def test_rmsnorm_gamma_is_elementwise_and_eps_matters():
    H = 32
    x = rand_bf16(H)
    g1 = to_bits(np.ones(H))
    gamma = np.ones(H, np.float32)
    gamma[5] = -2.0
    n1 = oracle.rmsnorm(x, g1, 0.0)
    n2 = oracle.rmsnorm(x, to_bits(gamma), 0.0)
    mask = np.arange(H) != 5
    assert np.array_equal(n1[mask], n2[mask])
    assert n2[5] == oracle.bf16_round(-2.0 * n1[5]) or abs(n2[5] + 2 * n1[5]) <= abs(n1[5]) * 2 ** -7
    # eps dominates for tiny inputs: n ~= x / sqrt(eps)
    xs = to_bits(np.full(H, 1e-6))
    n3 = oracle.rmsnorm(xs, g1, 1.0)
    np.testing.assert_allclose(n3, bf(xs) / 1.0, rtol=2 ** -8)


def test_rmsnorm_scale_invariant_without_eps():
    H = 128
    x = rand_bf16(H)
    x2 = to_bits(bf(x) * 2.0)                     # exact in bf16
    g = to_bits(1.0 + RNG.standard_normal(H) * 0.1)
    assert np.array_equal(oracle.rmsnorm(x, g, 0.0), oracle.rmsnorm(x2, g, 0.0))


# ---- router ----------------------------------------------------------------------------------

def selection_matrix(rows, cols, col_of_row, vals):
    """bf16 bits of a [rows, cols] matrix with one nonzero vals[r] at (r, col_of_row[r])."""
    m = np.zeros((rows, cols), np.float32)
    m[np.arange(rows), col_of_row] = vals
    return to_bits(m)


def test_router_closed_form_with_selection_matrix():
    H, E = 16, 12
    n = bf(rand_bf16(H))
    col = RNG.permutation(H)[:E]
    d = bf(rand_bf16(E))
    W = selection_matrix(E, H, col, d)
    lg = oracle.router(n, W)
    np.testing.assert_array_equal(lg, d * n[col])
    bias = RNG.standard_normal(E).astype(np.float32)
    lg2 = oracle.router(n, W, bias)
    np.testing.assert_array_equal(lg2, d * n[col] + bias.astype(np.float64))


def test_router_is_row_dot_not_column_dot():
    # Non-square, non-symmetric: a transposed access would read the wrong entries.
    H, E = 8, 3
    W = np.zeros((E, H), np.float32)
    W[0, 7] = 1.0
    W[1, 0] = 2.0
    W[2, 3] = -1.0
    n = np.arange(1, H + 1, dtype=np.float64)
    np.testing.assert_array_equal(oracle.router(n, to_bits(W)), [8.0, 2.0, -4.0])


# ---- SwiGLU expert ---------------------------------------------------------------------------

def silu(v):
    return v * expit(v)


def swiglu_closed_form(n, pg, dg, pu, du, pd, dd):
    g = dg * n[pg]
    u = du * n[pu]
    h = np.array([oracle.bf16_round(t) for t in silu(g) * u])
    return dd * h[pd]


@pytest.mark.parametrize("H,F", [(16, 8), (8, 16), (24, 24)])
def test_swiglu_closed_form_with_selection_matrices(H, F):
    n = bf(rand_bf16(H)) * 2
    pg = RNG.integers(0, H, F)
    pu = RNG.integers(0, H, F)
    pd = RNG.integers(0, F, H)
    dg, du, dd = bf(rand_bf16(F)), bf(rand_bf16(F)), bf(rand_bf16(H))
    out = oracle.swiglu(n, selection_matrix(F, H, pg, dg), selection_matrix(F, H, pu, du),
                        selection_matrix(H, F, pd, dd))
    want = swiglu_closed_form(n, pg, dg, pu, du, pd, dd)
    np.testing.assert_allclose(out, want, rtol=1e-13, atol=1e-300)


def test_swiglu_identity_weights():
    H = 32
    n = bf(rand_bf16(H))
    eye = to_bits(np.eye(H, dtype=np.float32))
    out = oracle.swiglu(n, eye, eye, eye)
    want = np.array([oracle.bf16_round(t) for t in silu(n) * n])
    np.testing.assert_allclose(out, want, rtol=1e-13, atol=1e-300)


def test_swiglu_gate_and_up_are_not_interchangeable():
    # silu is applied to the gate projection only: swapping gate/up changes the result.
    H = 16
    n = bf(rand_bf16(H))
    eye = to_bits(np.eye(H, dtype=np.float32))
    two = to_bits(2 * np.eye(H, dtype=np.float32))
    a = oracle.swiglu(n, eye, two, eye)
    b = oracle.swiglu(n, two, eye, eye)
    want_a = np.array([oracle.bf16_round(t) for t in silu(n) * 2 * n])
    np.testing.assert_allclose(a, want_a, rtol=1e-13, atol=1e-300)
    assert not np.allclose(a, b)


# ---- whole layer ------------------------------------------------------------------------------

def closed_form_layer(seed, force=None):
    """A tiny layer whose every matrix has one nonzero per row: the whole output
    has an elementwise closed form. force: a list of k distinct experts that
    replaces the row's top-k (the weights are then the softmax of the row's
    logits over that list)."""
    rng = np.random.default_rng(seed)
    H, E, k, I, Is, eps = 12, 6, 2, 5, 7, 1e-6
    x = to_bits(rng.standard_normal(H))
    gamma = to_bits(1 + 0.1 * rng.standard_normal(H))
    rcol = rng.permutation(H)[:E]
    rd = bf(to_bits(rng.standard_normal(E)))
    wr = selection_matrix(E, H, rcol, rd)
    bias = rng.standard_normal(E).astype(np.float32) * 0.5
    experts, maps = {}, {}
    for e in range(E):
        pg, pu, pd = rng.integers(0, H, I), rng.integers(0, H, I), rng.integers(0, I, H)
        dg, du, dd = (bf(to_bits(rng.standard_normal(I))), bf(to_bits(rng.standard_normal(I))),
                      bf(to_bits(rng.standard_normal(H))))
        experts[e] = (selection_matrix(I, H, pg, dg), selection_matrix(I, H, pu, du),
                      selection_matrix(H, I, pd, dd))
        maps[e] = (pg, dg, pu, du, pd, dd)
    spg, spu, spd = rng.integers(0, H, Is), rng.integers(0, H, Is), rng.integers(0, Is, H)
    sdg, sdu, sdd = (bf(to_bits(rng.standard_normal(Is))), bf(to_bits(rng.standard_normal(Is))),
                     bf(to_bits(rng.standard_normal(H))))
    W = dict(gamma=gamma, w_router=wr, router_bias=bias, experts=experts,
             ws_gate=selection_matrix(Is, H, spg, sdg), ws_up=selection_matrix(Is, H, spu, sdu),
             ws_down=selection_matrix(H, Is, spd, sdd))
    dims = dict(H=H, E=E, k=k, I=I, Is=Is, eps=eps)

    # closed form
    xf = bf(x)
    r = 1.0 / math.sqrt(np.sum(xf * xf) / H + eps)
    n = np.array([oracle.bf16_round(t) for t in xf * r * bf(gamma)])
    lg = rd * n[rcol] + bias.astype(np.float64)
    sel = sorted(range(E), key=lambda e: (-lg[e], e))[:k] if force is None else list(force)
    ws = softmax(lg[sel])
    s = swiglu_closed_form(n, spg, sdg, spu, sdu, spd, sdd)
    y = xf + s
    terms = []
    for j, e in enumerate(sel):
        terms.append(ws[j] * swiglu_closed_form(n, *maps[e]))
        y = y + terms[-1]
    return dims, W, x, dict(logits=lg, idx=np.array(sel), w=ws, y_pre=y, xs=xf + s, terms=terms)


@pytest.mark.parametrize("seed", range(8))
def test_layer_closed_form(seed):
    dims, W, x, want = closed_form_layer(seed)
    got = oracle.layer(dims, W, x)
    np.testing.assert_array_equal(got["logits"][0], want["logits"])
    np.testing.assert_array_equal(got["idx"][0], want["idx"])
    np.testing.assert_allclose(got["w"][0], want["w"], rtol=1e-13)
    np.testing.assert_allclose(got["y_pre"][0], want["y_pre"], rtol=1e-12, atol=1e-12)
    ybits = np.array([oracle.bf16_bits(t) for t in got["y_pre"][0]], np.uint16)
    np.testing.assert_array_equal(got["y"][0], ybits)


@pytest.mark.parametrize("seed", range(4))
def test_layer_with_given_selection_closed_form(seed):
    """A selection that is not the top-k: the output is the closed form evaluated on
    exactly that set, weighted by the softmax of the row's own logits over it."""
    rng = np.random.default_rng(100 + seed)
    force = [int(e) for e in rng.permutation(6)[:2]]
    dims, W, x, want = closed_form_layer(seed, force=force)
    got = oracle.layer(dims, W, x, selection=np.array([force]))
    np.testing.assert_array_equal(got["logits"][0], want["logits"])
    np.testing.assert_array_equal(got["idx"][0], force)
    np.testing.assert_allclose(got["w"][0], want["w"], rtol=1e-13)
    np.testing.assert_allclose(got["y_pre"][0], want["y_pre"], rtol=1e-12, atol=1e-12)


def test_layer_with_own_selection_equals_layer_bitwise():
    dims, W = tiny_random_layer(TINY)
    x = TINY.x_host()
    own = oracle.layer(dims, W, x)
    given = oracle.layer(dims, W, x, selection=own["idx"])
    for key in ("logits", "idx", "w", "y_pre", "y"):
        assert np.array_equal(own[key], given[key]), key


def test_layer_with_given_selection_is_order_free_and_rejects_bad_sets():
    dims, W = tiny_random_layer(TINY)
    x = TINY.x_host()
    own = oracle.layer(dims, W, x)
    # the same set in reverse order: the same weights per expert, the same output
    rev = oracle.layer(dims, W, x, selection=own["idx"][:, ::-1])
    np.testing.assert_allclose(rev["w"], own["w"][:, ::-1], rtol=1e-14)
    np.testing.assert_allclose(rev["y_pre"], own["y_pre"], rtol=1e-12, atol=1e-13)
    bad = own["idx"].copy()
    bad[0, 1] = bad[0, 0]                          # a repeated expert
    with pytest.raises(RuntimeError):
        oracle.layer(dims, W, x, selection=bad)
    bad = own["idx"].copy()
    bad[1, 0] = TINY.E                             # out of range
    with pytest.raises(RuntimeError):
        oracle.layer(dims, W, x, selection=bad)


@pytest.mark.parametrize("seed", range(4))
def test_layer_partial_closed_form(seed):
    """The part of the layer an expert range contributes: x + s when with_rs, plus the
    weighted outputs of the row's choices inside [e0, e1) -- against the closed form, with
    range ends placed on a selected expert (inclusive start, exclusive end)."""
    dims, W, x, want = closed_form_layer(seed)
    E, sel = dims["E"], [int(e) for e in want["idx"]]
    a = sel[0]
    cases = [(0, E, True), (0, E, False), (0, a, True), (a, E, False), (a, a + 1, False), (a, a, True),
             (0, 0, False)]
    for e0, e1, rs in cases:
        got = oracle.layer_partial(dims, W, x, e0, e1, rs)[0]
        ref = want["xs"].copy() if rs else np.zeros(dims["H"])
        for j, e in enumerate(sel):
            if e0 <= e < e1:
                ref = ref + want["terms"][j]
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12, err_msg=f"{(e0, e1, rs)}")


def test_layer_partials_over_a_partition_sum_to_the_layer():
    """Summed over a partition of the experts (residual and shared expert in one part),
    the parts are the layer's unrounded output; the whole range with them is that output
    bit for bit. Only each part's experts are given to it."""
    dims, W = tiny_random_layer(TINY)
    x = TINY.x_host()
    full = oracle.layer(dims, W, x)["y_pre"]
    whole = oracle.layer_partial(dims, W, x, 0, TINY.E, True)
    assert np.array_equal(whole, full)
    for cuts in ([0, 5, 16], [0, 1, 2, 9, 16], [0, 16]):
        total = np.zeros_like(full)
        for r, (e0, e1) in enumerate(zip(cuts[:-1], cuts[1:])):
            Wr = dict(W, experts={e: W["experts"][e] for e in range(e0, e1)})
            total += oracle.layer_partial(dims, Wr, x, e0, e1, r == 1 % (len(cuts) - 1))
        np.testing.assert_allclose(total, full, rtol=1e-12, atol=1e-12)


def test_layer_missing_expert_is_an_error():
    dims, W, x, want = closed_form_layer(0)
    W = dict(W)
    W["experts"] = {e: v for e, v in W["experts"].items() if e != int(want["idx"][0])}
    with pytest.raises(RuntimeError):
        oracle.layer(dims, W, x)


def tiny_random_layer(wl, seed=0):
    """Random tiny layer with the workload's generator (all experts present)."""
    dims = dict(H=wl.H, E=wl.E, k=wl.k, I=wl.I, Is=wl.Is, eps=wl.eps)
    sg, su, sd = wl.shared_host(0)
    W = dict(gamma=wl.gamma_host(0), w_router=wl.w_router_host(0), router_bias=wl.bias_host(0),
             experts={e: wl.expert_host(0, e) for e in range(wl.E)}, ws_gate=sg, ws_up=su, ws_down=sd)
    return dims, W


TINY = synth.Workload("pin_tiny", B=6, H=64, E=16, k=4, I=32, Is=48, seed=7)


def test_layer_batch_invariance_bitwise():
    dims, W = tiny_random_layer(TINY)
    x = TINY.x_host()
    together = oracle.layer(dims, W, x)
    for b in range(TINY.B):
        alone = oracle.layer(dims, W, x[b:b + 1])
        for key in ("logits", "idx", "w", "y_pre", "y"):
            assert np.array_equal(alone[key][0], together[key][b]), key


def test_layer_routing_invariants():
    dims, W = tiny_random_layer(TINY)
    got = oracle.layer(dims, W, TINY.x_host())
    B, k = TINY.B, TINY.k
    np.testing.assert_allclose(got["w"].sum(axis=1), 1.0, atol=1e-12)
    counts = np.bincount(got["idx"].ravel(), minlength=TINY.E)
    assert counts.sum() == B * k
    for b in range(B):
        assert len(set(got["idx"][b])) == k
        sel = got["logits"][b][got["idx"][b]]
        assert np.all(np.diff(sel) <= 0)
        assert sel[-1] >= np.max(np.delete(got["logits"][b], got["idx"][b]))


def test_layer_zero_down_weights_give_residual_exactly():
    dims, W = tiny_random_layer(TINY)
    W = dict(W)
    W["experts"] = {e: (g, u, np.zeros_like(d)) for e, (g, u, d) in W["experts"].items()}
    W["ws_down"] = np.zeros_like(W["ws_down"])
    x = TINY.x_host()
    got = oracle.layer(dims, W, x)
    assert np.array_equal(got["y"], x)


def test_layer_zero_routed_down_gives_shared_only():
    dims, W = tiny_random_layer(TINY)
    W = dict(W)
    W["experts"] = {e: (g, u, np.zeros_like(d)) for e, (g, u, d) in W["experts"].items()}
    x = TINY.x_host()
    got = oracle.layer(dims, W, x)
    for b in range(TINY.B):
        n = oracle.rmsnorm(x[b], W["gamma"], TINY.eps)
        s = oracle.swiglu(n, W["ws_gate"], W["ws_up"], W["ws_down"])
        np.testing.assert_array_equal(got["y_pre"][b], bf(x[b]) + s)


def test_layer_linear_in_down_weights():
    dims, W = tiny_random_layer(TINY)
    x = TINY.x_host()
    base = oracle.layer(dims, W, x)
    W2 = dict(W)
    W2["experts"] = {e: (g, u, to_bits(bf(d) * 2)) for e, (g, u, d) in W["experts"].items()}
    W2["ws_down"] = to_bits(bf(W["ws_down"]) * 2)
    dbl = oracle.layer(dims, W2, x)
    xf = bf(x)
    # linear in the down weights (up to the fp64 rounding of the residual add)
    np.testing.assert_allclose(dbl["y_pre"] - xf, 2 * (base["y_pre"] - xf), rtol=1e-12, atol=1e-13)


def test_layer_k_equals_E_weights_all_experts_by_full_softmax():
    wl = synth.Workload("pin_kE", B=2, H=32, E=5, k=5, I=16, Is=16, seed=9)
    dims, W = tiny_random_layer(wl)
    x = wl.x_host()
    got = oracle.layer(dims, W, x)
    for b in range(wl.B):
        n = oracle.rmsnorm(x[b], W["gamma"], wl.eps)
        lg = oracle.router(n, W["w_router"])
        p = softmax(lg)
        want = bf(x[b]) + oracle.swiglu(n, W["ws_gate"], W["ws_up"], W["ws_down"])
        for e in range(wl.E):
            want = want + p[e] * oracle.swiglu(n, *W["experts"][e])
        np.testing.assert_allclose(got["y_pre"][b], want, rtol=1e-12, atol=1e-12)


def test_layer_bias_enters_selection_and_weights():
    wl = synth.Workload("pin_bias", B=3, H=32, E=12, k=3, I=16, Is=16, seed=11, router="zipf")
    dims, W = tiny_random_layer(wl)
    x = wl.x_host()
    got = oracle.layer(dims, W, x)
    for b in range(wl.B):
        n = oracle.rmsnorm(x[b], W["gamma"], wl.eps)
        lg = oracle.router(n, W["w_router"]) + W["router_bias"].astype(np.float64)
        np.testing.assert_array_equal(got["logits"][b], lg)
        sel = sorted(range(wl.E), key=lambda e: (-lg[e], e))[:wl.k]
        np.testing.assert_array_equal(got["idx"][b], sel)
        np.testing.assert_allclose(got["w"][b], softmax(lg[sel]), rtol=1e-13)


# ---- FP8 expert weights ------------------------------------------------------------------

def test_e4m3_decode_matches_an_independent_table():
    """Every E4M3 code against torch's float8_e4m3fn conversion (NaN codes included)."""
    import torch

    codes = np.arange(256, dtype=np.uint8)
    mine = np.array([oracle.e4m3_value(c) for c in codes])
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    assert np.array_equal(mine[~np.isnan(mine)], ref[~np.isnan(ref)])


def test_e4m3_decode_closed_forms():
    # 1.0, the largest finite, the smallest subnormal and normal, signed zero and one
    assert oracle.e4m3_value(0x38) == 1.0 and oracle.e4m3_value(0x7E) == 448.0
    assert oracle.e4m3_value(0x01) == 2.0 ** -9 and oracle.e4m3_value(0x08) == 2.0 ** -6
    assert oracle.e4m3_value(0x07) == 7 * 2.0 ** -9 and oracle.e4m3_value(0x0F) == 1.875 * 2.0 ** -6
    assert oracle.e4m3_value(0xB8) == -1.0 and math.copysign(1.0, oracle.e4m3_value(0x80)) == -1.0
    assert math.isnan(oracle.e4m3_value(0x7F)) and math.isnan(oracle.e4m3_value(0xFF))


def test_dequant_applies_each_blocks_own_scale():
    """Codes of value 1 (and a few others) in a 3 x 2 grid of 128 x 128 blocks whose
    scales all differ: every weight is its code's value times its own block's scale."""
    rows, cols = 384, 256
    codes = np.full((rows, cols), 0x38, dtype=np.uint8)           # 1.0
    codes[5, 200] = 0x3C                                          # 1.5 in block (0, 1)
    codes[300, 7] = 0xC6                                          # -3.5 in block (2, 0)
    scales = np.ldexp(np.float32(1.0), np.array([[0, 3], [-2, 5], [7, -9]])).astype(np.float32)
    w = synth.bf16_bits_to_f32(oracle.dequant_e4m3(codes, scales)).astype(np.float64)
    want = np.repeat(np.repeat(scales.astype(np.float64), 128, axis=0), 128, axis=1)
    want[5, 200] *= 1.5
    want[300, 7] *= -3.5
    np.testing.assert_array_equal(w, want)


def test_dequant_rejects_weights_bf16_cannot_hold():
    codes = np.full((128, 128), 0x39, dtype=np.uint8)             # 1.125
    with pytest.raises(ValueError):
        oracle.dequant_e4m3(codes, np.array([[1.0 / 3.0]], dtype=np.float32))
    codes[0, 0] = 0x7F                                            # NaN
    with pytest.raises(ValueError):
        oracle.dequant_e4m3(codes, np.array([[1.0]], dtype=np.float32))


def test_fp8_layer_is_the_bf16_layer_on_the_dequantised_weights():
    """The workload's FP8 experts, dequantised, drive the same layer definition: the
    FP8 oracle layer equals oracle.layer given the dequantised expert matrices."""
    wl = synth.Workload("pin_fp8", B=2, H=256, E=8, k=2, I=128, Is=128, seed=13)
    x = wl.x_host()
    got = oracle.workload_layer(wl, 0, x, fp8=True)
    dims = dict(H=wl.H, E=wl.E, k=wl.k, I=wl.I, Is=wl.Is, eps=wl.eps)
    sg, su, sd = wl.shared_host(0)
    W = dict(gamma=wl.gamma_host(0), w_router=wl.w_router_host(0), router_bias=None, ws_gate=sg, ws_up=su,
             ws_down=sd, experts={e: oracle.fp8_expert(wl.expert_fp8_host(0, e)) for e in range(wl.E)})
    want = oracle.layer(dims, W, x)
    for key in ("logits", "idx", "w", "y"):
        assert np.array_equal(got[key], want[key]), key


PIN_CHECKS = [
    lambda: test_topk_matches_full_stable_sort(16, 4),
    test_softmax_selected_two_experts_is_logistic,
    test_rmsnorm_constant_vector,
    test_rmsnorm_one_hot_gives_sqrt_H_gamma,
    lambda: test_swiglu_closed_form_with_selection_matrices(16, 8),
    test_swiglu_gate_and_up_are_not_interchangeable,
    lambda: [test_layer_closed_form(s) for s in range(8)],
    lambda: [test_layer_with_given_selection_closed_form(s) for s in range(4)],
    test_layer_zero_routed_down_gives_shared_only,
    test_layer_bias_enters_selection_and_weights,
    test_e4m3_decode_matches_an_independent_table,
    test_dequant_applies_each_blocks_own_scale,
]


@pytest.mark.parametrize("mutant", sorted(oracle.MUTANTS))
def test_each_planted_mistake_fails_a_pin(mutant):
    """Plant one plausible mistake in the oracle; at least one pin must fail."""
    for check in PIN_CHECKS:                      # all pins pass on the real oracle
        check()
    failed = []
    oracle.set_mutant(mutant)
    try:
        for i, check in enumerate(PIN_CHECKS):
            try:
                check()
            except (AssertionError, ValueError, RuntimeError):
                failed.append(i)
    finally:
        oracle.set_mutant(0)
    assert failed, f"planted mistake {oracle.MUTANTS[mutant]} was not caught by any pin"


def test_shipped_oracle_has_no_mistake_switch():
    """The planted mistakes live only in the separately compiled mutant build: the
    oracle library itself exports no switch and carries no mistake branches."""
    import ctypes

    plain = ctypes.CDLL(oracle.LIB)
    assert not hasattr(plain, "oracle_set_mutant")
    assert hasattr(ctypes.CDLL(oracle.MUTANT_LIB), "oracle_set_mutant")

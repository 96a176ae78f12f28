"""Pins of the CPU oracle to facts other than itself (CPU only).

The pages print no worked example, so every pin here is a closed form, an
invariant, a special case that reduces to a library routine, or brute force
on tiny inputs.  Each ``pin_*`` takes an oracle build; ``test_pins`` runs them
on the reference build and ``test_mutants_are_caught`` rebuilds the oracle with
each deliberately planted mistake (oracle.c, ORACLE_MUTANT) and checks that at
least one pin fails for every one of them.
"""
import math
import os

import numpy as np
import pytest

import oracle
import synth

B16 = synth.f64_to_bf16_bits
F32 = synth.bf16_bits_to_f32


def dyadic(rng, shape, num=16, den=8):
    """bf16-exact values k/den with |k| <= num."""
    return rng.integers(-num, num + 1, size=shape).astype(np.float64) / den


# --- o_proj + residual ---------------------------------------------------------
def pin_oproj_permutation(o):
    # W_o = permutation matrix: h[i] = residual[i] + attn[pi(i)] exactly.
    rng = np.random.default_rng(1)
    d = 8
    pi = np.array([3, 0, 6, 1, 7, 2, 4, 5])  # no fixed points, not an involution
    W = np.zeros((d, d))
    W[np.arange(d), pi] = 1.0
    attn = dyadic(rng, (2, d))
    res = dyadic(rng, (2, d))
    h = o.oproj_residual(B16(W), B16(attn), B16(res), 2, d, d)
    assert np.array_equal(h, res + attn[:, pi])


def pin_oproj_single_entry(o):
    # Non-square W_o with one entry: only row 1 picks up 0.125 * attn[3].
    rng = np.random.default_rng(2)
    d, d_o = 3, 5
    W = np.zeros((d, d_o))
    W[1, 3] = 0.125
    attn = dyadic(rng, (2, d_o))
    res = dyadic(rng, (2, d))
    h = o.oproj_residual(B16(W), B16(attn), B16(res), 2, d, d_o)
    want = res.copy()
    want[:, 1] += 0.125 * attn[:, 3]
    assert np.array_equal(h, want)


def pin_oproj_token_permutation(o):
    # Tokens are independent: permuting the batch permutes h.
    rng = np.random.default_rng(3)
    d, d_o, B = 6, 10, 4
    W, attn, res = dyadic(rng, (d, d_o)), dyadic(rng, (B, d_o)), dyadic(rng, (B, d))
    p = np.array([2, 0, 3, 1])
    h = o.oproj_residual(B16(W), B16(attn), B16(res), B, d, d_o)
    hp = o.oproj_residual(B16(W), B16(attn[p]), B16(res[p]), B, d, d_o)
    assert np.array_equal(hp, h[p])


def pin_oproj_linearity(o):
    # h(W1 + W2) - r = (h(W1) - r) + (h(W2) - r), exactly for dyadic inputs.
    rng = np.random.default_rng(4)
    d, d_o = 5, 7
    W1, W2 = dyadic(rng, (d, d_o), 4, 8), dyadic(rng, (d, d_o), 4, 8)
    attn, res = dyadic(rng, (1, d_o)), np.zeros((1, d))
    f = lambda W: o.oproj_residual(B16(W), B16(attn), B16(res), 1, d, d_o)
    assert np.array_equal(f(W1 + W2), f(W1) + f(W2))


# --- RMSNorm ---------------------------------------------------------------------
def pin_rmsnorm_constant(o):
    # h = c everywhere: rstd = 1/sqrt(c^2 + eps), x_i = gamma_i * c * rstd.
    d = 16
    gamma = 1.0 + np.arange(d) / 64.0
    for c, eps in [(3.0, 1e-6), (1e-3, 1e-6), (-2.5, 0.25)]:
        h = np.full((1, d), c)
        rstd, x = o.rmsnorm(h, B16(gamma), eps)
        r = 1.0 / math.sqrt(c * c + eps)
        assert abs(rstd[0] - r) <= 1e-15 * r
        assert np.allclose(x[0], gamma * c * r, rtol=1e-15, atol=0)


def pin_rmsnorm_one_hot(o):
    # h = c e_j: mean(h^2) = c^2 / d.
    d, j, c, eps = 32, 5, 4.0, 1e-6
    gamma = np.full(d, 0.5)
    h = np.zeros((1, d))
    h[0, j] = c
    rstd, x = o.rmsnorm(h, B16(gamma), eps)
    r = 1.0 / math.sqrt(c * c / d + eps)
    assert abs(rstd[0] - r) <= 1e-15 * r
    want = np.zeros(d)
    want[j] = 0.5 * c * r
    assert np.allclose(x[0], want, rtol=1e-15, atol=0)


def pin_rmsnorm_zero(o):
    d = 8
    rstd, x = o.rmsnorm(np.zeros((1, d)), B16(np.ones(d)), 1e-6)
    assert abs(rstd[0] - 1000.0) < 1e-9 and np.all(x == 0)


def pin_rmsnorm_scale_invariance(o):
    # With eps -> 0, x(2^k h) = x(h) (power-of-two scaling is exact).
    rng = np.random.default_rng(5)
    d = 24
    h = rng.normal(size=(1, d))
    g = B16(1 + 0.1 * rng.normal(size=d))
    _, x1 = o.rmsnorm(h, g, 0.0)
    _, x2 = o.rmsnorm(h * 8.0, g, 0.0)
    assert np.allclose(x1, x2, rtol=1e-15, atol=0)


# --- router ---------------------------------------------------------------------
def pin_router_one_hot(o):
    # x = e_i gives the i-th column of W_r (W_r is [E][d]).
    rng = np.random.default_rng(6)
    E, d = 5, 7
    W = dyadic(rng, (E, d))
    x = np.zeros((2, d))
    x[0, 2] = 1.0
    x[1, 6] = -2.0
    lg = o.router(B16(W), x, E)
    assert np.array_equal(lg[0], W[:, 2]) and np.array_equal(lg[1], -2.0 * W[:, 6])


# --- top-k and gates -------------------------------------------------------------
def pin_topk_brute_force(o):
    # First k of a full stable sort on (-logit, index), with forced ties.
    rng = np.random.default_rng(7)
    for trial in range(300):
        E = int(rng.integers(2, 40))
        k = int(rng.integers(1, E + 1))
        B = int(rng.integers(1, 4))
        lg = rng.integers(-6, 7, size=(B, E)).astype(np.float32) / 4  # many ties
        if trial % 3 == 0:
            lg = rng.normal(size=(B, E)).astype(np.float32)
        idx, _ = o.topk_gates(lg, k)
        for b in range(B):
            want = sorted(range(E), key=lambda e: (-float(lg[b, e]), e))[:k]
            assert list(idx[b]) == want


def pin_gates_two(o):
    # k = 2: gate_0 = 1 / (1 + exp(l1 - l0)), gate_1 = 1 - gate_0.
    lg = np.array([[0.25, -1.5, 2.0, 0.75, -3.0]], np.float32)
    idx, gate = o.topk_gates(lg, 2)
    assert list(idx[0]) == [2, 3]
    g0 = 1.0 / (1.0 + math.exp(0.75 - 2.0))
    assert abs(gate[0, 0] - g0) < 1e-15 and abs(gate[0, 1] - (1 - g0)) < 1e-15


def pin_gates_invariants(o):
    rng = np.random.default_rng(8)
    lg = rng.normal(scale=2.0, size=(3, 50)).astype(np.float32)
    idx, gate = o.topk_gates(lg, 9)
    for b in range(3):
        assert abs(gate[b].sum() - 1.0) < 1e-14
        assert np.all(np.diff(gate[b]) <= 0)
        sel = lg[b, idx[b]].astype(np.float64)
        assert np.allclose(gate[b][1:] / gate[b][0], np.exp(sel[1:] - sel[0]), rtol=1e-13)
    one_idx, one = o.topk_gates(lg, 1)
    assert np.all(one == 1.0)


def pin_gates_dense_softmax(o):
    # k = E: the gates are the softmax of all logits (library routine), in sorted order.
    from scipy.special import softmax
    rng = np.random.default_rng(9)
    lg = rng.normal(size=(2, 12)).astype(np.float32)
    idx, gate = o.topk_gates(lg, 12)
    for b in range(2):
        sm = softmax(lg[b].astype(np.float64))
        assert np.allclose(gate[b], sm[idx[b]], rtol=1e-13, atol=0)


# --- SwiGLU expert ---------------------------------------------------------------
def pin_swiglu_scalar(o):
    # d = I = 1: y = w_d * silu(w_g x) * (w_u x), silu(g) = g / (1 + exp(-g)).
    for wg, wu, wd, x in [(0.5, -1.25, 0.75, 1.5), (-2.0, 0.25, -1.0, 0.75), (1.0, 1.0, 2.0, -3.0)]:
        a, y = o.expert(B16(np.array([wg, wu])), B16(np.array([wd])), np.array([x]), 1)
        g, u = wg * x, wu * x
        want_a = g / (1.0 + math.exp(-g)) * u
        assert abs(a[0] - want_a) <= 1e-15 * max(1, abs(want_a))
        assert abs(y[0] - wd * want_a) <= 1e-15 * max(1, abs(wd * want_a))


def pin_swiglu_zero_gate(o):
    # silu(0) = 0: zero gate rows give a = 0 and y = 0 whatever the rest is.
    rng = np.random.default_rng(10)
    d, I = 6, 3
    gu = dyadic(rng, (2 * I, d))
    gu[:I] = 0
    a, y = o.expert(B16(gu), B16(dyadic(rng, (d, I))), rng.normal(size=d), I)
    assert np.all(a == 0) and np.all(y == 0)


def pin_swiglu_down_single_entry(o):
    # W_down with one entry at (i=1, t=0): y = [0, w * a_0, 0].
    d, I = 3, 2
    gu = np.zeros((2 * I, d))
    gu[0, 0], gu[I + 0, 0] = 0.5, 1.5     # g_0 = 0.5 x_0, u_0 = 1.5 x_0
    gu[1, 1], gu[I + 1, 1] = -1.0, 2.0
    dn = np.zeros((d, I))
    dn[1, 0] = 0.25
    x = np.array([2.0, 1.0, 0.0])
    a, y = o.expert(B16(gu), B16(dn), x, I)
    a0 = 1.0 / (1 + math.exp(-1.0)) * 3.0
    a1 = -1.0 / (1 + math.exp(1.0)) * 2.0
    assert np.allclose(a, [a0, a1], rtol=1e-15, atol=0)
    assert np.allclose(y, [0.0, 0.25 * a0, 0.0], rtol=1e-15, atol=0)


def pin_swiglu_down_linear(o):
    # Doubling W_down doubles y exactly.
    rng = np.random.default_rng(11)
    d, I = 8, 4
    gu, dn, x = dyadic(rng, (2 * I, d)), dyadic(rng, (d, I), 8, 16), rng.normal(size=d)
    _, y1 = o.expert(B16(gu), B16(dn), x, I)
    _, y2 = o.expert(B16(gu), B16(2 * dn), x, I)
    assert np.array_equal(y2, 2 * y1)


# --- combine ------------------------------------------------------------------------
def pin_combine_closed_form(o):
    h = np.array([1.0, -2.0, 0.5])
    gate = np.array([0.75, 0.25])
    ys = [np.array([4.0, 0.0, -1.0]), np.array([-8.0, 2.0, 1.0])]
    out, ob = o.combine(h, gate, ys)
    want = np.array([1.0 + 3.0 - 2.0, -2.0 + 0.0 + 0.5, 0.5 - 0.75 + 0.25])
    assert np.array_equal(out, want)
    assert np.array_equal(ob, B16(want))


def pin_layer_relabel_invariance(o):
    # Relabelling experts (rows of W_r and the expert slabs permuted together)
    # relabels idx and leaves gates and the output unchanged.
    rng = np.random.default_rng(12)
    d, d_o, E, k, I = 16, 24, 6, 3, 4
    W_o, gamma, W_r = B16(rng.normal(0, .2, (d, d_o))), B16(1 + .1 * rng.normal(size=d)), \
        B16(rng.normal(0, .3, (E, d)))
    gu, dn = B16(rng.normal(0, .2, (E, 2 * I, d))), B16(rng.normal(0, .2, (E, d, I)))
    attn, res = B16(rng.normal(size=(1, d_o))), B16(rng.normal(size=(1, d)))
    perm = rng.permutation(E)

    def run(W_r, gu, dn):
        f = o.front(W_o, gamma, W_r, attn, res, B=1, d=d, d_o=d_o, E=E, k=k)
        sel = f["idx"][0]
        out, ob, _ = o.moe_token([gu[e] for e in sel], [dn[e] for e in sel], f["x"][0],
                                 f["h"][0], f["gate"][0], I)
        return f["idx"][0], f["gate"][0], out
    i1, g1, o1 = run(W_r, gu, dn)
    i2, g2, o2 = run(W_r[perm], gu[perm], dn[perm])
    assert np.array_equal(perm[i2], i1)
    assert np.array_equal(g1, g2) and np.array_equal(o1, o2)


# --- bf16 rounding of the output --------------------------------------------------------
def pin_bf16_rne(o):
    cases = [(1.0, 0x3F80), (1 + 2**-8, 0x3F80), (1 + 3 * 2**-8, 0x3F82),
             (1 + 2**-8 + 2**-20, 0x3F81), (-(1 + 2**-8 + 2**-20), 0xBF81), (0.0, 0x0000),
             (-0.0, 0x8000), (3.0, 0x4040), (254.5, 0x437E), (255.5, 0x4380), (255.75, 0x4380)]
    for v, want in cases:
        assert o.bf16_rne(v) == want, (v, hex(o.bf16_rne(v)), hex(want))
    # Agreement with a float32 round trip where float32 holds the value exactly.
    rng = np.random.default_rng(13)
    for v in rng.normal(scale=50, size=200).astype(np.float32):
        b = np.array([v], np.float32).view(np.uint32)[0]
        r = ((int(b) + 0x7FFF + ((int(b) >> 16) & 1)) >> 16) & 0xFFFF
        assert o.bf16_rne(float(v)) == r


PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pins(pin, oracle_ref):
    assert oracle_ref.mutant == 0
    pin(oracle_ref)


MUTANTS = list(range(1, 19))


@pytest.mark.parametrize("m", MUTANTS)
def test_mutants_are_caught(m, tmp_path):
    path = oracle.build(out=str(tmp_path / f"liboracle_m{m}.so"), mutant=m, force=True)
    om = oracle.Oracle(path)
    assert om.mutant == m
    failed = []
    for pin in PINS:
        try:
            pin(om)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"mutant {m} passes every pin"

"""Pins of the oracle's time-mix output epilogue (``oracle.timemix_out``).

The pages describe the epilogue in words only (Paper Review: RWKV-7 "Goose",
section "The approach": the receptance reads the state, the block also attends
to the current token without storing it, the result is normalised per head,
combined across heads and gated).  The oracle's reading of those words is pinned
here by facts that do not come from retyping its formula:
* a closed form of the normalisation (values 1..N: mean (N+1)/2, population
  variance (N^2-1)/12),
* exact cancellations of the current-token term built from the recurrence's own
  write (T = 1 from a zero state gives y = v (k . r)),
* invariances of a per-head layer normalisation (shift, scale, unit rms) and the
  linearity of the gate,
* that the term never enters the state,
and ``test_planted_mistakes_are_caught`` checks that plausible slips in the
oracle (sample variance, an unweighted current-token term, no centring, the
gate inside the affine, eps outside the square root, a dropped current-token
term) each fail one of them.
"""
import inspect

import numpy as np
import pytest

import oracle
from linear_rnn_sequence_wkv7_b200 import inputs

N = 64


def _single_token(r, k, v):
    """Inputs of a one-token sequence from a zero state (a = b = 0, w = 1):
    the state after the write is v k^T, so y = v (k . r)."""
    shape = (1, 1, 1, N)
    z = np.zeros(shape)
    return [np.asarray(r, float).reshape(shape), np.ones(shape), np.asarray(k, float).reshape(shape),
            np.asarray(v, float).reshape(shape), z, z]


def _recipe(B, T, H, seed):
    d = inputs.gen_sequence(B, T, H, N, seed=seed, dtype="f32", s0_std=0.1)
    return [inputs.to_f64(d[n]) for n in inputs.INPUT_NAMES], d["s0"].astype(np.float64)


def _params(H, seed):
    rng = np.random.default_rng(seed)
    return (rng.uniform(-1.5, 1.5, (H, N)), rng.uniform(0.5, 1.5, (H, N)), rng.uniform(-0.5, 0.5, (H, N)))


def check_norm_closed_form(fn):
    # r = k = e_0, rho = 0: y = v, o = v = (1, 2, ..., N)
    e0 = np.eye(N)[0]
    v = np.arange(1, N + 1, dtype=float)
    x = _single_token(e0, e0, v)
    y, _ = oracle.forward(*x)
    np.testing.assert_array_equal(y.reshape(-1), v)
    eps = 1e-3
    mu, var = (N + 1) / 2.0, (N * N - 1) / 12.0
    want = (v - mu) / np.sqrt(var + eps)
    z = fn(y, x[0], x[2], x[3], np.zeros((1, N)), eps=eps)
    return np.max(np.abs(z.reshape(-1) - want)) <= 1e-12 * np.max(np.abs(want))


def check_term_cancels_the_write(fn):
    # T = 1 from zero: o = v sum_j r_j k_j (1 + rho_j).  With rho_j = -1 wherever
    # r_j k_j != 0 the token's own contribution is cancelled exactly: o = 0 and
    # z = g * beta whatever the other rho_j are (up to rounding).
    rng = np.random.default_rng(5)
    r = np.zeros(N)
    k = np.zeros(N)
    r[:16], k[:16] = rng.standard_normal(16), rng.standard_normal(16)
    v = rng.standard_normal(N)
    rho = rng.uniform(-2.0, 2.0, (1, N))
    rho[0, :16] = -1.0
    gamma, beta = rng.uniform(0.5, 1.5, (1, N)), rng.uniform(-0.5, 0.5, (1, N))
    g = rng.standard_normal((1, 1, 1, N))
    x = _single_token(r, k, v)
    y, _ = oracle.forward(*x)
    z = fn(y, x[0], x[2], x[3], rho, gamma, beta, g, eps=1e-5)
    # o cancels up to the rounding of two sums of 16 products (~1e-16)
    return np.allclose(z, g * beta, rtol=0, atol=1e-12)


def check_term_scales_the_write(fn):
    # T = 1 from zero with a uniform rho: o = (1 + rho) y, and the per-head norm
    # (eps = 0) maps it to sign(1 + rho) times the norm of y
    rng = np.random.default_rng(6)
    x = _single_token(rng.standard_normal(N), rng.standard_normal(N), rng.standard_normal(N))
    y, _ = oracle.forward(*x)
    z0 = fn(y, x[0], x[2], x[3], np.zeros((1, N)), eps=0.0)
    zp = fn(y, x[0], x[2], x[3], np.full((1, N), 2.0), eps=0.0)        # o = 3 y
    zm = fn(y, x[0], x[2], x[3], np.full((1, N), -3.0), eps=0.0)       # o = -2 y
    return np.allclose(zp, z0, rtol=0, atol=1e-12) and np.allclose(zm, -z0, rtol=0, atol=1e-12)


def check_invariances(fn):
    B, T, H = 2, 9, 3
    (r, w, k, v, a, b), s0 = _recipe(B, T, H, seed=71)
    rho, gamma, beta = _params(H, 72)
    y, _ = oracle.forward(r, w, k, v, a, b, s0=s0)
    ok = True
    # unit rms and zero mean per head (gamma = 1, beta = 0, g = 1, eps = 0)
    z = fn(y, r, k, v, rho, eps=0.0)
    ok &= np.allclose(np.mean(z, axis=-1), 0.0, atol=1e-12)
    ok &= np.allclose(np.mean(z * z, axis=-1), 1.0, atol=1e-12)
    # shift of y by a constant per head-token, and scale of (y, v) by c > 0: unchanged
    shift = np.random.default_rng(73).standard_normal((B, T, H, 1))
    ok &= np.allclose(fn(y + shift, r, k, v, rho, eps=0.0), z, atol=1e-10)
    ok &= np.allclose(fn(3.5 * y, r, k, 3.5 * v, rho, eps=0.0), z, atol=1e-10)
    # the gate is linear; zero gate gives zero
    g1 = np.random.default_rng(74).standard_normal((B, T, H, N))
    g2 = np.random.default_rng(75).standard_normal((B, T, H, N))
    z1 = fn(y, r, k, v, rho, gamma, beta, g1)
    z2 = fn(y, r, k, v, rho, gamma, beta, g2)
    ok &= np.allclose(fn(y, r, k, v, rho, gamma, beta, g1 + g2), z1 + z2, atol=1e-12)
    ok &= np.array_equal(fn(y, r, k, v, rho, gamma, beta, np.zeros_like(g1)), np.zeros_like(g1))
    # the affine acts after the normalisation: g = 1 gives gamma * z(1, 0) + beta
    zn = fn(y, r, k, v, rho)
    ok &= np.allclose(fn(y, r, k, v, rho, gamma, beta), gamma * zn + beta, atol=1e-12)
    return bool(ok)


PINS = (check_norm_closed_form, check_term_cancels_the_write, check_term_scales_the_write, check_invariances)


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_oracle_satisfies(pin):
    assert pin(oracle.timemix_out)


def test_current_token_term_stays_out_of_the_state():
    """forward_timemix's final state is forward's: the current-token term is
    read, never written."""
    B, T, H = 1, 12, 2
    (r, w, k, v, a, b), s0 = _recipe(B, T, H, seed=81)
    rho, gamma, beta = _params(H, 82)
    z, sT = oracle.forward_timemix(r, w, k, v, a, b, s0, rho, gamma, beta)
    y, sT2 = oracle.forward(r, w, k, v, a, b, s0=s0)
    np.testing.assert_array_equal(sT, sT2)
    np.testing.assert_array_equal(z, oracle.timemix_out(y, r, k, v, rho, gamma, beta))


TIMEMIX_MUTANTS = {
    "sample_variance": ("var = float(np.sum((o - mu) ** 2)) / N", "var = float(np.sum((o - mu) ** 2)) / (N - 1)"),
    "unweighted_term": ("bonus = float(np.sum(r[bb, t, h] * rho[h] * k[bb, t, h]))",
                        "bonus = float(np.sum(r[bb, t, h] * k[bb, t, h])) * float(np.mean(rho[h]))"),
    "no_centring": ("(o - mu) / np.sqrt(var + eps)", "o / np.sqrt(var + eps)"),
    "gate_inside_affine": ("z[bb, t, h] = g[bb, t, h] * (gamma[h] * (o - mu) / np.sqrt(var + eps) + beta[h])",
                           "z[bb, t, h] = g[bb, t, h] * gamma[h] * (o - mu) / np.sqrt(var + eps) + beta[h]"),
    "eps_outside_sqrt": ("np.sqrt(var + eps)", "(np.sqrt(var) + eps)"),
    "dropped_term": ("o = y[bb, t, h] + bonus * v[bb, t, h]", "o = y[bb, t, h]"),
}


@pytest.mark.parametrize("mutant", sorted(TIMEMIX_MUTANTS))
def test_planted_mistakes_are_caught(mutant):
    src = inspect.getsource(oracle.timemix_out)
    old, new = TIMEMIX_MUTANTS[mutant]
    assert src.count(old) == 1, "mutation anchor not found"
    ns = dict(np=np, _f64=oracle._f64)
    exec(src.replace(old, new), ns)
    fn = ns["timemix_out"]
    assert not all(pin(fn) for pin in PINS), f"mutant {mutant} slipped through"

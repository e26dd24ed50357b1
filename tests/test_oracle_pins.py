"""Pins of the fp64 oracle against facts that do not come from the oracle.

The pages print no worked example of WKV7, so the oracle is pinned by
* hand-computed fixtures (tests/golden/, exact binary fractions),
* closed forms of degenerate cases (decayed linear attention, a = b = 0),
* the delta-rule replace / relaxed-replace semantics and the Householder case,
* agreement of two independently derived forms (sequential vs chunked),
* central finite differences for the backward,
and each is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign, a transposed operand, reading y before the write) fails one of
them; ``test_planted_mistakes_are_caught`` checks exactly that by compiling
mutated copies of the oracle.
"""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
from linear_rnn_sequence_wkv7_b200 import inputs
from tests._golden import load


def rel_err(x, ref):
    x, ref = np.asarray(x), np.asarray(ref)
    scale = np.sqrt(np.mean(ref ** 2))
    return float(np.max(np.abs(x - ref)) / (scale if scale > 0 else 1.0))


def unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def recipe(B, T, H, N, seed, x_mean=0.0, s0_std=0.1, dtype="f32"):
    d = inputs.gen_sequence(B, T, H, N, seed=seed, dtype=dtype, x_mean=x_mean, s0_std=s0_std)
    args = [inputs.to_f64(d[n]) for n in inputs.INPUT_NAMES]
    s0 = None if d["s0"] is None else d["s0"].astype(np.float64)
    return args, s0


# --- hand-computed fixtures --------------------------------------------------

@pytest.mark.parametrize("name", ["hand_n1_t3.txt", "hand_n2_t2.txt"])
def test_golden_forward(name):
    g = load(name)
    y, sT = oracle.forward(g["r"], g["w"], g["k"], g["v"], g["a"], g["b"], s0=g["s0"])
    np.testing.assert_array_equal(y, g["y"])
    np.testing.assert_array_equal(sT, g["sT"])


def test_golden_backward():
    g = load("hand_n1_t2_grad.txt")
    y, sT = oracle.forward(g["r"], g["w"], g["k"], g["v"], g["a"], g["b"], s0=g["s0"])
    np.testing.assert_array_equal(y, g["y"])
    np.testing.assert_array_equal(sT, g["sT"])
    dr, dw, dk, dv, da, db, ds0 = oracle.backward(g["r"], g["w"], g["k"], g["v"], g["a"], g["b"],
                                                  g["s0"], g["dy"], g["dsT"])
    for name, got in zip(("dr", "dw", "dk", "dv", "da", "db", "ds0"), (dr, dw, dk, dv, da, db, ds0)):
        np.testing.assert_array_equal(got, g[name], err_msg=name)


# --- closed form: a = b = 0 is linear attention with vector decay -------------

def test_closed_form_decayed_linear_attention():
    """With a = b = 0 the state is S_t = S_0 diag(prod_{m<=t} w_m)
    + sum_{s<=t} v_s (k_s * prod_{s<m<=t} w_m)^T, i.e. linear attention with a
    per-channel decay (Paper Review: RWKV-7 "Goose", section "Background
    information on delta rule").  Evaluated as an explicit double sum."""
    B, T, H, N = 1, 23, 2, 7
    (r, w, k, v, a, b), s0 = recipe(B, T, H, N, seed=11)
    a[:] = 0.0
    b[:] = 0.0
    y, sT = oracle.forward(r, w, k, v, a, b, s0=s0)
    for h in range(H):
        for t in range(T):
            decay0 = np.prod(w[0, :t + 1, h], axis=0)              # prod_{m<=t} w_m
            Y = s0[0, h] @ (decay0 * r[0, t, h])
            for s in range(t + 1):
                dec = np.prod(w[0, s + 1:t + 1, h], axis=0)         # empty product = 1
                Y = Y + v[0, s, h] * np.dot(k[0, s, h] * dec, r[0, t, h])
            assert rel_err(y[0, t, h], Y) < 1e-12
        Sref = s0[0, h] * np.prod(w[0, :, h], axis=0)[None, :]
        for s in range(T):
            Sref = Sref + np.outer(v[0, s, h], k[0, s, h] * np.prod(w[0, s + 1:, h], axis=0))
        assert rel_err(sT[0, h], Sref) < 1e-12


# --- delta rule: exact replace, relaxed replace, Householder -----------------

def _delta_inputs(T, N, seed):
    rng = np.random.default_rng(seed)
    kh = unit_rows(rng.standard_normal((1, T, 1, N)))
    v = rng.standard_normal((1, T, 1, N))
    s0 = rng.standard_normal((1, 1, N, N))
    return rng, kh, v, s0


def test_delta_rule_exact_replace():
    """w = 1, a = -k^, b = k^, k = k^ with unit k^: after the write S_t k^_t = v_t
    and S_t x = S_{t-1} x for x orthogonal to k^_t (the DeltaNet replace:
    Paper Review: RWKV-7 "Goose", section "Background information on delta
    rule"; separate removal and write keys set equal here)."""
    T, N = 12, 16
    rng, kh, v, s0 = _delta_inputs(T, N, 3)
    ones = np.ones_like(kh)
    # read-out along the key just written: y_t = S_t k^_t must equal v_t
    y, _ = oracle.forward(kh, ones, kh, v, -kh, kh, s0=s0)
    assert rel_err(y, v) < 1e-12
    # untouched directions are preserved, token by token
    S = s0
    for t in range(T):
        x = rng.standard_normal(N)
        x -= np.dot(x, kh[0, t, 0]) * kh[0, t, 0]
        sl = lambda z: z[:, t:t + 1]
        _, S_new = oracle.forward(sl(kh), sl(ones), sl(kh), sl(v), sl(-kh), sl(kh), s0=S)
        assert rel_err(S_new[0, 0] @ x, S[0, 0] @ x) < 1e-12
        assert rel_err(S_new[0, 0] @ kh[0, t, 0], v[0, t, 0]) < 1e-12
        S = S_new


def test_relaxed_value_replacement():
    """With a scalar learning rate lr in (0, 1), b = lr k^: S_t k^ = (1 - lr)
    S_{t-1} k^ + v (the relaxed value replacement named in the RWKV-7 "Goose"
    abstract)."""
    T, N = 10, 12
    rng, kh, v, s0 = _delta_inputs(T, N, 5)
    lr = rng.uniform(0.05, 0.95, size=(1, T, 1, 1))
    ones = np.ones_like(kh)
    S = s0
    for t in range(T):
        sl = lambda z: z[:, t:t + 1]
        y, S_new = oracle.forward(sl(kh), sl(ones), sl(kh), sl(v), sl(-kh), sl(kh * lr), s0=S)
        expect = (1.0 - lr[0, t, 0, 0]) * (S[0, 0] @ kh[0, t, 0]) + v[0, t, 0]
        assert rel_err(y[0, 0, 0], expect) < 1e-12
        S = S_new


def test_householder_transition_preserves_norm():
    """w = 1, a = -2k^, b = k^, v = 0: the transition I - 2 k^ k^T is an exact
    Householder reflection, so every state row keeps its Euclidean norm (the
    transition is described as a scaled Householder-like matrix: Paper Review:
    RWKV-7 "Goose", section "The approach")."""
    T, N = 64, 32
    rng, kh, _, s0 = _delta_inputs(T, N, 7)
    ones = np.ones_like(kh)
    zeros = np.zeros_like(kh)
    _, sT = oracle.forward(kh, ones, kh, zeros, -2.0 * kh, kh, s0=s0)
    np.testing.assert_allclose(np.linalg.norm(sT[0, 0], axis=1), np.linalg.norm(s0[0, 0], axis=1),
                               rtol=1e-12)
    # and the reflection is its own inverse: applying the same key twice restores S
    kk = np.repeat(kh[:, :1], 2, axis=1)
    _, s2 = oracle.forward(kk, np.ones_like(kk), kk, np.zeros_like(kk), -2.0 * kk, kk, s0=s0)
    assert rel_err(s2, s0) < 1e-12


def test_state_stays_bounded_without_inputs():
    """Workload recipe (w in (e^-0.6065, 1), a = -k^, b = k^ lr) with v = 0:
    the state must not grow over a long run (eigenvalues in a stable range:
    Paper Review: RWKV-7 "Goose", section "The approach")."""
    B, T, H, N = 1, 4096, 1, 64
    (r, w, k, v, a, b), s0 = recipe(B, T, H, N, seed=13)
    v[:] = 0.0
    S = s0
    n0 = np.linalg.norm(s0)
    for seg in range(0, T, 256):
        sl = lambda z: z[:, seg:seg + 256]
        _, S = oracle.forward(sl(r), sl(w), sl(k), sl(v), sl(a), sl(b), s0=S)
        assert np.linalg.norm(S) <= n0
    assert np.linalg.norm(S) < 1e-3 * n0


# --- structural: chunked form, state passing, step ---------------------------

@pytest.mark.parametrize("L", [1, 4, 16, 64])
def test_chunked_equals_sequential(L):
    B, T, H, N = 2, 150, 2, 16
    (r, w, k, v, a, b), s0 = recipe(B, T, H, N, seed=17)
    y, sT = oracle.forward(r, w, k, v, a, b, s0=s0)
    yc, sTc = oracle.forward_chunked(r, w, k, v, a, b, s0=s0, chunk_len=L)
    assert rel_err(yc, y) < 1e-11
    assert rel_err(sTc, sT) < 1e-11


def test_chunked_equals_sequential_full_width_long_memory():
    """N = 64, chunk 64, w near 1 (the long-context recipe) and a ragged tail."""
    B, T, H, N = 1, 200, 1, 64
    (r, w, k, v, a, b), s0 = recipe(B, T, H, N, seed=19, x_mean=-2.0)
    y, sT = oracle.forward(r, w, k, v, a, b, s0=s0)
    yc, sTc = oracle.forward_chunked(r, w, k, v, a, b, s0=s0, chunk_len=64)
    assert rel_err(yc, y) < 1e-11
    assert rel_err(sTc, sT) < 1e-11


@pytest.mark.parametrize("L", [1, 5, 16, 64])
def test_chunked_backward_equals_sequential(L):
    """The chunk-level backward (adjoint of the chunked form, matrix products
    per chunk) against the sequential C backward, which the central-difference
    pins below hold to the definition.  Ragged tails, nonzero s0 and dsT."""
    B, T, H, N = 1, 83, 2, 16
    (r, w, k, v, a, b), s0 = recipe(B, T, H, N, seed=29)
    rng = np.random.default_rng(31)
    dy = rng.standard_normal((B, T, H, N))
    dsT = rng.standard_normal((B, H, N, N))
    ref = oracle.backward(r, w, k, v, a, b, s0, dy, dsT)
    got = oracle.backward_chunked(r, w, k, v, a, b, s0, dy, dsT, chunk_len=L)
    for name, g, x in zip(("dr", "dw", "dk", "dv", "da", "db", "ds0"), got, ref):
        assert rel_err(g, x) < 1e-11, name


CHUNKED_BWD_MUTANTS = {
    "drop_removal_path_into_ds": ("dSin = dX + dY.T @ Rt + dZ.T @ At", "dSin = dX + dY.T @ Rt"),
    "untransposed_solve": ("dZ = np.linalg.solve(Mt.T, dU)", "dZ = np.linalg.solve(Mt, dU)"),
    "decay_index_shift": ("dgam[:-1] += (dAt * A)[1:]", "dgam += dAt * A"),
    "inclusive_removal_mask": ("dL_ab = (dZ @ U.T) * strict", "dL_ab = (dZ @ U.T) * incl"),
}


@pytest.mark.parametrize("mutant", sorted(CHUNKED_BWD_MUTANTS))
def test_chunked_backward_mutants_are_caught(mutant):
    import inspect
    src = inspect.getsource(oracle.backward_chunked)
    old, new = CHUNKED_BWD_MUTANTS[mutant]
    assert src.count(old) == 1, "mutation anchor not found"
    ns = dict(np=np, _f64=oracle._f64)
    exec(src.replace(old, new), ns)
    B, T, H, N = 1, 19, 1, 8
    (r, w, k, v, a, b), s0 = recipe(B, T, H, N, seed=37)
    rng = np.random.default_rng(41)
    dy = rng.standard_normal((B, T, H, N))
    dsT = rng.standard_normal((B, H, N, N))
    ref = oracle.backward(r, w, k, v, a, b, s0, dy, dsT)
    got = ns["backward_chunked"](r, w, k, v, a, b, s0, dy, dsT, chunk_len=8)
    assert max(rel_err(g, x) for g, x in zip(got, ref)) > 1e-6, f"mutant {mutant} slipped through"


def test_state_passing_split():
    B, T, H, N = 2, 37, 3, 8
    (r, w, k, v, a, b), s0 = recipe(B, T, H, N, seed=23)
    y, sT = oracle.forward(r, w, k, v, a, b, s0=s0)
    T1 = 15
    y1, s1 = oracle.forward(*(x[:, :T1] for x in (r, w, k, v, a, b)), s0=s0)
    y2, s2 = oracle.forward(*(x[:, T1:] for x in (r, w, k, v, a, b)), s0=s1)
    np.testing.assert_array_equal(np.concatenate([y1, y2], axis=1), y)
    np.testing.assert_array_equal(s2, sT)


def test_summary_is_the_affine_map_of_the_state():
    """The final state from any entry state is S_in M + E: checked against the
    C forward run from a random S_in (a reversed product order, a transposed
    M or a dropped a b^T term breaks it); T = 0 is the identity map."""
    B, T, H, N = 2, 23, 2, 8
    (r, w, k, v, a, b), _ = recipe(B, T, H, N, seed=43)
    S_in = np.random.default_rng(47).standard_normal((B, H, N, N))
    E, M = oracle.forward_summary(r, w, k, v, a, b)
    _, sT = oracle.forward(r, w, k, v, a, b, s0=S_in)
    assert rel_err(S_in @ M + E, sT) < 1e-12
    E0, M0 = oracle.forward_summary(*(x[:, :0] for x in (r, w, k, v, a, b)))
    np.testing.assert_array_equal(E0, 0.0)
    np.testing.assert_array_equal(M0, np.broadcast_to(np.eye(N), M0.shape))


def test_summary_closed_forms():
    """a = b = 0: M is the diagonal of the decay products.  w = 1 with
    a = -k_hat, b = 2 k_hat: every transition is a Householder reflection, so M
    is orthogonal (M M^T = I) with determinant (-1)^T."""
    B, T, H, N = 1, 9, 2, 8
    (r, w, k, v, a, b), _ = recipe(B, T, H, N, seed=53)
    zero = np.zeros_like(a)
    _, M = oracle.forward_summary(r, w, k, v, zero, zero)
    for h in range(H):
        np.testing.assert_allclose(M[0, h], np.diag(np.prod(w[0, :, h], axis=0)), rtol=1e-14, atol=0)
    kh = unit_rows(np.random.default_rng(59).standard_normal((B, T, H, N)))
    _, M = oracle.forward_summary(r, np.ones_like(w), k, v, -kh, 2.0 * kh)
    for h in range(H):
        np.testing.assert_allclose(M[0, h] @ M[0, h].T, np.eye(N), atol=1e-13)
        assert abs(np.linalg.det(M[0, h]) - (-1.0) ** T) < 1e-12


def test_compose_states_match_prefix_forwards():
    """Composing the summaries of consecutive stretches (ragged lengths, one
    empty) gives the state after every prefix, and the final state."""
    B, T, H, N = 2, 41, 2, 8
    (r, w, k, v, a, b), s0 = recipe(B, T, H, N, seed=61)
    cuts = [0, 13, 13, 30, 41]
    sums = []
    for c0, c1 in zip(cuts[:-1], cuts[1:]):
        E, M = oracle.forward_summary(*(x[:, c0:c1] for x in (r, w, k, v, a, b)))
        sums.append(np.stack([E, M]))
    states = oracle.compose_states(np.stack(sums), s0)
    assert states.shape == (len(cuts), B, H, N, N)
    np.testing.assert_array_equal(states[0], s0)
    for i, c in enumerate(cuts[1:], start=1):
        _, s_pref = oracle.forward(*(x[:, :c] for x in (r, w, k, v, a, b)), s0=s0)
        assert rel_err(states[i], s_pref) < 1e-12, i
    np.testing.assert_array_equal(oracle.compose_states(np.zeros((0, 2, B, H, N, N)))[0], 0.0)


def test_state_gradient_is_the_backward_ds0():
    """The state-gradient sweep equals ds0 of the C backward (an independent
    implementation pinned by central differences), for any k, v, s0."""
    B, T, H, N = 2, 29, 2, 8
    (r, w, k, v, a, b), s0 = recipe(B, T, H, N, seed=73)
    rng = np.random.default_rng(79)
    dy = rng.standard_normal((B, T, H, N))
    dsT = rng.standard_normal((B, H, N, N))
    g = oracle.state_gradient(r, w, a, b, dy, dsT)
    assert rel_err(g, oracle.backward(r, w, k, v, a, b, s0, dy, dsT)[6]) < 1e-12
    k2, v2 = rng.standard_normal(k.shape), rng.standard_normal(v.shape)
    assert rel_err(g, oracle.backward(r, w, k2, v2, a, b, None, dy, dsT)[6]) < 1e-12
    np.testing.assert_array_equal(oracle.state_gradient(*(x[:, :0] for x in (r, w, a, b, dy)), dsT), dsT)


def test_compose_adjoints_match_suffix_backwards():
    """Chaining (M_k, F_k) of consecutive stretches, last first, gives dL/dS
    before every stretch: ds0 of the C backward over the suffix from there."""
    B, T, H, N = 1, 37, 2, 8
    (r, w, k, v, a, b), s0 = recipe(B, T, H, N, seed=83)
    rng = np.random.default_rng(89)
    dy = rng.standard_normal((B, T, H, N))
    dsT = rng.standard_normal((B, H, N, N))
    cuts = [0, 11, 11, 25, 37]
    sums, F = [], []
    for c0, c1 in zip(cuts[:-1], cuts[1:]):
        sl = lambda x: x[:, c0:c1]
        E, M = oracle.forward_summary(*map(sl, (r, w, k, v, a, b)))
        sums.append(np.stack([E, M]))
        F.append(oracle.state_gradient(*map(sl, (r, w, a, b, dy))))
    adj = oracle.compose_adjoints(np.stack(sums), np.stack(F), dsT)
    np.testing.assert_array_equal(adj[-1], dsT)
    for i, c in enumerate(cuts[:-1]):
        sl = lambda x: x[:, c:]
        ref = oracle.backward(*map(sl, (r, w, k, v, a, b)), s0, sl(dy), dsT)[6]
        assert rel_err(adj[i], ref) < 1e-12, i


ADJOINT_MUTANTS = {
    "untransposed_transition": ("state_gradient", "G = G @ A.T", "G = G @ A"),
    "readout_after_transition": ("state_gradient",
                                 "G = G + np.outer(dy[bb, t, h], r[bb, t, h])\n                A = np.diag(w[bb, t, h]) + np.outer(a[bb, t, h], b[bb, t, h])\n                G = G @ A.T",
                                 "A = np.diag(w[bb, t, h]) + np.outer(a[bb, t, h], b[bb, t, h])\n                G = G @ A.T\n                G = G + np.outer(dy[bb, t, h], r[bb, t, h])"),
    "untransposed_summary": ("compose_adjoints", "np.swapaxes(summaries[kk, 1], -1, -2)", "summaries[kk, 1]"),
}


@pytest.mark.parametrize("mutant", sorted(ADJOINT_MUTANTS))
def test_adjoint_mutants_are_caught(mutant):
    import inspect
    fn, old, new = ADJOINT_MUTANTS[mutant]
    src = inspect.getsource(getattr(oracle, fn))
    assert src.count(old) == 1, "mutation anchor not found"
    ns = dict(np=np, _f64=oracle._f64)
    exec(src.replace(old, new), ns)
    B, T, H, N = 1, 9, 1, 8
    (r, w, k, v, a, b), s0 = recipe(B, T, H, N, seed=97)
    rng = np.random.default_rng(101)
    dy = rng.standard_normal((B, T, H, N))
    dsT = rng.standard_normal((B, H, N, N))
    ref = oracle.backward(r, w, k, v, a, b, s0, dy, dsT)[6]
    if fn == "state_gradient":
        got = ns["state_gradient"](r, w, a, b, dy, dsT)
    else:
        E, M = oracle.forward_summary(r, w, k, v, a, b)
        F = oracle.state_gradient(r, w, a, b, dy)
        got = ns["compose_adjoints"](np.stack([E, M])[None], F[None], dsT)[0]
    assert rel_err(got, ref) > 1e-6, f"mutant {mutant} slipped through"


SUMMARY_MUTANTS = {
    "reversed_product": ("P = P @ (np.diag(", "P = (np.diag("),
    "compose_left_multiply": ("states[kk] @ summaries[kk, 1]", "summaries[kk, 1] @ states[kk]"),
}


@pytest.mark.parametrize("mutant", sorted(SUMMARY_MUTANTS))
def test_summary_mutants_are_caught(mutant):
    import inspect
    fn = "forward_summary" if mutant == "reversed_product" else "compose_states"
    src = inspect.getsource(getattr(oracle, fn))
    old, new = SUMMARY_MUTANTS[mutant]
    assert src.count(old) == 1, "mutation anchor not found"
    if mutant == "reversed_product":
        new_src = src.replace(old, new).replace("b[bb, t, h]))", "b[bb, t, h])) @ P")
    else:
        new_src = src.replace(old, new)
    ns = dict(np=np, _f64=oracle._f64, forward=oracle.forward)
    exec(new_src, ns)
    B, T, H, N = 1, 7, 1, 8
    (r, w, k, v, a, b), s0 = recipe(B, T, H, N, seed=67)
    S_in = np.random.default_rng(71).standard_normal((B, H, N, N))
    if mutant == "reversed_product":
        E, M = ns["forward_summary"](r, w, k, v, a, b)
        _, sT = oracle.forward(r, w, k, v, a, b, s0=S_in)
        assert rel_err(S_in @ M + E, sT) > 1e-6
    else:
        E, M = oracle.forward_summary(r, w, k, v, a, b)
        states = ns["compose_states"](np.stack([E, M])[None], S_in)
        _, sT = oracle.forward(r, w, k, v, a, b, s0=S_in)
        assert rel_err(states[1], sT) > 1e-6


def test_step_equals_forward_t1():
    B, H, N = 3, 2, 8
    (r, w, k, v, a, b), s0 = recipe(B, 1, H, N, seed=29)
    y, sT = oracle.forward(r, w, k, v, a, b, s0=s0)
    ys, Ss = oracle.step(*(x[:, 0] for x in (r, w, k, v, a, b)), s0)
    np.testing.assert_array_equal(ys, y[:, 0])
    np.testing.assert_array_equal(Ss, sT)


def test_heads_and_batches_independent():
    """Heads are independent recurrences: permuting heads permutes outputs."""
    B, T, H, N = 2, 9, 3, 8
    (r, w, k, v, a, b), s0 = recipe(B, T, H, N, seed=31)
    y, sT = oracle.forward(r, w, k, v, a, b, s0=s0)
    perm = [2, 0, 1]
    yp, sTp = oracle.forward(*(x[:, :, perm] for x in (r, w, k, v, a, b)), s0=s0[:, perm])
    np.testing.assert_array_equal(yp, y[:, :, perm])
    np.testing.assert_array_equal(sTp, sT[:, perm])


def test_zero_initial_state_is_default():
    B, T, H, N = 1, 5, 1, 4
    (r, w, k, v, a, b), _ = recipe(B, T, H, N, seed=37)
    y0, s0T = oracle.forward(r, w, k, v, a, b, s0=None)
    y1, s1T = oracle.forward(r, w, k, v, a, b, s0=np.zeros((B, H, N, N)))
    np.testing.assert_array_equal(y0, y1)
    np.testing.assert_array_equal(s0T, s1T)


# --- backward: central finite differences ------------------------------------

def _loss(r, w, k, v, a, b, s0, dy, dsT):
    y, sT = oracle.forward(r, w, k, v, a, b, s0=s0)
    return float(np.sum(dy * y) + np.sum(dsT * sT))


@pytest.mark.parametrize("N,T", [(8, 16), (64, 16)])
def test_backward_matches_central_differences(N, T):
    B, H = 1, 1
    (r, w, k, v, a, b), s0 = recipe(B, T, H, N, seed=41)
    rng = np.random.default_rng(43)
    dy = rng.standard_normal((B, T, H, N))
    dsT = rng.standard_normal((B, H, N, N))
    grads = oracle.backward(r, w, k, v, a, b, s0, dy, dsT)
    tensors = [r, w, k, v, a, b, s0]
    h = 1e-6
    for idx, (x, g) in enumerate(zip(tensors, grads)):
        flat = x.reshape(-1)
        # every coordinate for N = 8; a fixed random subset for N = 64
        coords = np.arange(flat.size) if N <= 8 else rng.choice(flat.size, 96, replace=False)
        fd = np.empty(len(coords))
        for n, c in enumerate(coords):
            old = flat[c]
            flat[c] = old + h
            lp = _loss(*tensors, dy, dsT)
            flat[c] = old - h
            lm = _loss(*tensors, dy, dsT)
            flat[c] = old
            fd[n] = (lp - lm) / (2 * h)
        got = g.reshape(-1)[coords]
        scale = np.max(np.abs(got)) + 1e-30
        assert np.max(np.abs(got - fd)) / scale < 1e-7, f"input #{idx}"


def test_backward_zero_dsT_default():
    B, T, H, N = 1, 6, 2, 4
    (r, w, k, v, a, b), s0 = recipe(B, T, H, N, seed=47)
    dy = np.random.default_rng(1).standard_normal((B, T, H, N))
    g0 = oracle.backward(r, w, k, v, a, b, s0, dy, None)
    g1 = oracle.backward(r, w, k, v, a, b, s0, dy, np.zeros((B, H, N, N)))
    for x, y in zip(g0, g1):
        np.testing.assert_array_equal(x, y)


# --- the pins catch planted mistakes -----------------------------------------

MUTANTS = {
    "drop_write_term": ("p * bt[j] + vi * kt[j];\n                    acc", "p * bt[j];\n                    acc"),
    "removal_sign": ("S[j] * wt[j] + p * bt[j]", "S[j] * wt[j] - p * bt[j]"),
    "read_before_write": ("S[j] = S[j] * wt[j] + p * bt[j] + vi * kt[j];\n                    acc += S[j] * rt[j];",
                          "acc += S[j] * rt[j];\n                    S[j] = S[j] * wt[j] + p * bt[j] + vi * kt[j];"),
    "transposed_removal_key": ("p += S[j] * at[j];", "p += S[j] * at[i];"),
    "decay_on_value_axis": ("S[j] = S[j] * wt[j]", "S[j] = S[j] * wt[i]"),
}


def _pins_pass(lib):
    i = ctypes.c_int
    DP = ctypes.POINTER(ctypes.c_double)
    lib.oracle_forward.argtypes = [i, i, i, i] + [DP] * 9

    def fwd(r, w, k, v, a, b, s0):
        arrs = [np.ascontiguousarray(x, dtype=np.float64) for x in (r, w, k, v, a, b, s0)]
        B, T, H, N = arrs[0].shape
        y = np.empty((B, T, H, N))
        sT = np.empty((B, H, N, N))
        lib.oracle_forward(B, T, H, N, *[x.ctypes.data_as(DP) for x in arrs + [y, sT]])
        return y, sT

    ok = True
    for name in ("hand_n1_t3.txt", "hand_n2_t2.txt"):
        g = load(name)
        y, sT = fwd(g["r"], g["w"], g["k"], g["v"], g["a"], g["b"], g["s0"])
        ok &= np.array_equal(y, g["y"]) and np.array_equal(sT, g["sT"])
    T, N = 8, 8
    rng, kh, v, s0 = _delta_inputs(T, N, 3)
    y, _ = fwd(kh, np.ones_like(kh), kh, v, -kh, kh, s0)
    ok &= rel_err(y, v) < 1e-12
    return ok


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_planted_mistakes_are_caught(mutant, tmp_path):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "wkv7_oracle.c")).read()
    old, new = MUTANTS[mutant]
    assert src.count(old) == 1, "mutation anchor not found"
    path = tmp_path / "mut.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "mut.so"
    subprocess.check_call(["gcc", "-O1", "-fPIC", "-shared", "-std=c99", str(path), "-o", str(so), "-lm"])
    assert not _pins_pass(ctypes.CDLL(str(so))), f"mutant {mutant} slipped through the pins"


def test_unmutated_oracle_passes_mutation_harness():
    assert _pins_pass(oracle._load())

"""fp64 CPU oracle of the WKV7 recurrence.

TEST INFRASTRUCTURE ONLY: imported by the test suite, by the smoke check and
by the benchmark's CPU-baseline leg, never by the library's product path.  It
shares no code with the CUDA library; the only thing both sides use is the
seeded input generator, which holds none of the method's arithmetic.

What it computes, per batch b and head h (S is N x N, row i = value index,
column j = key index):

    S_t = S_{t-1} (diag(w_t) + a_t b_t^T) + v_t k_t^T,    y_t = S_t r_t

(the "diagonal plus rank one" generalised delta rule: Paper Review: RWKV-7
"Goose" with Expressive Dynamic State Evolution, sections "Architecture" and
"The approach"; vector decay, per-channel in-context learning rate and
separate removal / write keys: Elamur Research summary of RWKV-7 "Goose",
section "Summary").

* ``forward`` / ``backward`` call the plain C loops in ``wkv7_oracle.c``
  (fp64, one scalar loop per state row, OpenMP over heads).
* ``step`` is ``forward`` with T = 1 (a decode step is one token of the same
  recurrence: constant time and memory per token, RWKV-7 "Goose" abstract).
* ``forward_chunked`` is the chunked (parallel-in-time) form, written with
  numpy matrix products in fp64.  The pages only say that training stays
  parallelisable (RWKV-7 "Goose" abstract) and cite chunk-wise delta-rule
  parallelisation by title; the algebra here is our own derivation from the
  recurrence, applied chunk by chunk in the order of its definition.
* ``backward_chunked`` is the reverse-mode derivative of ``forward_chunked``,
  chunk by chunk (last chunk first), each line the adjoint of one line of the
  forward definition; pinned against ``backward``.
* ``forward_summary`` / ``compose_states``: the recurrence is affine in the
  state (the transition diag(w_t) + a_t b_t^T does not depend on S: paper
  review, section "Architecture"), so a stretch of tokens maps S_in to
  S_in M + E with M the ordered product of its transitions and E its final
  state from S = 0.  Both are written as those definitions: the product taken
  token by token, E from ``forward``.
* ``state_gradient`` / ``compose_adjoints``: the same affinity backwards.
  dL/dS before a stretch is (dL/dS after it) M^T + F, F being the stretch's
  own contribution (its outputs' gradient with nothing after it).
  ``state_gradient`` is the reverse sweep of the state gradient alone, token
  by token (the adjoint of S_t = S_{t-1} A_t + v_t k_t^T, y_t = S_t r_t, taken
  for S only): G <- G + dy_t r_t^T, then G <- G A_t^T.  ``compose_adjoints``
  chains those maps over stretches, last stretch first.
* ``timemix_out`` / ``forward_timemix``: the output epilogue of the time-mix
  block (the current-token term, the per-head normalisation and the gate; Paper
  Review, section "The approach").  The pages describe it in words only, so it
  is our plainest reading of them, written out token by token.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wkv7_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libwkv7_oracle.so")
_lib = None

_DP = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (fp64, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        i = ctypes.c_int
        lib.oracle_forward.argtypes = [i, i, i, i] + [_DP] * 9
        lib.oracle_forward.restype = None
        lib.oracle_backward.argtypes = [i, i, i, i] + [_DP] * 16
        lib.oracle_backward.restype = None
        lib.oracle_max_threads.restype = ctypes.c_int
        lib.oracle_set_threads.argtypes = [i]
        _lib = lib
    return _lib


def max_threads() -> int:
    return _load().oracle_max_threads()


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def _f64(x):
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(x):
    return None if x is None else x.ctypes.data_as(_DP)


def forward(r, w, k, v, a, b, s0=None):
    """y [B,T,H,N] and sT [B,H,N,N] in fp64 for inputs shaped [B,T,H,N]."""
    lib = _load()
    r, w, k, v, a, b = (_f64(x) for x in (r, w, k, v, a, b))
    B, T, H, N = r.shape
    for x in (w, k, v, a, b):
        assert x.shape == r.shape
    s0 = None if s0 is None else _f64(s0)
    if s0 is not None:
        assert s0.shape == (B, H, N, N)
    y = np.empty((B, T, H, N))
    sT = np.empty((B, H, N, N))
    lib.oracle_forward(B, T, H, N, *map(_ptr, (r, w, k, v, a, b, s0, y, sT)))
    return y, sT


def step(r, w, k, v, a, b, state):
    """One decode token: inputs [B,H,N], state [B,H,N,N] -> (y [B,H,N], new state)."""
    expand = [np.asarray(x)[:, None] for x in (r, w, k, v, a, b)]
    y, sT = forward(*expand, s0=state)
    return y[:, 0], sT


def backward(r, w, k, v, a, b, s0, dy, dsT=None):
    """Gradients (dr, dw, dk, dv, da, db, ds0) of sum(dy*y) + sum(dsT*sT)."""
    lib = _load()
    r, w, k, v, a, b, dy = (_f64(x) for x in (r, w, k, v, a, b, dy))
    B, T, H, N = r.shape
    s0 = None if s0 is None else _f64(s0)
    dsT = None if dsT is None else _f64(dsT)
    grads = [np.empty((B, T, H, N)) for _ in range(6)]
    ds0 = np.empty((B, H, N, N))
    lib.oracle_backward(B, T, H, N, *map(_ptr, (r, w, k, v, a, b, s0, dy, dsT)),
                        *map(_ptr, grads), _ptr(ds0))
    return (*grads, ds0)


def forward_chunked(r, w, k, v, a, b, s0=None, chunk_len=64):
    """Chunked form of ``forward`` (fp64, w > 0), chunk by chunk.

    Inside a chunk of L tokens (local index t = 0..L-1) starting from state
    S_in, with gamma_t = prod_{m<=t} w_m (elementwise, gamma_{-1} = 1):

      a~_t = a_t * gamma_{t-1},  r~_t = r_t * gamma_t,
      b^_s = b_s / gamma_s,      k^_s = k_s / gamma_s
      L_ab[t,s] = a~_t . b^_s,  L_ak[t,s] = a~_t . k^_s      (s <  t)
      L_rb[t,s] = r~_t . b^_s,  L_rk[t,s] = r~_t . k^_s      (s <= t)
      U = (I - L_ab)^{-1} (A~ S_in^T + L_ak V)     rows u_t = S_{t-1} a_t
      Y = R~ S_in^T + L_rb U + L_rk V
      S_out = S_in diag(gamma_{L-1}) + U^T B- + V^T K-,
          B-_s = b_s * gamma_{L-1} / gamma_s,  K-_s = k_s * gamma_{L-1} / gamma_s

    This follows from unrolling the recurrence inside the chunk:
      S_t = S_in diag(gamma_t) + sum_{s<=t} (u_s b_s^T + v_s k_s^T) diag(gamma_t / gamma_s).
    """
    r, w, k, v, a, b = (_f64(x) for x in (r, w, k, v, a, b))
    B, T, H, N = r.shape
    y = np.empty((B, T, H, N))
    sT = np.empty((B, H, N, N))
    for bb in range(B):
        for h in range(H):
            S = np.zeros((N, N)) if s0 is None else _f64(s0)[bb, h].copy()
            for c0 in range(0, T, chunk_len):
                c1 = min(T, c0 + chunk_len)
                L = c1 - c0
                R, W, K, V, A, Bm = (x[bb, c0:c1, h] for x in (r, w, k, v, a, b))
                gam = np.cumprod(W, axis=0)
                gam_prev = np.vstack([np.ones((1, N)), gam[:-1]])
                At = A * gam_prev
                Rt = R * gam
                Bh = Bm / gam
                Kh = K / gam
                strict = np.tril(np.ones((L, L)), -1)
                incl = np.tril(np.ones((L, L)), 0)
                L_ab = (At @ Bh.T) * strict
                L_ak = (At @ Kh.T) * strict
                L_rb = (Rt @ Bh.T) * incl
                L_rk = (Rt @ Kh.T) * incl
                U = np.linalg.solve(np.eye(L) - L_ab, At @ S.T + L_ak @ V)
                y[bb, c0:c1, h] = Rt @ S.T + L_rb @ U + L_rk @ V
                Bbar = Bh * gam[-1]
                Kbar = Kh * gam[-1]
                S = S * gam[-1][None, :] + U.T @ Bbar + V.T @ Kbar
            sT[bb, h] = S
    return y, sT


def backward_chunked(r, w, k, v, a, b, s0, dy, dsT=None, chunk_len=64):
    """Chunked form of ``backward`` (fp64, w > 0): the reverse-mode derivative
    of ``forward_chunked``, taken chunk by chunk, last chunk first.

    With the chunk quantities of ``forward_chunked`` (S = S_in, M = I - L_ab,
    Z = A~ S^T + L_ak V, U = M^{-1} Z, X = S + U^T B^ + V^T K^, S_out =
    X diag(gamma_{L-1})) and the upstream gradients dY (rows t) and dS_out:

      dX  = dS_out diag(gamma_{L-1});   dgamma_{L-1} += sum_i X * dS_out
      dS  = dX + dY^T R~ + dZ^T A~;     dU  = B^ dX^T + L_rb^T dY
      dZ  = M^{-T} dU
      dV  = K^ dX^T + L_rk^T dY + L_ak^T dZ
      dL_ab = (dZ U^T) strict,  dL_ak = (dZ V^T) strict,
      dL_rb = (dY U^T) incl,    dL_rk = (dY V^T) incl
      dA~ = dZ S + dL_ab B^ + dL_ak K^;    dR~ = dY S + dL_rb B^ + dL_rk K^
      dB^ = U dX + dL_ab^T A~ + dL_rb^T R~;  dK^ = V dX + dL_ak^T A~ + dL_rk^T R~

    then through the decay scalings (a~ = a gamma_{t-1}, r~ = r gamma_t,
    b^ = b / gamma_s, k^ = k / gamma_s) and gamma_t = prod_{m<=t} w_m.
    dS becomes dS_out of the previous chunk; at the start it is ds0.  Every
    line is the adjoint of one line of the forward definition.
    """
    r, w, k, v, a, b, dy = (_f64(x) for x in (r, w, k, v, a, b, dy))
    B, T, H, N = r.shape
    grads = [np.zeros((B, T, H, N)) for _ in range(6)]   # dr dw dk dv da db
    ds0 = np.zeros((B, H, N, N))
    for bb in range(B):
        for h in range(H):
            # forward pass, keeping the state entering each chunk
            S = np.zeros((N, N)) if s0 is None else _f64(s0)[bb, h].copy()
            starts = list(range(0, T, chunk_len))
            s_in = []
            for c0 in starts:
                c1 = min(T, c0 + chunk_len)
                s_in.append(S.copy())
                R, W, K, V, A, Bm = (x[bb, c0:c1, h] for x in (r, w, k, v, a, b))
                gam = np.cumprod(W, axis=0)
                gam_prev = np.vstack([np.ones((1, N)), gam[:-1]])
                L = c1 - c0
                strict = np.tril(np.ones((L, L)), -1)
                At, Bh, Kh = A * gam_prev, Bm / gam, K / gam
                L_ab = (At @ Bh.T) * strict
                L_ak = (At @ Kh.T) * strict
                U = np.linalg.solve(np.eye(L) - L_ab, At @ S.T + L_ak @ V)
                S = (S + U.T @ Bh + V.T @ Kh) * gam[-1][None, :]
            dS = np.zeros((N, N)) if dsT is None else _f64(dsT)[bb, h].copy()
            for ci in range(len(starts) - 1, -1, -1):
                c0 = starts[ci]
                c1 = min(T, c0 + chunk_len)
                L = c1 - c0
                S = s_in[ci]
                R, W, K, V, A, Bm = (x[bb, c0:c1, h] for x in (r, w, k, v, a, b))
                dY = dy[bb, c0:c1, h]
                # recompute the chunk
                gam = np.cumprod(W, axis=0)
                gam_prev = np.vstack([np.ones((1, N)), gam[:-1]])
                strict = np.tril(np.ones((L, L)), -1)
                incl = np.tril(np.ones((L, L)), 0)
                At, Rt, Bh, Kh = A * gam_prev, R * gam, Bm / gam, K / gam
                L_ab = (At @ Bh.T) * strict
                L_ak = (At @ Kh.T) * strict
                L_rb = (Rt @ Bh.T) * incl
                L_rk = (Rt @ Kh.T) * incl
                Mt = np.eye(L) - L_ab
                U = np.linalg.solve(Mt, At @ S.T + L_ak @ V)
                X = S + U.T @ Bh + V.T @ Kh
                # adjoints
                gL = gam[-1]
                dX = dS * gL[None, :]
                dgam = np.zeros((L, N))
                dgam[-1] += (X * dS).sum(axis=0)
                dU = Bh @ dX.T + L_rb.T @ dY
                dZ = np.linalg.solve(Mt.T, dU)
                dSin = dX + dY.T @ Rt + dZ.T @ At
                dV = Kh @ dX.T + L_rk.T @ dY + L_ak.T @ dZ
                dL_ab = (dZ @ U.T) * strict
                dL_ak = (dZ @ V.T) * strict
                dL_rb = (dY @ U.T) * incl
                dL_rk = (dY @ V.T) * incl
                dAt = dZ @ S + dL_ab @ Bh + dL_ak @ Kh
                dRt = dY @ S + dL_rb @ Bh + dL_rk @ Kh
                dBh = U @ dX + dL_ab.T @ At + dL_rb.T @ Rt
                dKh = V @ dX + dL_ak.T @ At + dL_rk.T @ Rt
                # decay scalings
                da = dAt * gam_prev
                dr = dRt * gam
                db = dBh / gam
                dk = dKh / gam
                dgam += dRt * R - dBh * Bh / gam - dKh * Kh / gam
                dgam[:-1] += (dAt * A)[1:]
                # gamma_t = prod_{m<=t} w_m: dw_m = sum_{t>=m} dgamma_t gamma_t / w_m
                dw = np.cumsum((dgam * gam)[::-1], axis=0)[::-1] / W
                for g, x in zip(grads, (dr, dw, dk, dV, da, db)):
                    g[bb, c0:c1, h] = x
                dS = dSin
            ds0[bb, h] = dS
    return (*grads, ds0)


def forward_summary(r, w, k, v, a, b):
    """(E, M), each [B,H,N,N] fp64, of a stretch shaped [B,T,H,N]:
    M = (diag(w_1) + a_1 b_1^T)(diag(w_2) + a_2 b_2^T)...(diag(w_T) + a_T b_T^T)
    (right-multiplied in token order, as S_t = S_{t-1} A_t applies them), and
    E = the final state of ``forward`` from S = 0.  T = 0 gives E = 0, M = I."""
    r, w, k, v, a, b = (_f64(x) for x in (r, w, k, v, a, b))
    B, T, H, N = r.shape
    M = np.empty((B, H, N, N))
    for bb in range(B):
        for h in range(H):
            P = np.eye(N)
            for t in range(T):
                P = P @ (np.diag(w[bb, t, h]) + np.outer(a[bb, t, h], b[bb, t, h]))
            M[bb, h] = P
    if T == 0:
        return np.zeros((B, H, N, N)), M
    _, E = forward(r, w, k, v, a, b, None)
    return E, M


def compose_states(summaries, s0=None):
    """states [nseg+1,B,H,N,N] from summaries [nseg,2,B,H,N,N] ([E; M] each):
    states[0] = s0 (or 0), states[k+1] = states[k] M_k + E_k."""
    summaries = _f64(summaries)
    nseg, _, B, H, N, _ = summaries.shape
    states = np.empty((nseg + 1, B, H, N, N))
    states[0] = 0.0 if s0 is None else _f64(s0)
    for kk in range(nseg):
        states[kk + 1] = states[kk] @ summaries[kk, 1] + summaries[kk, 0]
    return states


def state_gradient(r, w, a, b, dy, dsT=None):
    """dL/dS_0 [B,H,N,N] fp64 of L = sum(dy * y) + sum(dsT * S_T) for a stretch
    shaped [B,T,H,N]: the reverse sweep G_T = dsT (or 0), then for t = T-1..0
    G <- G + dy_t r_t^T and G <- G (diag(w_t) + a_t b_t^T)^T (the adjoint of
    S_t = S_{t-1} A_t + ..., y_t = S_t r_t, for the state alone).  k, v and the
    initial state play no part."""
    r, w, a, b, dy = (_f64(x) for x in (r, w, a, b, dy))
    B, T, H, N = r.shape
    out = np.empty((B, H, N, N))
    for bb in range(B):
        for h in range(H):
            G = np.zeros((N, N)) if dsT is None else _f64(dsT)[bb, h].copy()
            for t in range(T - 1, -1, -1):
                G = G + np.outer(dy[bb, t, h], r[bb, t, h])
                A = np.diag(w[bb, t, h]) + np.outer(a[bb, t, h], b[bb, t, h])
                G = G @ A.T
            out[bb, h] = G
    return out


def compose_adjoints(summaries, F, dsT=None):
    """adj [nseg+1,B,H,N,N] for consecutive stretches with summaries
    [nseg,2,B,H,N,N] ([E; M] each) and own state gradients F [nseg,B,H,N,N]:
    adj[nseg] = dsT (or 0), adj[k] = adj[k+1] M_k^T + F_k (adj[k] = dL/dS
    before stretch k)."""
    summaries, F = _f64(summaries), _f64(F)
    nseg, _, B, H, N, _ = summaries.shape
    adj = np.empty((nseg + 1, B, H, N, N))
    adj[nseg] = 0.0 if dsT is None else _f64(dsT)
    for kk in range(nseg - 1, -1, -1):
        adj[kk] = adj[kk + 1] @ np.swapaxes(summaries[kk, 1], -1, -2) + F[kk]
    return adj


def timemix_out(y, r, k, v, rho, gamma=None, beta=None, g=None, eps=1e-5):
    """Output epilogue of the time-mix block, fp64, for per-token tensors
    [B,T,H,N] and per-head parameters [H,N].  Paper Review: RWKV-7 "Goose"
    with Expressive Dynamic State Evolution, section "The approach": after the
    state update the receptance reads the state (y_t = S_t r_t, from
    ``forward``); the block also attends to the current token directly,
    without that token being stored in the state; the result is normalised,
    the heads are combined, gated, and a linear layer follows.  The pages give
    no formula; this is the plainest reading of those words:

        o_t   = y_t + (sum_j r_t[j] rho[j] k_t[j]) v_t     (current-token term)
        mu_t  = mean_i o_t[i],  var_t = mean_i (o_t[i] - mu_t)^2   (per head)
        z_t   = g_t * (gamma * (o_t - mu_t) / sqrt(var_t + eps) + beta)

    The heads are combined by concatenation (the [B,T,H,N] layout already is
    it); the gate g arrives as values (its projection, like the final linear
    layer, needs trained weights).  gamma / beta / g default to 1 / 0 / 1."""
    y, r, k, v = (_f64(x) for x in (y, r, k, v))
    B, T, H, N = y.shape
    rho = _f64(rho)
    gamma = np.ones((H, N)) if gamma is None else _f64(gamma)
    beta = np.zeros((H, N)) if beta is None else _f64(beta)
    g = np.ones((B, T, H, N)) if g is None else _f64(g)
    z = np.empty((B, T, H, N))
    for bb in range(B):
        for t in range(T):
            for h in range(H):
                bonus = float(np.sum(r[bb, t, h] * rho[h] * k[bb, t, h]))
                o = y[bb, t, h] + bonus * v[bb, t, h]
                mu = float(np.sum(o)) / N
                var = float(np.sum((o - mu) ** 2)) / N
                z[bb, t, h] = g[bb, t, h] * (gamma[h] * (o - mu) / np.sqrt(var + eps) + beta[h])
    return z


def forward_timemix(r, w, k, v, a, b, s0, rho, gamma=None, beta=None, g=None, eps=1e-5):
    """(z, sT): ``forward`` followed by ``timemix_out`` on its y."""
    y, sT = forward(r, w, k, v, a, b, s0=s0)
    return timemix_out(y, r, k, v, rho, gamma, beta, g, eps), sT

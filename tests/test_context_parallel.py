"""The sequence-parallel forward's and backward's host logic on CPU: gloo ranks
(one process each) hold consecutive stretches of one sequence, exchange their
summaries (and, backward, their own state gradients) by all-gather and compose
their entry states (and the state gradients after their stretches).  The
per-rank compute is the fp64 oracle, injected through ``StretchOps``, so the
test checks the orchestration (rank order = time order, the gathers, which
composed state each rank takes) against the oracle's forward and backward
over the whole sequence."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from linear_rnn_sequence_wkv7_b200 import inputs
from linear_rnn_sequence_wkv7_b200.context_parallel import (StretchOps, backward_context_parallel,
                                                            forward_context_parallel, split_lengths)
from linear_rnn_sequence_wkv7_b200.dist import Dist


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _np(t):
    return None if t is None else t.detach().cpu().numpy()


def oracle_ops():
    def summary(r, w, k, v, a, b):
        E, M = oracle.forward_summary(*map(_np, (r, w, k, v, a, b)))
        return torch.from_numpy(np.stack([E, M])), None

    def compose(sums, s0):
        return torch.from_numpy(oracle.compose_states(_np(sums), _np(s0)))

    def forward(r, w, k, v, a, b, s_in, ctx):
        y, _ = oracle.forward(*map(_np, (r, w, k, v, a, b)), s0=_np(s_in))
        return torch.from_numpy(y)

    def state_gradient(r, w, a, b, dy):
        return torch.from_numpy(oracle.state_gradient(*map(_np, (r, w, a, b, dy))))

    def compose_adjoints(sums, F, dsT):
        return torch.from_numpy(oracle.compose_adjoints(_np(sums), _np(F), _np(dsT)))

    def backward(r, w, k, v, a, b, s_in, dy, ds_out):
        return tuple(map(torch.from_numpy, oracle.backward(*map(_np, (r, w, k, v, a, b, s_in, dy, ds_out)))))

    return StretchOps(summary=summary, compose=compose, forward=forward, state_gradient=state_gradient,
                      compose_adjoints=compose_adjoints, backward=backward)


def _sequence(T, seed):
    d = inputs.gen_sequence(1, T, 2, 16, seed=seed, dtype="f32", s0_std=0.1)
    return [inputs.to_f64(d[n]) for n in inputs.INPUT_NAMES], d["s0"].astype(np.float64)


def _rank_main(rank, world, port, T, seed, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    d = Dist("gloo").init(timeout_s=60)
    try:
        args, s0 = _sequence(T, seed)
        lens = split_lengths(T, world, chunk=8)
        c0 = sum(lens[:rank])
        mine = [torch.from_numpy(np.ascontiguousarray(x[:, c0:c0 + lens[rank]])) for x in args]
        y, s_in, s_fin = forward_context_parallel(*mine, torch.from_numpy(s0), ops=oracle_ops())
        out.put((rank, c0, y.numpy(), s_in.numpy(), s_fin.numpy()))
    finally:
        d.close()


@pytest.mark.parametrize("world,T", [(2, 70), (3, 17)])
def test_gloo_ranks_match_whole_sequence(world, T):
    """Stretches of 8-token chunks (T = 17 over 3 ranks leaves the last one
    empty): every rank's y, its entry state and the shared final state equal
    the oracle's single forward over the whole sequence."""
    seed, port = 90 + world, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, T, seed, out)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted((out.get(timeout=120) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    args, s0 = _sequence(T, seed)
    y_ref, sT_ref = oracle.forward(*args, s0=s0)
    ys = []
    for rank, c0, y, s_in, s_fin in results:
        _, s_pref = oracle.forward(*(x[:, :c0] for x in args), s0=s0)
        np.testing.assert_allclose(s_in, s_pref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(s_fin, sT_ref, rtol=0, atol=1e-12)
        ys.append(y)
    np.testing.assert_allclose(np.concatenate(ys, axis=1), y_ref, rtol=0, atol=1e-12)


def _dy(T, seed):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((1, T, 2, 16)), 0.1 * rng.standard_normal((1, 2, 16, 16))


def _rank_main_bwd(rank, world, port, T, seed, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    d = Dist("gloo").init(timeout_s=60)
    try:
        args, s0 = _sequence(T, seed)
        dy, dsT = _dy(T, seed + 1)
        lens = split_lengths(T, world, chunk=8)
        c0 = sum(lens[:rank])
        cut = lambda x: torch.from_numpy(np.ascontiguousarray(x[:, c0:c0 + lens[rank]]))
        mine = [cut(x) for x in args]
        ops = oracle_ops()
        _, s_in, _, sums = forward_context_parallel(*mine, torch.from_numpy(s0), ops=ops, return_summaries=True)
        grads = backward_context_parallel(*mine, s_in, sums, cut(dy), torch.from_numpy(dsT), ops=ops)
        out.put((rank, [g.numpy() for g in grads]))
    finally:
        d.close()


@pytest.mark.parametrize("world,T", [(2, 70), (3, 17), (4, 45)])
def test_gloo_ranks_backward_match_whole_sequence(world, T):
    """Each rank's gradients from its stretch, the exchanged own state
    gradients F and the composed adjoints equal the oracle's single backward
    over the whole sequence (with a dL/dS_T term); dL/dS_0 agrees on every
    rank.  T = 17 over 3 ranks leaves the last stretch empty."""
    seed, port = 120 + world, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main_bwd, args=(r, world, port, T, seed, out)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted((out.get(timeout=120) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    args, s0 = _sequence(T, seed)
    dy, dsT = _dy(T, seed + 1)
    ref = oracle.backward(*args, s0, dy, dsT)
    for i in range(6):
        got = np.concatenate([g[i] for _, g in results], axis=1)
        np.testing.assert_allclose(got, ref[i], rtol=0, atol=1e-10 * max(1.0, np.abs(ref[i]).max()))
    for _, g in results:
        np.testing.assert_allclose(g[6], ref[6], rtol=0, atol=1e-10 * max(1.0, np.abs(ref[6]).max()))


def test_single_process_is_plain_forward():
    """Without a process group the orchestration is one stretch: compose
    returns [s0, sT] and y is the forward from s0."""
    args, s0 = _sequence(21, 5)
    y, s_in, s_fin = forward_context_parallel(*map(torch.from_numpy, args), torch.from_numpy(s0),
                                              ops=oracle_ops())
    y_ref, sT_ref = oracle.forward(*args, s0=s0)
    np.testing.assert_array_equal(s_in.numpy(), s0)
    np.testing.assert_allclose(s_fin.numpy(), sT_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(y.numpy(), y_ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("T,world", [(0, 3), (1, 2), (33, 2), (100, 2), (4096, 3), (65536, 8), (10, 4)])
def test_split_lengths(T, world):
    lens = split_lengths(T, world)
    assert len(lens) == world and sum(lens) == T and min(lens) >= 0
    nonempty = [i for i, n in enumerate(lens) if n]
    for i in nonempty[:-1]:
        assert lens[i] % 32 == 0                 # only the last stretch is ragged
    if nonempty:
        assert nonempty == list(range(len(nonempty)))
        full = [n // 32 for n in lens[:-1]] + [-(-lens[-1] // 32)]
        assert max(full) - min(full) <= 1 or T < 32 * world


def test_single_process_backward_is_plain_backward():
    """Without a process group the backward orchestration is one stretch: its
    gradients and ds0 are the oracle backward's; summaries for another world
    size are rejected."""
    args, s0 = _sequence(21, 6)
    dy, dsT = _dy(21, 7)
    ops = oracle_ops()
    t = [torch.from_numpy(x) for x in args]
    _, s_in, _, sums = forward_context_parallel(*t, torch.from_numpy(s0), ops=ops, return_summaries=True)
    got = backward_context_parallel(*t, s_in, sums, torch.from_numpy(dy), torch.from_numpy(dsT), ops=ops)
    ref = oracle.backward(*args, s0, dy, dsT)
    for g, r in zip(got, ref):
        np.testing.assert_allclose(g.numpy(), r, rtol=0, atol=1e-10 * max(1.0, np.abs(r).max()))
    with pytest.raises(ValueError):
        backward_context_parallel(*t, s_in, torch.cat([sums, sums]), torch.from_numpy(dy), ops=ops)

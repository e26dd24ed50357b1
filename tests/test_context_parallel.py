"""The sequence-parallel forward's host logic on CPU: gloo ranks (one process
each) hold consecutive stretches of one sequence, exchange their summaries by
all-gather and compose their entry states.  The per-rank compute is the fp64
oracle, injected through ``StretchOps``, so the test checks the orchestration
(rank order = time order, the gather, which composed state each rank takes)
against the oracle's forward over the whole sequence."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from linear_rnn_sequence_wkv7_b200 import inputs
from linear_rnn_sequence_wkv7_b200.context_parallel import StretchOps, forward_context_parallel, split_lengths
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

    return StretchOps(summary=summary, compose=compose, forward=forward)


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

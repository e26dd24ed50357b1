"""The sequence-parallel backward's per-rank steps on one GPU, through the C
ABI, vs the fp64 oracle: a stretch's own state gradient (wkv7_state_gradient),
the adjoint composition (wkv7_compose_adjoints), and a sequence split into
stretches whose backwards, run from the composed dL/dS after each, give the
whole sequence's gradients (the all-gathers replaced by stacking in order)."""
import numpy as np
import pytest
import torch

import oracle
from linear_rnn_sequence_wkv7_b200 import inputs, wkv7
from linear_rnn_sequence_wkv7_b200.context_parallel import (backward_context_parallel, forward_context_parallel,
                                                            split_lengths)
from tests._dev import to_dev, to_f64
from tests._tol import TAU_BF16, TAU_F32, assert_close

pytestmark = pytest.mark.gpu

GRADS = ("dr", "dw", "dk", "dv", "da", "db")


def _case(B, T, H, seed, dtype, dsT=True, **kw):
    N = 64
    d = inputs.gen_sequence(B, T, H, N, seed=seed, dtype=dtype, s0_std=0.1, **kw)
    d["dy"] = inputs.gen_dy(B, T, H, N, seed=seed, dtype=dtype)
    d["dsT"] = (inputs.gen_normal(B * H * N, N, seed=seed, stream=inputs.STREAM_DST, std=0.1)
                .reshape(B, H, N, N) if dsT else None)
    return d


def _dev_args(d):
    return [to_dev(d[n]) for n in inputs.INPUT_NAMES]


def _f64(d, names=inputs.INPUT_NAMES):
    return [inputs.to_f64(d[n]) for n in names]


def _opt64(x):
    return None if x is None else x.astype(np.float64)


@pytest.mark.parametrize("dtype,tau", [("bf16", TAU_BF16), ("f32", TAU_F32)])
@pytest.mark.parametrize("T,with_dsT", [(1, True), (32, False), (33, True), (200, False), (200, True)])
def test_state_gradient_matches_oracle(cuda_device, dtype, tau, T, with_dsT):
    """dL/dS_0 of one stretch from the reverse sweep alone: one token, a full
    chunk, a ragged tail, several chunks; with and without dL/dS_T."""
    B, H = 2, 3
    d = _case(B, T, H, 900 + T, dtype, dsT=with_dsT)
    r, w, k, v, a, b = _dev_args(d)
    ds0 = wkv7.state_gradient(r, w, a, b, to_dev(d["dy"]), to_dev(d["dsT"]))
    assert wkv7.device_status() == wkv7.OK
    rf, wf, kf, vf, af, bf = _f64(d)
    ref = oracle.state_gradient(rf, wf, af, bf, inputs.to_f64(d["dy"]), _opt64(d["dsT"]))
    assert_close(to_f64(ds0), ref, tau, "ds0")


@pytest.mark.parametrize("T", [700, 2001, 8192])
def test_segmented_sweep_matches_oracle(cuda_device, T):
    """Few heads over many tokens: with its workspace the sweep runs as
    segments (dual passes, then the chained adjoints); ds0 vs the oracle and
    vs the one-pass sweep, w near 1 so every segment's product matters."""
    B, H = 1, 2
    assert wkv7.state_gradient_workspace_size(B, T, H, 64) > 0
    d = _case(B, T, H, 930 + T, "bf16", x_mean=-4.0)
    r, w, k, v, a, b = _dev_args(d)
    dy, dsT = to_dev(d["dy"]), to_dev(d["dsT"])
    seg = wkv7.state_gradient(r, w, a, b, dy, dsT)
    one = wkv7.state_gradient(r, w, a, b, dy, dsT, workspace=False)
    assert wkv7.device_status() == wkv7.OK
    rf, wf, kf, vf, af, bf = _f64(d)
    ref = oracle.state_gradient(rf, wf, af, bf, inputs.to_f64(d["dy"]), d["dsT"].astype(np.float64))
    assert_close(to_f64(seg), ref, TAU_BF16, "segmented ds0")
    assert_close(to_f64(seg), to_f64(one), TAU_BF16, "segmented vs one pass")


def test_state_gradient_equals_backward_ds0(cuda_device):
    """The sweep's ds0 is the same quantity the full backward returns."""
    d = _case(1, 300, 4, 950, "bf16")
    args = _dev_args(d)
    r, w, k, v, a, b = args
    dy, dsT = to_dev(d["dy"]), to_dev(d["dsT"])
    ds0 = wkv7.state_gradient(r, w, a, b, dy, dsT)
    full = wkv7.backward(*args, to_dev(d["s0"]), dy, dsT)
    torch.cuda.synchronize()
    assert_close(to_f64(ds0), to_f64(full[6]), TAU_BF16, "sweep vs backward")


def test_state_gradient_of_empty_stretch(cuda_device):
    e = torch.empty(1, 0, 2, 64, dtype=torch.bfloat16, device="cuda")
    dsT = torch.randn(1, 2, 64, 64, device="cuda")
    assert torch.equal(wkv7.state_gradient(e, e, e, e, e, dsT), dsT)
    assert torch.equal(wkv7.state_gradient(e, e, e, e, e), torch.zeros_like(dsT))


@pytest.mark.parametrize("nseg", [0, 1, 5])
@pytest.mark.parametrize("with_dsT", [False, True])
def test_compose_adjoints_matches_oracle(cuda_device, nseg, with_dsT):
    """fp32, last stretch first: adj[k] = adj[k+1] M_k^T + F_k; an M that is
    not symmetric, so a missing transpose shows."""
    B, H, N = 2, 3, 64
    rng = np.random.default_rng(960 + nseg)
    sums = rng.standard_normal((nseg, 2, B, H, N, N)).astype(np.float32)
    sums[:, 1] *= np.float32(0.9 / np.sqrt(N))
    F = rng.standard_normal((nseg, B, H, N, N)).astype(np.float32)
    dsT = rng.standard_normal((B, H, N, N)).astype(np.float32) if with_dsT else None
    adj = wkv7.compose_adjoints(to_dev(sums), to_dev(F), to_dev(dsT))
    torch.cuda.synchronize()
    ref = oracle.compose_adjoints(sums.astype(np.float64), F.astype(np.float64), _opt64(dsT))
    for kk in range(nseg + 1):
        assert_close(to_f64(adj[kk]), ref[kk], TAU_F32, f"adj[{kk}]")


def _stretches_backward_on_one_gpu(d, world, lens=None):
    """Every rank's forward and backward steps in turn on this GPU (stretch
    lengths from split_lengths, or as given)."""
    args = _dev_args(d)
    dy, dsT = to_dev(d["dy"]), to_dev(d["dsT"])
    T = args[0].shape[1]
    bounds = np.cumsum([0] + (lens if lens is not None else split_lengths(T, world)))
    cut = lambda x, i: x[:, bounds[i]:bounds[i + 1]].contiguous()
    parts = [[cut(x, i) for x in args] for i in range(world)]
    sums = torch.stack([wkv7.forward_summary(*p) for p in parts])
    states = wkv7.compose_states(sums, to_dev(d["s0"]))
    F = torch.stack([wkv7.state_gradient(p[0], p[1], p[4], p[5], cut(dy, i)) for i, p in enumerate(parts)])
    adj = wkv7.compose_adjoints(sums, F, dsT)
    outs = [wkv7.backward(*p, states[i].contiguous(), cut(dy, i), adj[i + 1].contiguous())
            for i, p in enumerate(parts)]
    torch.cuda.synchronize()
    grads = [torch.cat([o[j] for o in outs], dim=1) for j in range(6)]
    return grads, adj, [o[6] for o in outs]


@pytest.mark.parametrize("T,world", [(700, 2), (2000, 3), (4097, 4)])
def test_stretch_backwards_match_whole_sequence(cuda_device, T, world):
    """Ragged last stretch, nonzero s0 and dsT, w near 1 so the adjoints carry
    far: the gradients vs the oracle's backward over the whole sequence and vs
    one wkv7.backward; each stretch's own ds_in equals the composed adj."""
    B, H = 1, 2
    d = _case(B, T, H, 970 + T, "bf16", x_mean=-4.0)
    grads, adj, ds_ins = _stretches_backward_on_one_gpu(d, world)
    assert wkv7.device_status() == wkv7.OK
    ref = oracle.backward(*_f64(d), d["s0"].astype(np.float64), inputs.to_f64(d["dy"]),
                          d["dsT"].astype(np.float64))
    for j, name in enumerate(GRADS):
        assert_close(to_f64(grads[j]), ref[j], TAU_BF16, name)
    assert_close(to_f64(adj[0]), ref[6], TAU_BF16, "ds0")
    whole = wkv7.backward(*_dev_args(d), to_dev(d["s0"]), to_dev(d["dy"]), to_dev(d["dsT"]))
    torch.cuda.synchronize()
    for j, name in enumerate(GRADS):
        assert_close(to_f64(grads[j]), to_f64(whole[j]), TAU_BF16, f"{name} vs whole")
    for i in range(world):
        assert_close(to_f64(ds_ins[i]), to_f64(adj[i]), TAU_BF16, f"stretch {i} ds_in vs adj")


def test_stretches_of_any_length(cuda_device):
    """Stretch boundaries off the 32-token chunk grid, a one-token stretch and
    an empty one: the composed forward and backward still equal the oracle's
    over the whole sequence."""
    lens = [333, 1, 0, 500, 77]
    T = sum(lens)
    d = _case(1, T, 2, 985, "bf16")
    grads, adj, ds_ins = _stretches_backward_on_one_gpu(d, len(lens), lens)
    assert wkv7.device_status() == wkv7.OK
    ref = oracle.backward(*_f64(d), d["s0"].astype(np.float64), inputs.to_f64(d["dy"]),
                          d["dsT"].astype(np.float64))
    for j, name in enumerate(GRADS):
        assert_close(to_f64(grads[j]), ref[j], TAU_BF16, name)
    assert_close(to_f64(adj[0]), ref[6], TAU_BF16, "ds0")
    for i in range(len(lens)):
        assert_close(to_f64(ds_ins[i]), to_f64(adj[i]), TAU_BF16, f"stretch {i} ds_in vs adj")


def test_backward_orchestration_without_process_group(cuda_device):
    """forward_context_parallel + backward_context_parallel on one process with
    the library's kernels equal the plain backward."""
    d = _case(1, 500, 3, 990, "bf16")
    args = _dev_args(d)
    s0, dy, dsT = to_dev(d["s0"]), to_dev(d["dy"]), to_dev(d["dsT"])
    _, s_in, _, sums = forward_context_parallel(*args, s0, return_summaries=True)
    got = backward_context_parallel(*args, s_in, sums, dy, dsT)
    ref = wkv7.backward(*args, s0, dy, dsT)
    torch.cuda.synchronize()
    for j, name in enumerate(GRADS + ("ds0",)):
        assert_close(to_f64(got[j]), to_f64(ref[j]), TAU_BF16, name)


def test_backward_orchestration_over_a_one_rank_nccl_group(cuda_device):
    """forward_context_parallel + backward_context_parallel inside an NCCL
    process group of one rank: both all-gathers go through NCCL on the GPU;
    the gradients equal the plain backward's."""
    import os
    import socket
    import torch.distributed as dist
    if dist.is_initialized():
        pytest.skip("a process group is already initialised")
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        d = _case(1, 1000, 4, 995, "bf16")
        args = _dev_args(d)
        s0, dy, dsT = to_dev(d["s0"]), to_dev(d["dy"]), to_dev(d["dsT"])
        _, s_in, _, sums = forward_context_parallel(*args, s0, return_summaries=True)
        got = backward_context_parallel(*args, s_in, sums, dy, dsT)
        ref = wkv7.backward(*args, s0, dy, dsT)
        torch.cuda.synchronize()
        for j, name in enumerate(GRADS + ("ds0",)):
            assert_close(to_f64(got[j]), to_f64(ref[j]), TAU_BF16, name)
    finally:
        dist.destroy_process_group()


def test_long_context_backward_over_eight_stretches(cuda_device):
    """B=1, T=65536, H=32, w near 1 (the long-context workload's inputs), split
    over 8 stretches of 8192 tokens (one per GPU of a node), with dy ~ N(0,1)
    and a dL/dS_T term: sampled heads vs the oracle's backward over the whole
    sequence, every head vs one wkv7.backward (which itself runs the
    segmented checkpoint pass and sweep)."""
    cfg = inputs.WORKLOADS["long_b1_t65536_h32_chunk32"]
    B, T, H, N = cfg["B"], cfg["T"], cfg["H"], cfg["N"]
    d = inputs.gen_sequence(B, T, H, N, seed=cfg["seed"], dtype="bf16", x_mean=cfg["x_mean"], s0_std=cfg["s0_std"])
    d["dy"] = inputs.gen_dy(B, T, H, N, seed=cfg["seed"], dtype="bf16")
    d["dsT"] = (inputs.gen_normal(B * H * N, N, seed=cfg["seed"], stream=inputs.STREAM_DST, std=0.1)
                .reshape(B, H, N, N))
    grads, adj, _ = _stretches_backward_on_one_gpu(d, 8)
    assert wkv7.device_status() == wkv7.OK
    heads = [7, 26]
    raw = [d[n][:, :, heads] for n in inputs.INPUT_NAMES]
    ref = oracle.backward(*map(inputs.to_f64, raw), d["s0"][:, heads].astype(np.float64),
                          inputs.to_f64(d["dy"][:, :, heads]), d["dsT"][:, heads].astype(np.float64))
    for j, name in enumerate(GRADS):
        assert_close(to_f64(grads[j][:, :, heads]), ref[j], TAU_BF16, f"{name} vs oracle")
    assert_close(to_f64(adj[0][:, heads]), ref[6], TAU_BF16, "ds0 vs oracle")
    whole = wkv7.backward(*_dev_args(d), to_dev(d["s0"]), to_dev(d["dy"]), to_dev(d["dsT"]))
    torch.cuda.synchronize()
    for j, name in enumerate(GRADS):
        for h in range(H):
            assert_close(to_f64(grads[j][:, :, h]), to_f64(whole[j][:, :, h]), TAU_BF16, f"{name} head {h} vs whole")
    assert_close(to_f64(adj[0]), to_f64(whole[6]), TAU_BF16, "ds0 vs whole")

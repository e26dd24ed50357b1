"""GPU stretch summaries and state composition (through the C ABI) vs the fp64
oracle, and a sequence split into stretches on one GPU vs the whole-sequence
forward: the per-rank steps of the sequence-parallel forward, with the
all-gather replaced by stacking the summaries in order."""
import numpy as np
import pytest
import torch

import oracle
from linear_rnn_sequence_wkv7_b200 import inputs, wkv7
from linear_rnn_sequence_wkv7_b200.context_parallel import forward_context_parallel, split_lengths
from tests._dev import to_dev, to_f64
from tests._tol import TAU_BF16, TAU_F32, assert_close

pytestmark = pytest.mark.gpu


def _dev_args(d):
    return [to_dev(d[n]) for n in inputs.INPUT_NAMES]


def _f64_args(d, heads=None, t0=0, t1=None):
    out = []
    for n in inputs.INPUT_NAMES:
        x = d[n][:, t0:t1]
        if heads is not None:
            x = x[:, :, heads]
        out.append(inputs.to_f64(x))
    return out


def _workspace(B, T, H, N=64):
    nbytes = wkv7.forward_summary_workspace_size(B, T, H, N)
    return torch.empty(nbytes, dtype=torch.uint8, device="cuda") if nbytes else None


@pytest.mark.parametrize("T", [1, 31, 32, 33, 200])
def test_summary_matches_oracle(cuda_device, T):
    """E (final state from 0) and M (ordered product of the transitions) of a
    bf16 stretch in one pass: one token, a full chunk, ragged tails, several
    chunks."""
    B, H, N = 2, 3, 64
    d = inputs.gen_sequence(B, T, H, N, seed=500 + T, dtype="bf16")
    summ = wkv7.forward_summary(*_dev_args(d))
    assert wkv7.device_status() == wkv7.OK
    E, M = oracle.forward_summary(*_f64_args(d))
    assert_close(to_f64(summ[0]), E, TAU_BF16, "E")
    assert_close(to_f64(summ[1]), M, TAU_BF16, "M")


@pytest.mark.parametrize("T", [700, 4097])
def test_segmented_summary_and_continue(cuda_device, T):
    """Few heads, long stretch: with the workspace the summary runs as
    segments chained into E and M (w near 1, so M stays far from zero), and
    forward_continue reuses them.  E, M vs the oracle and the one-pass
    summary; y and sT from a random entry state vs the oracle and wkv7.forward."""
    B, H, N = 1, 2, 64
    ws = _workspace(B, T, H)
    assert ws is not None
    d = inputs.gen_sequence(B, T, H, N, seed=550 + T, dtype="bf16", x_mean=-4.0, s0_std=0.1)
    args = _dev_args(d)
    summ = wkv7.forward_summary(*args, workspace=ws)
    one = wkv7.forward_summary(*args)
    s_in = to_dev(d["s0"])
    y, sT = wkv7.forward_continue(*args, s_in, workspace=ws, y_dtype=torch.float32, return_state=True)
    assert wkv7.device_status() == wkv7.OK
    f64 = _f64_args(d)
    E, M = oracle.forward_summary(*f64)
    assert_close(to_f64(summ[0]), E, TAU_BF16, "E")
    assert_close(to_f64(summ[1]), M, TAU_BF16, "M")
    assert_close(to_f64(summ), to_f64(one), TAU_BF16, "segmented vs one pass")
    y_ref, sT_ref = oracle.forward(*f64, s0=d["s0"].astype(np.float64))
    assert_close(to_f64(y), y_ref, TAU_BF16, "y")
    assert_close(to_f64(sT), sT_ref, TAU_BF16, "sT")
    yw, sw = wkv7.forward(*args, s0=s_in, y_dtype=torch.float32)
    torch.cuda.synchronize()
    assert_close(to_f64(y), to_f64(yw), TAU_BF16, "y vs wkv7.forward")
    assert_close(to_f64(sT), to_f64(sw), TAU_BF16, "sT vs wkv7.forward")


def test_summary_of_empty_stretch_is_identity(cuda_device):
    B, H, N = 2, 2, 64
    d = inputs.gen_sequence(B, 0, H, N, seed=1, dtype="bf16")
    summ = wkv7.forward_summary(*_dev_args(d))
    torch.cuda.synchronize()
    assert torch.equal(summ[0], torch.zeros_like(summ[0]))
    assert torch.equal(summ[1], torch.eye(N, device="cuda").expand(B, H, N, N))


def test_summary_rejects_fp32_inputs(cuda_device):
    d = inputs.gen_sequence(1, 40, 1, 64, seed=2, dtype="f32")
    with pytest.raises(wkv7.WKV7Error) as e:
        wkv7.forward_summary(*_dev_args(d))
    assert e.value.status == wkv7.ERR_UNSUPPORTED


@pytest.mark.parametrize("nseg", [0, 1, 5])
@pytest.mark.parametrize("with_s0", [False, True])
def test_compose_matches_oracle(cuda_device, nseg, with_s0):
    """fp32 composition: states[k+1] = states[k] M_k + E_k, every k."""
    B, H, N = 2, 3, 64
    rng = np.random.default_rng(600 + nseg)
    sums = rng.standard_normal((nseg, 2, B, H, N, N)).astype(np.float32)
    sums[:, 1] *= np.float32(0.9 / np.sqrt(N))           # keep the products O(1)
    s0 = rng.standard_normal((B, H, N, N)).astype(np.float32) if with_s0 else None
    states = wkv7.compose_states(to_dev(sums), to_dev(s0))
    torch.cuda.synchronize()
    ref = oracle.compose_states(sums.astype(np.float64), None if s0 is None else s0.astype(np.float64))
    for kk in range(nseg + 1):
        assert_close(to_f64(states[kk]), ref[kk], TAU_F32, f"states[{kk}]")


def _stretches_on_one_gpu(d, world):
    """The per-rank steps of the sequence-parallel forward, run one after
    another on this GPU: summaries, stacked in rank order, composed, then each
    stretch's forward from its entry state."""
    args = _dev_args(d)
    T = args[0].shape[1]
    lens = split_lengths(T, world)
    bounds = np.cumsum([0] + lens)
    parts = [[x[:, bounds[i]:bounds[i + 1]].contiguous() for x in args] for i in range(world)]
    wss = [_workspace(p[0].shape[0], p[0].shape[1], p[0].shape[2]) for p in parts]
    sums = torch.stack([wkv7.forward_summary(*p, workspace=ws) for p, ws in zip(parts, wss)])
    states = wkv7.compose_states(sums, to_dev(d["s0"]))
    ys = [wkv7.forward_continue(*p, states[i].contiguous(), workspace=wss[i], y_dtype=torch.float32)
          for i, p in enumerate(parts)]
    torch.cuda.synchronize()
    return torch.cat(ys, dim=1), states, bounds


@pytest.mark.parametrize("T,world", [(700, 2), (2000, 3), (4097, 4)])
def test_stretches_match_oracle(cuda_device, T, world):
    """Ragged last stretch, nonzero s0: y and every entry state vs the oracle."""
    B, H, N = 1, 2, 64
    d = inputs.gen_sequence(B, T, H, N, seed=700 + T, dtype="bf16", s0_std=0.1)
    y, states, bounds = _stretches_on_one_gpu(d, world)
    assert wkv7.device_status() == wkv7.OK
    args = _f64_args(d)
    y_ref, sT_ref = oracle.forward(*args, s0=d["s0"].astype(np.float64))
    assert_close(to_f64(y), y_ref, TAU_BF16, "y")
    assert_close(to_f64(states[world]), sT_ref, TAU_BF16, "final state")
    for i in range(1, world):
        _, s_pref = oracle.forward(*(x[:, :bounds[i]] for x in args), s0=d["s0"].astype(np.float64))
        assert_close(to_f64(states[i]), s_pref, TAU_BF16, f"entry state {i}")


def test_long_context_over_eight_stretches(cuda_device):
    """B=1, T=65536, H=32, w near 1, split over 8 stretches of 8192 tokens (one
    per GPU of a node): sampled heads vs the oracle, every head vs the whole
    sequence's chunked forward."""
    cfg = inputs.WORKLOADS["long_b1_t65536_h32_chunk32"]
    d = inputs.gen_sequence(cfg["B"], cfg["T"], cfg["H"], cfg["N"], seed=cfg["seed"], dtype="bf16",
                            x_mean=cfg["x_mean"], s0_std=cfg["s0_std"])
    y, states, _ = _stretches_on_one_gpu(d, 8)
    assert wkv7.device_status() == wkv7.OK
    heads = [3, 20]
    raw = [d[n][:, :, heads] for n in inputs.INPUT_NAMES]
    y_ref, sT_ref = oracle.forward(*map(inputs.to_f64, raw), s0=d["s0"][:, heads].astype(np.float64))
    assert_close(to_f64(y[:, :, heads]), y_ref, TAU_BF16, "y vs oracle")
    assert_close(to_f64(states[8][:, heads]), sT_ref, TAU_BF16, "sT vs oracle")
    yw, sw = wkv7.forward(*_dev_args(d), s0=to_dev(d["s0"]), y_dtype=torch.float32, algo="chunk")
    torch.cuda.synchronize()
    for h in range(cfg["H"]):
        assert_close(to_f64(y[:, :, h]), to_f64(yw[:, :, h]), TAU_BF16, f"y head {h} vs whole")
    assert_close(to_f64(states[8]), to_f64(sw), TAU_BF16, "sT vs whole")


def test_orchestration_without_process_group(cuda_device):
    """forward_context_parallel on one process with the library's kernels: the
    single stretch's y and final state equal the plain forward."""
    B, T, H, N = 1, 300, 2, 64
    d = inputs.gen_sequence(B, T, H, N, seed=801, dtype="bf16", s0_std=0.1)
    args = _dev_args(d)
    s0 = to_dev(d["s0"])
    y, s_in, s_fin = forward_context_parallel(*args, s0)
    y1, s1 = wkv7.forward(*args, s0=s0)
    torch.cuda.synchronize()
    assert torch.equal(s_in, s0)
    assert_close(to_f64(y), to_f64(y1), TAU_BF16, "y", bf16_out=True)
    assert_close(to_f64(s_fin), to_f64(s1), TAU_BF16, "sT")


def test_orchestration_over_a_one_rank_nccl_group(cuda_device):
    """forward_context_parallel inside an NCCL process group of one rank: the
    all-gather, composition and continue run on the GPU through NCCL and the
    library; the result, like the plain forward's, matches the oracle (the two
    bf16 outputs come from different launch sequences, so each is compared
    with the exact value rather than with the other)."""
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
        B, T, H, N = 1, 1000, 4, 64
        d = inputs.gen_sequence(B, T, H, N, seed=811, dtype="bf16", s0_std=0.1)
        args = _dev_args(d)
        s0 = to_dev(d["s0"])
        y, s_in, s_fin = forward_context_parallel(*args, s0)
        y1, s1 = wkv7.forward(*args, s0=s0)
        torch.cuda.synchronize()
        assert torch.equal(s_in, s0)
        yr, sr = oracle.forward(*(inputs.to_f64(d[n]) for n in inputs.INPUT_NAMES), s0=d["s0"].astype(np.float64))
        assert_close(to_f64(y), yr, TAU_BF16, "y", bf16_out=True)
        assert_close(to_f64(y1), yr, TAU_BF16, "y (plain forward)", bf16_out=True)
        assert_close(to_f64(s_fin), sr, TAU_BF16, "sT")
        assert_close(to_f64(s_fin), to_f64(s1), TAU_BF16, "sT vs the plain forward")
    finally:
        dist.destroy_process_group()

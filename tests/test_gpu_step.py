"""GPU decode step (through the C ABI) vs the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from linear_rnn_sequence_wkv7_b200 import inputs, wkv7
from tests._dev import oracle_args, to_dev, to_f64
from tests._tol import TAU_BF16, TAU_F32, assert_close

pytestmark = pytest.mark.gpu


def _run_steps(steps_in, state0, y_dtype, n_steps):
    state = to_dev(state0)
    ys = []
    for s in range(n_steps):
        args = [to_dev(steps_in[n][s]) for n in inputs.INPUT_NAMES]
        ys.append(to_f64(wkv7.step(*args, state, y_dtype=y_dtype)))
    torch.cuda.synchronize()
    return np.stack(ys), to_f64(state)


def _oracle_steps(steps_in, state0, n_steps, heads=None):
    S = state0.astype(np.float64)
    if heads is not None:
        S = S[:, heads]
    ys = []
    for s in range(n_steps):
        args = [inputs.to_f64(steps_in[n][s]) for n in inputs.INPUT_NAMES]
        if heads is not None:
            args = [x[:, heads] for x in args]
        y, S = oracle.step(*args, S)
        ys.append(y)
    return np.stack(ys), S


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_consecutive_steps_small(cuda_device, dtype):
    B, H, N, n = 3, 5, 64, 6
    st = inputs.gen_steps(n, B, H, N, seed=21, dtype=dtype)
    s0 = inputs.gen_normal(B * H * N, N, seed=21, stream=inputs.STREAM_S0, std=0.1).reshape(B, H, N, N)
    tau = TAU_F32 if dtype == "f32" else TAU_BF16
    y, S = _run_steps(st, s0, torch.float32, n)
    yr, Sr = _oracle_steps(st, s0, n)
    assert_close(y, yr, tau, "y")
    assert_close(S, Sr, tau, "state")
    if dtype == "bf16":
        yb, _ = _run_steps(st, s0, torch.bfloat16, n)
        assert_close(yb, yr, tau, "y(bf16 out)", bf16_out=True)


def test_step_matches_forward_t1(cuda_device):
    B, H, N = 2, 4, 64
    d = inputs.gen_sequence(B, 1, H, N, seed=22, dtype="f32", s0_std=0.1)
    args = [to_dev(d[n]) for n in inputs.INPUT_NAMES]
    y_f, s_f = wkv7.forward(*args, s0=to_dev(d["s0"]), algo="seq")
    state = to_dev(d["s0"])
    y_s = wkv7.step(*(x[:, 0].contiguous() for x in args), state)
    torch.cuda.synchronize()
    # two fp32 kernels with different summation orders: within the fp32 bound
    assert_close(to_f64(y_s), to_f64(y_f[:, 0]), TAU_F32, "y")
    assert_close(to_f64(state), to_f64(s_f), TAU_F32, "state")


def test_decode_workload_full_state(cuda_device):
    """B=256, H=40 (the benchmark's launch), 8 consecutive steps from the
    workload's seeds: every y and the whole 168 MB state vs the oracle."""
    cfg = inputs.WORKLOADS["decode_b256_h40_x1000"]
    B, H, N, n = cfg["B"], cfg["H"], cfg["N"], 8
    st = inputs.gen_steps(n, B, H, N, seed=cfg["seed"], dtype="bf16")
    s0 = inputs.gen_normal(B * H * N, N, seed=cfg["seed"], stream=inputs.STREAM_S0,
                           std=cfg["s0_std"]).reshape(B, H, N, N)
    y, S = _run_steps(st, s0, torch.bfloat16, n)
    yr, Sr = _oracle_steps(st, s0, n)
    assert_close(y, yr, TAU_BF16, "y", bf16_out=True)
    assert_close(S, Sr, TAU_BF16, "state")


def test_decode_workload_1000_steps_sampled_heads(cuda_device):
    """The decode workload as specified: B=256, H=40, all 1000 consecutive
    steps from the workload's seeds, through the step kernel in the benchmark's
    launch.  A random eighth of the (b, h) heads is checked: y of every step
    and the final state vs the oracle.  The steps of one head are one sequence
    of the recurrence (a decode step is one token of it), so the oracle runs
    them as a forward over the steps of each block, carrying its state."""
    cfg = inputs.WORKLOADS["decode_b256_h40_x1000"]
    B, H, N, n = cfg["B"], cfg["H"], cfg["N"], cfg["steps"]
    rng = np.random.default_rng(1000)
    flat = np.sort(rng.choice(B * H, size=B * H // 8, replace=False))
    sb, sh = flat // H, flat % H
    sel_b, sel_h = torch.as_tensor(sb, device="cuda"), torch.as_tensor(sh, device="cuda")
    s0 = inputs.gen_normal(B * H * N, N, seed=cfg["seed"], stream=inputs.STREAM_S0,
                           std=cfg["s0_std"]).reshape(B, H, N, N)
    state = to_dev(s0)
    S_ref = s0[sb, sh][:, None].astype(np.float64)          # [nsel, 1, N, N]
    y_got = np.empty((n, len(flat), N), np.float32)
    y_ref = np.empty((n, len(flat), N), np.float32)
    block = 100
    for s_lo in range(0, n, block):
        s_hi = min(n, s_lo + block)
        st = inputs.gen_steps_range(s_lo, s_hi, B, H, N, seed=cfg["seed"], dtype="bf16")
        dev = {nm: to_dev(st[nm]) for nm in inputs.INPUT_NAMES}
        y = torch.empty((s_hi - s_lo, B, H, N), dtype=torch.bfloat16, device="cuda")
        for s in range(s_hi - s_lo):
            wkv7.step(*(dev[nm][s] for nm in inputs.INPUT_NAMES), state, y=y[s])
        y_got[s_lo:s_hi] = y[:, sel_b, sel_h].float().cpu().numpy()
        # oracle: each sampled head is a batch row of a one-head sequence over these steps
        seq = [inputs.to_f64(np.ascontiguousarray(st[nm][:, sb, sh].transpose(1, 0, 2)))[:, :, None]
               for nm in inputs.INPUT_NAMES]
        yr, S_ref = oracle.forward(*seq, s0=S_ref)
        y_ref[s_lo:s_hi] = yr[:, :, 0].transpose(1, 0, 2)
        del dev, y
    torch.cuda.synchronize()
    assert wkv7.last_status() == wkv7.OK
    assert_close(y_got, y_ref, TAU_BF16, "y (every step, bf16 out)", bf16_out=True)
    assert_close(to_f64(state[sel_b, sel_h]), S_ref[:, 0], TAU_BF16, "state after 1000 steps")

"""The training pair: wkv7_forward_train (y, sT and the state before every
32-token chunk) and wkv7_backward_from_states (the backward without its own
checkpoint pass), against wkv7_forward / wkv7_backward and the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from linear_rnn_sequence_wkv7_b200 import inputs, wkv7
from tests._dev import to_dev, to_f64
from tests._tol import TAU_BF16, TAU_F32, assert_close

pytestmark = pytest.mark.gpu

GRAD_NAMES = ("dr", "dw", "dk", "dv", "da", "db", "ds0")


def _case(B, T, H, seed, dtype, x_mean=0.0):
    d = inputs.gen_sequence(B, T, H, 64, seed=seed, dtype=dtype, s0_std=0.1, x_mean=x_mean)
    d["dy"] = inputs.gen_dy(B, T, H, 64, seed=seed, dtype=dtype)
    d["dsT"] = inputs.gen_normal(B * H * 64, 64, seed=seed, stream=inputs.STREAM_DST, std=0.1).reshape(B, H, 64, 64)
    return d


def _dev(d):
    return [to_dev(d[n]) for n in inputs.INPUT_NAMES], to_dev(d["s0"]), to_dev(d["dy"]), to_dev(d["dsT"])


def _oracle_states(d):
    """The oracle's state before every 32-token chunk, [B, H, nck, N, N]."""
    args = [inputs.to_f64(d[n]) for n in inputs.INPUT_NAMES]
    B, T, H, N = d["r"].shape
    nck = (T + 31) // 32
    out = np.empty((B, H, nck, N, N))
    s = d["s0"].astype(np.float64)
    for c in range(nck):
        out[:, :, c] = s
        _, s = oracle.forward(*(x[:, 32 * c:32 * c + 32] for x in args), s0=s)
    return out


@pytest.mark.parametrize("dtype,B,T,H,algo", [("bf16", 2, 200, 3, "chunk"), ("bf16", 1, 2000, 2, "chunk"),
                                              ("f32", 2, 100, 2, "seq"), ("bf16", 1, 77, 2, "seq")])
def test_forward_train_matches_forward_and_oracle(cuda_device, dtype, B, T, H, algo):
    """y and sT equal wkv7_forward's (same kernels) and the saved states equal
    the oracle's state at every chunk start.  (1, 2000, 2) runs the chunked
    form as sequence segments, which write their own slots; there the plain
    forward takes the fix-up form (y = y0 + S_in q after one summary pass)
    while the training forward keeps the output runs that write the states,
    so the two agree within the bound rather than bit for bit."""
    d = _case(B, T, H, 970 + T, dtype)
    x, s0, _, _ = _dev(d)
    y, sT, states = wkv7.forward_train(*x, s0, y_dtype=torch.float32, algo=algo)
    y1, s1 = wkv7.forward(*x, s0=s0, y_dtype=torch.float32, algo=algo)
    torch.cuda.synchronize()
    assert wkv7.device_status() == wkv7.OK
    tau = TAU_F32 if dtype == "f32" else TAU_BF16
    segmented = algo == "chunk" and wkv7.forward_workspace_size(B, T, H, 64, torch.bfloat16, algo) > 0
    if segmented:
        assert_close(to_f64(y), to_f64(y1), tau, "y vs the plain forward")
        assert_close(to_f64(sT), to_f64(s1), tau, "sT vs the plain forward")
    else:
        assert torch.equal(y, y1) and torch.equal(sT, s1)
    ref = _oracle_states(d)
    for c in range(ref.shape[2]):
        assert_close(to_f64(states[:, :, c]), ref[:, :, c], tau, f"state before chunk {c}")


@pytest.mark.parametrize("dtype,B,T,H", [("bf16", 2, 200, 3), ("f32", 2, 100, 2), ("bf16", 1, 33, 1),
                                         ("bf16", 1, 1500, 2), ("f32", 1, 1100, 1)])
def test_backward_from_states_matches_oracle(cuda_device, dtype, B, T, H):
    """(1, 1500, 2) and (1, 1100, 1): few heads, so the forward keeps its
    states from sequence segments and the sweep runs as segments too."""
    d = _case(B, T, H, 990 + T, dtype)
    x, s0, dy, dsT = _dev(d)
    _, sT, states = wkv7.forward_train(*x, s0)
    got = wkv7.backward_from_states(*x, states, sT, dy, dsT)
    torch.cuda.synchronize()
    assert wkv7.device_status() == wkv7.OK
    args = [inputs.to_f64(d[n]) for n in inputs.INPUT_NAMES]
    ref = oracle.backward(*args, d["s0"].astype(np.float64), inputs.to_f64(d["dy"]), d["dsT"].astype(np.float64))
    tau = TAU_F32 if dtype == "f32" else TAU_BF16
    for name, g, r in zip(GRAD_NAMES, got, ref):
        assert_close(to_f64(g), r, tau, name)


def test_training_workload_equals_backward(cuda_device):
    """B=8, T=4096, H=32 bf16 (the training workload): the forward's saved
    states and chunk transitions are the backward's own checkpoint pass bit
    for bit, so every gradient equals that of wkv7_backward given its full
    workspace (dS by the transition chain in both).  wkv7_backward given its
    minimum workspace takes dS from the per-token sweep instead: the same
    gradients within the bf16 bound (its fp32 gradients against these bf16
    ones, so that one rounding separates them)."""
    cfg = inputs.WORKLOADS["train_bwd_b8_t4096_h32"]
    B, T, H = cfg["B"], cfg["T"], cfg["H"]
    d = inputs.gen_sequence(B, T, H, cfg["N"], seed=cfg["seed"], dtype="bf16", s0_std=cfg["s0_std"])
    x = [to_dev(d[n]) for n in inputs.INPUT_NAMES]
    s0 = to_dev(d["s0"])
    dy = to_dev(inputs.gen_dy(B, T, H, cfg["N"], seed=cfg["seed"], dtype="bf16"))
    _, sT, states = wkv7.forward_train(*x, s0)
    a = wkv7.backward_from_states(*x, states, sT, dy, None, grad_dtype=torch.bfloat16)
    b = wkv7.backward(*x, s0, dy, None, grad_dtype=torch.bfloat16)
    transitions = B * H * ((T + 31) // 32) * 24576
    ws_min = torch.empty(wkv7.backward_workspace_size(B, T, H, 64) - transitions, dtype=torch.uint8, device="cuda")
    c = wkv7.backward(*x, s0, dy, None, grad_dtype=torch.float32, workspace=ws_min)
    torch.cuda.synchronize()
    assert wkv7.device_status() == wkv7.OK
    for name, g1, g2 in zip(GRAD_NAMES, a, b):
        assert torch.equal(g1, g2), name
    for name, g1, g3 in zip(GRAD_NAMES, a, c):      # the bf16 bound of tests/_tol.py, on the device
        r = g1.double()
        bound = TAU_BF16 * r.pow(2).mean().sqrt() + (2.0 ** -8 if name != "ds0" else 0.0) * r.abs()
        excess = ((g3.double() - r).abs() - bound).max().item()
        assert excess <= 0.0, f"{name} (per-token sweep): excess over the bound {excess:.3e}"


def test_saved_states_buffer_size_is_checked(cuda_device):
    """The saved states carry the chunks' transitions after the states: a
    states tensor of the states' size alone is refused before any launch."""
    d = _case(1, 100, 2, 995, "bf16")
    x, s0, dy, _ = _dev(d)
    small = torch.empty(1, 2, 4, 64, 64, device="cuda")
    with pytest.raises(ValueError):
        wkv7.forward_train(*x, s0, states=small)
    _, sT, states = wkv7.forward_train(*x, s0)
    with pytest.raises(ValueError):
        wkv7.backward_from_states(*x, small, sT, dy)
    assert states.shape == (1, 2, 4, 64, 64)

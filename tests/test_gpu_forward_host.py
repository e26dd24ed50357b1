"""wkv7_forward_host (host tensors in and out, time slices pipelined against
the copies) vs the device forward and the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from linear_rnn_sequence_wkv7_b200 import inputs, wkv7
from tests._dev import to_dev, to_f64
from tests._tol import TAU_BF16, TAU_F32, assert_close

pytestmark = pytest.mark.gpu


def _host(x, pin=True):
    if x is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16) if x.dtype == np.uint16 \
        else torch.from_numpy(np.ascontiguousarray(x))
    return t.pin_memory() if pin else t.clone()


def run_host(d, y_dtype, algo="auto", pin=True, with_s0=True, want_sT=True):
    B, T, H, N = d["r"].shape
    hin = [_host(d[n], pin) for n in inputs.INPUT_NAMES]
    s0 = _host(d["s0"], pin) if with_s0 else None
    y = torch.empty(B, T, H, N, dtype=y_dtype)
    sT = torch.empty(B, H, N, N, dtype=torch.float32) if want_sT else None
    if pin:
        y = y.pin_memory()
        sT = sT.pin_memory() if sT is not None else None
    wkv7.forward_host(*hin, s0, y=y, sT=sT, algo=algo)
    torch.cuda.synchronize()
    return y, sT


def run_device(d, y_dtype, algo="auto", with_s0=True):
    args = [to_dev(d[n]) for n in inputs.INPUT_NAMES]
    y, sT = wkv7.forward(*args, s0=to_dev(d["s0"]) if with_s0 else None, y_dtype=y_dtype, algo=algo)
    torch.cuda.synchronize()
    return y.cpu(), sT.cpu()


def test_prefill_shape_is_bitwise_the_device_forward(cuda_device):
    """B=8, T=4096, H=32 bf16 (the prefill workload's shape, 8 slices of 512
    tokens): slices cut at chunk boundaries hand the fp32 state over exactly,
    so y and sT equal the one-call device forward bit for bit."""
    cfg = inputs.WORKLOADS["prefill_b8_t4096_h32_bf16"]
    d = inputs.gen_sequence(cfg["B"], cfg["T"], cfg["H"], cfg["N"], seed=cfg["seed"], dtype="bf16",
                            s0_std=cfg["s0_std"])
    y, sT = run_host(d, torch.bfloat16)
    yd, sd = run_device(d, torch.bfloat16)
    assert wkv7.device_status() == wkv7.OK
    assert torch.equal(y, yd)
    assert torch.equal(sT, sd)


@pytest.mark.parametrize("T", [1, 31, 300])
def test_fp32_sequential_is_bitwise_the_device_forward(cuda_device, T):
    B, H, N = 2, 2, 64
    d = inputs.gen_sequence(B, T, H, N, seed=900 + T, dtype="f32", s0_std=0.1)
    y, sT = run_host(d, torch.float32, algo="seq")
    yd, sd = run_device(d, torch.float32, algo="seq")
    assert torch.equal(y, yd) and torch.equal(sT, sd)
    yr, sr = oracle.forward(*(inputs.to_f64(d[n]) for n in inputs.INPUT_NAMES), s0=d["s0"].astype(np.float64))
    assert_close(to_f64(y), yr, TAU_F32, "y")
    assert_close(to_f64(sT), sr, TAU_F32, "sT")


@pytest.mark.parametrize("T", [97, 1000, 2049])
def test_few_heads_ragged_vs_oracle(cuda_device, T):
    """Few heads (the whole-sequence forward would split into segments; the
    slices choose their own), ragged last slice, fp32 y: vs the oracle."""
    B, H, N = 1, 3, 64
    d = inputs.gen_sequence(B, T, H, N, seed=950 + T, dtype="bf16", s0_std=0.1)
    y, sT = run_host(d, torch.float32)
    assert wkv7.device_status() == wkv7.OK
    yr, sr = oracle.forward(*(inputs.to_f64(d[n]) for n in inputs.INPUT_NAMES), s0=d["s0"].astype(np.float64))
    assert_close(to_f64(y), yr, TAU_BF16, "y")
    assert_close(to_f64(sT), sr, TAU_BF16, "sT")


def test_zero_state_no_final_state_pageable(cuda_device):
    """s0 = None (zeros), sT not requested, ordinary (pageable) host memory."""
    B, T, H, N = 2, 200, 2, 64
    d = inputs.gen_sequence(B, T, H, N, seed=991, dtype="bf16", s0_std=0.1)
    y, sT = run_host(d, torch.bfloat16, pin=False, with_s0=False, want_sT=False)
    assert sT is None
    yd, _ = run_device(d, torch.bfloat16, with_s0=False)
    assert_close(to_f64(y), to_f64(yd), TAU_BF16, "y", bf16_out=True)


def test_empty_sequence_copies_state(cuda_device):
    B, H, N = 2, 2, 64
    d = inputs.gen_sequence(B, 0, H, N, seed=992, dtype="bf16", s0_std=0.1)
    y, sT = run_host(d, torch.bfloat16)
    assert y.shape == (B, 0, H, N)
    assert torch.equal(sT, torch.from_numpy(d["s0"]))
    _, sT0 = run_host(d, torch.bfloat16, with_s0=False)
    assert torch.equal(sT0, torch.zeros_like(sT0))

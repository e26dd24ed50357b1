"""Run one WKV7 kernel on a chosen case, for profilers (ncu) and quick timing.

    python -m linear_rnn_sequence_wkv7_b200.profile_case --op fwd --algo chunk --B 2 --T 4096 --H 32
    python -m linear_rnn_sequence_wkv7_b200.profile_case --op step --B 256 --H 40 --reps 3
    python -m linear_rnn_sequence_wkv7_b200.profile_case --op bwd --B 1 --T 4096 --H 32
    python -m linear_rnn_sequence_wkv7_b200.profile_case --op timemix --B 8 --T 4096 --H 32

Inputs follow the prefill workload's distributions (bf16, s0 ~ N(0, 0.1)).
Runs ``--warmup`` untimed launches, then ``--reps`` launches timed with CUDA
events, and prints the mean device time per launch.
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

from linear_rnn_sequence_wkv7_b200 import inputs, wkv7  # noqa: E402


def to_dev(x):
    if x is None:
        return None
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(x).cuda()


def main():
    p = argparse.ArgumentParser()
    p.add_argument("--op", choices=["fwd", "step", "bwd", "timemix"], default="fwd")
    p.add_argument("--algo", choices=["auto", "seq", "chunk"], default="auto")
    p.add_argument("--B", type=int, default=2)
    p.add_argument("--T", type=int, default=4096)
    p.add_argument("--H", type=int, default=32)
    p.add_argument("--warmup", type=int, default=1)
    p.add_argument("--reps", type=int, default=2)
    a = p.parse_args()
    N = 64
    T = 1 if a.op == "step" else a.T
    d = inputs.gen_sequence(a.B, T, a.H, N, seed=1, dtype="bf16", s0_std=0.1)
    x = [to_dev(d[n]) for n in inputs.INPUT_NAMES]
    s0 = to_dev(d["s0"])
    if a.op == "fwd":
        y = torch.empty(a.B, T, a.H, N, dtype=torch.bfloat16, device="cuda")
        sT = torch.empty_like(s0)
        nws = wkv7.forward_workspace_size(a.B, T, a.H, N, torch.bfloat16, a.algo)
        ws = torch.empty(max(nws, 16), dtype=torch.uint8, device="cuda")
        run = lambda: wkv7.forward(*x, s0=s0, y=y, sT=sT, algo=a.algo, workspace=ws)
    elif a.op == "timemix":
        z = torch.empty(a.B, T, a.H, N, dtype=torch.bfloat16, device="cuda")
        sT = torch.empty_like(s0)
        rho, gamma, beta = (torch.from_numpy(t).cuda() for t in inputs.gen_timemix_params(a.H, N, seed=1))
        g = to_dev(inputs.gen_gate(a.B, T, a.H, N, seed=1))
        nws = wkv7.forward_timemix_workspace_size(a.B, T, a.H, N, torch.bfloat16, a.algo)
        ws = torch.empty(max(nws, 16), dtype=torch.uint8, device="cuda")
        run = lambda: wkv7.forward_timemix(*x, s0, rho=rho, gamma=gamma, beta=beta, g=g, z=z, sT=sT, algo=a.algo,
                                           workspace=ws)
    elif a.op == "step":
        xs = [t[:, 0].contiguous() for t in x]
        y = torch.empty(a.B, a.H, N, dtype=torch.bfloat16, device="cuda")
        run = lambda: wkv7.step(*xs, s0, y=y)
    else:
        dy = to_dev(inputs.gen_dy(a.B, T, a.H, N, seed=1))
        out = [torch.empty(a.B, T, a.H, N, dtype=torch.bfloat16, device="cuda") for _ in range(6)]
        out.append(torch.empty_like(s0))
        ws = torch.empty(wkv7.backward_workspace_size(a.B, T, a.H, N), dtype=torch.uint8, device="cuda")
        run = lambda: wkv7.backward(*x, s0, dy, None, grad_dtype=torch.bfloat16, workspace=ws, out=out)
    for _ in range(a.warmup):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.reps):
        run()
    e1.record()
    torch.cuda.synchronize()
    status = wkv7.device_status()
    print(f"{a.op} algo={a.algo} B={a.B} T={T} H={a.H}: {e0.elapsed_time(e1) / a.reps * 1e3:.1f} us/launch "
          f"status={status}")
    if status != wkv7.OK:
        sys.exit(1)


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Benchmark of the WKV7 hot path on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline (``value``): prefill forward throughput in head-tokens/s on the
B=8, T=4096, H=32, N=64 bf16 workload (fp32 state, s0 ~ N(0, 0.1)); one step
is one ``wkv7_forward`` call over the whole batch with inputs resident in
HBM.  The same run also measures, under ``parts``, the training backward on
the same shape (dy ~ N(0,1) bf16, dsT = 0) and the decode step (B=256, H=40,
1000 consecutive steps replayed from a CUDA graph) and the long-context
chunked forward (B=1, T=65536, H=32, decays near 1), where 32 heads cannot
fill the GPU and the sequence runs as parallel segments.

Multi-GPU: one process per GPU (torchrun); every rank runs its own batch
(weak scaling, no collective on the data path); times are the max over
ranks of device-side CUDA-event time.

``--impl reference`` times the fp64 CPU oracle on the host cores instead
(rank 0 only), each step a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_rnn_sequence_wkv7_b200 import inputs  # noqa: E402
from linear_rnn_sequence_wkv7_b200.dist import Dist, aggregate_throughput, shard_seed  # noqa: E402

METRIC = "WKV7 head-tokens/sec fwd/bwd + decode steps/sec; % of HBM/FP32/TC roofline"
N = 64
FWD = inputs.WORKLOADS["prefill_b8_t4096_h32_bf16"]
BWD = inputs.WORKLOADS["train_bwd_b8_t4096_h32"]
DEC = inputs.WORKLOADS["decode_b256_h40_x1000"]
LONG = inputs.WORKLOADS["long_b1_t65536_h32_chunk32"]
SM_COUNT = 148
TC_OPERANDS = ("bf16 hi/lo split (3 passes; 2 where one side is an exact bf16 input), fp32 accumulate "
               "in TMEM; state fp32")
FP32_LANES_PER_SM = 128
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "sm_max_mhz": 1965.0}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--algo", default="auto", choices=["auto", "seq", "chunk"])
    p.add_argument("--parts", default="fwd,bwd,train,decode,long,timemix")
    p.add_argument("--decode-steps", type=int, default=DEC["steps"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    return p.parse_args()


# ---------------------------------------------------------------------------
# peaks, algorithmic cost
# ---------------------------------------------------------------------------

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": float(pk["hbm_gbs"]), "bf16_tflops": float(pk["bf16_tflops"]),
                "sm_max_mhz": float(pk.get("sm_max_mhz", 1965.0)), "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


def fp32_peak_tflops(sm_mhz):
    """FP32 FMA peak: 148 SMs x 128 lanes x 2 flop x clock."""
    return SM_COUNT * FP32_LANES_PER_SM * 2 * sm_mhz * 1e6 / 1e12


def fwd_bytes(B, T, H, in_bytes=2, y_bytes=2):
    """Algorithmic HBM bytes of one forward call: six input tensors and y once,
    fp32 s0 in and sT out once."""
    return B * T * H * N * (6 * in_bytes + y_bytes) + 2 * B * H * N * N * 4


def fwd_flops(B, T, H):
    """9 N^2 flop per head-token: removal read 2N^2, update 5N^2, readout 2N^2."""
    return 9 * N * N * B * T * H


def fwd_chunk_flops(B, T, H, L=32):
    """Tensor-core flop the chunked form issues per call (bf16 passes counted):
    per 32-token chunk 3-pass Gram 64x64x64, W^T 64x32x32 (3), U~^T (2),
    M' 64x64x32 (3), Q'^T 64x32x32 (3), E 64x64x64 (3+2 over halves of K),
    Y_loc^T 64x32x64 (3+2), state 64x96x64 (3)."""
    per_chunk = 2 * (3 * 64 * 64 * 64 + 3 * 64 * 32 * 32 + 2 * 64 * 32 * 32 + 3 * 64 * 64 * 32
                     + 3 * 64 * 32 * 32 + 5 * 64 * 64 * 32 + 5 * 64 * 32 * 32 + 3 * 64 * 96 * 64)
    return per_chunk * B * H * ((T + L - 1) // L)


def bwd_bytes(B, T, H, in_bytes=2, g_bytes=2):
    """Six inputs + dy read, six gradients written, s0 read, ds0 written."""
    return B * T * H * N * (7 * in_bytes + 6 * g_bytes) + 2 * B * H * N * N * 4


def bwd_flops(B, T, H):
    """28 N^2 flop per head-token: 19 N^2 gradient recurrence + 9 N^2 recompute."""
    return 28 * N * N * B * T * H


def step_bytes(B, H, in_bytes=2, y_bytes=2):
    """One decode step: fp32 state read and written, six inputs read, y written."""
    return 2 * B * H * N * N * 4 + B * H * N * (6 * in_bytes + y_bytes)


def source_hash(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "linear_rnn_sequence_wkv7_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, src_hash):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current source of that kernel; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel)
    if not rec or rec.get("source_hash") != src_hash:
        return None
    return rec.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_uuid):
        self.uuid = device_uuid
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.uuid, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        if self.path and os.path.exists(self.path):
            with open(self.path) as f:
                for line in f:
                    parts = [x.strip() for x in line.split(",")]
                    if len(parts) == 8:
                        rows.append(parts)
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in rows for n, v in zip(names, r[4:]) if v.lower() == "active"})
        busy = [s for s in sm if s > 0.5 * max(sm)] if sm else []
        return {"sm_mhz": statistics.median(busy) if busy else None,
                "sm_max_mhz": float(rows[0][1]) if rows[0][1].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max([float(r[2]) for r in rows if r[2].replace(".", "").isdigit()] or [0.0])}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def to_dev(x, device):
    import torch
    if x is None:
        return None
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(x).to(device)


def to_pinned(x):
    import torch
    t = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16) if x.dtype == np.uint16 else torch.from_numpy(x)
    return t.pin_memory()


def require_ok_status(what, stream):
    """The library's device status word must read OK after a timed part: a
    bounded wait that ran out or a chunk outside the chunked form's range
    leaves outputs unspecified, so such a run is no measurement."""
    from linear_rnn_sequence_wkv7_b200 import wkv7
    st = wkv7.last_status(stream)
    if st != wkv7.OK:
        raise RuntimeError(f"{what}: device status {wkv7.status_string(st)} ({st}) after the timed run")


def timed(fn, steps, warmup, dist, stream, what="timed run"):
    """Device time of `steps` calls of fn (CUDA events on `stream`), max over ranks."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    require_ok_status(what + " (warm-up)", stream)
    dist.barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        fn()
    end.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    elapsed = start.elapsed_time(end) / 1e3
    require_ok_status(what, stream)
    return dist.max(elapsed)


def bench_forward(args, dist, peaks, device):
    import torch
    from linear_rnn_sequence_wkv7_b200 import wkv7
    cfg = FWD
    B, T, H = cfg["B"], cfg["T"], cfg["H"]
    d = inputs.gen_sequence(B, T, H, N, seed=shard_seed(cfg["seed"], dist.rank), dtype="bf16",
                            s0_std=cfg["s0_std"])
    dev = [to_dev(d[n], device) for n in inputs.INPUT_NAMES]
    s0 = to_dev(d["s0"], device)
    y = torch.empty(B, T, H, N, dtype=torch.bfloat16, device=device)
    sT = torch.empty(B, H, N, N, dtype=torch.float32, device=device)
    ws_n = wkv7.forward_workspace_size(B, T, H, N, torch.bfloat16, args.algo)
    ws = torch.empty(max(ws_n, 1), dtype=torch.uint8, device=device) if ws_n else None
    stream = torch.cuda.current_stream()

    def step():
        wkv7.forward(*dev, s0=s0, y=y, sT=sT, algo=args.algo, workspace=ws, stream=stream)

    uuid = str(torch.cuda.get_device_properties(device).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    with sampler:
        secs = timed(step, args.steps, args.warmup, dist, stream, "prefill forward")
    clocks = sampler.summary()

    # end to end through the host-buffer entry point: pinned host inputs in,
    # y and sT back to pinned host memory, copies pipelined against the
    # forward inside the call
    host_in = [to_pinned(d[n]) for n in inputs.INPUT_NAMES]
    host_s0 = to_pinned(d["s0"])
    host_y = torch.empty(B, T, H, N, dtype=torch.bfloat16).pin_memory()
    host_sT = torch.empty(B, H, N, N, dtype=torch.float32).pin_memory()
    del dev, y, ws
    torch.cuda.empty_cache()
    ws_host = torch.empty(wkv7.forward_host_workspace_size(B, T, H, N, torch.bfloat16, torch.bfloat16, args.algo),
                          dtype=torch.uint8, device=device)

    def e2e_step():
        wkv7.forward_host(*host_in, host_s0, y=host_y, sT=host_sT, algo=args.algo, workspace=ws_host,
                          stream=stream)

    e2e_steps = max(3, min(args.steps, 20))
    e2e_secs = timed(e2e_step, e2e_steps, 2, dist, stream, "prefill forward from host buffers")
    h2d = sum(t.numel() * t.element_size() for t in host_in) + host_s0.numel() * 4
    d2h = host_y.numel() * 2 + host_sT.numel() * 4

    head_tokens = B * T * H
    kernel = "fwd_" + wkv7.resolve_algo(T, torch.bfloat16, args.algo)
    per_launch = secs / args.steps
    nbytes = fwd_bytes(B, T, H)
    if kernel == "fwd_seq":
        pk = fp32_peak_tflops(peaks["sm_max_mhz"])
        ach = fwd_flops(B, T, H) / per_launch / 1e12
        roof = {"bound": "alu", "achieved": ach, "peak": pk, "unit": "TFLOP/s", "frac": ach / pk,
                "peak_source": "derived: 148 SM x 128 FP32 lanes x 2 x %.0f MHz" % peaks["sm_max_mhz"],
                "per_unit": "9*N^2 flop per head-token", "units_per_launch": head_tokens}
    else:
        pk = peaks["hbm_gbs"]
        ach = nbytes / per_launch / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": pk, "unit": "GB/s", "frac": ach / pk,
                "peak_source": peaks["source"], "per_unit": "896 B per head-token + 32 KiB state per head",
                "units_per_launch": head_tokens,
                "tensor_tflops": fwd_chunk_flops(B, T, H) / per_launch / 1e12}
    src = {"fwd_seq": ("fwd_seq.cu", "umma.cuh", "common.cuh"), "fwd_chunk": ("fwd_chunk.cu", "umma.cuh", "common.cuh")}[kernel]
    roof["traffic"] = recorded_traffic(kernel, source_hash(*src))
    roof["kernel"] = kernel
    roof["hbm_frac"] = nbytes / per_launch / 1e9 / peaks["hbm_gbs"]
    return {
        "value": aggregate_throughput(head_tokens * args.steps, secs, dist.world),
        "ms_per_step": secs / args.steps * 1e3,
        "roofline": roof,
        "clocks": clocks,
        "e2e": {"value": aggregate_throughput(head_tokens * e2e_steps, e2e_secs, dist.world), "unit": "head-tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "launches": args.steps,
        "sample": d,
    }


def bench_backward(args, dist, peaks, device, d):
    import torch
    from linear_rnn_sequence_wkv7_b200 import wkv7
    cfg = BWD
    B, T, H = cfg["B"], cfg["T"], cfg["H"]
    dev = [to_dev(d[n], device) for n in inputs.INPUT_NAMES]
    s0 = to_dev(d["s0"], device)
    dy = to_dev(inputs.gen_dy(B, T, H, N, seed=shard_seed(cfg["seed"], dist.rank), dtype="bf16"), device)
    out = [torch.empty(B, T, H, N, dtype=torch.bfloat16, device=device) for _ in range(6)]
    out.append(torch.empty(B, H, N, N, dtype=torch.float32, device=device))
    ws = torch.empty(wkv7.backward_workspace_size(B, T, H, N), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()

    def step():
        wkv7.backward(*dev, s0, dy, None, grad_dtype=torch.bfloat16, workspace=ws, out=out, stream=stream)

    steps = max(3, min(args.steps // 20, 10))
    secs = timed(step, steps, 2, dist, stream, "training backward")
    per = secs / steps
    pk = fp32_peak_tflops(peaks["sm_max_mhz"])
    ach_flops = bwd_flops(B, T, H) / per / 1e12
    nbytes = bwd_bytes(B, T, H)
    ach = nbytes / per / 1e9
    return {"value": aggregate_throughput(B * T * H, per, dist.world), "unit": "head-tokens/s",
            "ms_per_step": per * 1e3,
            "steps": steps, "launches": 3 * steps,
            "roofline": {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": ach / peaks["hbm_gbs"], "peak_source": peaks["source"],
                         "per_unit": "1664 B per head-token (6 inputs + dy read, 6 bf16 gradients written) "
                                     "+ 32 KiB state per head", "bytes_per_launch": nbytes,
                         "kernels": "checkpoints with every chunk's transition (chunked forward), dS by the "
                                    "transition chain (tcgen05), per-chunk gradients (tcgen05, bf16 hi/lo "
                                    "operands, fp32 accumulation)",
                         "fp32_alu": {"achieved": ach_flops, "peak": pk, "unit": "TFLOP/s", "frac": ach_flops / pk,
                                      "per_unit": "28*N^2 flop per head-token (the sequential scan's algebra)"},
                         "tensor_frac": ach_flops / peaks["bf16_tflops"]},
            "config": {"workload": "train_bwd_b8_t4096_h32", "B": B, "T": T, "H": H, "N": N,
                       "grad_dtype": "bf16", "dsT": "zero"}}


def bench_train(args, dist, peaks, device, d):
    """One training step of the recurrence on the training workload: the
    forward that keeps the chunk states, then the backward from them, against
    the forward followed by the self-contained backward."""
    import torch
    from linear_rnn_sequence_wkv7_b200 import wkv7
    cfg = BWD
    B, T, H = cfg["B"], cfg["T"], cfg["H"]
    dev = [to_dev(d[n], device) for n in inputs.INPUT_NAMES]
    s0 = to_dev(d["s0"], device)
    dy = to_dev(inputs.gen_dy(B, T, H, N, seed=shard_seed(cfg["seed"], dist.rank), dtype="bf16"), device)
    y = torch.empty(B, T, H, N, dtype=torch.bfloat16, device=device)
    sT = torch.empty(B, H, N, N, dtype=torch.float32, device=device)
    # the saved states (the state before every chunk), then the chunks' transitions
    states_buf = torch.empty(wkv7.saved_states_size(B, T, H, N) // 4, dtype=torch.float32, device=device)
    states = states_buf[: B * H * ((T + 31) // 32) * N * N].view(B, H, (T + 31) // 32, N, N)
    grads = [torch.empty(B, T, H, N, dtype=torch.bfloat16, device=device) for _ in range(6)]
    grads.append(torch.empty(B, H, N, N, dtype=torch.float32, device=device))
    ws_b = torch.empty(wkv7.backward_from_states_workspace_size(B, T, H, N), dtype=torch.uint8, device=device)
    ws_full = torch.empty(wkv7.backward_workspace_size(B, T, H, N), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()

    def step():
        wkv7.forward_train(*dev, s0, y=y, sT=sT, states=states, stream=stream)
        wkv7.backward_from_states(*dev, states, sT, dy, None, grad_dtype=torch.bfloat16, workspace=ws_b,
                                  out=grads, stream=stream)

    def step_separate():
        wkv7.forward(*dev, s0=s0, y=y, sT=sT, stream=stream)
        wkv7.backward(*dev, s0, dy, None, grad_dtype=torch.bfloat16, workspace=ws_full, out=grads, stream=stream)

    steps = max(3, min(args.steps // 20, 10))
    per = timed(step, steps, 2, dist, stream, "training step") / steps
    per_sep = timed(step_separate, steps, 2, dist, stream, "forward + backward") / steps
    return {"value": aggregate_throughput(B * T * H, per, dist.world), "unit": "head-tokens/s",
            "ms_per_step": per * 1e3, "steps": steps, "launches": 4 * steps,
            "separate_ms_per_step": per_sep * 1e3,
            "note": "wkv7_forward_train (states and chunk transitions kept) + wkv7_backward_from_states; "
                    "separate = wkv7_forward + wkv7_backward (which recomputes the chunk states)",
            "config": {"workload": "train_bwd_b8_t4096_h32", "B": B, "T": T, "H": H, "N": N,
                       "y_dtype": "bf16", "grad_dtype": "bf16", "dsT": "zero"}}


def bench_timemix(args, dist, peaks, device, d, plain_ms):
    """The prefill forward with the time-mix output epilogue (current-token
    term, per-head norm, gate) fused into the chunked kernel, bf16 z: its cost
    over the plain forward on the same inputs."""
    import torch
    from linear_rnn_sequence_wkv7_b200 import wkv7
    cfg = FWD
    B, T, H = cfg["B"], cfg["T"], cfg["H"]
    dev = [to_dev(d[n], device) for n in inputs.INPUT_NAMES]
    s0 = to_dev(d["s0"], device)
    rho, gamma, beta = (torch.from_numpy(x).to(device) for x in inputs.gen_timemix_params(H, N, seed=cfg["seed"]))
    g = to_dev(inputs.gen_gate(B, T, H, N, seed=shard_seed(cfg["seed"], dist.rank), dtype="bf16"), device)
    z = torch.empty(B, T, H, N, dtype=torch.bfloat16, device=device)
    sT = torch.empty(B, H, N, N, dtype=torch.float32, device=device)
    ws_n = wkv7.forward_timemix_workspace_size(B, T, H, N, torch.bfloat16, args.algo)
    ws = torch.empty(max(ws_n, 1), dtype=torch.uint8, device=device) if ws_n else None
    stream = torch.cuda.current_stream()

    def step():
        wkv7.forward_timemix(*dev, s0, rho=rho, gamma=gamma, beta=beta, g=g, z=z, sT=sT, algo=args.algo,
                             workspace=ws, stream=stream)

    steps = max(3, min(args.steps // 4, 50))
    per = timed(step, steps, 3, dist, stream, "time-mix forward") / steps
    nbytes = fwd_bytes(B, T, H) + B * T * H * N * 2          # + the gate read
    ach = nbytes / per / 1e9
    return {"value": aggregate_throughput(B * T * H, per, dist.world), "unit": "head-tokens/s",
            "ms_per_step": per * 1e3, "steps": steps, "launches": steps,
            "plain_forward_ms": plain_ms, "overhead_frac": per * 1e3 / plain_ms - 1.0,
            "roofline": {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": ach / peaks["hbm_gbs"],
                         "per_unit": "1024 B per head-token (six inputs, gate, z) + 32 KiB state per head",
                         "traffic": recorded_traffic("fwd_chunk_timemix",
                                                     source_hash("fwd_chunk.cu", "umma.cuh", "common.cuh"))},
            "config": {"workload": "prefill_b8_t4096_h32_bf16 + time-mix epilogue", "B": B, "T": T, "H": H,
                       "N": N, "z_dtype": "bf16", "eps": 1e-5,
                       "params": "rho ~ U(-1,1), gamma ~ U(0.5,1.5), beta ~ U(-0.5,0.5), g = sigmoid(N(0,1))"}}


def bench_decode(args, dist, peaks, device, steps_in):
    import torch
    from linear_rnn_sequence_wkv7_b200 import wkv7
    cfg = DEC
    B, H, n = cfg["B"], cfg["H"], args.decode_steps
    dev = {k: to_dev(v, device) for k, v in steps_in.items()}
    state = to_dev(inputs.gen_normal(B * H * N, N, seed=cfg["seed"], stream=inputs.STREAM_S0,
                                     std=cfg["s0_std"]).reshape(B, H, N, N), device)
    y = torch.empty(n, B, H, N, dtype=torch.bfloat16, device=device)
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap), wkv7.status_checks(False):     # no synchronizing check inside a capture
        for s in range(2):   # warm the launch path outside the capture
            wkv7.step(*(dev[nm][s] for nm in inputs.INPUT_NAMES), state, y=y[s], stream=cap)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=cap):
            for s in range(n):
                wkv7.step(*(dev[nm][s] for nm in inputs.INPUT_NAMES), state, y=y[s], stream=cap)
    torch.cuda.synchronize()
    reps = 3
    secs = timed(g.replay, reps, 1, dist, torch.cuda.current_stream(), "decode steps")
    per_step = secs / (reps * n)
    nbytes = step_bytes(B, H)
    ach = nbytes / per_step / 1e9
    del g
    return {"value": aggregate_throughput(1, per_step, dist.world), "unit": "steps/s",
            "us_per_step": per_step * 1e6,
            "graph_replays": reps, "steps_per_replay": n, "launches": reps * n,
            "head_tokens_per_s": aggregate_throughput(B * H, per_step, dist.world),
            "roofline": {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": ach / peaks["hbm_gbs"], "per_unit": "32 KiB state RMW + 896 B per head",
                         "units_per_launch": B * H,
                         "traffic": recorded_traffic("step", source_hash("step.cu", "common.cuh"))},
            "config": {"workload": "decode_b256_h40_x1000", "B": B, "H": H, "N": N, "steps": n,
                       "l2": "state 168 MB > 126 MB L2; inputs pre-staged, 7.9 GB"}}


def bench_long(args, dist, peaks, device):
    import torch
    from linear_rnn_sequence_wkv7_b200 import wkv7
    cfg = LONG
    B, T, H = cfg["B"], cfg["T"], cfg["H"]
    d = inputs.gen_sequence(B, T, H, N, seed=shard_seed(cfg["seed"], dist.rank), dtype="bf16",
                            x_mean=cfg["x_mean"], s0_std=cfg["s0_std"])
    dev = [to_dev(d[n], device) for n in inputs.INPUT_NAMES]
    s0 = to_dev(d["s0"], device)
    y = torch.empty(B, T, H, N, dtype=torch.bfloat16, device=device)
    sT = torch.empty(B, H, N, N, dtype=torch.float32, device=device)
    ws_n = wkv7.forward_workspace_size(B, T, H, N, torch.bfloat16, "chunk")
    ws = torch.empty(max(ws_n, 16), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()

    def step():
        wkv7.forward(*dev, s0=s0, y=y, sT=sT, algo="chunk", workspace=ws, stream=stream)

    steps = max(3, min(args.steps // 20, 10))
    secs = timed(step, steps, 2, dist, stream, "long-context forward")
    per = secs / steps
    nbytes = fwd_bytes(B, T, H)
    ach = nbytes / per / 1e9
    # launches per call: one pass, or the dual pass + the entry-state chain + the fix-up
    per_call = 3 if ws_n else 1
    return {"value": aggregate_throughput(B * T * H, per, dist.world), "unit": "head-tokens/s",
            "ms_per_step": per * 1e3, "steps": steps, "launches": per_call * steps,
            "workspace_bytes": ws_n,
            "roofline": {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": ach / peaks["hbm_gbs"], "per_unit": "896 B per head-token + 32 KiB state per head",
                         "units_per_launch": B * T * H},
            "config": {"workload": "long_b1_t65536_h32_chunk32", "B": B, "T": T, "H": H, "N": N, "algo": "chunk",
                       "chunk_len": cfg["chunk_len"],
                       "tc_operands": TC_OPERANDS,
                       "w": "exp(-0.6065 sigmoid(x)), x ~ N(-2, 1)",
                       "l2": "no flush: each step reads 1.6 GB of inputs (> 126 MB L2)"}}


def cpu_baseline(d, budget_s=10.0):
    """The oracle as it stands on this host's cores: forward over the first
    heads of the prefill workload (all T tokens), repeated up to budget_s."""
    import oracle
    cores = oracle.max_threads()
    nh = min(FWD["B"] * FWD["H"], max(8, 2 * cores))
    sel = [(b, h) for b in range(FWD["B"]) for h in range(FWD["H"])][:nh]
    bs = [b for b, _ in sel]
    hs = [h for _, h in sel]
    # each selected (b, h) becomes a batch row of a one-head problem: [nh, T, 1, N]
    args = [inputs.to_f64(d[n][bs, :, hs])[:, :, None] for n in inputs.INPUT_NAMES]
    s0 = d["s0"][bs, hs][:, None].astype(np.float64)
    done, t0 = 0, time.perf_counter()
    while True:
        oracle.forward(*args, s0=s0)
        done += 1
        el = time.perf_counter() - t0
        if el >= budget_s or done >= 50:
            break
    return {"value": done * nh * FWD["T"] / el, "unit": "head-tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{nh} heads x T={FWD['T']} of the prefill workload, fp64 C oracle, {done} pass(es), "
                      f"{el:.1f} s"}


def run_ours(args):
    import torch
    dist = Dist("nccl").init()
    device = torch.device("cuda", dist.local)
    from linear_rnn_sequence_wkv7_b200 import wkv7
    wkv7.load_library()
    peaks = load_peaks()
    parts = set(args.parts.split(","))

    steps_in = {}
    gen_thread = None
    if "decode" in parts:
        def gen():
            steps_in.update(inputs.gen_steps(args.decode_steps, DEC["B"], DEC["H"], N,
                                             seed=shard_seed(DEC["seed"], dist.rank), dtype="bf16"))
        gen_thread = threading.Thread(target=gen)
        gen_thread.start()

    fwd = bench_forward(args, dist, peaks, device)
    out_parts = {}
    launches = fwd["launches"]
    if "bwd" in parts:
        out_parts["backward"] = bench_backward(args, dist, peaks, device, fwd["sample"])
    if "train" in parts:
        out_parts["train_step"] = bench_train(args, dist, peaks, device, fwd["sample"])
    if gen_thread is not None:
        gen_thread.join()
        out_parts["decode"] = bench_decode(args, dist, peaks, device, steps_in)
    if "long" in parts:
        out_parts["long_context"] = bench_long(args, dist, peaks, device)
    if "timemix" in parts:
        out_parts["timemix"] = bench_timemix(args, dist, peaks, device, fwd["sample"], fwd["ms_per_step"])
    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(fwd["sample"])
    line = {
        "metric": METRIC,
        "value": fwd["value"],
        "unit": "head-tokens/s",
        "n_gpus": dist.world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": fwd["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": "prefill_b8_t4096_h32_bf16", "B": FWD["B"], "T": FWD["T"], "H": FWD["H"],
                   "N": N, "io_dtype": "bf16", "state_dtype": "f32", "algo": args.algo,
                   "kernel": fwd["roofline"]["kernel"],
                   "tc_operands": TC_OPERANDS if fwd["roofline"]["kernel"] == "fwd_chunk" else None,
                   "l2": "no flush: each step reads 805 MB of inputs (> 126 MB L2)",
                   "parallelism": f"dp{dist.world} (independent batches per GPU)"},
        "roofline": fwd["roofline"],
        "cpu_baseline": cpu,
        "e2e": fwd["e2e"],
        "gpu_launches": launches,
        "clocks": fwd["clocks"],
        "parts": out_parts,
    }
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()


# ---------------------------------------------------------------------------
# reference arm: the fp64 oracle on the host cores
# ---------------------------------------------------------------------------

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    cores = oracle.max_threads()
    # one step = forward over `nh` heads x `Ts` tokens of the prefill workload,
    # sized so that warmup + steps finish in about two minutes
    d = inputs.gen_sequence(1, FWD["T"], FWD["H"], N, seed=FWD["seed"], dtype="bf16", s0_std=FWD["s0_std"])
    nh = min(FWD["H"], max(1, cores))
    full = [inputs.to_f64(d[n][:, :, :nh]) for n in inputs.INPUT_NAMES]
    s0 = d["s0"][:, :nh].astype(np.float64)
    t0 = time.perf_counter()
    oracle.forward(*(x[:, :256] for x in full), s0=s0)
    rate = nh * 256 / max(time.perf_counter() - t0, 1e-6)
    budget = min(1.0, 120.0 / max(1, args.steps + args.warmup))
    Ts = int(min(FWD["T"], max(16, rate * budget / nh)))
    sample = [x[:, :Ts] for x in full]
    for _ in range(args.warmup):
        oracle.forward(*sample, s0=s0)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.forward(*sample, s0=s0)
    el = time.perf_counter() - t0
    value = args.steps * nh * Ts / el
    desc = f"{nh} heads x T={Ts} of the prefill workload per step, fp64 C oracle"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "head-tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "prefill_b8_t4096_h32_bf16", "B": FWD["B"], "T": FWD["T"], "H": FWD["H"],
                   "N": N, "sample": desc},
        "cpu_baseline": {"value": value, "unit": "head-tokens/s", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "head-tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

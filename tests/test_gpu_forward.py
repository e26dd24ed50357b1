"""GPU forward (through the C ABI) vs the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from linear_rnn_sequence_wkv7_b200 import inputs, wkv7
from tests._dev import oracle_args, to_dev, to_f64
from tests._tol import TAU_BF16, TAU_F32, assert_close

pytestmark = pytest.mark.gpu


def run_forward(d, y_dtype=None, algo="seq", s0=True):
    args = [to_dev(d[n]) for n in inputs.INPUT_NAMES]
    s0_t = to_dev(d["s0"]) if (s0 and d["s0"] is not None) else None
    y, sT = wkv7.forward(*args, s0=s0_t, y_dtype=y_dtype, algo=algo)
    torch.cuda.synchronize()
    return y, sT


def oracle_forward(d, heads=None):
    raw = [d[n] for n in inputs.INPUT_NAMES]
    s0 = d["s0"]
    if heads is not None:       # slice before widening to fp64
        raw = [x[:, :, heads] for x in raw]
        s0 = None if s0 is None else s0[:, heads]
    args = [inputs.to_f64(x) for x in raw]
    return oracle.forward(*args, s0=None if s0 is None else s0.astype(np.float64))


def test_fp32_reference_workload(cuda_device):
    """B=1, T=64, H=2, fp32 everywhere, zero s0: max err <= 1e-5 rms."""
    cfg = inputs.WORKLOADS["fwd_b1_t64_h2_f32"]
    d = inputs.gen_sequence(cfg["B"], cfg["T"], cfg["H"], cfg["N"], seed=cfg["seed"], dtype="f32")
    y, sT = run_forward(d)
    yr, sr = oracle_forward(d)
    assert_close(to_f64(y), yr, TAU_F32, "y")
    assert_close(to_f64(sT), sr, TAU_F32, "sT")


@pytest.mark.parametrize("T", [1, 2, 15, 16, 17, 63, 64, 65, 200])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_small_shapes(cuda_device, T, dtype):
    B, H, N = 2, 3, 64
    d = inputs.gen_sequence(B, T, H, N, seed=100 + T, dtype=dtype, s0_std=0.1)
    yr, sr = oracle_forward(d)
    tau = TAU_F32 if dtype == "f32" else TAU_BF16
    y, sT = run_forward(d, y_dtype=torch.float32)
    assert_close(to_f64(y), yr, tau, "y")
    assert_close(to_f64(sT), sr, tau, "sT")
    if dtype == "bf16":
        yb, _ = run_forward(d, y_dtype=torch.bfloat16)
        assert yb.dtype == torch.bfloat16
        assert_close(to_f64(yb), yr, tau, "y(bf16 out)", bf16_out=True)


def test_zero_initial_state_and_no_final_state(cuda_device):
    B, T, H, N = 1, 33, 2, 64
    d = inputs.gen_sequence(B, T, H, N, seed=7, dtype="bf16")
    args = [to_dev(d[n]) for n in inputs.INPUT_NAMES]
    y = wkv7.forward(*args, s0=None, y_dtype=torch.float32, algo="seq", return_state=False)
    yr, _ = oracle_forward(d)
    assert_close(to_f64(y), yr, TAU_BF16, "y")


def test_state_passing_in_place(cuda_device):
    """forward(T) == forward(T1) then forward(T - T1) continuing from sT (s0 aliasing sT)."""
    B, T, H, N = 2, 100, 2, 64
    d = inputs.gen_sequence(B, T, H, N, seed=9, dtype="f32", s0_std=0.1)
    args = [to_dev(d[n]) for n in inputs.INPUT_NAMES]
    s0 = to_dev(d["s0"])
    y_full, s_full = wkv7.forward(*args, s0=s0, algo="seq")
    state = s0.clone()
    y1 = wkv7.forward(*(x[:, :37].contiguous() for x in args), s0=state, sT=state, algo="seq")[0]
    y2 = wkv7.forward(*(x[:, 37:].contiguous() for x in args), s0=state, sT=state, algo="seq")[0]
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([y1, y2], dim=1), y_full)
    assert torch.equal(state, s_full)


def test_empty_sequence_copies_state(cuda_device):
    s0 = torch.randn(2, 3, 64, 64, device="cuda")
    e = torch.empty(2, 0, 3, 64, device="cuda")
    y, sT = wkv7.forward(e, e, e, e, e, e, s0=s0, algo="seq")
    torch.cuda.synchronize()
    assert y.shape == (2, 0, 3, 64)
    assert torch.equal(sT, s0)
    y, sT = wkv7.forward(e, e, e, e, e, e, s0=None, algo="seq")
    torch.cuda.synchronize()
    assert torch.count_nonzero(sT) == 0


def test_invalid_arguments_raise(cuda_device):
    x = torch.zeros(1, 4, 1, 32, device="cuda")
    with pytest.raises(wkv7.WKV7Error) as ei:
        wkv7.forward(x, x, x, x, x, x, algo="seq")
    assert ei.value.status == wkv7.ERR_UNSUPPORTED


def _sample_heads(H, n, seed):
    return sorted(np.random.default_rng(seed).choice(H, size=min(n, H), replace=False).tolist())


def test_prefill_workload_sampled_heads(cuda_device):
    """B=8, T=4096, H=32 bf16 prefill (the benchmark's launch): y (bf16) and sT on
    sampled heads of every batch row vs the oracle."""
    cfg = inputs.WORKLOADS["prefill_b8_t4096_h32_bf16"]
    d = inputs.gen_sequence(cfg["B"], cfg["T"], cfg["H"], cfg["N"], seed=cfg["seed"], dtype="bf16",
                            s0_std=cfg["s0_std"])
    assert wkv7.resolve_algo(cfg["T"], torch.bfloat16, "auto") == "chunk"
    y, sT = run_forward(d, algo="auto")
    assert wkv7.device_status() == wkv7.OK
    heads = _sample_heads(cfg["H"], cfg["H"] // 8, 0)      # an eighth of the heads of every batch row
    yr, sr = oracle_forward(d, heads)
    assert_close(to_f64(y[:, :, heads]), yr, TAU_BF16, "y", bf16_out=True)
    assert_close(to_f64(sT[:, heads]), sr, TAU_BF16, "sT")


def test_long_context_workload_sampled_heads(cuda_device):
    """B=1, T=65536, H=32 with w near 1 (long memory): sequential scan on sampled heads."""
    cfg = inputs.WORKLOADS["long_b1_t65536_h32_chunk32"]
    d = inputs.gen_sequence(cfg["B"], cfg["T"], cfg["H"], cfg["N"], seed=cfg["seed"], dtype="bf16",
                            x_mean=cfg["x_mean"], s0_std=cfg["s0_std"])
    y, sT = run_forward(d, y_dtype=torch.float32, algo="seq")
    heads = _sample_heads(cfg["H"], cfg["H"] // 8, 1)
    yr, sr = oracle_forward(d, heads)
    assert_close(to_f64(y[:, :, heads]), yr, TAU_BF16, "y")
    assert_close(to_f64(sT[:, heads]), sr, TAU_BF16, "sT")


# --- chunked tensor-core form ------------------------------------------------------

@pytest.mark.parametrize("T", [1, 15, 32, 33, 64, 65, 200])
def test_chunked_small_shapes(cuda_device, T):
    B, H, N = 2, 3, 64
    d = inputs.gen_sequence(B, T, H, N, seed=200 + T, dtype="bf16", s0_std=0.1)
    yr, sr = oracle_forward(d)
    y, sT = run_forward(d, y_dtype=torch.float32, algo="chunk")
    assert_close(to_f64(y), yr, TAU_BF16, "y")
    assert_close(to_f64(sT), sr, TAU_BF16, "sT")
    yb, _ = run_forward(d, y_dtype=torch.bfloat16, algo="chunk")
    assert_close(to_f64(yb), yr, TAU_BF16, "y(bf16 out)", bf16_out=True)
    assert wkv7.device_status() == wkv7.OK


def test_chunked_zero_state_and_in_place(cuda_device):
    B, T, H, N = 2, 130, 2, 64
    d = inputs.gen_sequence(B, T, H, N, seed=301, dtype="bf16", s0_std=0.1)
    args = [to_dev(d[n]) for n in inputs.INPUT_NAMES]
    y0 = wkv7.forward(*args, s0=None, y_dtype=torch.float32, algo="chunk", return_state=False)
    d0 = dict(d, s0=None)
    yr, _ = oracle_forward(d0)
    assert_close(to_f64(y0), yr, TAU_BF16, "y (zero s0)")
    state = to_dev(d["s0"])
    y1, _ = wkv7.forward(*args, s0=state, sT=state, y_dtype=torch.float32, algo="chunk")
    yr1, sr1 = oracle_forward(d)
    assert_close(to_f64(y1), yr1, TAU_BF16, "y")
    assert_close(to_f64(state), sr1, TAU_BF16, "sT in place")


def test_auto_picks_chunked_for_bf16():
    assert wkv7.resolve_algo(4096, torch.bfloat16, "auto") == "chunk"
    assert wkv7.resolve_algo(4096, torch.float32, "auto") == "seq"
    assert wkv7.resolve_algo(32, torch.bfloat16, "auto") == "seq"


def test_chunked_rejects_fp32_inputs(cuda_device):
    x = torch.zeros(1, 64, 1, 64, device="cuda")
    with pytest.raises(wkv7.WKV7Error) as ei:
        wkv7.forward(x, x, x, x, x, x, algo="chunk")
    assert ei.value.status == wkv7.ERR_UNSUPPORTED


def test_chunked_flags_out_of_domain_decay(cuda_device):
    """A chunk whose decay product underflows the fp32 range raises the RANGE
    status word (no fault); the sequential form handles the same input."""
    B, T, H, N = 1, 64, 1, 64
    d = inputs.gen_sequence(B, T, H, N, seed=5, dtype="bf16")
    d["w"] = inputs.f32_to_bf16_bits(np.full((B, T, H, N), 0.05, np.float32))
    assert wkv7.device_status() == wkv7.OK
    run_forward(d, y_dtype=torch.float32, algo="chunk")
    assert wkv7.last_status() == wkv7.ERR_RANGE
    assert wkv7.last_status() == wkv7.OK            # cleared by the read
    lib = wkv7.load_library()
    run_forward(d, y_dtype=torch.float32, algo="chunk")
    assert lib.wkv7_get_device_status(None) == wkv7.ERR_RANGE     # the earlier name of the same call
    with wkv7.status_checks(True):                  # the binding's per-call check raises instead
        with pytest.raises(wkv7.WKV7Error) as ei:
            run_forward(d, y_dtype=torch.float32, algo="chunk")
    assert ei.value.status == wkv7.ERR_RANGE
    assert wkv7.last_status() == wkv7.OK
    y, sT = run_forward(d, y_dtype=torch.float32, algo="seq")
    yr, sr = oracle_forward(d)
    assert_close(to_f64(y), yr, TAU_BF16, "y (seq)")


def test_long_context_chunked_matches_oracle_and_sequential(cuda_device):
    """B=1, T=65536, H=32, w near 1, chunked form: sampled heads vs the oracle,
    and every head vs the sequential scan."""
    cfg = inputs.WORKLOADS["long_b1_t65536_h32_chunk32"]
    d = inputs.gen_sequence(cfg["B"], cfg["T"], cfg["H"], cfg["N"], seed=cfg["seed"], dtype="bf16",
                            x_mean=cfg["x_mean"], s0_std=cfg["s0_std"])
    yc, sc = run_forward(d, y_dtype=torch.float32, algo="chunk")
    assert wkv7.device_status() == wkv7.OK
    heads = _sample_heads(cfg["H"], cfg["H"] // 8, 2)
    yr, sr = oracle_forward(d, heads)
    assert_close(to_f64(yc[:, :, heads]), yr, TAU_BF16, "y vs oracle")
    assert_close(to_f64(sc[:, heads]), sr, TAU_BF16, "sT vs oracle")
    ys, ss = run_forward(d, y_dtype=torch.float32, algo="seq")
    for h in range(cfg["H"]):
        assert_close(to_f64(yc[:, :, h]), to_f64(ys[:, :, h]), TAU_BF16, f"y head {h} vs seq")
    assert_close(to_f64(sc), to_f64(ss), TAU_BF16, "sT vs seq")


def test_chunked_wait_timeout_reports_and_recovers(cuda_device):
    """A device-side wait that runs out (limit forced to 1 cycle) makes the
    chunked kernel give up cleanly: WKV7_ERR_TIMEOUT in the status word, no
    fault, and the next launch with the default limit is correct."""
    B, T, H, N = 1, 96, 2, 64
    d = inputs.gen_sequence(B, T, H, N, seed=77, dtype="bf16", s0_std=0.1)
    assert wkv7.device_status() == wkv7.OK
    wkv7.set_wait_limit(1)
    try:
        run_forward(d, y_dtype=torch.float32, algo="chunk")
        status = wkv7.device_status()
    finally:
        wkv7.set_wait_limit(0)
    assert status == wkv7.ERR_TIMEOUT
    y, sT = run_forward(d, y_dtype=torch.float32, algo="chunk")
    assert wkv7.device_status() == wkv7.OK
    yr, sr = oracle_forward(d)
    assert_close(to_f64(y), yr, TAU_BF16, "y after recovery")
    assert_close(to_f64(sT), sr, TAU_BF16, "sT after recovery")


def test_scan_tile_wait_timeout_reports_and_recovers(cuda_device):
    """The sequential scan's wait for its TMA tile (the one-CTA-per-head
    layout: more heads than SMs) with the limit forced to 1 cycle: every CTA
    gives up on its first tile, lets that copy land and stops; the status word
    reads WKV7_ERR_TIMEOUT, nothing faults, and the next launch with the
    default limit is correct (sampled heads vs the oracle)."""
    B, T, H, N = 5, 40, 32, 64                   # 160 heads
    d = inputs.gen_sequence(B, T, H, N, seed=78, dtype="bf16", s0_std=0.1)
    assert wkv7.device_status() == wkv7.OK
    wkv7.set_wait_limit(1)
    try:
        run_forward(d, y_dtype=torch.float32, algo="seq")
        status = wkv7.device_status()
    finally:
        wkv7.set_wait_limit(0)
    assert status == wkv7.ERR_TIMEOUT
    y, sT = run_forward(d, y_dtype=torch.float32, algo="seq")
    assert wkv7.device_status() == wkv7.OK
    heads = [0, 31]
    raw = [d[n][:, :, heads] for n in inputs.INPUT_NAMES]
    yr, sr = oracle.forward(*map(inputs.to_f64, raw), s0=d["s0"][:, heads].astype(np.float64))
    assert_close(to_f64(y[:, :, heads]), yr, TAU_BF16, "y after recovery")
    assert_close(to_f64(sT[:, heads]), sr, TAU_BF16, "sT after recovery")


# --- chunked form over sequence segments (few heads, long sequences) -----------------

@pytest.mark.parametrize("T", [512, 700, 2000, 4097])
def test_chunked_segments_match_oracle_and_single_pass(cuda_device, T):
    """With B*H heads too few to fill the GPU the chunked form splits the
    sequence into segments (summary pass, entry-state scan, output pass).
    Ragged last segment, nonzero s0: y and sT vs the oracle, and vs the same
    call run in one pass (workspace too small)."""
    B, H, N = 1, 2, 64
    assert wkv7.forward_workspace_size(B, T, H, N, torch.bfloat16, "chunk") > 0
    d = inputs.gen_sequence(B, T, H, N, seed=400 + T, dtype="bf16", s0_std=0.1)
    yr, sr = oracle_forward(d)
    y, sT = run_forward(d, y_dtype=torch.float32, algo="chunk")
    assert wkv7.device_status() == wkv7.OK
    assert_close(to_f64(y), yr, TAU_BF16, "y")
    assert_close(to_f64(sT), sr, TAU_BF16, "sT")
    args = [to_dev(d[n]) for n in inputs.INPUT_NAMES]
    tiny = torch.empty(16, dtype=torch.uint8, device="cuda")
    y1, s1 = wkv7.forward(*args, s0=to_dev(d["s0"]), y_dtype=torch.float32, algo="chunk", workspace=tiny)
    torch.cuda.synchronize()
    assert_close(to_f64(y), to_f64(y1), TAU_BF16, "y segmented vs one pass")
    assert_close(to_f64(sT), to_f64(s1), TAU_BF16, "sT segmented vs one pass")


def test_chunked_segments_zero_state_in_place_and_bf16_out(cuda_device):
    B, T, H, N = 2, 1500, 1, 64
    assert wkv7.forward_workspace_size(B, T, H, N, torch.bfloat16, "chunk") > 0
    d = inputs.gen_sequence(B, T, H, N, seed=451, dtype="bf16", s0_std=0.1)
    args = [to_dev(d[n]) for n in inputs.INPUT_NAMES]
    y0 = wkv7.forward(*args, s0=None, y_dtype=torch.bfloat16, algo="chunk", return_state=False)
    torch.cuda.synchronize()
    yr0, _ = oracle_forward(dict(d, s0=None))
    assert_close(to_f64(y0), yr0, TAU_BF16, "y (zero s0, bf16 out)", bf16_out=True)
    state = to_dev(d["s0"])
    y1, _ = wkv7.forward(*args, s0=state, sT=state, y_dtype=torch.float32, algo="chunk")
    torch.cuda.synchronize()
    yr1, sr1 = oracle_forward(d)
    assert_close(to_f64(y1), yr1, TAU_BF16, "y")
    assert_close(to_f64(state), sr1, TAU_BF16, "sT in place")
    assert wkv7.device_status() == wkv7.OK


def test_forward_workspace_size_rules(cuda_device):
    """Scratch only for the chunked form with too few heads for the GPU."""
    assert wkv7.forward_workspace_size(8, 4096, 32, 64, torch.bfloat16, "chunk") == 0
    assert wkv7.forward_workspace_size(1, 65536, 32, 64, torch.bfloat16, "chunk") > 0
    assert wkv7.forward_workspace_size(1, 65536, 32, 64, torch.bfloat16, "seq") == 0
    assert wkv7.forward_workspace_size(1, 65536, 32, 64, torch.float32, "auto") == 0
    assert wkv7.forward_workspace_size(1, 200, 1, 64, torch.bfloat16, "chunk") == 0

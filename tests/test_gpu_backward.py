"""GPU backward (through the C ABI) vs the fp64 oracle and finite differences."""
import numpy as np
import pytest
import torch

import oracle
from linear_rnn_sequence_wkv7_b200 import inputs, wkv7
from tests._dev import oracle_args, to_dev, to_f64
from tests._tol import TAU_BF16, TAU_F32, assert_close

pytestmark = pytest.mark.gpu

GRAD_NAMES = ("dr", "dw", "dk", "dv", "da", "db", "ds0")


def _case(B, T, H, seed, dtype, dsT=True):
    N = 64
    d = inputs.gen_sequence(B, T, H, N, seed=seed, dtype=dtype, s0_std=0.1)
    d["dy"] = inputs.gen_dy(B, T, H, N, seed=seed, dtype=dtype)
    d["dsT"] = (inputs.gen_normal(B * H * N, N, seed=seed, stream=inputs.STREAM_DST, std=0.1)
                .reshape(B, H, N, N) if dsT else None)
    return d


def _gpu(d, grad_dtype=torch.float32, heads=None):
    args = [to_dev(d[n]) for n in inputs.INPUT_NAMES]
    out = wkv7.backward(*args, to_dev(d["s0"]), to_dev(d["dy"]), to_dev(d["dsT"]), grad_dtype=grad_dtype)
    torch.cuda.synchronize()
    if heads is not None:       # gather the sampled heads on the device first
        out = [x[:, :, heads] for x in out[:6]] + [out[6][:, heads]]
    return [to_f64(x) for x in out]


def _ref(d, heads=None):
    raw = [d[n] for n in inputs.INPUT_NAMES] + [d["dy"]]
    s0, dsT = d["s0"], d["dsT"]
    if heads is not None:       # slice before widening to fp64
        raw = [x[:, :, heads] for x in raw]
        s0 = s0[:, heads]
        dsT = None if dsT is None else dsT[:, heads]
    args = [inputs.to_f64(x) for x in raw]
    return oracle.backward(*args[:6], s0.astype(np.float64), args[6],
                           None if dsT is None else dsT.astype(np.float64))


@pytest.mark.parametrize("T", [1, 5, 16, 17, 48, 100])
def test_fp32_small(cuda_device, T):
    d = _case(2, T, 2, 300 + T, "f32")
    for name, got, ref in zip(GRAD_NAMES, _gpu(d), _ref(d)):
        assert_close(got, ref, TAU_F32, name)


@pytest.mark.parametrize("dtype,T", [("f32", 1000), ("bf16", 3000)])
def test_few_heads_long_sequence(cuda_device, dtype, T):
    """One head: the state-gradient sweep runs as segments (and, for bf16,
    the checkpoint pass as the segmented forward); the fp32 path keeps 1e-5."""
    d = _case(1, T, 1, 350 + T, dtype)
    assert wkv7.backward_workspace_size(1, T, 1, 64) > 2 * ((T + 31) // 32 + 1) * 64 * 64 * 4
    tau = TAU_F32 if dtype == "f32" else TAU_BF16
    for name, got, ref in zip(GRAD_NAMES, _gpu(d), _ref(d)):
        assert_close(got, ref, tau, name)


@pytest.mark.parametrize("T,with_dsT", [(1, True), (16, False), (32, True), (33, False), (77, False),
                                         (200, True)])
def test_bf16_inputs(cuda_device, T, with_dsT):
    """bf16 inputs (chunk gradients on the tensor cores): one token, a full
    chunk, ragged tails, several chunks, with and without dsT."""
    d = _case(2, T, 3, 400 + T, "bf16", dsT=with_dsT)
    ref = _ref(d)
    for name, got, r in zip(GRAD_NAMES, _gpu(d), ref):
        assert_close(got, r, TAU_BF16, name)
    for name, got, r in zip(GRAD_NAMES[:6], _gpu(d, torch.bfloat16)[:6], ref[:6]):
        assert_close(got, r, TAU_BF16, name + "(bf16 out)", bf16_out=True)


def test_empty_sequence_copies_dsT(cuda_device):
    e = torch.empty(1, 0, 2, 64, device="cuda")
    dsT = torch.randn(1, 2, 64, 64, device="cuda")
    out = wkv7.backward(e, e, e, e, e, e, None, e, dsT)
    torch.cuda.synchronize()
    assert torch.equal(out[-1], dsT)


def test_central_differences_slice(cuda_device):
    """B=1, T=16, H=1 (fp32): GPU gradients vs central differences of the fp64
    forward, independent of the oracle's own backward."""
    d = _case(1, 16, 1, 500, "f32")
    got = _gpu(d)
    args = oracle_args(d)
    s0, dy, dsT = d["s0"].astype(np.float64), inputs.to_f64(d["dy"]), d["dsT"].astype(np.float64)
    tensors = args + [s0]
    rng = np.random.default_rng(0)
    h = 1e-6

    def loss():
        y, sT = oracle.forward(*tensors[:6], s0=tensors[6])
        return float(np.sum(dy * y) + np.sum(dsT * sT))

    for x, g, name in zip(tensors, got, GRAD_NAMES):
        flat = x.reshape(-1)
        coords = rng.choice(flat.size, 64, replace=False)
        fd = np.empty(len(coords))
        for n, c in enumerate(coords):
            old = flat[c]
            flat[c] = old + h
            lp = loss()
            flat[c] = old - h
            lm = loss()
            flat[c] = old
            fd[n] = (lp - lm) / (2 * h)
        sel = g.reshape(-1)[coords]
        scale = np.sqrt(np.mean(g ** 2))
        assert np.max(np.abs(sel - fd)) <= 1e-5 * scale + 1e-7, name


def test_central_differences_training_slice_bf16(cuda_device):
    """The training workload's B=1, T=16, H=1 slice (first batch row, first 16
    tokens, head 0; bf16 inputs and dy, dsT = 0), whose chunk gradients run on
    the tensor cores: every GPU gradient vs central differences of the fp64
    forward at the same (bf16) input values, within the bf16-input bound
    2e-3 * rms of the oracle's gradient.  The differences use only the
    oracle's forward, not its backward."""
    cfg = inputs.WORKLOADS["train_bwd_b8_t4096_h32"]
    full = inputs.gen_sequence(cfg["B"], cfg["T"], cfg["H"], cfg["N"], seed=cfg["seed"], dtype="bf16",
                               s0_std=cfg["s0_std"])
    dy_full = inputs.gen_dy(cfg["B"], cfg["T"], cfg["H"], cfg["N"], seed=cfg["seed"], dtype="bf16")
    d = {n: np.ascontiguousarray(full[n][:1, :16, :1]) for n in inputs.INPUT_NAMES}
    d["s0"] = np.ascontiguousarray(full["s0"][:1, :1])
    d["dy"] = np.ascontiguousarray(dy_full[:1, :16, :1])
    d["dsT"] = None
    got = _gpu(d)
    ref = _ref(d)
    args = oracle_args(d)
    s0, dy = d["s0"].astype(np.float64), inputs.to_f64(d["dy"])
    tensors = args + [s0]
    rng = np.random.default_rng(1)
    h = 1e-6

    def loss():
        y, _ = oracle.forward(*tensors[:6], s0=tensors[6])
        return float(np.sum(dy * y))

    for x, g, r, name in zip(tensors, got, ref, GRAD_NAMES):
        flat = x.reshape(-1)
        coords = rng.choice(flat.size, min(flat.size, 256), replace=False)
        fd = np.empty(len(coords))
        for n, c in enumerate(coords):
            old = flat[c]
            flat[c] = old + h
            lp = loss()
            flat[c] = old - h
            lm = loss()
            flat[c] = old
            fd[n] = (lp - lm) / (2 * h)
        sel = g.reshape(-1)[coords]
        scale = np.sqrt(np.mean(r ** 2))
        assert np.max(np.abs(sel - fd)) <= TAU_BF16 * scale, (name, np.max(np.abs(sel - fd)) / scale)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_mid_head_count_sampled_heads(cuda_device, dtype):
    """B=4, T=1024, H=32 (128 heads): the state-gradient sweep takes four
    rows per thread with eight lanes per row; sampled heads vs the oracle,
    with a dL/dS_T term."""
    d = _case(4, 1024, 32, 360, dtype)
    heads = [5, 30]
    tau = TAU_F32 if dtype == "f32" else TAU_BF16
    for name, got, ref in zip(GRAD_NAMES, _gpu(d, heads=heads), _ref(d, heads=heads)):
        assert_close(got, ref, tau, name)


def test_training_workload_sampled_heads(cuda_device):
    """B=8, T=4096, H=32 bf16 with dy ~ N(0,1) bf16 and dsT = 0: a random eighth
    of the heads of every batch row vs the oracle's reverse-time pass."""
    cfg = inputs.WORKLOADS["train_bwd_b8_t4096_h32"]
    d = inputs.gen_sequence(cfg["B"], cfg["T"], cfg["H"], cfg["N"], seed=cfg["seed"], dtype="bf16",
                            s0_std=cfg["s0_std"])
    d["dy"] = inputs.gen_dy(cfg["B"], cfg["T"], cfg["H"], cfg["N"], seed=cfg["seed"], dtype="bf16")
    d["dsT"] = None
    heads = sorted(np.random.default_rng(4).choice(cfg["H"], cfg["H"] // 8, replace=False).tolist())
    got = _gpu(d, heads=heads)
    ref = _ref(d, heads)
    for name, g, r in zip(GRAD_NAMES, got, ref):
        assert_close(g, r, TAU_BF16, name)


def _transition_bytes(B, T, H):
    """Bytes of the chunks' transition images ([M^T; Q] per 32-token chunk,
    bf16 hi and lo: 24 KiB) that the backward's workspace holds on top of its
    minimum."""
    return B * H * ((T + 31) // 32) * 24576


def _kernel_names(fn):
    """Names of the CUDA kernels fn launches (empty when the profiler
    records no device activity in this PyTorch installation)."""
    from torch.profiler import ProfilerActivity, profile
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        fn()
        torch.cuda.synchronize()
    return {e.name for e in prof.events()}


@pytest.mark.parametrize("B,T,H", [(2, 40, 3), (2, 333, 3), (1, 4096, 40)])
def test_bf16_dS_by_transition_chain_and_by_sweep(cuda_device, B, T, H):
    """With the full workspace the checkpoint pass exports every chunk's
    transition and dS at the chunk ends comes from the tensor-core chain
    dS_in = dS_out M^T + dY^T Q; a workspace without room for the images takes
    the per-token sweep.  Both vs the oracle (sampled heads for the larger
    case), and the kernels each one launches."""
    d = _case(B, T, H, 480 + T, "bf16")
    full = wkv7.backward_workspace_size(B, T, H, 64)
    heads = None if H <= 3 else [0, 17, 39]
    ref = _ref(d, heads=heads)
    args = [to_dev(d[n]) for n in inputs.INPUT_NAMES]
    s0, dy, dsT = to_dev(d["s0"]), to_dev(d["dy"]), to_dev(d["dsT"])
    for ws, kernel in ((full, "bwd_dchain_kernel"), (full - _transition_bytes(B, T, H), "bwd_dstate_kernel")):
        buf = torch.empty(ws, dtype=torch.uint8, device="cuda")
        out = []
        names = _kernel_names(lambda: out.append(wkv7.backward(*args, s0, dy, dsT, workspace=buf)))
        assert wkv7.last_status() == wkv7.OK
        if names:
            assert any(kernel in n for n in names), (ws, sorted(names))
        got = out[0]
        if heads is not None:
            got = [x[:, :, heads] for x in got[:6]] + [got[6][:, heads]]
        for name, g, r in zip(GRAD_NAMES, [to_f64(x) for x in got], ref):
            assert_close(g, r, TAU_BF16, f"{name} ({kernel})")
    # below the minimum the call is rejected before any launch
    buf = torch.empty(full - _transition_bytes(B, T, H) - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(RuntimeError):
        wkv7.backward(*args, s0, dy, dsT, workspace=buf)


def test_bf16_wait_timeout_reports_and_recovers(cuda_device):
    """Device-side waits forced to run out (limit 1 cycle): the backward's
    tensor-core kernels report WKV7_ERR_TIMEOUT without a fault, and the next
    call at the default limit is correct."""
    d = _case(1, 70, 2, 450, "bf16")
    assert wkv7.device_status() == wkv7.OK
    wkv7.set_wait_limit(1)
    try:
        _gpu(d)
        status = wkv7.device_status()
    finally:
        wkv7.set_wait_limit(0)
    assert status == wkv7.ERR_TIMEOUT
    got = _gpu(d)
    assert wkv7.device_status() == wkv7.OK
    for name, g, r in zip(GRAD_NAMES, got, _ref(d)):
        assert_close(g, r, TAU_BF16, name)

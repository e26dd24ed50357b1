"""GPU time-mix output epilogue (wkv7_forward_timemix, through the C ABI) vs
the oracle's forward_timemix.

Tolerance.  The epilogue's input o_t = y_t + u_t v_t carries the forward's
error, bounded like y: |o - o_ref| <= D = tau * rms(o_ref) (tau = 2e-3 for
bf16 inputs, 1e-5 for fp32).  Per head-token row with sigma = sqrt(var + eps),
a perturbation of at most D per channel moves the mean by at most D and sigma
by at most D (both are 1-Lipschitz in the max norm), so to first order
    |z - z_ref| <= |g gamma| (2 D / sigma + |o - mean| D / sigma^2)
plus, for a bf16 z, one bf16 rounding (2^-8 |z_ref|).  That is the bound the
tests apply, element by element (and a small absolute floor for fp32 rounding
of the epilogue itself)."""
import numpy as np
import pytest
import torch

import oracle
from linear_rnn_sequence_wkv7_b200 import inputs, wkv7
from tests._dev import to_dev, to_f64
from tests._tol import TAU_BF16, TAU_F32, assert_close

pytestmark = pytest.mark.gpu

N = 64
EPS = 1e-5


def _case(B, T, H, seed, dtype, gate=True, s0=True):
    d = inputs.gen_sequence(B, T, H, N, seed=seed, dtype=dtype, s0_std=0.1 if s0 else None)
    d["rho"], d["gamma"], d["beta"] = inputs.gen_timemix_params(H, N, seed=seed)
    d["g"] = inputs.gen_gate(B, T, H, N, seed=seed, dtype=dtype) if gate else None
    return d


def _gpu(d, out_dtype, algo, heads=None, params=True, workspace=None):
    args = [to_dev(d[n]) for n in inputs.INPUT_NAMES]
    kw = dict(rho=to_dev(d["rho"]), out_dtype=out_dtype, algo=algo, eps=EPS)
    if params:
        kw.update(gamma=to_dev(d["gamma"]), beta=to_dev(d["beta"]), g=to_dev(d["g"]))
    if workspace is not None:
        kw["workspace"] = workspace
    z, sT = wkv7.forward_timemix(*args, to_dev(d["s0"]), **kw)
    torch.cuda.synchronize()
    assert wkv7.last_status() == wkv7.OK
    if heads is not None:
        z, sT = z[:, :, heads], sT[:, heads]
    return to_f64(z), to_f64(sT)


def _ref(d, heads=None, params=True):
    raw = [d[n] for n in inputs.INPUT_NAMES]
    s0, g, rho, gamma, beta = d["s0"], d["g"], d["rho"], d["gamma"], d["beta"]
    if heads is not None:
        raw = [x[:, :, heads] for x in raw]
        s0 = None if s0 is None else s0[:, heads]
        g = None if g is None else g[:, :, heads]
        rho, gamma, beta = rho[heads], gamma[heads], beta[heads]
    x = [inputs.to_f64(t) for t in raw]
    s0 = None if s0 is None else s0.astype(np.float64)
    gm, bt, gg = (gamma, beta, None if g is None else inputs.to_f64(g)) if params else (None, None, None)
    z, sT = oracle.forward_timemix(*x, s0, rho, gm, bt, gg, eps=EPS)
    # the pre-norm output o, for the tolerance
    y, _ = oracle.forward(*x, s0=s0)
    r, k, v = x[0], x[2], x[3]
    o = y + np.sum(r * rho.astype(np.float64) * k, axis=-1, keepdims=True) * v
    gfac = np.ones_like(z) if gg is None else gg
    gfac = gfac * (np.ones(z.shape[2:]) if gm is None else gm.astype(np.float64))
    return z, sT, o, gfac


def _assert_z(got, ref, o, gfac, tau, bf16_out, name="z"):
    D = tau * np.sqrt(np.mean(o * o))
    mu = o.mean(-1, keepdims=True)
    sig = np.sqrt(((o - mu) ** 2).mean(-1, keepdims=True) + EPS)
    bound = np.abs(gfac) * (2 * D / sig + np.abs(o - mu) * D / sig ** 2) + 1e-6 * (1 + np.abs(ref))
    if bf16_out:
        bound = bound + 2.0 ** -8 * np.abs(ref)
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    worst = np.argmax(err / bound)
    assert np.all(err <= bound), (f"{name}: err/bound = {np.max(err / bound):.3f} at {worst} "
                                  f"(got {got.flat[worst]!r}, ref {ref.flat[worst]!r})")


@pytest.mark.parametrize("T", [15, 33, 64, 200])
def test_chunked_fused_epilogue(cuda_device, T):
    """bf16 inputs, chunked form (the epilogue inside the chunked kernel):
    fp32 and bf16 z, ragged tails."""
    d = _case(2, T, 3, 600 + T, "bf16")
    z_ref, s_ref, o, gfac = _ref(d)
    for out_dtype, bf in ((torch.float32, False), (torch.bfloat16, True)):
        z, sT = _gpu(d, out_dtype, "chunk")
        _assert_z(z, z_ref, o, gfac, TAU_BF16, bf, f"z ({out_dtype})")
        assert_close(sT, s_ref, TAU_BF16, "sT")


@pytest.mark.parametrize("dtype,T", [("f32", 1), ("f32", 40), ("bf16", 70)])
def test_sequential_epilogue_pass(cuda_device, dtype, T):
    """The sequential scan plus the separate epilogue pass: fp32 inputs keep
    the fp32 bound; bf16 inputs forced onto the scan."""
    d = _case(2, T, 3, 650 + T, dtype)
    tau = TAU_F32 if dtype == "f32" else TAU_BF16
    z_ref, s_ref, o, gfac = _ref(d)
    z, sT = _gpu(d, torch.float32, "seq")
    _assert_z(z, z_ref, o, gfac, tau, False)
    assert_close(sT, s_ref, tau, "sT")


def test_defaults_give_the_normalised_readout(cuda_device):
    """gamma, beta, g left out (1, 0, 1), both paths."""
    d = _case(1, 96, 2, 700, "bf16")
    z_ref, _, o, gfac = _ref(d, params=False)
    for algo in ("chunk", "seq"):
        z, _ = _gpu(d, torch.float32, algo, params=False)
        _assert_z(z, z_ref, o, gfac, TAU_BF16, False, f"z ({algo})")


def test_state_is_the_plain_forward_state(cuda_device):
    """The current-token term is read, never written: sT equals wkv7_forward's
    (the same chunk algebra; only y's epilogue differs)."""
    d = _case(2, 130, 3, 710, "bf16")
    _, sT = _gpu(d, torch.float32, "chunk")
    args = [to_dev(d[n]) for n in inputs.INPUT_NAMES]
    _, s_plain = wkv7.forward(*args, s0=to_dev(d["s0"]), y_dtype=torch.float32, algo="chunk")
    torch.cuda.synchronize()
    assert_close(sT, to_f64(s_plain), 1e-6, "sT vs plain forward")


@pytest.mark.parametrize("T", [700, 2001])
def test_segmented_chunked_epilogue(cuda_device, T):
    """Few heads over many tokens: the chunked form runs as segments (dual
    summary runs, the first of them an output run, then output runs), each
    output run applying the epilogue."""
    B, H = 1, 2
    assert wkv7.forward_timemix_workspace_size(B, T, H, N, torch.bfloat16, "chunk") > 0
    d = _case(B, T, H, 720 + T, "bf16")
    z_ref, s_ref, o, gfac = _ref(d)
    z, sT = _gpu(d, torch.bfloat16, "chunk")
    _assert_z(z, z_ref, o, gfac, TAU_BF16, True)
    assert_close(sT, s_ref, TAU_BF16, "sT")


def test_prefill_workload_sampled_heads(cuda_device):
    """The prefill workload (B=8, T=4096, H=32 bf16) with the epilogue, bf16 z:
    an eighth of the heads of every batch row vs the oracle."""
    cfg = inputs.WORKLOADS["prefill_b8_t4096_h32_bf16"]
    B, T, H = cfg["B"], cfg["T"], cfg["H"]
    d = inputs.gen_sequence(B, T, H, N, seed=cfg["seed"], dtype="bf16", s0_std=cfg["s0_std"])
    d["rho"], d["gamma"], d["beta"] = inputs.gen_timemix_params(H, N, seed=cfg["seed"])
    d["g"] = inputs.gen_gate(B, T, H, N, seed=cfg["seed"], dtype="bf16")
    heads = sorted(np.random.default_rng(3).choice(H, H // 8, replace=False).tolist())
    z, sT = _gpu(d, torch.bfloat16, "auto", heads=heads)
    z_ref, s_ref, o, gfac = _ref(d, heads=heads)
    _assert_z(z, z_ref, o, gfac, TAU_BF16, True)
    assert_close(sT, s_ref, TAU_BF16, "sT")


def test_rejects_bad_arguments(cuda_device):
    x = torch.zeros(1, 64, 1, N, dtype=torch.bfloat16, device="cuda")
    rho = torch.zeros(1, N, device="cuda")
    lib = wkv7.load_library()
    ptr = [x.data_ptr()] * 6
    z = torch.empty_like(x)
    st = lib.wkv7_forward_timemix(1, 64, 1, N, wkv7.BF16, wkv7.BF16, *ptr, None, None, None, None, None, 1e-5,
                                  z.data_ptr(), None, wkv7.ALGO_CHUNK, 0, None, 0, None)
    assert st == wkv7.ERR_INVALID_ARG                            # rho is required
    st = lib.wkv7_forward_timemix(1, 64, 1, N, wkv7.BF16, wkv7.BF16, *ptr, None, rho.data_ptr(), None, None, None,
                                  -1.0, z.data_ptr(), None, wkv7.ALGO_CHUNK, 0, None, 0, None)
    assert st == wkv7.ERR_INVALID_ARG                            # eps < 0
    st = lib.wkv7_forward_timemix(1, 64, 1, N, wkv7.BF16, wkv7.BF16, *ptr, None, rho.data_ptr(), None, None, None,
                                  1e-5, z.data_ptr(), None, wkv7.ALGO_SEQ, 0, None, 0, None)
    assert st == wkv7.ERR_INVALID_ARG                            # the scan path needs its y workspace

"""Degenerate and extreme cases of the method through the GPU kernels, vs the
fp64 oracle: no removal (a = b = 0: decayed linear attention), exact delta
replacement, Householder transitions with no writes, decay exactly 1, and
the largest supported batch."""
import numpy as np
import pytest
import torch

import oracle
from linear_rnn_sequence_wkv7_b200 import inputs, wkv7
from tests._dev import to_dev, to_f64
from tests._tol import TAU_BF16, TAU_F32, assert_close

pytestmark = pytest.mark.gpu

N = 64


def _as(d, dtype):
    """Store float32 fields of d in the test dtype (bf16 bits or float32)."""
    out = dict(d)
    for n in inputs.INPUT_NAMES:
        x = np.asarray(d[n], np.float32)
        out[n] = inputs.f32_to_bf16_bits(x) if dtype == "bf16" else x
    return out


def _unit_keys(B, T, H, seed):
    rng = np.random.default_rng(seed)
    kh = rng.standard_normal((B, T, H, N)).astype(np.float32)
    return kh / np.linalg.norm(kh, axis=-1, keepdims=True)


def _run(d, algo, y_dtype=torch.float32):
    args = [to_dev(d[n]) for n in inputs.INPUT_NAMES]
    s0 = None if d["s0"] is None else to_dev(d["s0"])
    y, sT = wkv7.forward(*args, s0=s0, y_dtype=y_dtype, algo=algo)
    torch.cuda.synchronize()
    assert wkv7.device_status() == wkv7.OK
    return to_f64(y), to_f64(sT)


def _ref(d):
    args = [inputs.to_f64(d[n]) for n in inputs.INPUT_NAMES]
    return oracle.forward(*args, s0=None if d["s0"] is None else d["s0"].astype(np.float64))


def _check(d, algos, dtype):
    yr, sr = _ref(d)
    for algo in algos:
        tau = TAU_F32 if dtype == "f32" else TAU_BF16
        y, sT = _run(d, algo)
        assert_close(y, yr, tau, f"y ({algo})")
        assert_close(sT, sr, tau, f"sT ({algo})")


@pytest.mark.parametrize("dtype,algos", [("f32", ["seq"]), ("bf16", ["seq", "chunk"])])
def test_no_removal_is_decayed_linear_attention(cuda_device, dtype, algos):
    B, T, H = 1, 150, 2
    d = inputs.gen_sequence(B, T, H, N, seed=61, dtype="f32", s0_std=0.1)
    d["a"] = np.zeros_like(d["a"])
    d["b"] = np.zeros_like(d["b"])
    _check(_as(d, dtype), algos, dtype)


@pytest.mark.parametrize("dtype,algos", [("f32", ["seq"]), ("bf16", ["seq", "chunk"])])
def test_delta_rule_replacement(cuda_device, dtype, algos):
    """w = 1, a = -k, b = k, unit keys: each token replaces the value stored
    under its key (the oracle pins the exact property)."""
    B, T, H = 1, 130, 2
    d = inputs.gen_sequence(B, T, H, N, seed=62, dtype="f32", s0_std=0.1)
    kh = _unit_keys(B, T, H, 63)
    d.update(w=np.ones_like(kh), a=-kh, b=kh, k=kh)
    _check(_as(d, dtype), algos, dtype)
    if dtype == "f32":
        y, sT = _run(_as(d, dtype), "seq")
        # after the last token, S k_T = v_T
        Sk = np.einsum("bhij,bhj->bhi", sT, kh[:, -1].astype(np.float64))
        assert np.abs(Sk - d["v"][:, -1]).max() < 1e-4


@pytest.mark.parametrize("algo", ["seq", "chunk"])
def test_householder_transitions_without_writes(cuda_device, algo):
    """w = 1, a = -2k, b = k, v = 0: a long product of reflections (no decay,
    so no error is forgotten), T = 2048, vs the oracle on the same bf16 keys."""
    B, T, H = 1, 2048, 1
    d = inputs.gen_sequence(B, T, H, N, seed=64, dtype="f32", s0_std=0.1)
    kh = _unit_keys(B, T, H, 65)
    d.update(w=np.ones_like(kh), a=-2 * kh, b=kh, v=np.zeros_like(kh))
    _check(_as(d, "bf16"), [algo], "bf16")


@pytest.mark.parametrize("algo", ["seq", "chunk"])
def test_decay_exactly_one(cuda_device, algo):
    """w = 1 everywhere (no forgetting): the chunk's decay products are all 1."""
    B, T, H = 1, 200, 2
    d = inputs.gen_sequence(B, T, H, N, seed=66, dtype="f32", s0_std=0.1)
    d["w"] = np.ones_like(d["w"])
    _check(_as(d, "bf16"), [algo], "bf16")


def test_largest_batch(cuda_device):
    """B = 65535 (the largest the library accepts), H = 1, T = 3, zero initial
    state: sampled batch entries vs the oracle; B = 65536 is rejected."""
    B, T, H = 65535, 3, 1
    d = inputs.gen_sequence(B, T, H, N, seed=67, dtype="bf16")
    y, sT = _run(d, "seq")
    rows = [0, 1, 4097, B // 2, B - 1]
    sub = {n: d[n][rows] for n in inputs.INPUT_NAMES}
    sub["s0"] = None
    yr, sr = _ref(sub)
    assert_close(y[rows], yr, TAU_BF16, "y")
    assert_close(sT[rows], sr, TAU_BF16, "sT")
    x = torch.zeros(B + 1, T, H, N, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(wkv7.WKV7Error) as ei:
        wkv7.forward(x, x, x, x, x, x, algo="seq")
    assert ei.value.status == wkv7.ERR_UNSUPPORTED

"""Parity tolerances.

Per output tensor x with oracle value x_ref (fp64):
  max |x - x_ref| <= tau * rms(x_ref)
with tau = 1e-5 when every input is fp32 and tau = 2e-3 for bf16 inputs with
an fp32 state.  Outputs stored in bf16 are compared with the rounded oracle
value and allowed one extra bf16 rounding step: |x - x_ref| <= tau * rms +
2^-8 |x_ref| (RNE to 8 significant bits is within half an ulp, 2^-8 |x|).
"""
import numpy as np

TAU_F32 = 1e-5
TAU_BF16 = 2e-3


def rms(x):
    x = np.asarray(x, dtype=np.float64)
    return float(np.sqrt(np.mean(x * x))) if x.size else 0.0


def max_err_over_rms(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    s = rms(ref)
    return float(np.max(np.abs(got - ref)) / (s if s > 0 else 1.0)) if ref.size else 0.0


def assert_close(got, ref, tau, name="", bf16_out=False):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    if ref.size == 0:
        return
    bound = tau * rms(ref) + (2.0 ** -8) * np.abs(ref) * (1.0 if bf16_out else 0.0)
    err = np.abs(got - ref)
    worst = np.argmax(err - bound)
    assert np.all(err <= bound), (
        f"{name}: max|err|/rms = {max_err_over_rms(got, ref):.3e} > tau = {tau:.1e}"
        f" (worst at flat index {worst}: got {got.flat[worst]!r}, ref {ref.flat[worst]!r})")

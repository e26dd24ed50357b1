"""wkv7_backward_noalloc, the backward that takes its scratch from the
library's fixed device array instead of a workspace (for callers that cannot
allocate device memory where they run the backward).  It must give the same
gradients as wkv7_backward with a workspace, call after call, although every
call reuses the same array.  This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import oracle
from linear_rnn_sequence_wkv7_b200 import inputs, wkv7
from tests._dev import to_dev, to_f64
from tests._tol import TAU_BF16, TAU_F32, assert_close

pytestmark = pytest.mark.gpu

NAMES = ("dr", "dw", "dk", "dv", "da", "db", "ds0")


def _case(seed, B=2, T=77, H=3, dtype="f32"):
    N = 64
    d = inputs.gen_sequence(B, T, H, N, seed=seed, dtype=dtype, s0_std=0.1)
    x = [to_dev(d[n]) for n in inputs.INPUT_NAMES]
    dy = to_dev(inputs.gen_dy(B, T, H, N, seed=seed, dtype=dtype))
    dsT = to_dev(inputs.gen_normal(B * H * N, N, seed=seed, stream=inputs.STREAM_DST, std=0.1)
                 .reshape(B, H, N, N))
    return x, to_dev(d["s0"]), dy, dsT


def test_noalloc_backward_matches_workspace_backward(cuda_device):
    # two calls in a row on different inputs: the second must not see the first's scratch
    for seed in (910, 911):
        x, s0, dy, dsT = _case(seed)
        ref = wkv7.backward(*x, s0, dy, dsT)
        got = wkv7.backward_noalloc(*x, s0, dy, dsT)
        torch.cuda.synchronize()
        for name, g, r in zip(NAMES, got, ref):
            assert_close(to_f64(g), to_f64(r), TAU_F32, name)


def test_noalloc_backward_bf16_segmented_then_small(cuda_device):
    """bf16 inputs (checkpoints by the chunked forward, chunk gradients on the
    tensor cores).  First a few-head long sequence (B=1, T=1024, H=2) whose
    checkpoint pass and state-gradient sweep run as segments, so their
    per-segment scratch lives in the fixed array too; then a smaller problem
    on the same array.  Each call vs the backward with a workspace, and vs
    the oracle."""
    for seed, (B, T, H) in ((920, (1, 1024, 2)), (921, (2, 77, 3))):
        assert wkv7.backward_workspace_size(B, T, H, 64) <= (32 << 20)
        x, s0, dy, dsT = _case(seed, B=B, T=T, H=H, dtype="bf16")
        ref = wkv7.backward(*x, s0, dy, dsT)
        got = wkv7.backward_noalloc(*x, s0, dy, dsT)
        torch.cuda.synchronize()
        assert wkv7.last_status() == wkv7.OK
        args = [to_f64(t) for t in x]
        want = oracle.backward(*args, to_f64(s0), to_f64(dy), to_f64(dsT))
        for name, g, r, o in zip(NAMES, got, ref, want):
            assert_close(to_f64(g), to_f64(r), TAU_BF16, name + " vs workspace backward")
            assert_close(to_f64(g), o, TAU_BF16, name + " vs oracle")


def test_noalloc_backward_rejects_oversized_problems(cuda_device):
    B, T, H, N = 8, 4096, 32, 64
    assert wkv7.backward_workspace_size(B, T, H, N) > (32 << 20)
    x = torch.empty(1, device="cuda")     # never touched: rejected before any launch
    lib = wkv7.load_library()
    p = [None] * 16
    for i in (0, 1, 2, 3, 4, 5, 7, 9, 10, 11, 12, 13, 14, 15):
        p[i] = x.data_ptr()
    st = lib.wkv7_backward_noalloc(B, T, H, N, wkv7.BF16, wkv7.F32, *p, None)
    assert st == wkv7.ERR_TOO_LARGE
    assert "fixed scratch" in wkv7.status_string(st)

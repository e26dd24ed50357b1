"""The C-ABI library: it builds, loads without a GPU, exports every symbol that
include/wkv7.h declares, and rejects invalid arguments on the host (these
calls return before any CUDA call, so they run on a CPU-only machine)."""
import ctypes
import os
import re

import pytest

from linear_rnn_sequence_wkv7_b200 import build as libbuild
from linear_rnn_sequence_wkv7_b200 import wkv7

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    libbuild.build()
    return wkv7.load_library()


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"WKV7_API[^;(]*?\b(wkv7_\w+)\s*\(", src))
    return names


def test_header_declares_the_api():
    assert set(wkv7.EXPORTED_SYMBOLS) <= declared_symbols()


def test_every_declared_symbol_is_exported(lib):
    for name in sorted(declared_symbols()):
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_version_and_status_strings(lib):
    assert lib.wkv7_abi_version() == 1
    for code in range(6):
        assert wkv7.status_string(code)
    assert wkv7.status_string(99) == "unknown status"


def test_workspace_sizes(lib):
    assert lib.wkv7_forward_workspace_size(1, 64, 2, 64, wkv7.F32, wkv7.ALGO_SEQ, 0) == 0
    ws = lib.wkv7_backward_workspace_size(8, 4096, 32, 64)
    # per head: the state before every 32-token chunk, dL/dS at every chunk end, the final state,
    # and every chunk's transition image ([M^T; Q], bf16 hi and lo: 24 KiB)
    assert ws >= 8 * 32 * ((2 * (4096 // 32) + 1) * 64 * 64 * 4 + (4096 // 32) * 24576)
    assert lib.wkv7_backward_workspace_size(0, 10, 1, 64) == 0


P = ctypes.c_void_p(16)   # aligned, never dereferenced: validation fails first


def _fwd(lib, B=1, T=4, H=1, N=64, in_dt=0, y_dt=0, ptrs=None, algo=1, chunk=0):
    ptrs = ptrs or [P] * 9
    return lib.wkv7_forward(B, T, H, N, in_dt, y_dt, *ptrs, algo, chunk, None, 0, None)


def test_forward_rejects_invalid_arguments(lib):
    assert _fwd(lib, N=32) == wkv7.ERR_UNSUPPORTED
    assert _fwd(lib, B=-1) == wkv7.ERR_INVALID_ARG
    assert _fwd(lib, T=-3) == wkv7.ERR_INVALID_ARG
    assert _fwd(lib, in_dt=7) == wkv7.ERR_INVALID_ARG
    assert _fwd(lib, algo=9) == wkv7.ERR_INVALID_ARG
    assert _fwd(lib, chunk=64) == wkv7.ERR_UNSUPPORTED     # the chunked form's chunk is 32
    bad = [P] * 9
    bad[0] = None                                    # r missing
    assert _fwd(lib, ptrs=bad) == wkv7.ERR_INVALID_ARG
    bad = [P] * 9
    bad[2] = ctypes.c_void_p(18)                     # k misaligned
    assert _fwd(lib, ptrs=bad) == wkv7.ERR_INVALID_ARG
    assert _fwd(lib, B=0) == wkv7.OK                 # empty batch: nothing to do
    assert _fwd(lib, H=0) == wkv7.OK


def test_step_and_backward_reject_invalid_arguments(lib):
    assert lib.wkv7_step(1, 1, 16, 0, 0, *([P] * 8), None) == wkv7.ERR_UNSUPPORTED
    bad = [P] * 8
    bad[6] = None                                    # state missing
    assert lib.wkv7_step(1, 1, 64, 0, 0, *bad, None) == wkv7.ERR_INVALID_ARG
    assert lib.wkv7_step(0, 4, 64, 0, 0, *([P] * 8), None) == wkv7.OK
    ptrs = [P] * 16
    # workspace too small
    assert lib.wkv7_backward(1, 32, 1, 64, 0, 0, *ptrs, P, 16, None) == wkv7.ERR_INVALID_ARG
    ptrs[15] = None                                  # ds0 is required
    assert lib.wkv7_backward(1, 32, 1, 64, 0, 0, *ptrs, P, 1 << 40, None) == wkv7.ERR_INVALID_ARG


def test_summary_and_compose_reject_invalid_arguments(lib):
    summ = lambda B=1, T=64, H=1, N=64, dt=wkv7.BF16, ptrs=None, ws=None: lib.wkv7_forward_summary(
        B, T, H, N, dt, *(ptrs or [P] * 7), ws, 0, None)
    assert summ(N=32) == wkv7.ERR_UNSUPPORTED
    assert summ(dt=wkv7.F32) == wkv7.ERR_UNSUPPORTED     # computed by the chunked form
    assert summ(dt=5) == wkv7.ERR_INVALID_ARG
    assert summ(T=-1) == wkv7.ERR_INVALID_ARG
    bad = [P] * 7
    bad[6] = None                                        # summary output missing
    assert summ(ptrs=bad) == wkv7.ERR_INVALID_ARG
    bad = [P] * 7
    bad[3] = ctypes.c_void_p(24)                         # v misaligned
    assert summ(ptrs=bad) == wkv7.ERR_INVALID_ARG
    assert summ(ws=ctypes.c_void_p(40)) == wkv7.ERR_INVALID_ARG  # workspace misaligned
    assert summ(B=0) == wkv7.OK
    cont = lambda B=1, T=64, H=1, N=64, dt=wkv7.BF16, ydt=wkv7.BF16, ptrs=None: lib.wkv7_forward_continue(
        B, T, H, N, dt, ydt, *(ptrs or [P] * 9), None, 0, None)
    assert cont(N=128) == wkv7.ERR_UNSUPPORTED
    assert cont(dt=wkv7.F32) == wkv7.ERR_UNSUPPORTED
    assert cont(ydt=3) == wkv7.ERR_INVALID_ARG
    bad = [P] * 9
    bad[7] = None                                        # y missing
    assert cont(ptrs=bad) == wkv7.ERR_INVALID_ARG
    bad = [P] * 9
    bad[6] = ctypes.c_void_p(36)                         # s_in misaligned
    assert cont(ptrs=bad) == wkv7.ERR_INVALID_ARG
    assert cont(H=0) == wkv7.OK
    assert lib.wkv7_forward_summary_workspace_size(1, 64, 1, 32) == 0
    comp = lambda nseg=2, B=1, H=1, N=64, s0=None, sums=P, out=P: lib.wkv7_compose_states(
        nseg, B, H, N, s0, sums, out, None)
    assert comp(N=16) == wkv7.ERR_UNSUPPORTED
    assert comp(nseg=-1) == wkv7.ERR_INVALID_ARG
    assert comp(sums=None) == wkv7.ERR_INVALID_ARG       # nseg > 0 needs summaries
    assert comp(out=None) == wkv7.ERR_INVALID_ARG
    assert comp(s0=ctypes.c_void_p(20)) == wkv7.ERR_INVALID_ARG
    assert comp(H=0) == wkv7.OK


def test_forward_host_rejects_invalid_arguments(lib):
    fh = lambda B=1, T=64, H=1, N=64, dt=wkv7.BF16, ydt=wkv7.BF16, ptrs=None, algo=0, chunk=0, ws=P, nb=1 << 40: (
        lib.wkv7_forward_host(B, T, H, N, dt, ydt, *(ptrs or [P] * 9), algo, chunk, ws, nb, None))
    assert fh(N=32) == wkv7.ERR_UNSUPPORTED
    assert fh(dt=4) == wkv7.ERR_INVALID_ARG
    assert fh(algo=5) == wkv7.ERR_INVALID_ARG
    assert fh(chunk=16) == wkv7.ERR_UNSUPPORTED
    assert fh(dt=wkv7.F32, algo=wkv7.ALGO_CHUNK) == wkv7.ERR_UNSUPPORTED
    assert fh(ws=None) == wkv7.ERR_INVALID_ARG                     # device workspace is required
    assert fh(nb=16) == wkv7.ERR_INVALID_ARG                       # ... and must be large enough
    bad = [P] * 9
    bad[7] = None                                                  # y missing
    assert fh(ptrs=bad) == wkv7.ERR_INVALID_ARG
    assert fh(B=0) == wkv7.OK
    # two slots of 8 slices' inputs and y, the state, no forward scratch for 256 heads
    B, T, H = 8, 4096, 32
    need = lib.wkv7_forward_host_workspace_size(B, T, H, 64, wkv7.BF16, wkv7.BF16, wkv7.ALGO_CHUNK, 0)
    assert need >= 2 * 7 * B * (T // 8) * H * 64 * 2 + B * H * 64 * 64 * 4
    assert lib.wkv7_forward_host_workspace_size(B, T, H, 16, wkv7.BF16, wkv7.BF16, 0, 0) == 0


def test_training_pair_rejects_invalid_arguments(lib):
    ft = lambda B=1, T=64, H=1, N=64, ptrs=None: lib.wkv7_forward_train(
        B, T, H, N, wkv7.BF16, wkv7.BF16, *(ptrs or [P] * 10), 0, 0, None, 0, None)
    assert ft(N=32) == wkv7.ERR_UNSUPPORTED
    bad = [P] * 10
    bad[8] = None                                        # sT is required
    assert ft(ptrs=bad) == wkv7.ERR_INVALID_ARG
    bad = [P] * 10
    bad[9] = None                                        # states are required
    assert ft(ptrs=bad) == wkv7.ERR_INVALID_ARG
    assert ft(B=0) == wkv7.OK
    bs = lambda T=64, ptrs=None, nb=1 << 40: lib.wkv7_backward_from_states(
        1, T, 1, 64, wkv7.BF16, wkv7.F32, *(ptrs or [P] * 17), P, nb, None)
    assert bs(nb=16) == wkv7.ERR_INVALID_ARG             # workspace too small
    bad = [P] * 17
    bad[6] = None                                        # states missing
    assert bs(ptrs=bad) == wkv7.ERR_INVALID_ARG
    bad = [P] * 17
    bad[16] = None                                       # ds0 is required
    assert bs(ptrs=bad) == wkv7.ERR_INVALID_ARG
    # the state before every chunk, then every chunk's transition image (24 KiB)
    assert lib.wkv7_saved_states_size(2, 100, 3, 64) == 2 * 3 * 4 * 64 * 64 * 4 + 2 * 3 * 4 * 24576
    assert lib.wkv7_backward_from_states_workspace_size(2, 100, 3, 64) >= 2 * 3 * 4 * 64 * 64 * 4


def test_state_gradient_and_adjoints_reject_invalid_arguments(lib):
    sg = lambda B=1, T=64, H=1, N=64, dt=wkv7.BF16, ptrs=None, ws=None: lib.wkv7_state_gradient(
        B, T, H, N, dt, *(ptrs or [P] * 7), ws, 0, None)
    assert sg(N=32) == wkv7.ERR_UNSUPPORTED
    assert sg(dt=7) == wkv7.ERR_INVALID_ARG
    assert sg(T=-2) == wkv7.ERR_INVALID_ARG
    bad = [P] * 7
    bad[6] = None                                        # ds0 is required
    assert sg(ptrs=bad) == wkv7.ERR_INVALID_ARG
    bad = [P] * 7
    bad[4] = None                                        # dy missing
    assert sg(ptrs=bad) == wkv7.ERR_INVALID_ARG
    bad = [P] * 7
    bad[5] = ctypes.c_void_p(12)                         # dsT misaligned
    assert sg(ptrs=bad) == wkv7.ERR_INVALID_ARG
    assert sg(ws=ctypes.c_void_p(40)) == wkv7.ERR_INVALID_ARG     # workspace misaligned
    assert sg(H=0) == wkv7.OK
    # the segmented sweep's scratch: 3 states per segment, none for many heads
    assert lib.wkv7_state_gradient_workspace_size(1, 65536, 32, 64) % (3 * 32 * 64 * 64 * 4) == 0
    assert lib.wkv7_state_gradient_workspace_size(1, 65536, 32, 64) > 0
    assert lib.wkv7_state_gradient_workspace_size(16, 4096, 32, 64) == 0
    assert lib.wkv7_state_gradient_workspace_size(1, 64, 1, 16) == 0
    ca = lambda nseg=2, B=1, H=1, N=64, dsT=None, sums=P, F=P, adj=P: lib.wkv7_compose_adjoints(
        nseg, B, H, N, dsT, sums, F, adj, None)
    assert ca(N=128) == wkv7.ERR_UNSUPPORTED
    assert ca(nseg=-1) == wkv7.ERR_INVALID_ARG
    assert ca(sums=None) == wkv7.ERR_INVALID_ARG         # nseg > 0 needs summaries ...
    assert ca(F=None) == wkv7.ERR_INVALID_ARG            # ... and the stretches' F
    assert ca(adj=None) == wkv7.ERR_INVALID_ARG
    assert ca(dsT=ctypes.c_void_p(8)) == wkv7.ERR_INVALID_ARG
    assert ca(B=0) == wkv7.OK


def test_last_status_without_a_device(lib):
    """wkv7_get_last_status (and its earlier name wkv7_get_device_status)
    synchronize the stream first; without a usable device that fails and the
    call says so instead of reporting a status word it could not read."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present (the GPU tests read the status word)")
    lib.wkv7_get_last_status.argtypes = [ctypes.c_void_p]
    lib.wkv7_get_device_status.argtypes = [ctypes.c_void_p]
    assert lib.wkv7_get_last_status(None) == wkv7.ERR_CUDA
    assert lib.wkv7_get_device_status(None) == wkv7.ERR_CUDA


def test_timemix_rejects_invalid_arguments(lib):
    """wkv7_forward_timemix validates on the host before any CUDA call."""
    lib.wkv7_forward_timemix.argtypes = ([ctypes.c_int] * 6 + [ctypes.c_void_p] * 11 + [ctypes.c_float] +
                                         [ctypes.c_void_p] * 2 + [ctypes.c_int] * 2 +
                                         [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p])

    def call(N=64, rho=P, eps=1e-5, algo=2, ws=None, wsb=0, g=None, T=64):
        return lib.wkv7_forward_timemix(1, T, 1, N, wkv7.BF16, wkv7.BF16, P, P, P, P, P, P, None, rho, None, None,
                                        g, eps, P, None, algo, 0, ws, wsb, None)

    assert call(rho=None) == wkv7.ERR_INVALID_ARG                  # rho is required
    assert call(eps=-1.0) == wkv7.ERR_INVALID_ARG
    assert call(eps=float("nan")) == wkv7.ERR_INVALID_ARG
    assert call(N=32) == wkv7.ERR_UNSUPPORTED
    assert call(g=ctypes.c_void_p(18)) == wkv7.ERR_INVALID_ARG      # misaligned gate
    assert call(algo=1) == wkv7.ERR_INVALID_ARG                    # the scan path needs its fp32 y workspace
    assert call(algo=7) == wkv7.ERR_INVALID_ARG
    assert lib.wkv7_forward_timemix_workspace_size(2, 100, 3, 64, wkv7.BF16, wkv7.ALGO_SEQ, 0) == 2 * 100 * 3 * 64 * 4

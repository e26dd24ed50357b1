"""Python binding of libwkv7.so (ctypes): argument marshalling only.

Each function takes torch CUDA tensors, checks dtype / shape / contiguity,
and passes raw device pointers and the current CUDA stream to the C ABI
declared in include/wkv7.h.  Every step of the computation runs in the
library's kernels; there is no fallback of any kind.  If the shared library
is missing or fails to load, the first call raises.
"""
from __future__ import annotations

import contextlib
import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libwkv7.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_RANGE, ERR_TOO_LARGE = range(7)
F32, BF16 = 0, 1
ALGO_AUTO, ALGO_SEQ, ALGO_CHUNK = 0, 1, 2
ALGOS = {"auto": ALGO_AUTO, "seq": ALGO_SEQ, "chunk": ALGO_CHUNK}

EXPORTED_SYMBOLS = (
    "wkv7_abi_version", "wkv7_status_string", "wkv7_forward_workspace_size", "wkv7_forward",
    "wkv7_step", "wkv7_backward_workspace_size", "wkv7_backward", "wkv7_get_device_status",
    "wkv7_forward_resolve_algo", "wkv7_backward_noalloc", "wkv7_set_wait_limit",
    "wkv7_forward_summary", "wkv7_compose_states", "wkv7_forward_summary_workspace_size",
    "wkv7_forward_continue", "wkv7_forward_host_workspace_size", "wkv7_forward_host",
    "wkv7_saved_states_size", "wkv7_forward_train", "wkv7_backward_from_states_workspace_size",
    "wkv7_backward_from_states", "wkv7_state_gradient", "wkv7_state_gradient_workspace_size",
    "wkv7_compose_adjoints", "wkv7_get_last_status", "wkv7_forward_timemix",
    "wkv7_forward_timemix_workspace_size",
)

_lib = None


class WKV7Error(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {status_string(status)} ({status})")


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libwkv7.so and declare the C signatures (raises if absent)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libwkv7.so not built at {path}; run linear_rnn_sequence_wkv7_b200/build.py")
    lib = ctypes.CDLL(path)
    i, z, vp = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
    lib.wkv7_abi_version.restype = i
    lib.wkv7_status_string.argtypes = [i]
    lib.wkv7_status_string.restype = ctypes.c_char_p
    lib.wkv7_forward_workspace_size.argtypes = [i, i, i, i, i, i, i]
    lib.wkv7_forward_workspace_size.restype = z
    lib.wkv7_forward.argtypes = [i, i, i, i, i, i] + [vp] * 9 + [i, i, vp, z, vp]
    lib.wkv7_forward.restype = i
    lib.wkv7_step.argtypes = [i, i, i, i, i] + [vp] * 8 + [vp]
    lib.wkv7_step.restype = i
    lib.wkv7_backward_workspace_size.argtypes = [i, i, i, i]
    lib.wkv7_backward_workspace_size.restype = z
    lib.wkv7_backward.argtypes = [i, i, i, i, i, i] + [vp] * 16 + [vp, z, vp]
    lib.wkv7_backward.restype = i
    lib.wkv7_backward_noalloc.argtypes = [i, i, i, i, i, i] + [vp] * 16 + [vp]
    lib.wkv7_backward_noalloc.restype = i
    lib.wkv7_forward_summary_workspace_size.argtypes = [i, i, i, i]
    lib.wkv7_forward_summary_workspace_size.restype = z
    lib.wkv7_forward_summary.argtypes = [i, i, i, i, i] + [vp] * 8 + [z, vp]
    lib.wkv7_forward_summary.restype = i
    lib.wkv7_forward_continue.argtypes = [i, i, i, i, i, i] + [vp] * 10 + [z, vp]
    lib.wkv7_forward_continue.restype = i
    lib.wkv7_compose_states.argtypes = [i, i, i, i, vp, vp, vp, vp]
    lib.wkv7_compose_states.restype = i
    lib.wkv7_forward_host_workspace_size.argtypes = [i, i, i, i, i, i, i, i]
    lib.wkv7_forward_host_workspace_size.restype = z
    lib.wkv7_forward_host.argtypes = [i, i, i, i, i, i] + [vp] * 9 + [i, i, vp, z, vp]
    lib.wkv7_forward_host.restype = i
    lib.wkv7_saved_states_size.argtypes = [i, i, i, i]
    lib.wkv7_saved_states_size.restype = z
    lib.wkv7_forward_train.argtypes = [i, i, i, i, i, i] + [vp] * 10 + [i, i, vp, z, vp]
    lib.wkv7_forward_train.restype = i
    lib.wkv7_backward_from_states_workspace_size.argtypes = [i, i, i, i]
    lib.wkv7_backward_from_states_workspace_size.restype = z
    lib.wkv7_backward_from_states.argtypes = [i, i, i, i, i, i] + [vp] * 17 + [vp, z, vp]
    lib.wkv7_backward_from_states.restype = i
    lib.wkv7_state_gradient.argtypes = [i, i, i, i, i] + [vp] * 8 + [z, vp]
    lib.wkv7_state_gradient_workspace_size.argtypes = [i, i, i, i]
    lib.wkv7_state_gradient_workspace_size.restype = z
    lib.wkv7_state_gradient.restype = i
    lib.wkv7_compose_adjoints.argtypes = [i, i, i, i, vp, vp, vp, vp, vp]
    lib.wkv7_compose_adjoints.restype = i
    lib.wkv7_forward_resolve_algo.argtypes = [i, i, i]
    lib.wkv7_forward_resolve_algo.restype = i
    lib.wkv7_set_wait_limit.argtypes = [ctypes.c_longlong]
    lib.wkv7_set_wait_limit.restype = None
    lib.wkv7_get_device_status.argtypes = [vp]
    lib.wkv7_get_device_status.restype = i
    lib.wkv7_get_last_status.argtypes = [vp]
    lib.wkv7_get_last_status.restype = i
    lib.wkv7_forward_timemix_workspace_size.argtypes = [i, i, i, i, i, i, i]
    lib.wkv7_forward_timemix_workspace_size.restype = z
    lib.wkv7_forward_timemix.argtypes = ([i, i, i, i, i, i] + [vp] * 11 + [ctypes.c_float] + [vp, vp] +
                                         [i, i, vp, z, vp])
    lib.wkv7_forward_timemix.restype = i
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().wkv7_status_string(int(status)).decode()


# Status checks after every call: off by default (a check synchronizes the
# stream).  WKV7_CHECK_STATUS=1 in the environment, set_status_checks(True) or
# the status_checks() context turn them on; then each call also reads the
# device status word (wkv7_get_last_status) and raises on a device-side
# condition such as a chunk outside the chunked form's range.
_status_checks = os.environ.get("WKV7_CHECK_STATUS", "") not in ("", "0")


def set_status_checks(on: bool) -> bool:
    """Turn the per-call device status check on or off; returns the old setting."""
    global _status_checks
    old, _status_checks = _status_checks, bool(on)
    return old


@contextlib.contextmanager
def status_checks(on: bool):
    old = set_status_checks(on)
    try:
        yield
    finally:
        set_status_checks(old)


def _check(fn, status, stream=None):
    if status != OK:
        raise WKV7Error(fn, status)
    if _status_checks:
        dev = load_library().wkv7_get_last_status(_stream(stream))
        if dev != OK:
            raise WKV7Error(fn, dev)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _tdt(code: int) -> torch.dtype:
    return torch.float32 if code == F32 else torch.bfloat16


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("tensors must be contiguous CUDA tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _same(ts, shape, dtype):
    for t in ts:
        if tuple(t.shape) != tuple(shape) or t.dtype != dtype:
            raise ValueError(f"expected {tuple(shape)} {dtype}, got {tuple(t.shape)} {t.dtype}")


def forward_workspace_size(B, T, H, N, in_dtype=torch.bfloat16, algo="auto", chunk_len=0) -> int:
    code = F32 if in_dtype == torch.float32 else BF16
    return load_library().wkv7_forward_workspace_size(B, T, H, N, code, ALGOS[algo], chunk_len)


def forward(r, w, k, v, a, b, s0=None, *, y=None, sT=None, y_dtype=None, algo="auto",
            chunk_len=0, workspace=None, return_state=True, stream=None):
    """y [B,T,H,N] (and sT [B,H,N,N] fp32) for inputs [B,T,H,N] (fp32 or bf16)."""
    lib = load_library()
    B, T, H, N = r.shape
    _same((w, k, v, a, b), r.shape, r.dtype)
    ycode = _dt(r) if y_dtype is None else (F32 if y_dtype == torch.float32 else BF16)
    if y is None:
        y = torch.empty((B, T, H, N), dtype=_tdt(ycode), device=r.device)
    if return_state and sT is None:
        sT = torch.empty((B, H, N, N), dtype=torch.float32, device=r.device)
    if s0 is not None:
        _same((s0,), (B, H, N, N), torch.float32)
    ws_bytes = lib.wkv7_forward_workspace_size(B, T, H, N, _dt(r), ALGOS[algo], chunk_len)
    if ws_bytes and workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=r.device)
    st = lib.wkv7_forward(B, T, H, N, _dt(r), ycode, *map(_ptr, (r, w, k, v, a, b, s0, y, sT)),
                          ALGOS[algo], chunk_len, _ptr(workspace),
                          0 if workspace is None else workspace.numel(), _stream(stream))
    _check("wkv7_forward", st, stream)
    return (y, sT) if return_state else y


def forward_timemix_workspace_size(B, T, H, N, in_dtype=torch.bfloat16, algo="auto", chunk_len=0) -> int:
    code = F32 if in_dtype == torch.float32 else BF16
    return load_library().wkv7_forward_timemix_workspace_size(B, T, H, N, code, ALGOS[algo], chunk_len)


def forward_timemix(r, w, k, v, a, b, s0=None, *, rho, gamma=None, beta=None, g=None, eps=1e-5, z=None, sT=None,
                    out_dtype=None, algo="auto", chunk_len=0, workspace=None, return_state=True, stream=None):
    """wkv7_forward_timemix: z [B,T,H,N] (and sT) of the forward followed by the
    time-mix output epilogue (current-token term with weight ``rho`` [H,N],
    per-head normalisation with ``gamma``/``beta`` [H,N], gate ``g`` [B,T,H,N])."""
    lib = load_library()
    B, T, H, N = r.shape
    _same((w, k, v, a, b), r.shape, r.dtype)
    _same((rho,), (H, N), torch.float32)
    for p in (gamma, beta):
        if p is not None:
            _same((p,), (H, N), torch.float32)
    if g is not None:
        _same((g,), r.shape, r.dtype)
    ocode = _dt(r) if out_dtype is None else (F32 if out_dtype == torch.float32 else BF16)
    if z is None:
        z = torch.empty((B, T, H, N), dtype=_tdt(ocode), device=r.device)
    if return_state and sT is None:
        sT = torch.empty((B, H, N, N), dtype=torch.float32, device=r.device)
    if s0 is not None:
        _same((s0,), (B, H, N, N), torch.float32)
    ws_bytes = lib.wkv7_forward_timemix_workspace_size(B, T, H, N, _dt(r), ALGOS[algo], chunk_len)
    if ws_bytes and workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=r.device)
    st = lib.wkv7_forward_timemix(B, T, H, N, _dt(r), ocode, *map(_ptr, (r, w, k, v, a, b, s0, rho, gamma, beta, g)),
                                  float(eps), _ptr(z), _ptr(sT), ALGOS[algo], chunk_len, _ptr(workspace),
                                  0 if workspace is None else workspace.numel(), _stream(stream))
    _check("wkv7_forward_timemix", st, stream)
    return (z, sT) if return_state else z


def forward_summary_workspace_size(B, T, H, N) -> int:
    return load_library().wkv7_forward_summary_workspace_size(B, T, H, N)


def forward_summary(r, w, k, v, a, b, *, out=None, workspace=None, stream=None):
    """[2,B,H,N,N] fp32 summary [E; M] of a bf16 stretch [B,T,H,N]: its final
    state is S_in @ M + E for entry state S_in.  Pass the same ``workspace``
    (or None) to the ``forward_continue`` of this stretch."""
    lib = load_library()
    B, T, H, N = r.shape
    _same((w, k, v, a, b), r.shape, r.dtype)
    if out is None:
        out = torch.empty((2, B, H, N, N), dtype=torch.float32, device=r.device)
    _same((out,), (2, B, H, N, N), torch.float32)
    st = lib.wkv7_forward_summary(B, T, H, N, _dt(r), *map(_ptr, (r, w, k, v, a, b, out)), _ptr(workspace),
                                  0 if workspace is None else workspace.numel(), _stream(stream))
    _check("wkv7_forward_summary", st, stream)
    return out


def forward_continue(r, w, k, v, a, b, s_in=None, *, workspace=None, y=None, sT=None, y_dtype=None,
                     return_state=False, stream=None):
    """y [B,T,H,N] of a bf16 stretch from entry state ``s_in``, reusing what
    ``forward_summary`` left in ``workspace`` (same inputs, same workspace)."""
    lib = load_library()
    B, T, H, N = r.shape
    _same((w, k, v, a, b), r.shape, r.dtype)
    ycode = _dt(r) if y_dtype is None else (F32 if y_dtype == torch.float32 else BF16)
    if y is None:
        y = torch.empty((B, T, H, N), dtype=_tdt(ycode), device=r.device)
    if return_state and sT is None:
        sT = torch.empty((B, H, N, N), dtype=torch.float32, device=r.device)
    if s_in is not None:
        _same((s_in,), (B, H, N, N), torch.float32)
    st = lib.wkv7_forward_continue(B, T, H, N, _dt(r), ycode, *map(_ptr, (r, w, k, v, a, b, s_in, y, sT)),
                                   _ptr(workspace), 0 if workspace is None else workspace.numel(),
                                   _stream(stream))
    _check("wkv7_forward_continue", st, stream)
    return (y, sT) if return_state else y


def compose_states(summaries, s0=None, *, out=None, stream=None):
    """states [nseg+1,B,H,N,N]: states[0] = s0 (or 0), states[k+1] = states[k] @ M_k + E_k
    for summaries [nseg,2,B,H,N,N]."""
    lib = load_library()
    nseg, two, B, H, N, _ = summaries.shape
    if two != 2:
        raise ValueError("summaries must be [nseg, 2, B, H, N, N]")
    _same((summaries,), summaries.shape, torch.float32)
    if s0 is not None:
        _same((s0,), (B, H, N, N), torch.float32)
    if out is None:
        out = torch.empty((nseg + 1, B, H, N, N), dtype=torch.float32, device=summaries.device)
    _same((out,), (nseg + 1, B, H, N, N), torch.float32)
    st = lib.wkv7_compose_states(nseg, B, H, N, _ptr(s0), _ptr(summaries), _ptr(out), _stream(stream))
    _check("wkv7_compose_states", st, stream)
    return out


def _host_ptr(t):
    if t is None:
        return None
    if t.is_cuda or not t.is_contiguous():
        raise ValueError("host tensors must be contiguous CPU tensors")
    return ctypes.c_void_p(t.data_ptr())


def forward_host_workspace_size(B, T, H, N, in_dtype=torch.bfloat16, y_dtype=None, algo="auto", chunk_len=0) -> int:
    ic = F32 if in_dtype == torch.float32 else BF16
    yc = ic if y_dtype is None else (F32 if y_dtype == torch.float32 else BF16)
    return load_library().wkv7_forward_host_workspace_size(B, T, H, N, ic, yc, ALGOS[algo], chunk_len)


def forward_host(r, w, k, v, a, b, s0=None, *, y, sT=None, algo="auto", chunk_len=0, workspace=None,
                 device=None, stream=None):
    """wkv7_forward_host: inputs and outputs are CPU tensors (pinned for
    overlap), ``y`` [B,T,H,N] and optional ``sT`` written in place once the
    stream reaches the call; ``workspace`` is a CUDA uint8 tensor (allocated
    on ``device`` when None)."""
    lib = load_library()
    B, T, H, N = r.shape
    _same((w, k, v, a, b), r.shape, r.dtype)
    ycode = _dt(y)
    if tuple(y.shape) != (B, T, H, N):
        raise ValueError("y must be [B, T, H, N]")
    if s0 is not None:
        _same((s0,), (B, H, N, N), torch.float32)
    if sT is not None:
        _same((sT,), (B, H, N, N), torch.float32)
    ws_bytes = lib.wkv7_forward_host_workspace_size(B, T, H, N, _dt(r), ycode, ALGOS[algo], chunk_len)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8,
                                device=device if device is not None else torch.cuda.current_device())
    st = lib.wkv7_forward_host(B, T, H, N, _dt(r), ycode, *map(_host_ptr, (r, w, k, v, a, b, s0, y, sT)),
                               ALGOS[algo], chunk_len, _ptr(workspace), workspace.numel(), _stream(stream))
    _check("wkv7_forward_host", st, stream)
    return y, sT


def state_gradient_workspace_size(B, T, H, N) -> int:
    return load_library().wkv7_state_gradient_workspace_size(B, T, H, N)


def state_gradient(r, w, a, b, dy, dsT=None, *, out=None, workspace=None, stream=None):
    """dL/dS_0 [B,H,N,N] fp32 of a stretch [B,T,H,N] given dL/dS_T (dsT, None = 0).
    ``workspace=False`` runs the sweep unsegmented."""
    lib = load_library()
    B, T, H, N = r.shape
    _same((w, a, b, dy), r.shape, r.dtype)
    if dsT is not None:
        _same((dsT,), (B, H, N, N), torch.float32)
    if out is None:
        out = torch.empty((B, H, N, N), dtype=torch.float32, device=r.device)
    if workspace is None:
        nbytes = lib.wkv7_state_gradient_workspace_size(B, T, H, N)
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=r.device) if nbytes else None
    elif workspace is False:
        workspace = None
    st = lib.wkv7_state_gradient(B, T, H, N, _dt(r), *map(_ptr, (r, w, a, b, dy, dsT, out, workspace)),
                                 0 if workspace is None else workspace.numel(), _stream(stream))
    _check("wkv7_state_gradient", st, stream)
    return out


def compose_adjoints(summaries, F, dsT=None, *, out=None, stream=None):
    """adj [nseg+1,B,H,N,N]: adj[nseg] = dsT (or 0), adj[k] = adj[k+1] @ M_k^T + F_k."""
    lib = load_library()
    nseg, two, B, H, N, _ = summaries.shape
    if two != 2:
        raise ValueError("summaries must be [nseg, 2, B, H, N, N]")
    _same((F,), (nseg, B, H, N, N), torch.float32)
    if dsT is not None:
        _same((dsT,), (B, H, N, N), torch.float32)
    if out is None:
        out = torch.empty((nseg + 1, B, H, N, N), dtype=torch.float32, device=summaries.device)
    st = lib.wkv7_compose_adjoints(nseg, B, H, N, _ptr(dsT), _ptr(summaries), _ptr(F), _ptr(out), _stream(stream))
    _check("wkv7_compose_adjoints", st, stream)
    return out


def resolve_algo(T, in_dtype=torch.bfloat16, algo="auto") -> str:
    """Which forward algorithm ("seq" or "chunk") the library runs for these arguments."""
    code = load_library().wkv7_forward_resolve_algo(T, F32 if in_dtype == torch.float32 else BF16, ALGOS[algo])
    if code < 0:
        raise ValueError("invalid dtype or algorithm")
    return {ALGO_SEQ: "seq", ALGO_CHUNK: "chunk"}[code]


def step(r, w, k, v, a, b, state, *, y=None, y_dtype=None, stream=None):
    """One decode token: inputs [B,H,N]; the fp32 state [B,H,N,N] is updated in place."""
    lib = load_library()
    B, H, N = r.shape
    _same((w, k, v, a, b), r.shape, r.dtype)
    _same((state,), (B, H, N, N), torch.float32)
    ycode = _dt(r) if y_dtype is None else (F32 if y_dtype == torch.float32 else BF16)
    if y is None:
        y = torch.empty((B, H, N), dtype=_tdt(ycode), device=r.device)
    st = lib.wkv7_step(B, H, N, _dt(r), ycode, *map(_ptr, (r, w, k, v, a, b, state, y)), _stream(stream))
    _check("wkv7_step", st, stream)
    return y


def backward_workspace_size(B, T, H, N) -> int:
    return load_library().wkv7_backward_workspace_size(B, T, H, N)


def backward(r, w, k, v, a, b, s0, dy, dsT=None, *, grad_dtype=torch.float32, workspace=None,
             out=None, stream=None):
    """(dr, dw, dk, dv, da, db, ds0) of L = sum(dy*y) + sum(dsT*sT)."""
    lib = load_library()
    B, T, H, N = r.shape
    _same((w, k, v, a, b, dy), r.shape, r.dtype)
    gcode = F32 if grad_dtype == torch.float32 else BF16
    if out is None:
        out = [torch.empty((B, T, H, N), dtype=grad_dtype, device=r.device) for _ in range(6)]
        out.append(torch.empty((B, H, N, N), dtype=torch.float32, device=r.device))
    ws_bytes = lib.wkv7_backward_workspace_size(B, T, H, N)
    if workspace is None and ws_bytes:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=r.device)
    st = lib.wkv7_backward(B, T, H, N, _dt(r), gcode,
                           *map(_ptr, (r, w, k, v, a, b, s0, dy, dsT, *out)),
                           _ptr(workspace), 0 if workspace is None else workspace.numel(), _stream(stream))
    _check("wkv7_backward", st, stream)
    return tuple(out)


def saved_states_size(B, T, H, N) -> int:
    return load_library().wkv7_saved_states_size(B, T, H, N)


def backward_from_states_workspace_size(B, T, H, N) -> int:
    return load_library().wkv7_backward_from_states_workspace_size(B, T, H, N)


def _saved_states_capacity_ok(states, B, T, H, N):
    """The saved-states buffer holds wkv7_saved_states_size bytes from the
    tensor's first element on (the states, then the chunks' transitions)."""
    need = load_library().wkv7_saved_states_size(B, T, H, N)
    have = states.untyped_storage().nbytes() - states.storage_offset() * states.element_size()
    return states.is_contiguous() and have >= need


def forward_train(r, w, k, v, a, b, s0=None, *, y=None, sT=None, states=None, y_dtype=None, algo="auto",
                  chunk_len=0, workspace=None, stream=None):
    """(y, sT, states): the forward plus the state before every 32-token chunk,
    [B, H, ceil(T/32), N, N] fp32, for ``backward_from_states``.  ``states`` is
    a view of the first part of a buffer of ``saved_states_size`` bytes whose
    remainder holds every chunk's transition (bf16 inputs); pass it to
    ``backward_from_states`` as returned."""
    lib = load_library()
    B, T, H, N = r.shape
    _same((w, k, v, a, b), r.shape, r.dtype)
    ycode = _dt(r) if y_dtype is None else (F32 if y_dtype == torch.float32 else BF16)
    if y is None:
        y = torch.empty((B, T, H, N), dtype=_tdt(ycode), device=r.device)
    if sT is None:
        sT = torch.empty((B, H, N, N), dtype=torch.float32, device=r.device)
    if states is None:
        nck = (T + 31) // 32
        buf = torch.empty(max(lib.wkv7_saved_states_size(B, T, H, N), 4) // 4, dtype=torch.float32,
                          device=r.device)
        states = buf[: B * H * nck * N * N].view(B, H, nck, N, N)
    elif T > 0 and not _saved_states_capacity_ok(states, B, T, H, N):
        raise ValueError("states: needs saved_states_size(B, T, H, N) bytes of contiguous storage")
    if s0 is not None:
        _same((s0,), (B, H, N, N), torch.float32)
    ws_bytes = lib.wkv7_forward_workspace_size(B, T, H, N, _dt(r), ALGOS[algo], chunk_len)
    if ws_bytes and workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=r.device)
    st = lib.wkv7_forward_train(B, T, H, N, _dt(r), ycode, *map(_ptr, (r, w, k, v, a, b, s0, y, sT, states)),
                                ALGOS[algo], chunk_len, _ptr(workspace),
                                0 if workspace is None else workspace.numel(), _stream(stream))
    _check("wkv7_forward_train", st, stream)
    return y, sT, states


def backward_from_states(r, w, k, v, a, b, states, sT, dy, dsT=None, *, grad_dtype=torch.float32,
                         workspace=None, out=None, stream=None):
    """(dr, dw, dk, dv, da, db, ds0) from the states and sT of ``forward_train``."""
    lib = load_library()
    B, T, H, N = r.shape
    _same((w, k, v, a, b, dy), r.shape, r.dtype)
    if T > 0 and not _saved_states_capacity_ok(states, B, T, H, N):
        raise ValueError("states: pass the tensor forward_train returned (saved_states_size bytes)")
    gcode = F32 if grad_dtype == torch.float32 else BF16
    if out is None:
        out = [torch.empty((B, T, H, N), dtype=grad_dtype, device=r.device) for _ in range(6)]
        out.append(torch.empty((B, H, N, N), dtype=torch.float32, device=r.device))
    ws_bytes = lib.wkv7_backward_from_states_workspace_size(B, T, H, N)
    if workspace is None and ws_bytes:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=r.device)
    st = lib.wkv7_backward_from_states(B, T, H, N, _dt(r), gcode,
                                       *map(_ptr, (r, w, k, v, a, b, states, sT, dy, dsT, *out)),
                                       _ptr(workspace), 0 if workspace is None else workspace.numel(),
                                       _stream(stream))
    _check("wkv7_backward_from_states", st, stream)
    return tuple(out)


def backward_noalloc(r, w, k, v, a, b, s0, dy, dsT=None, *, grad_dtype=torch.float32, out=None, stream=None):
    """wkv7_backward_noalloc: the backward with the library's fixed 32 MiB device
    scratch instead of a workspace, for callers that cannot allocate device
    memory where they run it (see include/wkv7.h).  Output tensors are still the
    caller's; pass ``out`` to avoid any allocation here as well."""
    lib = load_library()
    B, T, H, N = r.shape
    _same((w, k, v, a, b, dy), r.shape, r.dtype)
    gcode = F32 if grad_dtype == torch.float32 else BF16
    if out is None:
        out = [torch.empty((B, T, H, N), dtype=grad_dtype, device=r.device) for _ in range(6)]
        out.append(torch.empty((B, H, N, N), dtype=torch.float32, device=r.device))
    st = lib.wkv7_backward_noalloc(B, T, H, N, _dt(r), gcode,
                                   *map(_ptr, (r, w, k, v, a, b, s0, dy, dsT, *out)), _stream(stream))
    _check("wkv7_backward_noalloc", st, stream)
    return tuple(out)


def set_wait_limit(cycles: int = 0) -> None:
    """Bound (SM cycles) on device-side waits of later launches; 0 = default (~1 s)."""
    load_library().wkv7_set_wait_limit(int(cycles))


def last_status(stream=None) -> int:
    """Synchronize and read/clear the library's sticky device status word."""
    return load_library().wkv7_get_last_status(_stream(stream))


device_status = last_status

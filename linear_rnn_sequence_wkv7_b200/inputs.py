"""Seeded synthetic inputs for the WKV7 recurrence.

This module draws the tensors r, w, k, v, a, b (and s0, dy) with the
distributions the workloads specify; it holds none of the recurrence's own
arithmetic, so both the fp64 oracle and the CUDA path can consume its output
without sharing any part of the method.

Distributions (per head-token, an N-vector per tensor):
  r, k, v ~ N(0, 1)
  w = exp(-0.6065 * sigmoid(x)),  x ~ N(x_mean, 1)   (x_mean = 0, or -2 for
      the long-context workload, which keeps w near 1)
  k_hat = z / ||z||_2 with a fresh z ~ N(0, 1)      (the removal key, drawn
      independently of k: the pages describe separate removal and write keys,
      RWKV-7 "Goose" paper review, section "Architecture")
  lr = sigmoid(N(0, 1)) per channel                 (in-context learning rate)
  a = -k_hat,  b = k_hat * lr
  s0 ~ N(0, 0.1) (standard deviation 0.1), dy ~ N(0, 1)

All draws and the recipe are evaluated in float32, then stored.
Random numbers come from numpy's Philox bit generator.  The flat stream of
N-vectors of each tensor is cut into fixed blocks of ``BLOCK_VECS`` vectors,
block ``c`` of stream ``s`` under seed ``seed`` is drawn from
``Philox(key=[seed * 65536 + s, c])``; so the values do not depend on the
thread count, and any block can be regenerated alone.

bf16 tensors are stored as uint16 bit patterns (round-to-nearest-even from
fp32); fp32 tensors as float32.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

BLOCK_VECS = 16384

STREAM_R, STREAM_W, STREAM_K, STREAM_V, STREAM_KHAT, STREAM_LR = 1, 2, 3, 4, 5, 6
STREAM_S0, STREAM_DY, STREAM_DST = 7, 8, 9
STREAM_GATE, STREAM_PARAMS = 10, 11

INPUT_NAMES = ("r", "w", "k", "v", "a", "b")


def _rng(seed: int, stream: int, block: int) -> np.random.Generator:
    key = np.array([seed * 65536 + stream, block], dtype=np.uint64)
    return np.random.Generator(np.random.Philox(key=key))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest-even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    return (np.asarray(u, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def to_f64(x: np.ndarray) -> np.ndarray:
    """Exact fp64 copy of a stored tensor (uint16 = bf16 bits, else float)."""
    if x.dtype == np.uint16:
        return bf16_bits_to_f32(x).astype(np.float64)
    return np.asarray(x, dtype=np.float64)


def _store(x: np.ndarray, dtype: str) -> np.ndarray:
    x32 = np.asarray(x, dtype=np.float32)
    if dtype == "bf16":
        return f32_to_bf16_bits(x32)
    if dtype == "f32":
        return x32
    raise ValueError(f"unknown dtype {dtype!r}")


def _empty(nvec: int, N: int, dtype: str) -> np.ndarray:
    return np.empty((nvec, N), dtype=np.uint16 if dtype == "bf16" else np.float32)


def _blocks(nvec: int):
    return [(c, c * BLOCK_VECS, min(nvec, (c + 1) * BLOCK_VECS))
            for c in range((nvec + BLOCK_VECS - 1) // BLOCK_VECS)]


def _run(fn, blocks, threads):
    if threads is None:
        threads = min(32, os.cpu_count() or 1)
    if threads <= 1 or len(blocks) == 1:
        for blk in blocks:
            fn(blk)
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(fn, blocks))


def gen_vectors(nvec: int, N: int, *, seed: int, dtype: str = "bf16",
                x_mean: float = 0.0, threads: int | None = None) -> dict:
    """Draw ``nvec`` head-token vectors of length N for r, w, k, v, a, b.

    Returns a dict of arrays shaped [nvec, N] (uint16 bf16 bits or float32).
    """
    return gen_vectors_range(0, nvec, N, seed=seed, dtype=dtype, x_mean=x_mean, threads=threads)


def gen_vectors_range(first: int, stop: int, N: int, *, seed: int, dtype: str = "bf16",
                      x_mean: float = 0.0, threads: int | None = None) -> dict:
    """Vectors ``first`` .. ``stop - 1`` of the flat stream that ``gen_vectors``
    draws (the same values, regenerating only the blocks that hold them)."""
    nvec = stop - first
    out = {name: _empty(nvec, N, dtype) for name in INPUT_NAMES}
    c0 = first // BLOCK_VECS
    c1 = (stop + BLOCK_VECS - 1) // BLOCK_VECS
    blocks = [(c, max(first, c * BLOCK_VECS), min(stop, (c + 1) * BLOCK_VECS)) for c in range(c0, c1)]

    def block(blk):
        c, lo_abs, hi_abs = blk
        off = lo_abs - c * BLOCK_VECS      # the block's leading vectors are drawn and dropped
        n = hi_abs - c * BLOCK_VECS        # draws up to the last vector needed
        lo, hi = lo_abs - first, hi_abs - first
        buf = np.empty((n, N), dtype=np.float32)
        for name, stream in (("r", STREAM_R), ("k", STREAM_K), ("v", STREAM_V)):
            _rng(seed, stream, c).standard_normal(out=buf, dtype=np.float32)
            out[name][lo:hi] = _store(buf[off:], dtype)
        _rng(seed, STREAM_W, c).standard_normal(out=buf, dtype=np.float32)
        buf += np.float32(x_mean)
        out["w"][lo:hi] = _store(np.exp(np.float32(-0.6065) / (np.float32(1.0) + np.exp(-buf[off:]))), dtype)
        _rng(seed, STREAM_KHAT, c).standard_normal(out=buf, dtype=np.float32)
        kb = buf[off:]
        khat = kb / np.sqrt(np.einsum("ij,ij->i", kb, kb))[:, None]
        lr = np.empty((n, N), dtype=np.float32)
        _rng(seed, STREAM_LR, c).standard_normal(out=lr, dtype=np.float32)
        lr = np.float32(1.0) / (np.float32(1.0) + np.exp(-lr[off:]))
        out["a"][lo:hi] = _store(-khat, dtype)
        out["b"][lo:hi] = _store(khat * lr, dtype)

    _run(block, blocks, threads)
    return out


def gen_normal(nvec: int, N: int, *, seed: int, stream: int, std: float = 1.0,
               dtype: str = "f32", threads: int | None = None) -> np.ndarray:
    """``nvec`` vectors of N(0, std^2) values, shaped [nvec, N]."""
    out = _empty(nvec, N, dtype)

    def block(blk):
        c, lo, hi = blk
        buf = np.empty((hi - lo, N), dtype=np.float32)
        _rng(seed, stream, c).standard_normal(out=buf, dtype=np.float32)
        out[lo:hi] = _store(buf * np.float32(std), dtype)

    _run(block, _blocks(nvec), threads)
    return out


def gen_sequence(B: int, T: int, H: int, N: int, *, seed: int, dtype: str = "bf16",
                 x_mean: float = 0.0, s0_std: float | None = None,
                 threads: int | None = None) -> dict:
    """Inputs of one forward call: r..b shaped [B, T, H, N]; s0 [B, H, N, N]
    float32 when ``s0_std`` is given (else None, meaning a zero state)."""
    vecs = gen_vectors(B * T * H, N, seed=seed, dtype=dtype, x_mean=x_mean, threads=threads)
    out = {name: arr.reshape(B, T, H, N) for name, arr in vecs.items()}
    out["s0"] = None
    if s0_std is not None:
        out["s0"] = gen_normal(B * H * N, N, seed=seed, stream=STREAM_S0, std=s0_std,
                               dtype="f32", threads=threads).reshape(B, H, N, N)
    return out


def gen_steps(steps: int, B: int, H: int, N: int, *, seed: int, dtype: str = "bf16",
              threads: int | None = None) -> dict:
    """Per-token inputs of ``steps`` consecutive decode steps, [steps, B, H, N]."""
    vecs = gen_vectors(steps * B * H, N, seed=seed, dtype=dtype, threads=threads)
    return {name: arr.reshape(steps, B, H, N) for name, arr in vecs.items()}


def gen_steps_range(first: int, stop: int, B: int, H: int, N: int, *, seed: int, dtype: str = "bf16",
                    threads: int | None = None) -> dict:
    """Steps ``first`` .. ``stop - 1`` of ``gen_steps`` (same values), [stop - first, B, H, N]."""
    vecs = gen_vectors_range(first * B * H, stop * B * H, N, seed=seed, dtype=dtype, threads=threads)
    return {name: arr.reshape(stop - first, B, H, N) for name, arr in vecs.items()}


def gen_dy(B: int, T: int, H: int, N: int, *, seed: int, dtype: str = "bf16",
           threads: int | None = None) -> np.ndarray:
    return gen_normal(B * T * H, N, seed=seed, stream=STREAM_DY, dtype=dtype,
                      threads=threads).reshape(B, T, H, N)


def gen_gate(B: int, T: int, H: int, N: int, *, seed: int, dtype: str = "bf16",
             threads: int | None = None) -> np.ndarray:
    """Gate values of the time-mix output, sigmoid(N(0, 1)) per channel, [B, T, H, N]."""
    x = gen_normal(B * T * H, N, seed=seed, stream=STREAM_GATE, dtype="f32", threads=threads)
    return _store(np.float32(1.0) / (np.float32(1.0) + np.exp(-x)), dtype).reshape(B, T, H, N)


def gen_timemix_params(H: int, N: int, *, seed: int):
    """Per-head parameters of the time-mix output, float32 [H, N] each: the
    current-token weight rho ~ U(-1, 1), the norm's gamma ~ U(0.5, 1.5) and
    beta ~ U(-0.5, 0.5)."""
    u = _rng(seed, STREAM_PARAMS, 0).random((3, H, N), dtype=np.float32)
    return (u[0] * np.float32(2.0) - np.float32(1.0), u[1] + np.float32(0.5), u[2] - np.float32(0.5))


# Named workloads: (kind, shape, recipe).  Sizes follow the workload list of
# the method's benchmark plan; the seed of workload c is c.
WORKLOADS = {
    "fwd_b1_t64_h2_f32": dict(kind="forward", B=1, T=64, H=2, N=64, dtype="f32",
                              x_mean=0.0, s0_std=None, seed=0),
    "prefill_b8_t4096_h32_bf16": dict(kind="forward", B=8, T=4096, H=32, N=64, dtype="bf16",
                                      x_mean=0.0, s0_std=0.1, seed=1),
    "decode_b256_h40_x1000": dict(kind="step", B=256, H=40, N=64, dtype="bf16",
                                  steps=1000, s0_std=0.1, seed=2),
    # served by the chunked form's 32-token chunks (the result does not depend
    # on the chunk length; a 64-token chunk is not implemented)
    "long_b1_t65536_h32_chunk32": dict(kind="forward", B=1, T=65536, H=32, N=64, dtype="bf16",
                                       x_mean=-2.0, s0_std=0.1, seed=3, chunk_len=32),
    "train_bwd_b8_t4096_h32": dict(kind="backward", B=8, T=4096, H=32, N=64, dtype="bf16",
                                   x_mean=0.0, s0_std=0.1, seed=4),
}

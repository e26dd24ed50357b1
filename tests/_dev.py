"""numpy <-> torch CUDA tensors for the GPU parity tests."""
import numpy as np
import torch

from linear_rnn_sequence_wkv7_b200 import inputs


def to_dev(x, device="cuda"):
    if x is None:
        return None
    if x.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)


def to_f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def oracle_args(d, names=inputs.INPUT_NAMES):
    return [inputs.to_f64(d[n]) for n in names]

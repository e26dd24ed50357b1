"""WKV7 (RWKV-7 time-mix recurrence) on B200: a C-ABI CUDA library (libwkv7.so,
sm_100a) with a thin Python binding.

    from linear_rnn_sequence_wkv7_b200 import forward, step, backward

``forward``/``step``/``backward`` live in ``wkv7.py`` and are imported lazily
so that ``inputs`` (the seeded workload generator) can be used without torch.
"""
_EXPORTS = ("forward", "step", "backward", "forward_workspace_size", "backward_workspace_size",
            "device_status", "load_library", "WKV7Error")


def __getattr__(name):
    if name in _EXPORTS:
        from . import wkv7
        return getattr(wkv7, name)
    raise AttributeError(name)

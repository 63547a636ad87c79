"""Single-GPU Megatron tensor-parallel block for B200 (sm_100a).

``tp`` is the ctypes binding of libtp.so (include/tp.h); ``block`` holds the
buffer management and call sequences of the MLP / attention / SP steps on top
of it. Build the library with ``python -m megatron_tensor_transformer_gemm_b200.build``.
The binding is imported on first use of one of its names, and that import
raises ImportError when libtp.so is missing.
"""
_EXPORTS = ("Plan", "TPError", "device_status", "launch_count")


def __getattr__(name):
    if name in _EXPORTS:
        from . import tp
        return getattr(tp, name)
    raise AttributeError(name)

"""int4 group-quantized (q4f16) dequantizing GEMV for NVIDIA B200 (sm_100a).

The compute entry points live in ``zt_q4`` (a ctypes binding of the in-tree
``libzt_q4.so``).  They are imported lazily so that ``synth`` and ``build``
work on a machine where the library has not been built yet; touching any
compute name without the library raises ImportError.
"""
_BINDING = ("gemv", "gate_up_silu", "lmhead_argmax", "lmhead_workspace_bytes",
            "pack_host", "unpack_host", "strerror", "version", "ZtError")


def __getattr__(name):
    if name in _BINDING:
        from . import zt_q4
        return getattr(zt_q4, name)
    raise AttributeError(name)

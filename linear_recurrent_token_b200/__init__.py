"""B200-native mLSTM / retention recurrence: chunkwise prefill and decode step.

``linear_recurrent_token_b200.mlstm``   binding of libmlstm.so (the C ABI in include/mlstm.h)
``linear_recurrent_token_b200.inputs``  seeded synthetic workloads
``linear_recurrent_token_b200.build``   nvcc build of libmlstm.so for sm_100a
"""
from . import inputs  # noqa: F401

__all__ = ["inputs", "mlstm", "build"]


def __getattr__(name):
    if name in ("mlstm", "build"):
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)

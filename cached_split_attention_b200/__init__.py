"""FlashBlock denoise-step attention on B200 (sm_100a).

The compute path is the C-ABI library ``libflashblock.so`` built from ``csrc/``;
``binding`` marshals arguments to it.  ``workloads`` draws seeded synthetic
inputs and is importable without the library.
"""
import importlib

__all__ = ["binding", "workloads"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)

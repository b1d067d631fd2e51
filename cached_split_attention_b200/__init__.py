"""FlashBlock denoise-step attention on B200 (sm_100a).

The compute path is the C-ABI library ``libflashblock.so`` built from ``csrc/``;
``binding`` marshals arguments to it.  ``workloads`` draws seeded synthetic
inputs and is importable without the library.
"""
__all__ = ["binding", "workloads"]


def __getattr__(name):
    if name == "binding":
        from . import binding
        return binding
    raise AttributeError(name)

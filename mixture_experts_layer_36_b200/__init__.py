"""libmoe: the forward pass of a sparse Mixture-of-Experts layer on one B200.

The C-ABI library (``libmoe.so``, declared in ``include/moe.h``) holds every
kernel; ``binding`` is its ctypes front end with the same function names
(``moe_route``, ``moe_permute``, ``moe_expert_gate_up``, ``moe_expert_down``,
``moe_expert_mlp``, ``moe_combine``, ``moe_layer_forward`` and the size
queries).  Those names are re-exported here on first access, which loads the
library and raises ImportError if it has not been built.  ``configs`` and
``synth`` (workload shapes and seeded inputs) import without it.
"""
import importlib

# submodules load on their own (``from ... import configs`` must not need the library)
_SUBMODULES = {"binding", "build", "configs", "ep", "synth"}


def __getattr__(name):
    if name.startswith("__"):
        raise AttributeError(name)
    if name in _SUBMODULES:
        return importlib.import_module("." + name, __name__)
    binding = importlib.import_module(".binding", __name__)
    if hasattr(binding, name):
        return getattr(binding, name)
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")

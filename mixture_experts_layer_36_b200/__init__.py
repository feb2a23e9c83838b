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

def __getattr__(name):
    if name.startswith("__"):
        raise AttributeError(name)
    binding = importlib.import_module(".binding", __name__)
    if hasattr(binding, name):
        return getattr(binding, name)
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")

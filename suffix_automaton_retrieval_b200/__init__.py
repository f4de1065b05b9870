"""B200-native ROSA retrieval step (suffix-automaton retrieval of ROSA-Tuning).

The compute path lives in the CUDA library ``librosa_b200.so`` built from
``csrc/``; ``binding`` marshals torch tensors into its C ABI.  The binding is
imported lazily so that ``workloads`` (input generators) can be used without
touching the CUDA library.
"""
from importlib import import_module

__all__ = ["discretize", "match", "gather", "match_workspace_size", "status_string",
           "RosaError", "binding", "workloads"]


def __getattr__(name):
    if name in ("binding", "workloads"):
        return import_module(f"{__name__}.{name}")
    if name in __all__:
        return getattr(import_module(f"{__name__}.binding"), name)
    raise AttributeError(name)

"""B200-native KDA (Kimi Delta Attention) recurrence.

The compute lives in ``libkda.so`` (CUDA for sm_100a, C ABI in ``include/kda.h``);
``gated_delta_rule_62_b200.kda`` is the thin ctypes binding over it (argument
marshalling only). ``gated_delta_rule_62_b200.workloads`` holds the seeded
synthetic input recipes. Importing this package does not load the library.
"""

__all__ = ["kda", "workloads", "build"]


def __getattr__(name):
    if name in __all__:
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)

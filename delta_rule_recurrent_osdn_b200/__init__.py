"""B200-native forward pass of the Online Scaled DeltaNet (OSDN) token mixer.

The compute lives in ``libosdn.so`` (hand-written sm_100a CUDA kernels behind a C ABI,
declared in ``include/osdn.h``).  ``delta_rule_recurrent_osdn_b200.osdn`` is the thin
Python binding; it is imported lazily so that the input generators can be used on
machines without a GPU.
"""
__all__ = ["inputs", "osdn"]


def __getattr__(name):
    if name == "osdn":
        from . import osdn as _osdn
        return _osdn
    if name == "inputs":
        from . import inputs as _inputs
        return _inputs
    raise AttributeError(name)

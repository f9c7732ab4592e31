"""Tile-routed FP16/INT8 fused prefill attention for B200 (sm_100a).

The compute path is the C-ABI library ``libtm.so`` (hand-written CUDA for
sm_100a) built in this package directory; ``ops`` is its thin Python binding.
``inputs`` draws seeded synthetic workloads and imports neither.

Importing this package does not load the CUDA library; ``ops`` does, and it
raises if the library is missing.
"""

__all__ = ["inputs", "ops"]


def __getattr__(name):
    if name in ("ops", "inputs", "metrics"):
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)

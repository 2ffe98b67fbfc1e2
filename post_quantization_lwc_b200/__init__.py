"""libomq: a B200 (sm_100a) implementation of OmniQuant's fake-quantized linear calibration
step (learnable equivalent transformation, learnable weight clipping, per-token activation
fake-quant, tcgen05 GEMMs, MSE, straight-through backward, fold/pack).

The compute lives in the CUDA shared library ``libomq.so`` behind a C ABI (include/omq.h).
``post_quantization_lwc_b200.omq`` is the thin ctypes binding; importing it loads the library
and raises if it is missing. ``synth`` holds the seeded input recipes.
"""
__all__ = ["omq", "synth"]


def __getattr__(name):
    if name in __all__:
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)

"""Dynamic Bifocal RoPE attention (Jet-Long) for NVIDIA B200 (sm_100a).

The compute lives in the CUDA shared library ``libjetlong.so`` (C ABI in
``include/jetlong.h``); :mod:`zero_shot_rope_b200.jetlong` is its thin Python
binding and :mod:`zero_shot_rope_b200.synth` makes seeded synthetic inputs.
"""
__version__ = "0.1.0"


def __getattr__(name):
    # the binding is imported lazily so that `synth` works without the library
    if name in ("jetlong",):
        import importlib

        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)

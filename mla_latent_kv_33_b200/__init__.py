"""B200-native absorbed-form MLA decode (DeepSeek-V2 Multi-head Latent Attention).

The compute path lives in the CUDA library ``libmla.so`` (csrc/), called
through the C ABI declared in include/mla.h. ``mla_latent_kv_33_b200.mla`` is
the thin ctypes binding; submodules are imported on first use so that the
seeded input generator (``synth``) stays importable on machines without a GPU.
"""
import importlib

__all__ = ["mla", "synth"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)

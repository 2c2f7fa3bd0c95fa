"""B200-native ART run-time-terminated decode attention.

The compute path is ``libart.so`` (CUDA, sm_100a) behind the C ABI in
``include/art.h``; this package holds its ctypes binding, its build script and
the seeded synthetic workload generator.  The binding is imported lazily so
that the generator can be used on machines where the library is not built;
calling any attention entry point without the library raises ImportError.
"""
from importlib import import_module

_BINDING_NAMES = {
    "art_decode_attention", "art_decode_attention_ex", "art_decode_attention_multi",
    "art_build_order_sink_recency", "art_strerror",
    "art_page_summary", "art_build_order_importance",
    "art_version", "art_workspace_bytes", "art_decode_attention_no_alloc", "ArtError", "descriptor", "raw_library", "ENGINE_AUTO", "ENGINE_CUDA", "ENGINE_MMA",
    "STATUS", "ArtParams", "ArtTensor", "ArtLaunchInfo", "LIB_PATH",
}

__all__ = sorted(_BINDING_NAMES) + ["workloads", "build"]


def __getattr__(name):
    if name in _BINDING_NAMES:
        return getattr(import_module(".binding", __name__), name)
    if name in ("workloads", "build"):
        return import_module("." + name, __name__)
    raise AttributeError(name)

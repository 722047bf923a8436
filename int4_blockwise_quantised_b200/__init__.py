"""int4 blockwise-quantised Qwen2 decoder step on NVIDIA B200 (sm_100a).

The product is libvv.so (C ABI, include/vv.h) built from csrc/; this package is its Python
binding.  ``_vv`` exposes one function per C entry point with the same name; ``model`` packs
weights on the GPU and wraps the decoder handle.  Importing the binding requires the built
library: there is no CPU fallback.
"""

__all__ = ["_vv", "model"]


def __getattr__(name):
    # Lazy: `import int4_blockwise_quantised_b200.build` must work before libvv.so exists.
    if name in ("_vv", "model"):
        import importlib

        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)

"""Low-bit quantized linear layers with a low-rank adapter, for B200 (sm_100a).

The library is the C ABI in include/lbq.h, implemented by CUDA kernels in
csrc/ and built into liblbq.so (see build.py).  `qlora_quantized_linear_b200.lbq`
is its Python binding; `synthetic` draws the seeded benchmark inputs.
The binding is imported lazily so that `synthetic` works without the library.
"""

__all__ = ["lbq", "synthetic"]


def __getattr__(name):
    if name in ("lbq", "synthetic"):
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)

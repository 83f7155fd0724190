"""B200-native Clebsch-Gordan tensor-product convolution.

``equivariant_mlip_clebsch_b200.cgtp`` binds the C ABI of libcgtp
(include/cgtp.h); ``workloads`` draws the seeded synthetic inputs.  The
binding is imported lazily so that the input generators work without the
compiled library.
"""
import importlib

__all__ = ["cgtp", "workloads", "build"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)

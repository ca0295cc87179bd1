"""B200-native (sm_100a) block-sparse video attention.

VSA-style trainable block-sparse attention over 4x4x4 cube tiles of a video
latent grid, with an optional SLA/RoLA-style linear branch, as a C-ABI CUDA
library (libvsa.so, declared in include/vsa.h) plus a thin torch front-end.
"""
from .workloads import WORKLOADS, HEADLINE, Workload  # noqa: F401


def __getattr__(name):
    # the CUDA front-end loads libvsa.so lazily, on first use
    if name in ("ops", "_lib"):
        import importlib
        return importlib.import_module(f".{name}", __name__)
    raise AttributeError(name)

"""Mixed-format paged KV cache (FP8 anchor pages + packed 3-bit TQ3 pages) with decode
attention run directly over it, as hand-written CUDA kernels for sm_100a behind a C ABI
(``include/mkv.h``).  ``api.Pool`` is the Python binding; ``workloads`` draws seeded inputs."""
from .api import FMT_FP8, FMT_TQ3, MkvError, Pool, lib  # noqa: F401

__all__ = ["Pool", "MkvError", "lib", "FMT_FP8", "FMT_TQ3"]

"""Star Attention two-phase attention hot path for one B200 (sm_100a).

The compute lives in ``lib/libstar.so`` (C ABI: include/star_attention.h);
``api`` is a thin ctypes/PyTorch binding; ``workloads`` draws the seeded
synthetic inputs.  Importing the package does not load the library; the
first use of ``StarCache``, ``star_lse_merge`` or ``star_rope`` does, and raises if the
library or a CUDA device is missing.
"""

__all__ = ["StarCache", "star_lse_merge", "star_rope", "workloads", "build"]


def __getattr__(name):
    if name in ("StarCache", "star_lse_merge", "star_rope"):
        from . import api
        return getattr(api, name)
    raise AttributeError(name)

"""Group-wise affine quantized matmul for NVIDIA B200 (sm_100a).

The product is libaq.so (C ABI: include/aq.h); ``api`` is its thin Python
binding and ``inputs`` the seeded synthetic workloads.  Importing the package
loads nothing; the first call of an ``aq_*`` function loads libaq.so.
"""
__version__ = "0.1.0"


def __getattr__(name):
    if name.startswith("aq_") or name in ("AqError", "Workspace", "AQ_MODE_AFFINE", "AQ_MODE_FP4"):
        from . import api
        return getattr(api, name)
    raise AttributeError(name)

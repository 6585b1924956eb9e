"""DFSAttn block-sparse spatiotemporal attention on B200 (sm_100a).

The CUDA library ``libdfsattn.so`` (C ABI declared in include/dfsattn.h)
implements the whole path; ``dfsattn`` binds it with ctypes and
``pipeline.DfsLayer`` chains the calls for one attention layer.
"""
from . import dfsattn  # noqa: F401  (raises if the library is missing)
from .dfsattn import Shape  # noqa: F401
from .pipeline import DfsLayer  # noqa: F401

__version__ = "0.1.0"

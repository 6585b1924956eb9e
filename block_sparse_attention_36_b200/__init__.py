"""DFSAttn block-sparse spatiotemporal attention on B200 (sm_100a).

The CUDA library ``libdfsattn.so`` (C ABI declared in include/dfsattn.h)
implements the whole path; ``dfsattn`` binds it with ctypes and
``pipeline.DfsLayer`` chains the calls for one attention layer.

The library is loaded on first use of ``dfsattn``, ``Shape`` or
``DfsLayer`` (so that ``block_sparse_attention_36_b200.build`` can run
before it exists); loading raises if it is missing.
"""
import importlib

__version__ = "0.1.0"
__all__ = ["dfsattn", "pipeline", "Shape", "DfsLayer"]


def __getattr__(name):
    if name in ("dfsattn", "pipeline"):
        return importlib.import_module(f".{name}", __name__)
    if name == "Shape":
        return importlib.import_module(".dfsattn", __name__).Shape
    if name == "DfsLayer":
        return importlib.import_module(".pipeline", __name__).DfsLayer
    raise AttributeError(name)

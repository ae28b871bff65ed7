"""Decode-step hash-score -> top-k select -> exact sparse attention on B200.

``hash_indexed_top_b200.dashkv`` is the Python binding over the C-ABI
library ``libdashkv.so`` (built from ``csrc/``); ``workloads`` draws seeded
synthetic inputs.  Importing the package loads neither.
"""
__all__ = ["dashkv", "workloads"]

"""SSA block-sparse attention on NVIDIA B200 (sm_100a).

The hot path of "SSA: Sparse Sparse Attention by Aligning Full and Sparse
Attention Outputs in Feature Space" (arXiv 2511.20102): block pooling, causal
top-k block selection, sparse and full attention forward/backward, and the
bidirectional output-alignment loss, as hand-written CUDA behind the C ABI of
include/ssa.h (libssa.so).  ``_lib`` is the thin ctypes binding; ``ops``
holds allocation helpers on top of it; ``inputs`` draws seeded synthetic
workloads.  Importing the package loads nothing; the library is loaded on the
first call.
"""

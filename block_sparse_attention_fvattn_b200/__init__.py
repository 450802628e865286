"""B200-native adaptive block-sparse attention (FVAttn-style routing + sparse kernel).

The compute path is a C-ABI CUDA library (`libfvattn.so`, built from `csrc/`)
with a thin ctypes binding in `fvattn.py`. Importing this package does not load
the library; `block_sparse_attention_fvattn_b200.fvattn` does, and raises if it
is missing.
"""

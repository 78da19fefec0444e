"""SAS gated block-sparse causal attention for NVIDIA B200 (sm_100a).

The compute lives in a C-ABI CUDA library (include/sas.h, built by
``block_sparse_attention_sas_b200.build``); ``_lib`` is its Python binding.
``workloads`` draws the seeded synthetic inputs, ``dist`` holds the
multi-process plumbing.
"""
__all__ = ["build", "workloads", "dist"]

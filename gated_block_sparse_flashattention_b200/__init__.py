"""SAS gated block-sparse attention for NVIDIA B200 (sm_100a).

The compute path is the CUDA library ``libsas_b200.so`` built from ``csrc/``;
``binding`` marshals torch tensors into its C ABI. Importing this package does
not load the library; the first call through ``binding`` does, and raises if it
is missing.
"""

__all__ = ["binding", "workloads"]

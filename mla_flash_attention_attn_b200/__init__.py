"""B200-native (sm_100a) flash attention for Multi-head Latent Attention (MLA).

The computation lives in libmla_fa.so (C ABI: include/mla_fa.h); ``binding``
marshals torch tensors to it. ``workloads`` holds the seeded synthetic inputs.
Importing the package loads nothing; the library is loaded on first use.
"""

__all__ = ["binding", "workloads", "build"]

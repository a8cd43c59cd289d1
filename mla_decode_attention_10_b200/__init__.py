"""Fused MLA decode epilogue for NVIDIA B200 (sm_100a).

Per token: H latent query rows (ql_nope[512] || q_pe[64], optional RoPE on the
64 pe dims, optional per-tensor e4m3) and one latent KV row scattered into a
paged cache at slot_mapping[t], in one CUDA kernel behind a C ABI
(``include/mla_epilogue.h``).  ``epilogue`` is the ctypes binding,
``workloads`` the seeded synthetic inputs, ``build`` the nvcc build.

Importing the package does not load the CUDA library; the first call into
``epilogue`` does, and raises if it has not been built.
"""

__all__ = ["epilogue", "workloads", "build"]

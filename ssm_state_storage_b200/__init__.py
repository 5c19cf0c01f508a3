"""ReplaySSM SSM-layer decode on B200 (sm_100a).

The compute lives in the C-ABI library ``libreplayssm.so`` (CUDA kernels built
for sm_100a); ``ssm_state_storage_b200.replayssm`` is the thin ctypes binding
over it.  ``workloads`` draws the seeded synthetic inputs.
"""
__all__ = ["workloads", "replayssm"]

"""B200-native batched speculative-decoding verification.

The compute path is the CUDA library ``libspecverify.so`` (sm_100a) behind a
C ABI (``include/spec_verify.h``); :mod:`.binding` marshals PyTorch tensors
and streams into it.  :mod:`.workloads` draws the seeded synthetic inputs.
"""
__all__ = ["binding", "workloads"]

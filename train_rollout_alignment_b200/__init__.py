"""NVFP4 block quantization with train/rollout rounding alignment on B200.

The compute lives in ``libnvfp4trace.so`` (hand-written sm_100a CUDA behind the
C ABI of ``include/nvfp4_trace.h``); ``_binding`` exposes the same entry points
for torch CUDA tensors.  ``synthetic`` holds the seeded workload generators.
"""

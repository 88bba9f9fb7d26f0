"""TTQ (activation-aware test-time quantization) hot path for B200 (sm_100a).

The compute lives in ``libttq.so`` (hand-written CUDA behind the C ABI in
``include/ttq.h``); :mod:`test_weight_quantization_b200.ttq` is the thin
ctypes binding with the same call names. Import of the package itself loads
nothing, so CPU-only tools (the input generator) work without a GPU.
"""
__all__ = ["inputs", "ttq"]

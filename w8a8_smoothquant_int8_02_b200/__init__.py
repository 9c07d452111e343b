"""SmoothQuant W8A8 linear layer for B200 (sm_100a).

Y = X W = (X diag(s)^-1)(diag(s) W): per-channel calibration, smoothing
factors, offline per-output-channel weight quantization, a fused runtime
activation smooth + per-token quantization kernel, and an 8-bit tcgen05
tensor-core GEMM with a fused dequantization epilogue. All compute runs in the
CUDA library ``libsq.so`` behind the C ABI declared in ``include/sq.h``; the
Python layer (``ops``) only marshals arguments.
"""
__all__ = ["ops", "synth", "workloads"]

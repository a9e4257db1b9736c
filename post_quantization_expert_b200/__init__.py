"""B200 (sm_100a) implementation of CLHA calibration: Cross-Layer Hessian Aggregation for quantizing
weight-shared Mixture-of-Experts transformers.

    clha      ctypes binding of libclha.so (the C ABI in include/clha.h), same names as the C calls
    pipeline  the collect -> aggregate -> quantize sequence for dense and MoE weight groups
    build     nvcc build of libclha.so for sm_100a
"""
__all__ = ["clha", "pipeline", "build"]

"""B200 (sm_100a) fused residual-add + RMSNorm + activation quantization.

`mxfp4_quantization_b200.fusednorm` is the binding of libfusednorm.so (the
kernels and their C ABI, include/fusednorm.h).  It is not imported here, so
that `mxfp4_quantization_b200.synth` and `.build` work before the library is
built; importing `fusednorm` without the library raises ImportError.
"""
__all__ = ["fusednorm", "synth", "build"]

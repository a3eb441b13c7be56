"""Quantised Mamba2 mixer (FastMamba's W8A8 + power-of-two scheme) on one B200.

`lib` is the ctypes binding of the C ABI (include/fastmamba.h), `model` holds
device-resident layers and stacks, `synth` the seeded synthetic inputs and
`build` the in-tree nvcc build of libfastmamba.so.
"""
__all__ = ["lib", "model", "synth", "build"]

"""B200-native FNO spectral-convolution block: C-ABI CUDA library + thin binding.

``synth`` (seeded inputs) imports nothing else from this package.  The CUDA
binding (``capi``) loads ``libfno.so`` on first use and raises if it is
missing; there is no fallback path.
"""
__all__ = ["synth", "capi"]

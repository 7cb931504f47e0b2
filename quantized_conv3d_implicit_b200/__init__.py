"""B200-native Conv3D implicit GEMM with fused NVFP4 activation fake-quantisation.

The compute path is a C-ABI shared library (``libq3d.so``, built from
``csrc/`` for sm_100a by ``build.py``); ``api`` only marshals torch tensors
into its calls and raises if the library is missing.  ``workloads`` draws the
seeded synthetic inputs.
"""
from .api import (Q3DError, check_device_error, conv3d_implicit_gemm, fp4_fake_quant,  # noqa: F401
                  load_library, out_shape)

__all__ = ["conv3d_implicit_gemm", "fp4_fake_quant", "check_device_error", "load_library", "out_shape", "Q3DError"]

"""B200-native Conv3D implicit GEMM with fused NVFP4 activation fake-quantisation.

The compute path is a C-ABI shared library (``libq3d.so``, built from
``csrc/`` for sm_100a); this package only marshals torch tensors into its
calls.  ``workloads`` draws the seeded synthetic inputs.
"""

"""B200-native SPIN-4DGS per-Gaussian attribute decoder.

The compute path is the C-ABI library ``libspin4d.so`` (hand-written CUDA
kernels for sm_100a) declared in ``include/spin4d.h``; ``spin4d`` is its thin
ctypes binding.  Import it explicitly::

    from spatiotemporal_neural_field_b200 import spin4d

``synthetic`` draws seeded inputs and holds none of the decoder's arithmetic.
"""
__all__ = ["spin4d", "synthetic"]

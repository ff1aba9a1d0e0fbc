"""CPU oracle for the SPIN-4DGS attribute decoder -- TEST INFRASTRUCTURE ONLY.

A plain, slow, obviously correct numpy implementation of what the decoder
computes, written from *Implicit 4D Gaussian Splatting for Fast Motion with
Large Inter-Frame Displacements* (SPIN-4DGS), section 3.1 Eq. 2 and section
3.3 Eqs. 7-11, from the 4D Gaussian Splatting reading notes (sections
2.2 and 3.1-3.2: HexPlane and the deformation network), and from the
KineticGS notes (double-sigmoid temporal window, "learnable energy-flow
activation"; Z-order space-filling curve), and, for the renderer behind the
decoder, from section 3.1 Eqs. 1, 3 and 4 (EWA projection and alpha
compositing).  Floating point is fp64 except where the method decides an
integer (the interpolation cell of each position), which is taken in fp32
exactly as the CUDA path takes it.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path never calls it and
shares no code with it; the only shared module is the seeded input generator
``spatiotemporal_neural_field_b200.synthetic``, which draws data and holds
none of the decoder's arithmetic.

Every function here is pinned by ``tests/test_oracle_*.py`` against values
and properties fixed by the pages or by mathematics (closed forms, brute
force, finite differences), not against itself.
"""
from . import hashgrid, decoder, hexplane, ordering, heads, render  # noqa: F401

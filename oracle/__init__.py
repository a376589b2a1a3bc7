"""CPU oracle for the weight-only quantized linear layer.

TEST INFRASTRUCTURE ONLY.  Two independent restatements of what the layer
computes -- ``oracle_c`` (a ctypes wrapper over the plain C99 ``oracle.c``)
and ``oracle_np`` (NumPy) -- used by the tests, by the smoke check and by the
benchmark's CPU-baseline leg.  The CUDA library never imports, links or calls
anything here, and nothing here imports the library.

Every function is pinned by ``tests/test_oracle_*.py`` against facts fixed by
the source pages and by mathematics (bits-per-weight closed forms, exhaustive
round trips, hand-derived byte patterns, exact rational dequantisation,
brute-force rational dot products, symmetry and linearity).
"""

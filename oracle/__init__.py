"""Plain fp64 CPU oracle for the DFSAttn hot path.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or
execute anything in this package: only the tests, ``__graft_entry__.smoke()``
and the benchmark's CPU-baseline / reference arm use it. It shares no code,
tables or constants with the CUDA library; the two meet only on the seeded
inputs drawn by the separate ``synth`` module.

Each function computes the plain definition of one stage, in the order the
pages give the method:

* ``hilbert``   -- global 3D Hilbert-curve token order and its inverse
                   (DFSAttn, Methodology item 1).
* ``scoring``   -- sub-block mean pooling and the hierarchical block score
                   (DFSAttn, Methodology item 2).
* ``selection`` -- per-query-block top-k and cumulative-mass threshold
                   selection (DFSAttn, Methodology item 3; VMoBA abstract,
                   modification 3).
* ``lvsa``      -- rotating global anchors plus expanded adaptive windows
                   (LVSA, section 2, core mechanism).
* ``schedule``  -- monotonically decreasing keep budget with masks refreshed
                   at a fixed interval (DFSAttn, Methodology item 3).
* ``attention`` -- softmax attention restricted to the kept key blocks, in
                   fp64, and dense attention.

Readings of passages the pages leave open are stated in each module header.
"""

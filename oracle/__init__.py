"""FP64 CPU oracle for block-sparse video attention -- TEST INFRASTRUCTURE ONLY.

Only the test suite, the smoke check and the benchmark's CPU-baseline leg may import
this package.  The product path (the CUDA library and its Python binding) never calls
it, and it shares no code with that path: the two meet only on the seeded inputs from
``synthetic``.

It is a plain, slow, obviously-correct restatement of what the hot path computes:

* ``reorder``   -- the 3D-tile token permutation and its inverse, by explicit loops
                   over tiles and tokens;
* ``mask``      -- the block masks (local window + rotating global anchors, SQuad-style
                   two-stage windows, all-ones, given static masks) as dense boolean
                   matrices, and their per-query-block CSR lists;
* ``attention`` -- masked softmax attention in float64, both block-wise (rows of one
                   query block share their key set) and by brute force over an explicit
                   token-level mask;
* ``calib``     -- the offline calibration of static masks: block energies of dense
                   softmax attention, the minimal-prefix selection reaching a cumulative
                   energy threshold, and the cross-prompt agreement threshold.

Every function is pinned by tests under ``-m "not gpu"`` against hand-worked examples,
closed forms, library routines and invariants; none is "parity unpinned".
"""

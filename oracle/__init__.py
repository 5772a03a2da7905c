"""CPU oracle for Sol block-sparse attention -- test infrastructure only.

Only the tests, the smoke check and the bench's CPU-baseline leg may import
this package.  The CUDA path never imports it and shares no code with it.
``sol_ref`` is the fp64 NumPy oracle; ``brute`` is an independent scalar
restatement used to pin it on tiny inputs.
"""

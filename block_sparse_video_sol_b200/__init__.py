"""B200-native Sol block-sparse attention (pool -> route -> exact + centroid attention).

The compute path is the C-ABI library ``libsol.so`` (hand-written CUDA for
sm_100a); ``block_sparse_video_sol_b200.sol`` is its thin ctypes binding.
Importing this package does not load the library; ``sol`` does, and fails
loudly if it is missing.
"""

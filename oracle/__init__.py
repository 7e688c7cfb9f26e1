"""Float64 CPU oracle for the DraftAttention2 attention hot path.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg are the only callers.  The product path never imports it.
"""

"""CPU oracle for the fused MoE layer: test infrastructure only.

Only the tests, the graft entry point's smoke check and bench.py's CPU
baseline / reference legs may import it; the product path never does.
"""

"""CPU oracle for the fused MoE layer: test infrastructure only.

Only the tests, `__graft_entry__.smoke()` and bench.py's CPU
baseline / reference legs may import it; the product path never does.
"""

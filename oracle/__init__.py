"""CPU oracle for the Q4_0 decode hot path (test infrastructure only).

Only tests/, the smoke check and the bench's CPU-baseline leg may import it.
"""

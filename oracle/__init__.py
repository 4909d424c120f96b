"""CPU oracle for causal prefill attention with the ZYFA FP8 method.

Test infrastructure only (tests/, the smoke check, the bench's CPU-baseline
leg).  The product package never imports it.
"""

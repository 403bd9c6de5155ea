"""CPU oracle of the routed MoE layer, forward and bf16 backward (test
infrastructure only).

Imported by the tests, the smoke check and the benchmark's CPU-baseline leg;
never by the library itself.
"""

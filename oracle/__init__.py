"""Independent CPU oracle of the MoE layer forward (plain C + ctypes).

TEST INFRASTRUCTURE ONLY: tests/, the package smoke check and the CPU-baseline
leg of bench.py use it; the product path never imports it.
"""

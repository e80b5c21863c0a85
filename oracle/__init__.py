"""CPU oracle of Prism's sparse video self-attention.

Test infrastructure only: imported by tests/, by the package's smoke() check
and by the CPU-baseline leg of bench.py, never by the library itself.
"""

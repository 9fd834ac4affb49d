"""CPU oracle for block-scaled FP4 quantization -- test infrastructure only.

Importable by the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py``; never by the library itself.
"""

"""CPU oracle of the record-and-replay discrete adjoint -- TEST INFRASTRUCTURE ONLY.

Importable only by tests/, the smoke check and the benchmark's CPU-baseline leg.  The product
path (the CUDA library and its Python binding) never imports, links or runs anything here.
"""

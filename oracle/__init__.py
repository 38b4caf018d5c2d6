"""float64 CPU oracle of the RG-LRU block core -- test infrastructure only.

Importable by tests, the smoke check and the benchmark's CPU-baseline leg;
never by the product package.
"""

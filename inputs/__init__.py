"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle's callers.

``inputs.workloads`` draws random numbers and lays them out (pages, block tables);
it holds none of the attention arithmetic and imports only numpy, so importing it
never loads the CUDA library.
"""

"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle's
callers.

A package of its own, outside the library: importing it loads no CUDA code,
so a process that only runs the CPU oracle never maps the library.  It holds
no arithmetic of the quantizer or of the layer (see ``inputs/synthetic.py``).
"""

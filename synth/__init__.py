"""Seeded synthetic inputs (token streams, table values, workload configs).

Shared by tests, the bench and the oracle checks; it contains no arithmetic of
the N-gram embedding layer itself. `synth.device` (optional, needs the built
`libngram_synth.so`) fills device tables with the same generator.
"""
from . import configs, gen, workloads  # noqa: F401

"""CPU oracle for the quantized fused-MoE experts path (test infrastructure).

This package is test infrastructure. Only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.
The product path (``bit_weight_quantization_moeq_b200``) never imports, links or
executes anything under ``oracle/``, and the oracle imports nothing from it.
"""
from .moeq_oracle import *  # noqa: F401,F403

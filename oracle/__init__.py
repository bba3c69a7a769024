"""fp64 CPU oracle for SAS gated block-sparse attention (test infrastructure only).

Only the tests, the smoke check and the benchmark's CPU-baseline leg import
this package. It shares no code with the CUDA library and imports nothing from
it.
"""
from .sas_oracle import *  # noqa: F401,F403

"""CPU oracle (test infrastructure only; see llama_oracle's docstring).

Only tests, the smoke check and the benchmark's CPU-baseline leg import it.
"""
from . import llama_oracle  # noqa: F401

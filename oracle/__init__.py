"""CPU oracle for the GPT training step (test infrastructure only).

Nothing in the ``decoder_only_gpt_b200`` package imports this package, and
this package imports nothing from it.  Callers: ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference arm.
"""
from .gpt_oracle import *  # noqa: F401,F403
from .gpt_oracle import OracleConfig, StepResult, from_workload, step  # noqa: F401

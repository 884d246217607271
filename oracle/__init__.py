"""CPU oracle of the LongFlow decode step — test infrastructure only.

Imported by the tests, by ``__graft_entry__.smoke()`` and by the CPU-baseline
leg of ``bench.py``; never by the library.  See ``oracle/longflow.py``.
"""
from .longflow import (SCORES, RowStep, StepResult, decode_attention,  # noqa: F401
                       decode_row, decode_step, prefill)

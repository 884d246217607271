"""CPU oracle of the LongFlow decode step — test infrastructure only.

Imported by the tests, by ``__graft_entry__.smoke()`` and by the CPU-baseline
leg of ``bench.py``; never by the library.  See ``oracle/longflow.py``.
"""
from .longflow import (SCORES, RowStep, StepResult, decode_attention,  # noqa: F401
                       decode_row, decode_step, prefill)
from .kvfp8 import (E4M3_MAX, decode_step_fp8, dequantize, e4m3_decode,  # noqa: F401
                    e4m3_encode, prefill_fp8, quantize)

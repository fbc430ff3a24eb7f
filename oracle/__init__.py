"""fp64 CPU oracle for the sparse MLA prefill attend block (test infrastructure).

Only the tests, the smoke check and the benchmark's CPU-baseline leg may
import this package. The CUDA library never does.
"""
from .oracle import (  # noqa: F401
    attend_rows,
    attend_rows_threaded,
    build,
    bf16_from_double,
    bf16_to_double,
    e4m3_from_float,
    e4m3_to_double,
    host_threads,
    prefill_rows,
    prefill_rows_threaded,
    project_rows,
    quantize_act,
    upproject_rows,
)

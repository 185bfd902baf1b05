"""CPU oracle for KDA multi-token recurrent prefill (test infrastructure).

Only the tests, the smoke check and the CPU-baseline leg of the benchmark may
import this package.  It is independent of the CUDA path: it shares no code,
header, helper or constant with it, and the product never calls it.

Two independent implementations of the same definition live here:

* ``prefill``  — the per-token FP64 recurrence in plain C (kda_oracle.c), the
  reference every GPU result is compared against;
* ``chunked_prefill`` — the chunked (UT/WY) form in NumPy FP64, derived by hand
  from the per-token recurrence and used only to pin it: the chunked and the
  per-token forms must agree.

Both compute the Kimi Delta Attention recurrence written out in the module
header of kda_oracle.c.
"""
from .kda_oracle import (build_oracle, oracle_library_path, prefill, prefill_f64,
                         max_threads)
from .kda_chunked import chunked_prefill_f64

__all__ = ["build_oracle", "oracle_library_path", "prefill", "prefill_f64", "max_threads",
           "chunked_prefill_f64"]

"""CPU oracle for KDA multi-token recurrent prefill (test infrastructure).

Only the tests, the smoke check and the CPU-baseline leg of the benchmark may
import this package.  It is independent of the CUDA path: it shares no code,
header, helper or constant with it, and the product never calls it.

Two independent implementations of the same definition live here:

* ``prefill``  — the per-token FP64 recurrence in plain C (kda_oracle.c), the
  reference every GPU result is compared against;
* ``chunked_prefill`` — the chunked (UT/WY) form in NumPy FP64, derived by hand
  from the per-token recurrence and used only to pin it: the chunked and the
  per-token forms must agree;
* ``frontend_f64`` — the input front end (q/k L2 norm, gate from A_log and
  dt_bias under a lower bound, beta from its logit) in NumPy FP64, whose
  formula is this library's stated reading (kda_frontend.py).

Both compute the Kimi Delta Attention recurrence written out in the module
header of kda_oracle.c.
"""
from .kda_oracle import (build_oracle, oracle_library_path, prefill, prefill_f64,
                         max_threads)
from .kda_chunked import chunked_prefill_f64
from .kda_frontend import frontend_f64, QK_L2NORM, GATE_IN_KERNEL, BETA_IS_LOGIT

__all__ = ["build_oracle", "oracle_library_path", "prefill", "prefill_f64", "max_threads",
           "chunked_prefill_f64", "frontend_f64", "QK_L2NORM", "GATE_IN_KERNEL",
           "BETA_IS_LOGIT"]

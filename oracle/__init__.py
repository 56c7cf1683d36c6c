"""CPU oracle package: test infrastructure only (see ``rlt_oracle``).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import it.  It shares no code with the CUDA library.
"""
from .rlt_oracle import (RLTOracle, RowState, argmax_lowest, attend, rmsnorm, rope,
                         round_bf16, run_sequence, sample_inverse_cdf, softmax)

__all__ = ["RLTOracle", "RowState", "argmax_lowest", "attend", "rmsnorm", "rope",
           "round_bf16", "run_sequence", "sample_inverse_cdf", "softmax"]

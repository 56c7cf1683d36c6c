"""bf16 drift over recurrent steps, measured on the oracle: the bf16-mirrored
mode (rounding where the bf16 CUDA path stores bf16) against the fp64 mode,
position by position.  The pages concede that the recurrence's Jacobian
products are unbounded in general (jiphyeonjeon review §4.3); at the
workloads' random N(0, 0.02) weights the rounding error does not grow with
the number of transitions, which is what lets one tolerance serve every
position of the parity tests."""
import numpy as np
import pytest

import rlt_inputs as ri
from oracle import RLTOracle


@pytest.mark.parametrize("name,T", [("parity_bf16", 128), ("rlt2_mod5_bf16", 64)])
def test_bf16_rounding_does_not_accumulate_over_positions(name, T):
    cfg = ri.CONFIGS[name]
    W = ri.generate_weights(cfg)
    mirror, exact = RLTOracle(cfg, W, "bf16"), RLTOracle(cfg, W, "fp64")
    toks = ri.make_tokens(cfg, 2, T)
    err = np.zeros(T)
    for r in range(2):
        a, b = mirror.new_state(), exact.new_state()
        mirror.encode(a, toks[r])
        exact.encode(b, toks[r])
        for t in range(T):
            mirror.transition(a)
            exact.transition(b)
            err[t] = max(err[t], float(np.max(np.abs(mirror.readout(a) - exact.readout(b)))))
    q = T // 4
    print(f"{name}: |dlogit| bf16 mirror vs fp64, max over positions 1-{q}: "
          f"{err[:q].max():.2e}, {T - q + 1}-{T}: {err[-q:].max():.2e}")
    assert err.max() < 3e-2                        # inside the bf16 parity tolerance
    assert err[-q:].max() < 2.0 * err[:q].max()    # no growth along the recurrence

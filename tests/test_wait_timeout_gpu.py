"""Failure detection on the device without a fault: a kernel whose wait can
never be satisfied must give up after its poll limit, record the timeout in
the state's error word and return, leaving the context usable.

rlt_selftest_wait launches one CTA that waits (kind 0) on an mbarrier
nobody arrives on -- no copy in flight, no tensor memory held -- or (kind 1)
on a global word nobody sets, through the same bounded-wait helpers as the
library's pipelines.  rlt_state_check must then report RLT_E_TIMEOUT once,
and the state must go on computing what the oracle computes.
"""
import time

import numpy as np
import pytest

import rlt_inputs as ri
from oracle import RLTOracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sd():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tests.conftest import build_library
    build_library()
    import stateful_decoding_b200 as sd
    return sd


@pytest.mark.parametrize("kind,polls", [(0, 64), (0, 1024), (1, 4096)])
def test_wait_gives_up_and_reports_timeout(sd, kind, polls):
    import torch
    cfg = ri.CONFIGS["tiny_fp32"]
    W = ri.generate_weights(cfg)
    model = sd.Model(ri.write_blob(cfg, W))
    B, T = 2, 8
    st = sd.State(model, B, T + 1)
    toks = ri.make_tokens(cfg, B, T)
    st.encode(toks)
    st.prefill(T // 2)
    st.check()
    t0 = time.perf_counter()
    assert sd.rlt_selftest_wait(st.handle, kind, polls) == sd.RLT_OK
    assert sd.rlt_state_check(st.handle) == sd.RLT_E_TIMEOUT
    dt = time.perf_counter() - t0
    print(f"kind {kind}: {polls} polls gave up after {dt * 1e3:.2f} ms "
          f"({dt / polls * 1e6:.2f} us per poll)")
    assert sd.rlt_state_check(st.handle) == sd.RLT_OK        # reported once, then cleared
    # the context and the state still work: finish the prefill, match the oracle
    st.prefill(T - T // 2)
    lg = np.zeros((B, cfg.vocab), np.float32)
    st.readout(lg)
    torch.cuda.synchronize()
    st.check()
    orc = RLTOracle(cfg, W, "fp64")
    for b in range(B):
        r = orc.new_state()
        orc.encode(r, toks[b])
        orc.prefill(r, T)
        assert np.max(np.abs(lg[b] - orc.readout(r))) <= 1e-4
    st.close()
    model.close()


def test_selftest_rejects_bad_arguments(sd):
    cfg = ri.CONFIGS["tiny_fp32"]
    model = sd.Model(ri.write_blob(cfg, ri.generate_weights(cfg)))
    st = sd.State(model, 1, 4)
    for kind, polls in ((2, 10), (-1, 10), (0, 0), (1, (1 << 24) + 1)):
        assert sd.rlt_selftest_wait(st.handle, kind, polls) == sd.RLT_E_ARG
    assert sd.rlt_selftest_wait(None, 0, 10) == sd.RLT_E_ARG
    st.check()
    st.close()
    model.close()

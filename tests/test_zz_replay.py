"""Replay log-probabilities (rlt_replay_logprobs) through the C ABI.

log p(y_j | everything before y_j), each read from the state that precedes the
token and followed by one transition (jiphyeonjeon review "Recurrent Looped
Transformer" §6.2, eq. 5.3-5.5; greeksharifa "Recurrent Looped Transformer 요약
설명" App. D.3, F.4), against the oracle's replay; against the log-softmax of
rlt_readout's own logits; the state it leaves against encode + prefill; host
and device buffers; error paths.  Tolerance: a logit error of tol moves a
log-probability by at most 2 tol / temperature.
"""
import numpy as np
import pytest

import rlt_inputs as ri
from oracle import RLTOracle
from oracle.rlt_oracle import replay_logprobs
from tests.rlt_testlib import TOL_BF16, oracle_mode, tol_for

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


def _log_softmax_rows(lg, temperature):
    z = lg.astype(np.float64) / temperature
    z = z - z.max(axis=1, keepdims=True)
    return z - np.log(np.exp(z).sum(axis=1, keepdims=True))


@pytest.mark.parametrize("name,temp", [("tiny_fp32", 1.0), ("parity_bf16", 1.0),
                                       ("s5_bf16", 0.7), ("rlt2_mod5_bf16", 0.8)])
def test_replay_matches_oracle_and_readout(sd, name, temp):
    import torch
    cfg = ri.CONFIGS[name]
    B, n = 3, 17
    W = ri.generate_weights(cfg)
    model = sd.Model(ri.write_blob(cfg, W))
    toks = ri.make_tokens(cfg, B, n)
    st = sd.State(model, B, n + 1)
    lp = st.replay_logprobs(toks, temperature=temp)          # from H_0
    pe, pd = st.positions()
    assert list(pe) == [n] * B and list(pd) == [n] * B
    assert np.isfinite(lp).all() and (lp <= 1e-6).all()

    orc = RLTOracle(cfg, W, oracle_mode(cfg))
    tol = 2 * tol_for(cfg) / temp
    worst = 0.0
    for b in range(B):
        want = replay_logprobs(orc, orc.new_state(), toks[b], temp)
        err = float(np.max(np.abs(lp[b] - want)))
        worst = max(worst, err)
        assert err <= tol, f"row {b}: |dlogp| {err} > {tol}"
    print(f"{name}: max |dlogp| vs oracle {worst:.3e} (tol {tol:.1e})")

    # the state it leaves = encode + prefill of the same tokens
    ref = sd.State(model, B, n + 1)
    ref.encode(toks)
    ref.prefill(n)
    if cfg.variant == 1:
        np.testing.assert_array_equal(st.read(sd.PART_S), ref.read(sd.PART_S))
    else:
        # RLT-2 prefill runs each chunk's positions together while the replay
        # steps token by token: equal up to rounding, as in the serving-split
        # test, so the readouts agree to the bf16 tolerance
        la = np.zeros((B, cfg.vocab), np.float32)
        lb = np.zeros((B, cfg.vocab), np.float32)
        st.readout(la)
        ref.readout(lb)
        torch.cuda.synchronize()
        np.testing.assert_allclose(la, lb, atol=TOL_BF16, rtol=0)

    # one more token: its log-probability is the log-softmax of the logits
    # rlt_readout gives for the same state
    lg = np.zeros((B, cfg.vocab), np.float32)
    st.readout(lg, temperature=temp)
    torch.cuda.synchronize()
    extra = np.ascontiguousarray((toks[:, -1:] + 1) % cfg.vocab).astype(np.int32)
    lp1 = st.replay_logprobs(extra, temperature=temp)
    want1 = _log_softmax_rows(lg, temp)[np.arange(B), extra[:, 0]]
    np.testing.assert_allclose(lp1[:, 0], want1, atol=2e-5, rtol=0)
    st.check()
    for s_ in (st, ref):
        s_.close()
    model.close()


def test_replay_device_buffers_and_errors(sd):
    import torch
    cfg = ri.CONFIGS["parity_bf16"]
    B, n = 2, 6
    model = sd.Model(ri.write_blob(cfg, ri.generate_weights(cfg)))
    toks = ri.make_tokens(cfg, B, n)
    a = sd.State(model, B, n + 2)
    b = sd.State(model, B, n + 2)
    lp_h = a.replay_logprobs(toks)
    lp_d = torch.empty((B, n), dtype=torch.float32, device="cuda")
    b.replay_logprobs(torch.from_numpy(toks).cuda(), logprobs=lp_d)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(lp_d.cpu().numpy(), lp_h)

    one = np.ascontiguousarray(toks[:, :1])
    out = np.zeros((B, 1), np.float32)
    # encoded tokens not yet consumed
    a.encode(one)
    with pytest.raises(sd.RLTError) as e:
        a.replay_logprobs(one)
    assert e.value.code == sd.RLT_E_ORDER
    a.prefill(1)
    # temperature, host token outside the vocabulary, capacity: nothing runs
    assert sd.rlt_replay_logprobs(a.handle, one, 1, out, 0.0) == sd.RLT_E_ARG
    bad = np.full((B, 1), cfg.vocab, np.int32)
    assert sd.rlt_replay_logprobs(a.handle, bad, 1, out, 1.0) == sd.RLT_E_ARG
    two = np.ascontiguousarray(toks[:, :2])
    assert sd.rlt_replay_logprobs(a.handle, two, 2, np.zeros((B, 2), np.float32),
                                  1.0) == sd.RLT_E_CAPACITY
    pe, pd = a.positions()
    assert list(pe) == [n + 1] * B and list(pd) == [n + 1] * B
    # a device token outside the vocabulary: NaN, and the state's error word
    bad_d = torch.full((B, 1), cfg.vocab + 3, dtype=torch.int32, device="cuda")
    got = b.replay_logprobs(bad_d)
    assert np.isnan(got).all()
    with pytest.raises(sd.RLTError) as e:
        b.check()
    assert e.value.code == sd.RLT_E_ARG
    b.check()
    a.check()
    for s_ in (a, b):
        s_.close()
    model.close()

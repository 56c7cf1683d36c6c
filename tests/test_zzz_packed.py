"""Packed documents (rlt_prefill_packed) through the C ABI.

Each row holds independent documents one after another; at a document start
the row restarts from H_0 (jiphyeonjeon review "Recurrent Looped
Transformer" §6.1; greeksharifa "Recurrent Looped Transformer 요약 설명"
App. F).  After the call a row must equal its last document encoded and
prefilled alone in a fresh row (the GPU against itself) and the oracle's
packed run.  Rows start documents at different columns, so they run at
different positions.  Named to be collected after the other GPU tests.
"""
import numpy as np
import pytest

import rlt_inputs as ri
from oracle import RLTOracle
from oracle.rlt_oracle import prefill_packed
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


def _logits(st, cfg):
    import torch
    lg = np.zeros((st.batch, cfg.vocab), np.float32)
    st.readout(lg)
    torch.cuda.synchronize()
    return lg


STARTS = {0: [0, 9], 1: [0, 4, 17], 2: [0]}      # row -> columns where documents start
RLT2_SCHEDULE_GAP = TOL_BF16 / 3


@pytest.mark.parametrize("name", ["tiny_fp32", "parity_bf16", "rlt2_mod5_bf16"])
def test_packed_rows_equal_their_last_document_alone(sd, name):
    import torch
    cfg = ri.CONFIGS[name]
    B, n = 3, 26
    W = ri.generate_weights(cfg)
    model = sd.Model(ri.write_blob(cfg, W))
    toks = ri.make_tokens(cfg, B, n)
    starts = np.zeros((B, n), np.uint8)
    for b, cols in STARTS.items():
        starts[b, cols] = 1
    st = sd.State(model, B, n)
    st.prefill_packed(toks, starts)
    pe, pd = st.positions()
    want = [n - max(STARTS[b]) for b in range(B)]
    assert list(pe) == want and list(pd) == want
    lg = _logits(st, cfg)

    tol = tol_for(cfg)
    orc = RLTOracle(cfg, W, oracle_mode(cfg))
    for b in range(B):
        j = max(STARTS[b])
        alone = sd.State(model, 1, n)
        alone.encode(np.ascontiguousarray(toks[b:b + 1, j:]))
        alone.prefill(n - j)
        la = _logits(alone, cfg)[0]
        # RLT-2: the lone prefill runs whole chunks together, the packed one
        # meets chunks cut at document starts (rows at different positions);
        # the two schedules differ by rounding only, well inside the bf16
        # tolerance (the bound is a third of it)
        gap = float(np.max(np.abs(lg[b] - la)))
        print(f"{name} row {b}: packed vs alone max|dlogit| {gap:.3e}")
        assert gap <= (0 if cfg.variant != 2 else RLT2_SCHEDULE_GAP)
        ref = prefill_packed(orc, toks[b], starts[b].astype(bool))
        assert np.max(np.abs(lg[b] - orc.readout(ref))) <= tol
        alone.close()

    # device tokens: the same results, bit for bit
    st2 = sd.State(model, B, n)
    st2.prefill_packed(torch.from_numpy(toks).cuda(), starts)
    np.testing.assert_array_equal(_logits(st2, cfg), lg)
    st.check()
    st2.check()
    for s_ in (st, st2):
        s_.close()
    model.close()


def test_packed_continues_and_rejects(sd):
    cfg = ri.CONFIGS["tiny_fp32"]
    B, n = 2, 10
    model = sd.Model(ri.write_blob(cfg, ri.generate_weights(cfg)))
    toks = ri.make_tokens(cfg, B, 2 * n)
    # a row without a start at column 0 continues its current document
    st = sd.State(model, B, 2 * n)
    first = np.zeros((B, n), np.uint8)
    first[:, 0] = 1
    st.prefill_packed(np.ascontiguousarray(toks[:, :n]), first)
    st.prefill_packed(np.ascontiguousarray(toks[:, n:]), np.zeros((B, n), np.uint8))
    whole = sd.State(model, B, 2 * n)
    whole.encode(toks)
    whole.prefill(2 * n)
    np.testing.assert_array_equal(_logits(st, cfg), _logits(whole, cfg))
    # errors, checked before anything runs
    short = sd.State(model, B, n)
    with pytest.raises(sd.RLTError) as e:
        short.prefill_packed(np.ascontiguousarray(toks[:, :n + 1]), np.zeros((B, n + 1), np.uint8))
    assert e.value.code == sd.RLT_E_CAPACITY
    bad = np.full((B, 3), cfg.vocab, np.int32)
    assert sd.rlt_prefill_packed(short.handle, bad, np.zeros((B, 3), np.uint8), 3) == sd.RLT_E_ARG
    import torch
    dev_starts = torch.zeros((B, 3), dtype=torch.uint8, device="cuda")   # must be host memory
    assert sd.rlt_prefill_packed(short.handle, np.ascontiguousarray(toks[:, :3]), dev_starts,
                                 3) == sd.RLT_E_ARG
    short.encode(np.ascontiguousarray(toks[:, :1]))
    with pytest.raises(sd.RLTError) as e:
        short.prefill_packed(np.ascontiguousarray(toks[:, :2]), np.zeros((B, 2), np.uint8))
    assert e.value.code == sd.RLT_E_ORDER
    pe, pd = short.positions()
    assert list(pe) == [1, 1] and list(pd) == [0, 0]
    for s_ in (st, whole, short):
        s_.check()
        s_.close()
    model.close()

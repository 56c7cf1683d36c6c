"""rlt_readout_rows: reading out state vectors the caller supplies, with no
device allocation inside the call.

Who needs it: a serving process that scores exported or candidate state
vectors while its memory pool already holds the rest of the device (a
cudaMalloc there fails or forces an eviction), or while other streams run
(cudaMalloc and cudaFree can synchronise the device and stall them).  The
call therefore works out of a fixed file-scope device array instead of
allocating.

Checked here against rlt_readout on the same s_t, two calls in a row (they
share the one array), with device and host outputs, for both dtypes; the
device's free memory is the same before and after a call; oversize requests
and bad arguments are rejected.  The file name sorts last, so a run that
stops at the first failure has run every other test before this one; it
also passes alone in a fresh process.
"""
import numpy as np
import pytest

import rlt_inputs as ri

pytestmark = pytest.mark.gpu

TOL = 1e-6      # same kernels on the same inputs: equal in practice


@pytest.fixture(scope="module")
def sd():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tests.conftest import build_library
    build_library()
    import stateful_decoding_b200 as sd
    return sd


@pytest.mark.parametrize("name,B,T", [("parity_bf16", 7, 20), ("tiny_fp32", 3, 9)])
def test_readout_rows_matches_readout(sd, name, B, T):
    import torch
    cfg = ri.CONFIGS[name]
    W = ri.generate_weights(cfg)
    model = sd.Model(ri.write_blob(cfg, W))
    st = sd.State(model, B, T)
    st.encode(ri.make_tokens(cfg, B, T))
    st.prefill(T)
    seed, step, temp = ri.SAMPLE_SEED, 3, 0.8
    lg = np.zeros((B, cfg.vocab), np.float32)
    am = np.zeros(B, np.int32)
    sp = np.zeros(B, np.int32)
    st.readout(lg, am, sp, seed=seed, step=step, temperature=temp)
    torch.cuda.synchronize()
    s_rows = torch.from_numpy(st.read(sd.PART_S).view(np.float32).reshape(B, cfg.d).copy()).cuda()

    stream = torch.cuda.Stream()
    # every buffer exists before the calls, so that only the library could
    # change the device's free memory during one
    lg_d = torch.empty((B, cfg.vocab), device="cuda")
    am_d = torch.empty((B,), dtype=torch.int32, device="cuda")
    sp_d = torch.empty((B,), dtype=torch.int32, device="cuda")
    lg_h = np.empty((B, cfg.vocab), np.float32)
    am_h = np.empty(B, np.int32)
    sp_h = np.empty(B, np.int32)
    for call in range(2):          # two calls in a row reuse the one scratch
        # device outputs
        lg_d.fill_(float("nan"))
        am_d.fill_(-1)
        sp_d.fill_(-1)
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        model.readout_rows(s_rows, lg_d, am_d, sp_d, seed=seed, step=step, temperature=temp,
                           stream=stream)
        stream.synchronize()
        free1 = torch.cuda.mem_get_info()[0]
        if call == 1:               # the first call may load the module on this device
            assert free1 == free0, f"device free memory moved by {free0 - free1} bytes"
        np.testing.assert_allclose(lg_d.cpu().numpy(), lg, atol=TOL, rtol=0)
        np.testing.assert_array_equal(am_d.cpu().numpy(), am)
        np.testing.assert_array_equal(sp_d.cpu().numpy(), sp)
        # host outputs: logits and ids pass through the scratch, valid on return
        lg_h.fill(np.nan)
        am_h.fill(-1)
        sp_h.fill(-1)
        free0 = torch.cuda.mem_get_info()[0]
        model.readout_rows(s_rows, lg_h, am_h, sp_h, seed=seed, step=step, temperature=temp,
                           stream=stream)
        free1 = torch.cuda.mem_get_info()[0]
        assert free1 == free0, f"device free memory moved by {free0 - free1} bytes"
        np.testing.assert_allclose(lg_h, lg, atol=TOL, rtol=0)
        np.testing.assert_array_equal(am_h, am)
        np.testing.assert_array_equal(sp_h, sp)
    st.close()
    model.close()


def test_readout_rows_rejects_oversize_and_bad_args(sd):
    import torch
    cfg = ri.CONFIGS["parity_bf16"]
    model = sd.Model(ri.write_blob(cfg, ri.generate_weights(cfg)))
    limit = sd.READOUT_ROWS_SCRATCH_BYTES
    fits = max(r for r in range(15000, 17000)
               if sd.readout_rows_scratch_bytes(r, cfg.d, cfg.vocab, True, False) <= limit)
    s_big = torch.zeros(fits + 1, cfg.d, device="cuda")
    am = torch.empty(fits + 1, dtype=torch.int32, device="cuda")
    lg = torch.empty(fits + 1, cfg.vocab, device="cuda")
    with pytest.raises(ValueError, match="static scratch"):
        model.readout_rows(s_big, lg, am)
    # the largest request that fits runs
    model.readout_rows(s_big[:fits], lg[:fits], am[:fits])
    torch.cuda.synchronize()
    assert (am[:fits].cpu().numpy() >= 0).all()
    # host input, non-positive temperature
    code = sd.rlt_readout_rows(model.handle, np.zeros((2, cfg.d), np.float32), 2, None, None,
                               None)
    assert code == sd.RLT_E_ARG
    code = sd.rlt_readout_rows(model.handle, s_big, 2, None, am, None, 0, 0, 0.0)
    assert code == sd.RLT_E_ARG
    assert sd.rlt_readout_rows(model.handle, s_big, 0) == 0
    model.close()

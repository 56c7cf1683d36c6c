"""GPU parity: the CUDA library through its C ABI against the CPU oracle.

Same seeded weights and tokens on both sides.  Sizes span several tiles and
ragged tails; the bench launch configuration is checked at full size on
sampled rows.  Tolerances: |delta logit| <= 1e-4 (fp32 path vs fp64 oracle),
<= 3e-2 (bf16 path vs bf16-mirrored oracle); argmax / sampled ids exact up to
the tie rule of rlt_testlib.
"""
import numpy as np
import pytest

import rlt_inputs as ri
from oracle import RLTOracle
from tests.rlt_testlib import TOL_BF16, Tally, check_argmax, check_sample, oracle_mode, tol_for

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


def make(sd, cfg, batch, max_len, seed=ri.WEIGHT_SEED):
    W = ri.generate_weights(cfg, seed=seed)
    model = sd.Model(ri.write_blob(cfg, W, seed=seed))
    return W, model, sd.State(model, batch, max_len)


def readout_host(st, cfg, seed=0, step=0, temperature=1.0):
    B = st.batch
    lg = np.zeros((B, cfg.vocab), np.float32)
    am = np.zeros(B, np.int32)
    sp = np.zeros(B, np.int32)
    st.readout(lg, am, sp, seed=seed, step=step, temperature=temperature)
    import torch
    torch.cuda.synchronize()
    return lg, am, sp


def state_vec(st, part, B, d):
    return st.read(part).view(np.float32).reshape(B, d)


# ----------------------------------------------------------------------------
def run_stepwise_and_compare(sd, cfg, B, T, n_decode=0, temperature=1.0, seed_tok=ri.TOKEN_SEED):
    """Step the GPU one position at a time, read out after every position, and
    compare each row with the oracle; then generate n_decode sampled tokens
    (the oracle follows the GPU's sampled ids and checks each)."""
    tol = tol_for(cfg)
    W, model, st = make(sd, cfg, B, T + n_decode)
    toks = ri.make_tokens(cfg, B, T, seed=seed_tok)
    orc = RLTOracle(cfg, W, oracle_mode(cfg))
    exact = RLTOracle(cfg, W, "fp64")
    rows = [orc.new_state() for _ in range(B)]
    rows_x = [exact.new_state() for _ in range(B)]
    for b in range(B):
        orc.encode(rows[b], toks[b])
        exact.encode(rows_x[b], toks[b])
    st.encode(toks)
    tally = Tally()
    for t in range(1, T + 1):
        st.step()
        lg, am, _ = readout_host(st, cfg)
        for b in range(B):
            orc.transition(rows[b])
            exact.transition(rows_x[b])
            ol = orc.readout(rows[b])
            err = float(np.max(np.abs(lg[b] - ol)))
            tally.max_err = max(tally.max_err, err)
            tally.max_err_exact = max(tally.max_err_exact,
                                      float(np.max(np.abs(lg[b] - exact.readout(rows_x[b])))))
            assert err <= tol, f"row {b} t={t}: |dlogit| {err} > {tol}"
            check_argmax(int(am[b]), ol, tol, tally, f"row {b} t={t}")
    for k in range(n_decode):
        lg, am, sp = readout_host(st, cfg, seed=ri.SAMPLE_SEED, step=k, temperature=temperature)
        for b in range(B):
            ol = orc.readout(rows[b])
            u = ri.sample_uniform(ri.SAMPLE_SEED, b, k)
            check_sample(int(sp[b]), ol, u, temperature, tol, tally, f"row {b} decode {k}")
        st.encode(sp.reshape(B, 1).astype(np.int32))
        st.step()
        lg, _, _ = readout_host(st, cfg)
        for b in range(B):
            orc.encode(rows[b], [int(sp[b])])
            orc.transition(rows[b])
            err = float(np.max(np.abs(lg[b] - orc.readout(rows[b]))))
            tally.max_err = max(tally.max_err, err)
            assert err <= tol, f"row {b} decode {k}: |dlogit| {err} > {tol}"
    s_gpu = state_vec(st, sd.PART_S, B, cfg.d)
    for b in range(B):
        np.testing.assert_allclose(s_gpu[b], rows[b].s, atol=max(10 * tol, 1e-3), rtol=0)
    st.check()
    print(f"{cfg.name}: max|dlogit| vs mirrored {tally.max_err:.3e}, vs fp64 "
          f"{tally.max_err_exact:.3e}, argmax ties {tally.argmax_ties}, sample ties "
          f"{tally.sample_ties}")
    return tally


def test_tiny_fp32_full_workload(sd):
    """The tiny fp32 workload at full size: 2 rows x 16 tokens, 6 sampled."""
    cfg = ri.CONFIGS["tiny_fp32"]
    t = run_stepwise_and_compare(sd, cfg, cfg.batch, cfg.prompt, cfg.decode)
    assert t.argmax_ties == 0 and t.sample_ties == 0


def test_tiny_fp32_temperature_and_ragged(sd):
    cfg = ri.CONFIGS["tiny_fp32"].replace(window=3)
    run_stepwise_and_compare(sd, cfg, 5, 37, n_decode=4, temperature=0.7, seed_tok=11)


@pytest.mark.parametrize("name,B,T", [("parity_bf16", 3, 37), ("s5_bf16", 2, 37),
                                      ("rlt2_mod5_bf16", 3, 23)])
def test_bf16_configs_stepwise(sd, name, B, T):
    cfg = ri.CONFIGS[name]
    run_stepwise_and_compare(sd, cfg, B, T, n_decode=2)


@pytest.mark.parametrize("name,B,T", [("parity_bf16", 3, 70), ("s5_bf16", 3, 41),
                                      ("rlt2_mod5_bf16", 5, 23), ("tiny_fp32", 3, 29)])
def test_prefill_matches_oracle(sd, name, B, T):
    """rlt_prefill (chunked for RLT-2) against the oracle's token-by-token run."""
    cfg = ri.CONFIGS[name]
    tol = tol_for(cfg)
    W, model, st = make(sd, cfg, B, T)
    toks = ri.make_tokens(cfg, B, T)
    st.encode(toks)
    st.prefill(T)
    lg, am, _ = readout_host(st, cfg)
    orc = RLTOracle(cfg, W, oracle_mode(cfg))
    tally = Tally()
    for b in range(B):
        r = orc.new_state()
        orc.encode(r, toks[b])
        orc.prefill(r, T)
        ol = orc.readout(r)
        assert np.max(np.abs(lg[b] - ol)) <= tol
        check_argmax(int(am[b]), ol, tol, tally)
        if cfg.variant == 2:
            R_gpu = state_vec(st, sd.PART_R, B, cfg.d)[b]
            np.testing.assert_allclose(R_gpu, r.R, atol=max(10 * tol, 1e-3), rtol=0)


@pytest.mark.parametrize("chunk", [2, 3, 8, 16])
def test_rlt2_chunk_blocks_match_oracle(sd, chunk):
    """RLT-2 at other chunk sizes B_c (greeksharifa App. J.10): rlt_prefill
    runs each chunk as one block of B_c positions -- the multi-query tile
    products at d_h 64, one or two query rows per lane -- against the
    oracle's chunked run of the same
    blocks; logits, argmax and the held register R."""
    cfg = ri.CONFIGS["rlt2_mod5_bf16"].replace(name=f"rlt2_chunk{chunk}", chunk=chunk)
    B, T = 3, 40
    tol = tol_for(cfg)
    W, model, st = make(sd, cfg, B, T)
    toks = ri.make_tokens(cfg, B, T)
    st.encode(toks)
    st.prefill(T)
    lg, am, _ = readout_host(st, cfg)
    R_gpu = state_vec(st, sd.PART_R, B, cfg.d)
    orc = RLTOracle(cfg, W, oracle_mode(cfg))
    tally = Tally()
    for b in range(B):
        r = orc.new_state()
        orc.encode(r, toks[b])
        orc.prefill(r, T, chunked=True)
        ol = orc.readout(r)
        err = float(np.max(np.abs(lg[b] - ol)))
        assert err <= tol, f"chunk {chunk} row {b}: |dlogit| {err}"
        check_argmax(int(am[b]), ol, tol, tally, f"row {b}")
        rel = float(np.linalg.norm(R_gpu[b] - r.R) / np.linalg.norm(r.R))
        assert rel <= tol, f"chunk {chunk} row {b}: |dR|/|R| {rel}"
    st.check()
    st.close()
    model.close()


def test_large_config_slice(sd):
    """The large tied workload at full width (d=2048, 16 heads x 128, vocab
    32000, W=256) on a 2+2-layer slice, 2 rows x 12 tokens + 2 sampled."""
    cfg = ri.CONFIGS["large_bf16"].replace(n_enc=2, n_dec=2)
    run_stepwise_and_compare(sd, cfg, 2, 12, n_decode=2)


# ----------------------------------------------------------------------------
# identities the pages state, on the GPU path itself (bit-exact)
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("name", ["parity_bf16", "rlt2_mod5_bf16", "tiny_fp32"])
def test_serving_split_bitexact(sd, name):
    """Prop. 3.1: prefill of a prefix then token-by-token = one prefill."""
    cfg = ri.CONFIGS[name]
    B, T = 3, 21
    W, model, a = make(sd, cfg, B, T)
    b_ = sd.State(model, B, T)
    toks = ri.make_tokens(cfg, B, T)
    a.encode(toks)
    a.prefill(T)
    k = 9
    b_.encode(np.ascontiguousarray(toks[:, :k]))
    b_.prefill(k)
    for t in range(k, T):
        b_.encode(np.ascontiguousarray(toks[:, t:t + 1]))
        b_.step()
    la, _, _ = readout_host(a, cfg)
    lb, _, _ = readout_host(b_, cfg)
    if cfg.variant == 2:
        # RLT-2: the one-shot prefill runs whole chunks in one block while the
        # split schedule steps token by token, so the window attention folds
        # its keys in another order: equal up to rounding, which bf16 storage
        # amplifies to its noise floor (the bf16 tolerance)
        np.testing.assert_allclose(la, lb, atol=TOL_BF16, rtol=0)
    else:
        np.testing.assert_array_equal(la, lb)
        np.testing.assert_array_equal(a.read(sd.PART_S), b_.read(sd.PART_S))


def test_batch_independence_bitexact(sd):
    cfg = ri.CONFIGS["s5_bf16"]
    B, T = 6, 19
    W, model, big = make(sd, cfg, B, T)
    toks = ri.make_tokens(cfg, B, T)
    big.encode(toks)
    big.prefill(T)
    lbig, _, _ = readout_host(big, cfg)
    for r in (0, 4):
        one = sd.State(model, 1, T)
        one.encode(np.ascontiguousarray(toks[r:r + 1]))
        one.prefill(T)
        l1, _, _ = readout_host(one, cfg)
        np.testing.assert_array_equal(l1[0], lbig[r])


def test_batch_independence_across_gemm_tiles(sd):
    """A batch large enough for the wide GEMM tiles (M = 130 x 16 rows) against
    the same rows run alone (narrow tiles): bit-identical logits."""
    cfg = ri.CONFIGS["parity_bf16"]
    B, T = 130, 16
    W, model, big = make(sd, cfg, B, T)
    toks = ri.make_tokens(cfg, B, T)
    big.encode(toks)
    big.prefill(T)
    lbig, _, _ = readout_host(big, cfg)
    for r in (0, 129):
        one = sd.State(model, 1, T)
        one.encode(np.ascontiguousarray(toks[r:r + 1]))
        one.prefill(T)
        l1, _, _ = readout_host(one, cfg)
        np.testing.assert_array_equal(l1[0], lbig[r])


def test_causality_bitexact(sd):
    """Prop. B.1: tokens after t do not change the state at t."""
    cfg = ri.CONFIGS["parity_bf16"]
    B, T, t = 2, 24, 13
    W, model, a = make(sd, cfg, B, T)
    b_ = sd.State(model, B, T)
    toks = ri.make_tokens(cfg, B, T)
    alt = toks.copy()
    alt[:, t:] = 1 - np.minimum(alt[:, t:], 1)
    a.encode(toks)
    b_.encode(alt)
    a.prefill(t)
    b_.prefill(t)
    la, _, _ = readout_host(a, cfg)
    lb, _, _ = readout_host(b_, cfg)
    np.testing.assert_array_equal(la, lb)


def test_reset_rows_restarts_from_h0(sd):
    cfg = ri.CONFIGS["tiny_fp32"]
    B, T = 3, 10
    W, model, st = make(sd, cfg, B, 2 * T)
    toks = ri.make_tokens(cfg, B, T)
    st.encode(toks)
    st.prefill(T)
    ref, _, _ = readout_host(st, cfg)
    st.reset()
    st.encode(toks)
    st.prefill(T)
    again, _, _ = readout_host(st, cfg)
    np.testing.assert_array_equal(ref, again)
    st.reset(rows=[1])
    pe, pd = st.positions()
    assert list(pe) == [T, 0, T] and list(pd) == [T, 0, T]


def test_error_codes(sd):
    cfg = ri.CONFIGS["tiny_fp32"]
    W, model, st = make(sd, cfg, 2, 4)
    with pytest.raises(sd.RLTError) as e:
        st.step()
    assert e.value.code == sd.RLT_E_ORDER
    with pytest.raises(sd.RLTError) as e:
        st.encode(np.zeros((2, 5), np.int32))
    assert e.value.code == sd.RLT_E_CAPACITY
    with pytest.raises(sd.RLTError) as e:
        st.encode(np.full((2, 1), 99, np.int32))
    assert e.value.code == sd.RLT_E_ARG
    import torch
    bad = torch.full((2, 1), 99, dtype=torch.int32, device="cuda")
    st.encode(bad)                      # device tokens: the kernel flags the bad id
    with pytest.raises(sd.RLTError) as e:
        st.check()
    assert e.value.code == sd.RLT_E_ARG
    st.check()                          # the error word was cleared
    per_row, total = st.bytes()
    c = cfg
    want = 2 * 4 * ((c.n_enc + c.groups) * 4 * c.d + c.n_dec * (c.window - 1) * c.d) + 4 * c.d
    assert per_row == want             # eq. 3.3 terms, fp32 storage

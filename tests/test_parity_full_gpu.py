"""GPU parity at the sizes the benchmarks run, and on the paths only those
sizes reach, against the CPU oracle.

* Every d=512 bf16 workload at its full batch and length in the bench's
  launch configuration (one encode call, one prefill call): parity 256 x 256,
  S5 512 x 256 (its encoder runs in two 128-position blocks), RLT-2 1024 x 64
  (chunk blocks of 4); the oracle recomputes sampled rows spread over the
  batch and across 128-row GEMM tiles.
* The large tied model at full depth (24 + 24 layers, d 2048, 16 heads of 128,
  vocab 32000, W 256): 2 rows x (256-token prompt + 32 sampled tokens), so the
  encoder attention runs over several 64-key stages and the cross-attention
  over t up to 288 at d_h 128.
* RLT-0 (no feedback, greeksharifa "Recurrent Looped Transformer 요약 설명"
  §2.7) through rlt_prefill's 16-position blocks and replayed graphs, and
  one position at a time.
* A snapshot restored into another row of another state, continued through
  an appended turn and sampled generation, against the oracle's
  uninterrupted row (jiphyeonjeon review "Recurrent Looped Transformer"
  §6.5; greeksharifa App. E).

Tolerances: |delta logit| <= 3e-2 (bf16 path vs the bf16-mirrored oracle),
1e-4 (fp32 path vs the fp64 oracle); argmax and sampled ids exact up to the
tie rule of rlt_testlib; the state vector s within the same figure (3e-2,
or 1e-4 for fp32) relative in the Euclidean norm: the readout normalises s,
so this carries the logit tolerance over to the state.
"""
import numpy as np
import pytest

import rlt_inputs as ri
from oracle import RLTOracle
from tests.rlt_testlib import Tally, check_argmax, check_sample, oracle_mode, tol_for
from tests.test_parity_gpu import make, readout_host, run_stepwise_and_compare, state_vec

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


def check_state(s_gpu, s_orc, what, tol):
    rel = float(np.linalg.norm(s_gpu - s_orc) / np.linalg.norm(s_orc))
    assert rel <= tol, f"{what}: |ds| / |s| = {rel:.3e} > {tol}"
    return rel


# rows recomputed by the oracle: both ends, both sides of every 128-row tile
# boundary the batch has, and a spread in between
SAMPLED_ROWS = {
    "parity_bf16": [0, 1, 63, 64, 100, 127, 128, 129, 131, 170, 191, 200, 223, 250, 254, 255],
    "s5_bf16": [0, 127, 128, 255, 256, 383, 384, 511],
    "rlt2_mod5_bf16": [0, 1, 127, 128, 255, 256, 383, 511, 512, 640, 767, 768, 895, 896, 1022,
                       1023],
}


@pytest.mark.parametrize("name", ["parity_bf16", "s5_bf16", "rlt2_mod5_bf16"])
def test_full_size_bench_launch_sampled_rows(sd, name):
    """The workload at its full batch and length, one encode call and one
    prefill call on a stream of its own as the bench runs it (the prefill
    replays captured graphs of 16 transition blocks); sampled rows against
    the oracle."""
    import torch
    cfg = ri.CONFIGS[name]
    B, T = cfg.batch, cfg.prompt
    W, model, st = make(sd, cfg, B, T)
    toks = ri.make_tokens(cfg)
    stream = torch.cuda.Stream()
    st.encode(toks, stream=stream)
    st.prefill(T, stream=stream)
    stream.synchronize()
    lg, am, _ = readout_host(st, cfg)
    s_gpu = state_vec(st, sd.PART_S, B, cfg.d)
    R_gpu = state_vec(st, sd.PART_R, B, cfg.d)
    st.check()
    orc = RLTOracle(cfg, W, oracle_mode(cfg))
    tol = tol_for(cfg)
    tally = Tally()
    worst, worst_s = 0.0, 0.0
    for b in SAMPLED_ROWS[name]:
        r = orc.new_state()
        orc.encode(r, toks[b])
        orc.prefill(r, T, chunked=True)
        ol = orc.readout(r)
        err = float(np.max(np.abs(lg[b] - ol)))
        worst = max(worst, err)
        assert err <= tol, f"{name} row {b}: |dlogit| {err}"
        check_argmax(int(am[b]), ol, tol, tally, f"row {b}")
        worst_s = max(worst_s, check_state(s_gpu[b], r.s, f"{name} row {b} s", tol))
        if cfg.variant == 2:
            check_state(R_gpu[b], r.R, f"{name} row {b} R", tol)
    print(f"{name} {B}x{T}: max|dlogit| {worst:.3e}, max |ds|/|s| {worst_s:.3e}, "
          f"argmax ties {tally.argmax_ties}")
    st.close()
    model.close()


def test_encode_split_into_blocks(sd, monkeypatch):
    """One rlt_encode call split into several encoder blocks (RLT_MAX_ROWS
    bounds the rows of one block: 4 rows x 200 positions become blocks of 64
    positions), so later blocks attend over cache prefixes written by earlier
    blocks of the same call: equal, bit for bit, to the same call as one
    block, and to the oracle."""
    cfg = ri.CONFIGS["parity_bf16"]
    B, T = 4, 200
    W = ri.generate_weights(cfg)
    model = sd.Model(ri.write_blob(cfg, W))
    toks = ri.make_tokens(cfg, B, T)
    one = sd.State(model, B, T)
    monkeypatch.setenv("RLT_MAX_ROWS", "256")          # read when a state is created
    blocks = sd.State(model, B, T)
    monkeypatch.delenv("RLT_MAX_ROWS")
    for st in (one, blocks):
        st.encode(toks)
        st.prefill(T)
    l1, _, _ = readout_host(one, cfg)
    lb, _, _ = readout_host(blocks, cfg)
    np.testing.assert_array_equal(lb, l1)
    orc = RLTOracle(cfg, W, "bf16")
    for b in (0, B - 1):
        r = orc.new_state()
        orc.encode(r, toks[b])
        orc.prefill(r, T)
        assert np.max(np.abs(lb[b] - orc.readout(r))) <= tol_for(cfg)
    for st in (one, blocks):
        st.check()
        st.close()
    model.close()


@pytest.mark.parametrize("name,B,T", [("rlt2_mod5_bf16", 300, 12), ("parity_bf16", 1030, 3)])
def test_many_row_products_match_rows_alone(sd, name, B, T):
    """From 1024 rows on, a split product keeps its split runs in one CTA's
    tensor memory and adds them in run order in its epilogue; below, the runs
    are separate CTAs whose slabs the consumer adds.  The two must agree bit
    for bit: rows of a big batch (RLT-2 chunks of 4 -> 1200 rows per product;
    RLT-1, 1030 rows) against the same rows run alone."""
    cfg = ri.CONFIGS[name]
    W, model, big = make(sd, cfg, B, T)
    toks = ri.make_tokens(cfg, B, T)
    big.encode(toks)
    big.prefill(T)
    lbig, _, _ = readout_host(big, cfg)
    for r in (0, B - 1):
        one = sd.State(model, 1, T)
        one.encode(np.ascontiguousarray(toks[r:r + 1]))
        one.prefill(T)
        l1, _, _ = readout_host(one, cfg)
        np.testing.assert_array_equal(l1[0], lbig[r])
        one.close()
    big.check()
    big.close()
    model.close()


def test_rope_scatter_epilogue_wide_heads(sd):
    """From 2048 rows on, the encoder's q|k|v and memory products apply RoPE
    and scatter into the caches in the GEMM epilogue; below, a row kernel
    does it from the stored product.  At d_h 128 (the large model's width on
    a 2 + 2 layer slice, 8 rows x 256 positions = 2048 rows per product) the
    two must agree bit for bit, and the big batch must match the oracle."""
    cfg = ri.CONFIGS["large_bf16"].replace(n_enc=2, n_dec=2)
    B, T = 8, 256
    W, model, big = make(sd, cfg, B, T)
    toks = ri.make_tokens(cfg, B, T)
    big.encode(toks)
    big.prefill(T)
    lbig, _, _ = readout_host(big, cfg)
    for r in (0, B - 1):
        one = sd.State(model, 1, T)
        one.encode(np.ascontiguousarray(toks[r:r + 1]))
        one.prefill(T)
        l1, _, _ = readout_host(one, cfg)
        np.testing.assert_array_equal(l1[0], lbig[r])
        one.close()
    orc = RLTOracle(cfg, W, oracle_mode(cfg))
    r = orc.new_state()
    orc.encode(r, toks[3])
    orc.prefill(r, T)
    err = float(np.max(np.abs(lbig[3] - orc.readout(r))))
    assert err <= tol_for(cfg), f"row 3: |dlogit| {err}"
    big.check()
    big.close()
    model.close()


def test_large_full_depth_prompt_and_sampled_generation(sd):
    """large_bf16 at full depth on 2 rows: a 256-token prompt encoded and
    prefilled in one call each, then 32 tokens sampled one at a time and fed
    back (the oracle follows the GPU's ids); every readout compared.

    Through 48 bf16 layers the mirrored oracle is itself chaotic at the level
    of single rounding flips: a second mirror whose embeddings are nudged by a
    relative 1e-6 (a perturbation the size of fp32 summation-order noise)
    moves its logits by a floor of ~2-3e-2, the size of the 3e-2 bar.  So
    each readout must agree within max(3e-2, 2 x that floor), measured at the
    same readout; the worst gap and the floors are printed."""
    import torch
    cfg = ri.CONFIGS["large_bf16"]
    B, T, G = 2, 256, 32
    W, model, st = make(sd, cfg, B, T + G)
    toks = ri.make_tokens(cfg, B, T)
    st.encode(toks)
    st.prefill(T)
    Wn = dict(W)
    Wn["embed"] = W["embed"].astype(np.float64) * (1.0 + 1e-6)
    orc, nud = RLTOracle(cfg, W, "bf16"), RLTOracle(cfg, Wn, "bf16")
    rows, rows_n = [], []
    for b in range(B):
        for o, lst in ((orc, rows), (nud, rows_n)):
            r = o.new_state()
            o.encode(r, toks[b])
            o.prefill(r, T)
            lst.append(r)
    tally = Tally()
    tol = tol_for(cfg)
    gaps, floors = [], []
    temp = 1.0
    for k in range(G + 1):
        lg, am, sp = readout_host(st, cfg, seed=ri.SAMPLE_SEED, step=k, temperature=temp)
        for b in range(B):
            ol = orc.readout(rows[b])
            floor = float(np.max(np.abs(nud.readout(rows_n[b]) - ol)))
            err = float(np.max(np.abs(lg[b] - ol)))
            gaps.append(err)
            floors.append(floor)
            bound = max(tol, 2.0 * floor)
            assert err <= bound, f"row {b} t={T + k}: |dlogit| {err} > {bound} (floor {floor})"
            check_argmax(int(am[b]), ol, bound, tally, f"row {b} t={T + k}")
            check_sample(int(sp[b]), ol, ri.sample_uniform(ri.SAMPLE_SEED, b, k), temp, bound,
                         tally, f"row {b} t={T + k}")
        if k == G:
            break
        st.encode(torch.from_numpy(sp.reshape(B, 1)).cuda())
        st.step()
        for b in range(B):
            for o, lst in ((orc, rows), (nud, rows_n)):
                o.encode(lst[b], [int(sp[b])])
                o.transition(lst[b])
    s_gpu = state_vec(st, sd.PART_S, B, cfg.d)
    rel = max(check_state(s_gpu[b], rows[b].s, f"row {b} s", tol) for b in range(B))
    st.check()
    g, f = np.array(gaps), np.array(floors)
    print(f"large_bf16 24+24, 2 x (256 + 32): GPU vs mirror max|dlogit| {g.max():.3e} "
          f"(median {np.median(g):.3e}, {int((g > tol).sum())} of {g.size} readouts above "
          f"{tol}); mirror floor max {f.max():.3e} median {np.median(f):.3e}; worst gap/floor "
          f"{(g / np.maximum(f, 1e-12)).max():.2f}; |ds|/|s| {rel:.3e}; argmax ties "
          f"{tally.argmax_ties}, sample ties {tally.sample_ties}")
    st.close()
    model.close()


def _rlt0(name):
    base = ri.CONFIGS[name]
    return base.replace(name=f"rlt0_{name}", variant=0)


@pytest.mark.parametrize("name,B,T", [("parity_bf16", 3, 290), ("tiny_fp32", 2, 45)])
def test_rlt0_prefill_blocks_against_oracle(sd, name, B, T):
    """RLT-0 prefill: blocks of 16 positions per pass (16 such blocks replayed
    as one graph when the prefill is long enough, then the ragged rest),
    against the oracle's token-by-token run."""
    cfg = _rlt0(name)
    tol = tol_for(cfg)
    W, model, st = make(sd, cfg, B, T)
    toks = ri.make_tokens(cfg, B, T)
    st.encode(toks)
    st.prefill(T)
    lg, am, _ = readout_host(st, cfg)
    s_gpu = state_vec(st, sd.PART_S, B, cfg.d)
    st.check()
    orc = RLTOracle(cfg, W, oracle_mode(cfg))
    tally = Tally()
    for b in range(B):
        r = orc.new_state()
        orc.encode(r, toks[b])
        orc.prefill(r, T)
        ol = orc.readout(r)
        err = float(np.max(np.abs(lg[b] - ol)))
        assert err <= tol, f"row {b}: |dlogit| {err}"
        check_argmax(int(am[b]), ol, tol, tally, f"row {b}")
        check_state(s_gpu[b], r.s, f"row {b} s", tol)
    st.close()
    model.close()


def test_rlt0_stepwise_against_oracle(sd):
    """RLT-0 one position at a time (rlt_step), with sampled continuations."""
    run_stepwise_and_compare(sd, _rlt0("parity_bf16"), 3, 21, n_decode=2)


@pytest.mark.parametrize("name", ["parity_bf16", "rlt2_mod5_bf16", "tiny_fp32"])
def test_snapshot_continuation_matches_oracle(sd, name):
    """Rows saved after a prefix with encoded-but-unconsumed positions,
    restored swapped into a state of another capacity that was running other
    sequences, then continued through the next turn and sampled generation:
    each must match the oracle's uninterrupted run of the original row."""
    import torch
    cfg = ri.CONFIGS[name]
    tol = tol_for(cfg)
    B, T, P, Pd, gen, temp = 2, 30, 17, 13, 3, 0.9
    W, model, a = make(sd, cfg, B, T)
    toks = ri.make_tokens(cfg, B, T)
    a.encode(np.ascontiguousarray(toks[:, :P]))
    a.prefill(Pd)
    snaps = [a.save(r) for r in range(B)]
    # b: another capacity, other sequences in flight; a's row 1 goes to b's
    # row 0 and a's row 0 to b's row 1
    b_ = sd.State(model, B, T + gen + 7)
    other = ri.make_tokens(cfg, B, 6, seed=ri.TOKEN_SEED + 5)
    b_.encode(other)
    b_.prefill(4)
    src = [1, 0]
    for i in range(B):
        b_.load(i, snaps[src[i]])
    b_.encode(np.ascontiguousarray(toks[src, P:]))
    b_.prefill(T - Pd)
    orc = RLTOracle(cfg, W, oracle_mode(cfg))
    rows = []
    for i in range(B):
        # the same encode calls as the GPU's (the bf16 mirror's attention
        # rounding follows the call size), uninterrupted by any snapshot
        r = orc.new_state()
        orc.encode(r, toks[src[i], :P])
        orc.encode(r, toks[src[i], P:])
        orc.prefill(r, T, chunked=True)
        rows.append(r)
    tally = Tally()
    for k in range(gen + 1):
        lg, am, sp = readout_host(b_, cfg, seed=ri.SAMPLE_SEED, step=k, temperature=temp)
        for i in range(B):
            ol = orc.readout(rows[i])
            err = float(np.max(np.abs(lg[i] - ol)))
            assert err <= tol, f"row {i} step {k}: |dlogit| {err}"
            check_argmax(int(am[i]), ol, tol, tally, f"row {i} step {k}")
            check_sample(int(sp[i]), ol, ri.sample_uniform(ri.SAMPLE_SEED, i, k), temp, tol,
                         tally, f"row {i} step {k}")
        if k == gen:
            break
        b_.encode(torch.from_numpy(sp.reshape(B, 1)).cuda())
        b_.step()
        for i in range(B):
            orc.encode(rows[i], [int(sp[i])])
            orc.transition(rows[i])
    s_gpu = state_vec(b_, sd.PART_S, B, cfg.d)
    for i in range(B):
        check_state(s_gpu[i], rows[i].s, f"row {i} s", tol)
    b_.check()
    for s_ in (a, b_):
        s_.close()
    model.close()

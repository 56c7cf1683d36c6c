"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: an identity
the pages state (serving-split invariance, causality, encoder schedules,
B=1 RLT-2 = RLT-1), an independent formulation written here (masked parallel
passes, full-history windows), a closed form (saturated gates, single keys,
W=1), a number printed on the pages (parameter counts, init loss) or a library
routine (torch's bf16 cast, scipy's softmax).
"""
import json
import math
import os

import numpy as np
import pytest

import rlt_inputs as ri
from oracle import RLTOracle, argmax_lowest, attend, rmsnorm, rope, round_bf16
from oracle.rlt_oracle import (log_softmax_at, prefill_packed, replay_logprobs, run_sequence,
                               sample_inverse_cdf, softmax)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def small_cfg(**kw):
    base = dict(name="pin", vocab=11, d=32, heads=4, n_enc=2, n_dec=2, ffn=48, window=3,
                groups=1, dtype=ri.DT_F32, batch=1, prompt=9)
    base.update(kw)
    c = ri.RLTConfig(**base)
    c.validate()
    return c


def weights(cfg, seed=7, std=0.2):
    """Seeded weights with a larger std than the workloads' 0.02, and gains and
    the gate bias drawn away from 1 and 0, so that every term and every norm's
    own gain is visible in the outputs."""
    W = ri.generate_weights(cfg, seed=seed, std=std)
    rng = np.random.default_rng(seed)
    for k in W:
        if k.endswith("norm"):
            W[k] = (1.0 + 0.3 * rng.standard_normal(W[k].shape)).astype(np.float32)
        elif k == "merge.bg":
            W[k] = (0.5 * rng.standard_normal(W[k].shape)).astype(np.float32)
    return W


def toks(cfg, n, seed=3):
    return ri.make_tokens(cfg.replace(token_recipe="uniform"), 1, n, seed=seed)[0]


def logits_token_by_token(m, tokens):
    st = m.new_state()
    out = []
    for x in tokens:
        m.encode(st, [x])
        m.transition(st)
        out.append(m.readout(st))
    return np.array(out), st


def logits_parallel_then_prefill(m, tokens, k):
    """Encode the first k tokens in one block, prefill them, then go token by token."""
    st = m.new_state()
    out = []
    m.encode(st, tokens[:k])
    for _ in range(k):
        m.transition(st)
        out.append(m.readout(st))
    for x in tokens[k:]:
        m.encode(st, [x])
        m.transition(st)
        out.append(m.readout(st))
    return np.array(out), st


# ----------------------------------------------------------------------------
# input generator
# ----------------------------------------------------------------------------


def test_splitmix64_published_outputs():
    g = json.load(open(os.path.join(GOLDEN, "splitmix64.json")))
    want = [int(h, 16) for h in g["first_outputs_hex"]]
    assert ri.splitmix64_stream_int(g["seed"], 3) == want
    assert [int(x) for x in ri.splitmix64_stream(g["seed"], 0, 3)] == want


def test_token_recipes_follow_the_documented_structure():
    """The synthetic token streams that stand in for the pages' task suites
    have the structure the workload table documents, and a row's tokens do
    not depend on the batch it is drawn in."""
    C = ri.CONFIGS
    sizes = {n: (c.batch, c.prompt, c.decode) for n, c in C.items()}
    assert sizes == {"tiny_fp32": (2, 16, 6), "parity_bf16": (256, 256, 0),
                     "s5_bf16": (512, 256, 0), "rlt2_mod5_bf16": (1024, 64, 0),
                     "large_bf16": (64, 4096, 512)}
    x = ri.make_tokens(C["parity_bf16"])                   # [BOS=2, bits, SEP=3]
    assert x.dtype == np.int32 and x.shape == (256, 256)
    assert (x[:, 0] == 2).all() and (x[:, -1] == 3).all()
    bits = x[:, 1:-1]
    assert set(np.unique(bits)) == {0, 1} and abs(bits.mean() - 0.5) < 0.01
    x = ri.make_tokens(C["s5_bf16"])                       # [BOS=11, ops 0..10]
    assert (x[:, 0] == 11).all() and x[:, 1:].min() == 0 and x[:, 1:].max() == 10
    counts = np.bincount(x[:, 1:].ravel(), minlength=11)
    assert counts.min() > 0.9 * counts.mean()
    x = ri.make_tokens(C["rlt2_mod5_bf16"])                # BOS=9, digit, op, ..., '=', digit
    assert (x[:, 0] == 9).all() and (x[:, -2] == 8).all()
    digits = x[:, 1:-2:2]
    ops = x[:, 2:-2:2]
    assert digits.min() == 0 and digits.max() == 4 and ops.min() == 5 and ops.max() == 7
    assert x[:, -1].max() <= 4
    big = C["large_bf16"]
    x = ri.make_tokens(big, 8, 4096)                       # BOS=0, then Zipf(1.1) over 1..V-1
    assert (x[:, 0] == 0).all() and x[:, 1:].min() >= 1 and x[:, 1:].max() < big.vocab
    f = np.bincount(x[:, 1:].ravel(), minlength=big.vocab)
    assert f[1] > f[2] > f[3] > f[10]
    assert abs(f[1] / f[2] - 2 ** 1.1) < 0.15               # rank-frequency slope
    x = ri.make_tokens(C["tiny_fp32"], 4, 50)
    assert x.min() >= 0 and x.max() < 32
    for name in C:                                          # rows independent of the batch
        a = ri.make_tokens(C[name], 5, 12)
        b = ri.make_tokens(C[name], 1, 12, row0=3)
        np.testing.assert_array_equal(a[3], b[0])


def test_box_muller_moments():
    z = ri.normal(123, 200000, 1.0)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1.0) < 0.01
    assert abs(np.mean(z ** 4) - 3.0) < 0.05            # Gaussian kurtosis


def test_normal_draws_by_range_and_threads():
    """Draw i of a stream uses its outputs 2i+1, 2i+2: any range of draws
    equals the same slice of the whole stream, and weights generated in
    pieces on a thread pool equal the single-thread ones bit for bit."""
    z = ri.normal(77, 1000, 0.5)
    for i0, i1 in ((0, 1), (3, 500), (999, 1000)):
        np.testing.assert_array_equal(ri.normal(77, i1 - i0, 0.5, start=i0), z[i0:i1])
    # the first draw from its published definition: SplitMix64 outputs 1 and 2
    o1, o2 = ri.splitmix64_stream_int(77, 2)
    u1 = ((o1 >> 11) + 1) / 9007199254740992.0
    u2 = (o2 >> 11) / 9007199254740992.0
    assert z[0] == 0.5 * np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)
    cfg = ri.CONFIGS["parity_bf16"].replace(vocab=50)
    old = ri._GEN_CHUNK
    try:
        ri._GEN_CHUNK = 1000                    # many pieces per tensor
        a = ri.generate_weights(cfg, threads=8)
    finally:
        ri._GEN_CHUNK = old
    b = ri.generate_weights(cfg, threads=1)
    for k in b:
        np.testing.assert_array_equal(a[k], b[k])


def test_blob_roundtrip_and_checksum():
    for name in ("tiny_fp32", "rlt2_mod5_bf16"):
        cfg = ri.CONFIGS[name].replace(d=32, heads=4, ffn=40, vocab=10)
        W = ri.generate_weights(cfg, seed=9)
        blob = ri.write_blob(cfg, W)
        cfg2, W2 = ri.read_blob(blob)
        assert cfg2.d == cfg.d and cfg2.variant == cfg.variant and cfg2.chunk == cfg.chunk
        for k in W:
            np.testing.assert_array_equal(W[k], W2[k])
        bad = bytearray(blob)
        bad[-70] ^= 1
        with pytest.raises(AssertionError):
            ri.read_blob(bytes(bad))


# ----------------------------------------------------------------------------
# parameter counts printed on the pages
# ----------------------------------------------------------------------------


def _paper_cfg(ne, nd, variant=1, vocab=16):
    return ri.RLTConfig("p", vocab=vocab, d=512, heads=4, n_enc=ne, n_dec=nd, ffn=1365, window=8,
                        groups=1, variant=variant)


def test_merge_block_parameter_count():
    g = json.load(open(os.path.join(GOLDEN, "pages_numbers.json")))
    want = g["merge_block_params_d512"]["value"]
    c1, c0 = _paper_cfg(4, 4, 1), _paper_cfg(4, 4, 0)
    assert ri.param_count(c1) - ri.param_count(c0) == want


def test_layer_split_parameter_deltas():
    """Successive RLT-1 splits 4+4 .. 8+0 differ as the pages print (to 0.01M):
    a decoder block carries cross-attention (2 d^2) and one norm more than an
    encoder block, and 8+0 also drops the memory projection."""
    g = json.load(open(os.path.join(GOLDEN, "pages_numbers.json")))["rlt1_params_8layer_M"]
    splits = ["4+4", "5+3", "6+2", "7+1", "8+0"]
    counts = {s: ri.param_count(_paper_cfg(int(s[0]), int(s[2]))) for s in splits}
    for a, b in zip(splits, splits[1:]):
        ours = (counts[a] - counts[b]) / 1e6
        paper = g["value"][a] - g["value"][b]
        assert abs(ours - paper) <= 2 * g["rounding"] + 1e-9, (a, b, ours, paper)


def _no_vocab_count(cfg):
    """Parameters outside the vocabulary matrices (embedding and readout)."""
    return ri.param_count(cfg) - 2 * cfg.vocab * cfg.d


def test_printed_totals_share_one_constant():
    """Every total the pages print -- RLT-0 4+4 exactly, the five RLT-1 splits
    and the GPT Layer 8 baseline to 0.01M -- equals our count of the layers,
    memory and merge plus one constant C shared by all of them (the
    vocabulary matrices and whatever else the pages' model carries outside
    the layers).  GPT Layer 8 has the shape of RLT-0 8+0 in our manifest
    (eight causal self-attention + FFN blocks, no memory, no merge), so its
    printed count checks the decoder's cross-attention and memory terms
    against a model without them."""
    g = json.load(open(os.path.join(GOLDEN, "pages_numbers.json")))
    C = g["rlt0_params_4p4"]["value"] - _no_vocab_count(_paper_cfg(4, 4, 0))
    r1 = g["rlt1_params_8layer_M"]
    for split, want in r1["value"].items():
        ours = (_no_vocab_count(_paper_cfg(int(split[0]), int(split[2]))) + C) / 1e6
        assert abs(ours - want) <= r1["rounding"] + 1e-9, (split, ours, want)
    gpt = g["gpt8_params_M"]
    ours = (_no_vocab_count(_paper_cfg(8, 0, 0)) + C) / 1e6
    assert abs(ours - gpt["value"]) <= gpt["rounding"] + 1e-9, ours
    # the constant is not a whole number of untied (or tied) vocabulary rows
    # of width 512: 1024 * 141 + 128 -- the departure the readings record
    assert C == 144512 and C % 512 == 128


# ----------------------------------------------------------------------------
# helpers: closed forms and library routines
# ----------------------------------------------------------------------------


def test_round_bf16_matches_torch():
    torch = pytest.importorskip("torch")
    x = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 3
    x = np.concatenate([x, np.float32([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.5 - 2 ** -9, 0.0])])
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(round_bf16(x.astype(np.float64)), want)
    assert round_bf16(np.float64(1.0 + 2 ** -8)) == 1.0            # tie goes to even
    assert round_bf16(np.float64(1.0 + 3 * 2 ** -8)) == 1.0 + 2 ** -6


def test_rmsnorm_closed_form():
    c, eps = -0.7, 1e-6
    x = np.full(10, c)
    g = np.arange(1, 11, dtype=np.float64)
    np.testing.assert_allclose(rmsnorm(x, g, eps), g * c / math.sqrt(c * c + eps), rtol=1e-14)


def test_rope_rotation_and_relative_position():
    rng = np.random.default_rng(1)
    # dh = 2: one pair, angle = pos * base^0 = pos radians
    v = np.array([[[1.0, 0.0]]])
    for p in (1, 2, 5):
        np.testing.assert_allclose(rope(v, np.array([p]), 10000.0)[0, 0],
                                   [math.cos(p), math.sin(p)], atol=1e-15)
    # second pair of dh=4 turns by pos / base^(1/2)
    v = np.array([[[0.0, 1.0, 0.0, 0.0]]])
    ang = 3 / 10000.0 ** 0.5
    np.testing.assert_allclose(rope(v, np.array([3]), 10000.0)[0, 0],
                               [0.0, math.cos(ang), 0.0, math.sin(ang)], atol=1e-15)
    q, k = rng.standard_normal((1, 2, 16)), rng.standard_normal((1, 2, 16))
    d1 = np.sum(rope(q, np.array([7]), 100.0) * rope(k, np.array([3]), 100.0))
    d2 = np.sum(rope(q, np.array([24]), 100.0) * rope(k, np.array([20]), 100.0))
    assert abs(d1 - d2) < 1e-12                                   # depends on m - n only
    np.testing.assert_allclose(np.linalg.norm(rope(q, np.array([9]), 100.0)), np.linalg.norm(q))


def test_attend_closed_forms_and_scipy():
    scipy_special = pytest.importorskip("scipy.special")
    rng = np.random.default_rng(2)
    q = rng.standard_normal((3, 8))
    V = rng.standard_normal((1, 3, 8))
    np.testing.assert_allclose(attend(q, rng.standard_normal((1, 3, 8)), V), V[0])
    K = np.repeat(rng.standard_normal((1, 3, 8)), 5, axis=0)
    V = rng.standard_normal((5, 3, 8))
    np.testing.assert_allclose(attend(q, K, V), V.mean(0), atol=1e-14)
    K, V = rng.standard_normal((6, 3, 8)), rng.standard_normal((6, 3, 8))
    p = scipy_special.softmax(np.einsum("hd,mhd->hm", q, K) / math.sqrt(8), axis=1)
    np.testing.assert_allclose(attend(q, K, V), np.einsum("hm,mhd->hd", p, V), atol=1e-14)


def test_sampling_inverse_cdf_brute_force():
    logits = np.log(np.array([0.1, 0.2, 0.3, 0.4]))
    edges = [0.1, 0.3, 0.6, 1.0]
    for u in np.linspace(0, 0.999, 97):
        if any(abs(u - e) < 1e-9 for e in edges):
            continue
        want = next(i for i, e in enumerate(edges) if e > u)
        assert sample_inverse_cdf(logits, u) == want
    # empirical frequencies over the shared uniforms
    us = [ri.sample_uniform(42, r, 0) for r in range(20000)]
    ids = np.array([sample_inverse_cdf(logits, u) for u in us])
    np.testing.assert_allclose(np.bincount(ids, minlength=4) / len(ids), [0.1, 0.2, 0.3, 0.4],
                               atol=0.015)
    assert argmax_lowest(np.array([1.0, 3.0, 3.0, 2.0])) == 1
    np.testing.assert_allclose(softmax(np.array([0.0, math.log(3.0)]), 1.0), [0.25, 0.75])
    # temperature 1/2 squares the probabilities: [1, 4, 9, 16] / 30
    edges = np.cumsum([1, 4, 9, 16]) / 30.0
    np.testing.assert_allclose(softmax(logits, 0.5), np.array([1, 4, 9, 16]) / 30.0, rtol=1e-12)
    for u in np.linspace(0, 0.999, 101):
        if np.min(np.abs(edges - u)) < 1e-9:
            continue
        assert sample_inverse_cdf(logits, u, 0.5) == int(np.searchsorted(edges, u, side="right"))


# ----------------------------------------------------------------------------
# identities the pages state
# ----------------------------------------------------------------------------


@pytest.mark.parametrize("variant,chunk", [(1, 1), (2, 3), (0, 1)])
@pytest.mark.parametrize("mode", ["fp64", "bf16"])
def test_serving_split_invariance(variant, chunk, mode):
    """Prop. 3.1 (jiphyeonjeon review §4.1): any prompt/response split gives the
    same states and next-token distributions."""
    cfg = small_cfg(variant=variant, chunk=chunk)
    m = RLTOracle(cfg, weights(cfg), mode=mode)
    x = toks(cfg, 9)
    ref, st_ref = logits_token_by_token(m, x)
    for k in range(0, len(x) + 1):
        got, st = logits_parallel_then_prefill(m, x, k)
        np.testing.assert_allclose(got, ref, atol=1e-12, rtol=0)
        np.testing.assert_allclose(st.s, st_ref.s, atol=1e-12, rtol=0)


def test_causality_future_tokens_do_not_change_earlier_logits():
    """Prop. B.1 (jiphyeonjeon review §4.1, App. B)."""
    cfg = small_cfg()
    m = RLTOracle(cfg, weights(cfg))
    x = toks(cfg, 9)
    base, _ = logits_parallel_then_prefill(m, x, len(x))
    for t in range(1, len(x)):
        y = x.copy()
        y[t:] = (y[t:] + 1 + np.arange(len(x) - t)) % cfg.vocab
        pert, _ = logits_parallel_then_prefill(m, y, len(y))
        np.testing.assert_allclose(pert[:t], base[:t], atol=1e-12, rtol=0)
        assert np.max(np.abs(pert[t:] - base[t:])) > 1e-6


def test_encoder_parallel_equals_stepwise_any_split():
    """Parallel encoding and E^step stepping are one causal computation
    (jiphyeonjeon review §3.2)."""
    cfg = small_cfg()
    m = RLTOracle(cfg, weights(cfg))
    x = toks(cfg, 10)
    st_a = m.new_state()
    m.encode(st_a, x)
    for splits in ([1] * 10, [3, 4, 3], [9, 1], [2, 8]):
        st_b = m.new_state()
        i = 0
        for n in splits:
            m.encode(st_b, x[i:i + n])
            i += n
        np.testing.assert_allclose(np.array(st_b.e), np.array(st_a.e), atol=1e-12, rtol=0)
        np.testing.assert_allclose(st_b.mem_k[0], st_a.mem_k[0], atol=1e-12, rtol=0)


def test_rlt2_with_chunk_one_is_rlt1():
    """B = 1 makes RLT-2 exactly RLT-1 (greeksharifa §2.7)."""
    c1 = small_cfg(variant=1)
    c2 = small_cfg(variant=2, chunk=1)
    W = weights(c1)
    x = toks(c1, 9)
    a, _ = logits_token_by_token(RLTOracle(c1, W), x)
    b, _ = logits_token_by_token(RLTOracle(c2, W), x)
    np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("chunk", [2, 4])
def test_rlt2_chunk_parallel_equals_token_by_token(chunk):
    """Chunk positions run together per layer with the held register
    (greeksharifa App. I.2) = token-by-token with the same register."""
    cfg = small_cfg(variant=2, chunk=chunk, window=3)
    m = RLTOracle(cfg, weights(cfg))
    x = toks(cfg, 11)
    st_a, st_b = m.new_state(), m.new_state()
    m.encode(st_a, x)
    m.encode(st_b, x)
    sa = m.prefill(st_a, len(x), chunked=False)
    sb = m.prefill(st_b, len(x), chunked=True)
    np.testing.assert_allclose(np.array(sb), np.array(sa), atol=1e-12, rtol=0)
    np.testing.assert_allclose(st_b.R, st_a.R, atol=1e-12, rtol=0)


def test_depth_counts():
    """Sequential decoder passes: T for RLT-1, ceil(T/B) for chunked RLT-2
    (greeksharifa §2.7, Table 1)."""
    cfg = small_cfg(variant=2, chunk=4)
    m = RLTOracle(cfg, weights(cfg))
    calls = []
    orig = m._dec_layer
    m._dec_layer = lambda st, l, z, pos: (calls.append(len(pos)) if l == 0 else None) or orig(st, l, z, pos)
    st = m.new_state()
    m.encode(st, toks(cfg, 10))
    m.prefill(st, 10, chunked=True)
    assert len(calls) == math.ceil(10 / 4) and sum(calls) == 10
    st = m.new_state()
    m.encode(st, toks(cfg, 10))
    calls.clear()
    m.prefill(st, 10, chunked=False)
    assert len(calls) == 10


# ----------------------------------------------------------------------------
# independent parallel formulation: RLT-0 as one masked pass per layer
# ----------------------------------------------------------------------------


def _rms(x, g, eps):
    return x / np.sqrt((x ** 2).mean(-1, keepdims=True) + eps) * g


def _rot(x, pos, base):
    T, h, dh = x.shape
    half = dh // 2
    freq = np.array([base ** (-(2.0 * i) / dh) for i in range(half)])
    out = np.empty_like(x)
    for t in range(T):
        for i in range(half):
            a = pos[t] * freq[i]
            ca, sa = math.cos(a), math.sin(a)
            out[t, :, i] = x[t, :, i] * ca - x[t, :, i + half] * sa
            out[t, :, i + half] = x[t, :, i + half] * ca + x[t, :, i] * sa
    return out


def _masked_attention(Q, K, V, mask):
    S = np.einsum("ihd,jhd->hij", Q, K) / math.sqrt(Q.shape[-1])
    S = np.where(mask[None], S, -np.inf)
    S = S - S.max(-1, keepdims=True)
    P = np.exp(S)
    P /= P.sum(-1, keepdims=True)
    return np.einsum("hij,jhd->ihd", P, V)


def parallel_teacher_forced(cfg, W, tokens, window=None):
    """Whole-sequence pass: causal encoder, memory, then (RLT-0) each decoder
    layer over all positions with a window mask and a prefix cross mask."""
    T, d, h = len(tokens), cfg.d, cfg.heads
    dh, eps, base = d // h, cfg.eps, cfg.rope_base
    pos = np.arange(1, T + 1)
    ii, jj = np.meshgrid(np.arange(T), np.arange(T), indexing="ij")
    causal = jj <= ii
    Wn = window if window is not None else cfg.window
    win = causal & (jj >= ii - Wn + 1)
    f64 = {k: v.astype(np.float64) for k, v in W.items()}
    E = lambda l, n: f64[(f"dec.{l}." if cfg.tied else f"enc.{l}.") + n]
    x = f64["embed"][tokens]
    for l in range(cfg.n_enc):
        y = _rms(x, f64[f"enc.{l}.attn_norm"], eps)
        Q = _rot((y @ E(l, "wq").T).reshape(T, h, dh), pos, base)
        K = _rot((y @ E(l, "wk").T).reshape(T, h, dh), pos, base)
        V = (y @ E(l, "wv").T).reshape(T, h, dh)
        x = x + _masked_attention(Q, K, V, causal).reshape(T, d) @ E(l, "wo").T
        y = _rms(x, f64[f"enc.{l}.ffn_norm"], eps)
        a1, a3 = y @ E(l, "w1").T, y @ E(l, "w3").T
        x = x + (a1 / (1 + np.exp(-a1)) * a3) @ E(l, "w2").T
    e = x.copy()
    nu = _rms(e, f64["mem_norm"], eps)
    mem = [(_rot((nu @ f64[f"mem.{g}.wk"].T).reshape(T, h, dh), pos, base),
            (nu @ f64[f"mem.{g}.wv"].T).reshape(T, h, dh)) for g in range(cfg.groups)]
    z = e.copy()
    for l in range(cfg.n_dec):
        p = f"dec.{l}."
        y = _rms(z, f64[p + "swa_norm"], eps)
        Q = _rot((y @ f64[p + "wq"].T).reshape(T, h, dh), pos, base)
        K = _rot((y @ f64[p + "wk"].T).reshape(T, h, dh), pos, base)
        V = (y @ f64[p + "wv"].T).reshape(T, h, dh)
        z = z + _masked_attention(Q, K, V, win).reshape(T, d) @ f64[p + "wo"].T
        y = _rms(z, f64[p + "x_norm"], eps)
        Qx = _rot((y @ f64[p + "xq"].T).reshape(T, h, dh), pos, base)
        mk, mv = mem[l if cfg.groups > 1 else 0]
        z = z + _masked_attention(Qx, mk, mv, causal).reshape(T, d) @ f64[p + "xo"].T
        y = _rms(z, f64[p + "ffn_norm"], eps)
        a1, a3 = y @ f64[p + "w1"].T, y @ f64[p + "w3"].T
        z = z + (a1 / (1 + np.exp(-a1)) * a3) @ f64[p + "w2"].T
    logits = _rms(z, f64["out_norm"], eps) @ f64["out"].T
    return e, z, logits


@pytest.mark.parametrize("window,groups,tied", [(3, 1, False), (1, 1, False), (100, 2, False),
                                                (4, 1, True)])
def test_rlt0_sequential_equals_parallel_pass(window, groups, tied):
    """RLT-0 has no feedback, so its T sequential transitions equal one masked
    parallel pass per decoder layer (greeksharifa §2.7, App. J.3)."""
    cfg = small_cfg(variant=0, window=window, groups=groups, tied=tied)
    W = weights(cfg)
    x = toks(cfg, 10)
    e_ref, z_ref, lg_ref = parallel_teacher_forced(cfg, W, x)
    got, st = logits_token_by_token(RLTOracle(cfg, W), x)
    np.testing.assert_allclose(np.array(st.e), e_ref, atol=1e-11, rtol=0)
    np.testing.assert_allclose(got, lg_ref, atol=1e-11, rtol=0)


def test_rlt0_chunked_block_equals_parallel_pass():
    cfg = small_cfg(variant=0, window=4)
    W = weights(cfg)
    x = toks(cfg, 10)
    _, z_ref, _ = parallel_teacher_forced(cfg, W, x)
    m = RLTOracle(cfg, W)
    st = m.new_state()
    m.encode(st, x)
    z = np.concatenate([m.transition_chunk(st, 6), m.transition_chunk(st, 4)])
    np.testing.assert_allclose(z, z_ref, atol=1e-11, rtol=0)


def test_alpha_zero_is_rlt0():
    """With alpha = 0 the merge returns e_t (greeksharifa §2.5 merge equations)."""
    c1 = small_cfg(variant=1, alpha=0.0)
    c0 = small_cfg(variant=0)
    W1 = weights(c1)
    W0 = {k: v for k, v in W1.items() if not (k.startswith("merge") or k == "s_star")}
    x = toks(c1, 8)
    a, _ = logits_token_by_token(RLTOracle(c1, W1), x)
    b, _ = logits_token_by_token(RLTOracle(c0, W0), x)
    np.testing.assert_allclose(a, b, atol=1e-13, rtol=0)


def test_window_at_least_T_is_full_causal_attention():
    """W >= T: nothing is evicted, so the window attention is full causal
    attention over decoder activations (jiphyeonjeon §3.3 retention rule)."""
    cfg = small_cfg(variant=0, window=50)
    W = weights(cfg)
    x = toks(cfg, 10)
    full = small_cfg(variant=0, window=10 ** 6)
    _, _, lg = parallel_teacher_forced(full, W, x, window=10 ** 6)
    got, _ = logits_token_by_token(RLTOracle(cfg, W), x)
    np.testing.assert_allclose(got, lg, atol=1e-11, rtol=0)


# ----------------------------------------------------------------------------
# closed forms with switched-off sub-layers
# ----------------------------------------------------------------------------


def _zero(W, cfg, names):
    W = {k: v.copy() for k, v in W.items()}
    for l in range(cfg.n_dec):
        for n in names:
            W[f"dec.{l}.{n}"][:] = 0
    return W


def test_merge_saturated_gate_recursion():
    """L_D = 0 makes s_t = u_t.  With W_g = 0 and b_g = +40 the gate is 1 and
    s_t = e_t + alpha W_s RMSNorm_s(s_{t-1}) from s_0 = s_star; with b_g = -40
    the gate closes and s_t = e_t (greeksharifa §2.5)."""
    cfg = small_cfg(n_dec=0, variant=1, alpha=0.3)
    W = weights(cfg)
    W["merge.wg"][:] = 0
    x = toks(cfg, 7)
    for bg, open_gate in ((40.0, True), (-40.0, False)):
        W["merge.bg"][:] = bg
        m = RLTOracle(cfg, W)
        st = m.new_state()
        e = m.encode(st, x)
        s = W["s_star"].astype(np.float64)
        for t in range(len(x)):
            r = s / np.sqrt(np.mean(s * s) + cfg.eps) * W["merge.norm"]
            s_want = e[t] + (cfg.alpha * (W["merge.ws"].astype(np.float64) @ r) if open_gate else 0)
            got = m.transition(st)
            np.testing.assert_allclose(got, s_want, atol=1e-12)
            s = s_want


def test_merge_gate_reads_e_then_r():
    """g = sigmoid(W_g [e_t; r] + b_g), u = e_t + alpha g (W_s r) (greeksharifa
    §2.5): the first d columns of W_g take e_t, the last d take r.  With the
    r-half zero the gate depends on e_t alone, so (u - e) : (W_s r) is one
    vector for every previous state; with the e-half zero, u - e does not
    change with e_t.  A swapped [r; e] fails both."""
    cfg = small_cfg(alpha=0.3)
    d = cfg.d
    W = weights(cfg)
    rng = np.random.default_rng(5)
    e1, e2 = rng.normal(size=(2, d))
    f1, f2 = rng.normal(size=(2, d))

    def with_half_zero(cols):
        Wz = dict(W)
        Wz["merge.wg"] = W["merge.wg"].copy()
        Wz["merge.wg"][:, cols] = 0
        return RLTOracle(cfg, Wz)

    ws = W["merge.ws"].astype(np.float64)
    wsr = lambda fb: ws @ rmsnorm(fb, W["merge.norm"].astype(np.float64), cfg.eps)  # noqa: E731
    m = with_half_zero(slice(d, 2 * d))             # gate from e_t only
    du1, du2 = m.merge(e1, f1)[0] - e1, m.merge(e1, f2)[0] - e1
    # du_k = alpha g(e1) * (W_s r_k): cross-multiplied, g(e1) cancels
    np.testing.assert_allclose(du1 * wsr(f2), du2 * wsr(f1), atol=1e-12, rtol=0)
    assert np.max(np.abs(m.merge(e2, f1)[0] - e2 - du1)) > 1e-3      # the gate does read e_t
    m = with_half_zero(slice(0, d))                 # gate from r only
    np.testing.assert_allclose(m.merge(e1, f1)[0] - e1, m.merge(e2, f1)[0] - e2, atol=1e-12,
                               rtol=0)
    assert np.max(np.abs(m.merge(e1, f1)[0] - m.merge(e1, f2)[0])) > 1e-3


def test_rlt2_register_timing_closed_form():
    """RLT-2 with L_D = 0 and an open gate: s_t = e_t + alpha W_s RMSNorm(R) where
    R = s at the last complete chunk end before t (s_star before the first)."""
    cfg = small_cfg(n_dec=0, variant=2, chunk=3, alpha=0.5)
    W = weights(cfg)
    W["merge.wg"][:] = 0
    W["merge.bg"][:] = 40.0
    m = RLTOracle(cfg, W)
    st = m.new_state()
    x = toks(cfg, 8)
    e = m.encode(st, x)
    R = W["s_star"].astype(np.float64)
    for t in range(1, 9):
        r = R / np.sqrt(np.mean(R * R) + cfg.eps) * W["merge.norm"]
        s = e[t - 1] + cfg.alpha * (W["merge.ws"].astype(np.float64) @ r)
        np.testing.assert_allclose(m.transition(st), s, atol=1e-12)
        if t % 3 == 0:
            R = s


def test_cross_attention_at_t1_reads_single_key():
    """At t = 1 the memory holds one key, so cross-attention returns v_1 and the
    block adds W_xo v_1 (prefix restriction, jiphyeonjeon §2)."""
    cfg = small_cfg(n_dec=1, variant=0)
    W = _zero(weights(cfg), cfg, ["wo", "w2"])
    m = RLTOracle(cfg, W)
    st = m.new_state()
    e = m.encode(st, toks(cfg, 4))
    s1 = m.transition(st)
    nu = e[0] / np.sqrt(np.mean(e[0] ** 2) + cfg.eps) * W["mem_norm"]
    v1 = W["mem.0.wv"].astype(np.float64) @ nu
    np.testing.assert_allclose(s1, e[0] + W["dec.0.xo"].astype(np.float64) @ v1, atol=1e-12)


def test_window_one_attends_only_current_token():
    """W = 1 keeps no cache: the window attention returns v_t at every t."""
    cfg = small_cfg(n_dec=1, variant=0, window=1)
    W = _zero(weights(cfg), cfg, ["xo", "w2"])
    m = RLTOracle(cfg, W)
    st = m.new_state()
    e = m.encode(st, toks(cfg, 6))
    for t in range(6):
        u = e[t]
        y = u / np.sqrt(np.mean(u ** 2) + cfg.eps) * W["dec.0.swa_norm"]
        want = u + W["dec.0.wo"].astype(np.float64) @ (W["dec.0.wv"].astype(np.float64) @ y)
        np.testing.assert_allclose(m.transition(st), want, atol=1e-12)
        assert len(st.swa[0]) == 0


def test_window_retention_and_full_history_reference():
    """Independent windowed decoder on a full history (no eviction) for RLT-1:
    position t attends t-W+1..t; the oracle's cache keeps at most W-1 entries."""
    cfg = small_cfg(variant=1, window=3, n_dec=1)
    W = weights(cfg)
    f = {k: v.astype(np.float64) for k, v in W.items()}
    x = toks(cfg, 9)
    m = RLTOracle(cfg, W)
    st = m.new_state()
    e = m.encode(st, x)
    h, dh = cfg.heads, cfg.d // cfg.heads
    s, Ks, Vs = f["s_star"], [], []
    mk = _rot((_rms(e, f["mem_norm"], cfg.eps) @ f["mem.0.wk"].T).reshape(-1, h, dh),
              np.arange(1, 10), cfg.rope_base)
    mv = (_rms(e, f["mem_norm"], cfg.eps) @ f["mem.0.wv"].T).reshape(-1, h, dh)
    for t in range(1, 10):
        r = _rms(s, f["merge.norm"], cfg.eps)
        gte = 1 / (1 + np.exp(-(f["merge.wg"] @ np.concatenate([e[t - 1], r]) + f["merge.bg"])))
        z = e[t - 1] + cfg.alpha * gte * (f["merge.ws"] @ r)
        y = _rms(z, f["dec.0.swa_norm"], cfg.eps)
        q = _rot((f["dec.0.wq"] @ y).reshape(1, h, dh), [t], cfg.rope_base)
        Ks.append(_rot((f["dec.0.wk"] @ y).reshape(1, h, dh), [t], cfg.rope_base)[0])
        Vs.append((f["dec.0.wv"] @ y).reshape(h, dh))
        lo = max(1, t - cfg.window + 1)
        K, V = np.stack(Ks[lo - 1:t]), np.stack(Vs[lo - 1:t])
        mask = np.ones((1, t - lo + 1), bool)
        z = z + f["dec.0.wo"] @ _masked_attention(q, K, V, mask).reshape(-1)
        y = _rms(z, f["dec.0.x_norm"], cfg.eps)
        qx = _rot((f["dec.0.xq"] @ y).reshape(1, h, dh), [t], cfg.rope_base)
        z = z + f["dec.0.xo"] @ _masked_attention(qx, mk[:t], mv[:t], np.ones((1, t), bool)).reshape(-1)
        y = _rms(z, f["dec.0.ffn_norm"], cfg.eps)
        a1, a3 = f["dec.0.w1"] @ y, f["dec.0.w3"] @ y
        s = z + f["dec.0.w2"] @ (a1 / (1 + np.exp(-a1)) * a3)
        np.testing.assert_allclose(m.transition(st), s, atol=1e-12)
        assert sorted(st.swa[0]) == list(range(max(1, t - cfg.window + 2), t + 1))


# ----------------------------------------------------------------------------
# structural identities
# ----------------------------------------------------------------------------


def test_groups_with_equal_projections_equal_shared_memory():
    c1 = small_cfg(groups=1, n_dec=3)
    cg = small_cfg(groups=3, n_dec=3)
    W1 = weights(c1)
    Wg = dict(W1)
    for g in range(3):
        Wg[f"mem.{g}.wk"], Wg[f"mem.{g}.wv"] = W1["mem.0.wk"], W1["mem.0.wv"]
    x = toks(c1, 8)
    a, _ = logits_token_by_token(RLTOracle(c1, W1), x)
    b, _ = logits_token_by_token(RLTOracle(cg, Wg), x)
    np.testing.assert_allclose(a, b, atol=1e-13, rtol=0)


def test_tied_equals_untied_with_copied_weights():
    """Tying (greeksharifa App. A.1): encoder layer l uses decoder layer l's
    attention and FFN matrices; norms stay separate."""
    ct = small_cfg(tied=True)
    cu = small_cfg(tied=False)
    Wt = weights(ct)
    Wu = dict(Wt)
    for l in range(2):
        for n in ("wq", "wk", "wv", "wo", "w1", "w3", "w2"):
            Wu[f"enc.{l}.{n}"] = Wt[f"dec.{l}.{n}"]
    x = toks(ct, 8)
    a, _ = logits_token_by_token(RLTOracle(ct, Wt), x)
    b, _ = logits_token_by_token(RLTOracle(cu, Wu), x)
    np.testing.assert_array_equal(a, b)


def test_random_init_loss_is_about_ln_vocab():
    """The pages' random-init loss of a vocab-32 model is 3.467 ~ ln 32 (tistory
    §5): near-uniform softmax at init.  Same for the tiny workload here."""
    g = json.load(open(os.path.join(GOLDEN, "pages_numbers.json")))["tiny_init_loss"]
    cfg = ri.CONFIGS["tiny_fp32"]
    m = RLTOracle(cfg, ri.generate_weights(cfg))
    x = ri.make_tokens(cfg)
    ces = []
    for row in x:
        lg, _ = logits_token_by_token(m, row)
        for t in range(len(row) - 1):
            z = lg[t] - lg[t].max()
            ces.append(-(z[row[t + 1]] - math.log(np.exp(z).sum())))
    assert abs(np.mean(ces) - math.log(g["vocab"])) < 0.02
    assert abs(g["value"] - math.log(g["vocab"])) < 0.002


def test_bf16_mode_rounds_stored_keys_and_stays_close():
    cfg = small_cfg(dtype=ri.DT_BF16)
    W = {k: ri.bf16_bits_to_f32(ri.to_bf16_bits(v)).reshape(v.shape)
         for k, v in weights(cfg, seed=5).items()}
    x = toks(cfg, 8)
    a, st = logits_token_by_token(RLTOracle(cfg, W, "bf16"), x)
    b, _ = logits_token_by_token(RLTOracle(cfg, W, "fp64"), x)
    for arr in st.mem_k + st.enc_k:
        np.testing.assert_array_equal(round_bf16(arr), arr)
    assert 0 < np.max(np.abs(a - b)) < 0.1


def test_bf16_mode_rounds_every_cache_and_product_input():
    """Reading c14: in bf16 mode every stored key and value (encoder cache,
    memory, window ring) is a bf16 value, and every matrix-product input is
    rounded -- rounding it before the call changes nothing (rounding is
    idempotent), while the fp64 mode's product does change."""
    cfg = small_cfg(dtype=ri.DT_BF16, window=3)
    W = {k: ri.bf16_bits_to_f32(ri.to_bf16_bits(v)).reshape(v.shape)
         for k, v in weights(cfg, seed=5).items()}
    m = RLTOracle(cfg, W, "bf16")
    _, st = logits_token_by_token(m, toks(cfg, 8))
    ring = [a for cache in st.swa for kv in cache.values() for a in kv]
    assert ring
    for arr in st.enc_k + st.enc_v + st.mem_k + st.mem_v + ring:
        np.testing.assert_array_equal(round_bf16(arr), arr)
    y = np.random.default_rng(3).normal(size=(3, cfg.d))
    for name in ("dec.0.wq", "dec.1.w1", "mem.0.wk", "out"):
        np.testing.assert_array_equal(m._lin(y, name), m._lin(round_bf16(y), name))
    f64 = RLTOracle(cfg, W, "fp64")
    assert not np.array_equal(f64._lin(y, "out"), f64._lin(round_bf16(y), "out"))
    # the encoder attention's products take a bf16 query and bf16
    # probabilities: rounding q first changes nothing, the unrounded
    # attention differs, and one key still returns its value exactly
    rng = np.random.default_rng(4)
    q, K, V = rng.normal(size=(2, 8)), rng.normal(size=(5, 2, 8)), rng.normal(size=(5, 2, 8))
    np.testing.assert_array_equal(attend(q, K, V, rounded=True),
                                  attend(round_bf16(q), K, V, rounded=True))
    assert not np.array_equal(attend(q, K, V, rounded=True), attend(q, K, V))
    np.testing.assert_allclose(attend(q, K[:1], V[:1], rounded=True), V[0], rtol=1e-15)
    # and encode() uses it in bf16 mode: at head size 64 with short prefixes
    # for any call, otherwise for calls of at least ENC_TC_MIN_POSITIONS
    # tokens (the pin model's head size is 8, so the call size decides)
    import oracle.rlt_oracle as ro
    seen = []
    real = ro.attend

    def spy(q_, K_, V_, rounded=False):
        seen.append(rounded)
        return real(q_, K_, V_, rounded)
    ro.attend = spy
    try:
        n_tc = ro.ENC_TC_MIN_POSITIONS
        st_ = m.new_state()
        m.encode(st_, toks(cfg, n_tc))
        assert seen and all(seen)
        seen.clear()
        m.encode(st_, toks(cfg, n_tc - 1))
        assert seen and not any(seen)
        seen.clear()
        f64.encode(f64.new_state(), toks(cfg, n_tc))
        assert seen and not any(seen)
    finally:
        ro.attend = real


def test_decoder_blocks_round_attention_inputs_like_the_tile_products():
    """bf16 mode, head size 64: a decoder block of 2..16 positions (an RLT-2
    chunk) passes rounded q and probabilities to both attentions (the window
    only when W exceeds the block); a one-position transition does not; the
    fp64 mode never does."""
    import oracle.rlt_oracle as ro
    cfg = ri.CONFIGS["rlt2_mod5_bf16"].replace(name="pin_mq", n_enc=1, n_dec=1, vocab=64)
    W = ri.generate_weights(cfg)
    seen = []
    real = ro.attend

    def spy(q_, K_, V_, rounded=False):
        seen.append(rounded)
        return real(q_, K_, V_, rounded)
    ro.attend = spy
    try:
        tok = (np.arange(12) % 60 + 1).astype(np.int64)
        for mode, want_block in (("bf16", True), ("fp64", False)):
            m = RLTOracle(cfg, W, mode)
            st_ = m.new_state()
            m.encode(st_, tok)
            seen.clear()
            m.transition_chunk(st_, cfg.chunk)          # positions 1..4: one block
            assert len(seen) == 2 * cfg.chunk and all(x == want_block for x in seen)
            seen.clear()
            m.transition(st_)                           # position 5 alone
            assert len(seen) == 2 and not any(seen)
        # a window no longer than the block keeps the window's inputs unrounded
        narrow = cfg.replace(name="pin_mq_w", window=cfg.chunk)
        m = RLTOracle(narrow, W, "bf16")
        st_ = m.new_state()
        m.encode(st_, tok)
        seen.clear()
        m.transition_chunk(st_, narrow.chunk)
        assert seen[:narrow.chunk] == [False] * narrow.chunk and all(seen[narrow.chunk:])
    finally:
        ro.attend = real


# ----------------------------------------------------------------------------
# replay log-probabilities (jiphyeonjeon review §6.2, eq. 5.3-5.5)
# ----------------------------------------------------------------------------


def test_log_softmax_at_closed_forms_and_scipy():
    from scipy.special import log_softmax
    # equal logits: every token has probability 1/V
    for V in (1, 2, 7, 32000):
        assert abs(log_softmax_at(np.full(V, 3.25), V // 2) + math.log(V)) < 1e-12
    # two logits: the logistic, log p_0 = -log(1 + exp((l_1 - l_0) / T))
    for l0, l1, T in ((0.3, -1.2, 1.0), (2.0, 5.0, 0.7), (-4.0, 4.0, 3.0)):
        want = -math.log1p(math.exp((l1 - l0) / T))
        assert abs(log_softmax_at(np.array([l0, l1]), 0, T) - want) < 1e-12
    # any logits and temperature against scipy's log_softmax
    rng = np.random.default_rng(11)
    for T in (1.0, 0.6, 2.5):
        lg = rng.normal(0, 4, 513)
        ref = log_softmax(lg / T)
        got = np.array([log_softmax_at(lg, i, T) for i in range(len(lg))])
        np.testing.assert_allclose(got, ref, atol=1e-12, rtol=0)
        # a distribution: the probabilities sum to one, the argmax is the largest
        assert abs(np.exp(got).sum() - 1.0) < 1e-12
        assert int(np.argmax(got)) == argmax_lowest(lg)


@pytest.mark.parametrize("variant,chunk", [(1, 1), (2, 2), (0, 1)])
def test_replay_probabilities_of_all_continuations_sum_to_one(variant, chunk):
    """Eq. 5.3: pi(y | c) = prod_i p(y_i | c, y_<i).  Summed over every
    continuation y of a fixed length the product is 1 only if each factor is
    read from the state that has consumed exactly c and y_<i (reading it
    after consuming y_i, or from a stale state, breaks the sum).  Brute force
    over all V^3 continuations of a small model."""
    cfg = small_cfg(vocab=5, variant=variant, chunk=chunk)
    m = RLTOracle(cfg, weights(cfg))
    prompt = toks(cfg, 4)
    st = m.new_state()
    replay_logprobs(m, st, prompt)
    total = 0.0
    for a in range(cfg.vocab):
        for b in range(cfg.vocab):
            for c in range(cfg.vocab):
                total += math.exp(replay_logprobs(m, st.copy(), [a, b, c]).sum())
    assert abs(total - 1.0) < 1e-12


def test_replay_equals_readouts_of_the_prefilled_sequence():
    """Replay token by token = one parallel encode and a prefill, read out
    after every position (the logits after position t give token t+1), and it
    ends in the same state (Prop. 3.1 applied to the replay schedule)."""
    cfg = small_cfg(variant=2, chunk=3)
    m = RLTOracle(cfg, weights(cfg))
    x = toks(cfg, 10)
    for T in (1.0, 0.8):
        st = m.new_state()
        got = replay_logprobs(m, st, x, T)
        ref_st = m.new_state()
        first = m.readout(ref_st)
        seq = [first] + run_sequence(m, list(x))[:-1]
        want = [log_softmax_at(seq[j], int(x[j]), T) for j in range(len(x))]
        np.testing.assert_allclose(got, want, atol=1e-12, rtol=0)
        full = m.new_state()
        m.encode(full, x)
        m.prefill(full, len(x))
        np.testing.assert_allclose(st.s, full.s, atol=1e-12, rtol=0)
        np.testing.assert_allclose(st.R, full.R, atol=1e-12, rtol=0)


# ----------------------------------------------------------------------------
# packed documents (jiphyeonjeon review §6.1: independent documents reset the
# recurrent output, the decoder window cache, the encoder cache and positions)
# ----------------------------------------------------------------------------


@pytest.mark.parametrize("variant,chunk", [(1, 1), (2, 3), (0, 1)])
def test_packed_documents_are_independent(variant, chunk):
    cfg = small_cfg(variant=variant, chunk=chunk)
    m = RLTOracle(cfg, weights(cfg))
    x = toks(cfg, 20)
    starts = np.zeros(20, bool)
    starts[[0, 7, 12]] = True
    st = prefill_packed(m, x, starts)
    # the last document alone, from a fresh state, in one encode + prefill
    alone = m.new_state()
    m.encode(alone, x[12:])
    m.prefill(alone, 8)
    assert (st.pos_enc, st.pos_dec) == (8, 8)
    np.testing.assert_allclose(st.s, alone.s, atol=1e-12, rtol=0)
    np.testing.assert_allclose(m.readout(st), m.readout(alone), atol=1e-12, rtol=0)
    # earlier documents leave no trace: change every token before the start
    y = x.copy()
    y[:12] = (y[:12] + 5) % cfg.vocab
    other = prefill_packed(m, y, starts)
    np.testing.assert_array_equal(m.readout(other), m.readout(st))
    # one document from column 0 is the plain run
    one = prefill_packed(m, x, np.eye(1, 20, 0, dtype=bool)[0])
    plain = m.new_state()
    m.encode(plain, x)
    m.prefill(plain, 20)
    np.testing.assert_allclose(one.s, plain.s, atol=1e-12, rtol=0)
    # a start at every column: the last token alone
    last = prefill_packed(m, x, np.ones(20, bool))
    solo = m.new_state()
    m.encode(solo, x[-1:])
    m.prefill(solo, 1)
    np.testing.assert_allclose(last.s, solo.s, atol=1e-12, rtol=0)

"""Exact prefix snapshots (rlt_state_save / rlt_state_load).

A row saved after a prefix and restored -- into another row of a state that
already held other sequences, into a state of another max_len, from host or
device memory -- continues bit for bit like the row it was taken from:
through an appended turn (encode + prefill), sampled generation fed back in,
and the readout (jiphyeonjeon review "Recurrent Looped Transformer" §6.5;
greeksharifa "Recurrent Looped Transformer 요약 설명" App. E).  Named to be
collected after the parity tests.
"""
import numpy as np
import pytest

import rlt_inputs as ri

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


def _model(sd, cfg, seed=ri.WEIGHT_SEED):
    return sd.Model(ri.write_blob(cfg, ri.generate_weights(cfg, seed=seed), seed=seed))


def _readout(st, cfg, step=0):
    import torch
    B = st.batch
    lg = np.zeros((B, cfg.vocab), np.float32)
    am = np.zeros(B, np.int32)
    sp = np.zeros(B, np.int32)
    st.readout(lg, am, sp, seed=ri.SAMPLE_SEED, step=step, temperature=0.9)
    torch.cuda.synchronize()
    return lg, am, sp


def _row_parts(sd, st, cfg, P):
    """Bit patterns of every state component, per row, restricted to the
    positions 1..P a snapshot carries."""
    B, Tc, d, dh = st.batch, st.max_len, cfg.d, cfg.d // cfg.heads
    el = np.uint16 if cfg.dtype == ri.DT_BF16 else np.uint32
    out = {
        "s": st.read(sd.PART_S).view(np.uint32).reshape(B, d),
        "R": st.read(sd.PART_R).view(np.uint32).reshape(B, d),
        "e": st.read(sd.PART_E).view(np.uint32).reshape(B, Tc, d)[:, :P],
    }
    for key, part in (("enc", sd.PART_ENC), ("mem", sd.PART_MEM)):
        a = st.read(part).view(el)
        if a.size:
            out[key] = a.reshape(B, -1, Tc, dh)[:, :, :P]
    ring = st.read(sd.PART_RING).view(el)
    if ring.size:
        out["ring"] = ring.reshape(B, -1)
    return out


@pytest.mark.parametrize("name", ["parity_bf16", "s5_bf16", "rlt2_mod5_bf16", "tiny_fp32"])
def test_restored_rows_continue_bitexact(sd, name):
    import torch
    cfg = ri.CONFIGS[name]
    B, T, P, Pd, gen = 3, 26, 14, 11, 3
    model = _model(sd, cfg)
    toks = ri.make_tokens(cfg, B, T)
    a = sd.State(model, B, T + gen)
    a.encode(np.ascontiguousarray(toks[:, :P]))
    a.prefill(Pd)                         # positions P - Pd encoded but not yet consumed
    snaps = [a.save(r) for r in range(B)]
    for r in range(B):
        c, pe, pd = sd.snapshot_info(snaps[r])
        assert (pe, pd) == (P, Pd) and c.d == cfg.d
    dev_snaps = []
    for r in range(B):
        buf = torch.empty(snaps[r].nbytes, dtype=torch.uint8, device="cuda")
        dev_snaps.append(a.save(r, dst=buf))
        np.testing.assert_array_equal(buf.cpu().numpy(), snaps[r])
    parts_a = _row_parts(sd, a, cfg, P)

    # b: same shape, already running other sequences; rows restored permuted
    perm = [2, 0, 1]
    b = sd.State(model, B, T + gen)
    other = ri.make_tokens(cfg, B, 5, seed=ri.TOKEN_SEED + 17)
    b.encode(other)
    b.prefill(5)
    for i in range(B):
        b.load(i, snaps[perm[i]])
    pe, pd = b.positions()
    assert list(pe) == [P] * B and list(pd) == [Pd] * B
    parts_b = _row_parts(sd, b, cfg, P)
    for key, va in parts_a.items():
        np.testing.assert_array_equal(parts_b[key], va[perm], err_msg=key)

    # c: a longer max_len, restored from device memory in row order
    c = sd.State(model, B, T + gen + 9)
    for i in range(B):
        c.load(i, dev_snaps[i])

    # the next turn, appended onto the cached prefix and consumed
    a.encode(np.ascontiguousarray(toks[:, P:]))
    a.prefill(T - Pd)
    b.encode(np.ascontiguousarray(toks[perm, P:]))
    b.prefill(T - Pd)
    c.encode(np.ascontiguousarray(toks[:, P:]))
    c.prefill(T - Pd)
    la, aa, _ = _readout(a, cfg)
    lb, ab, _ = _readout(b, cfg)
    np.testing.assert_array_equal(lb, la[perm])
    np.testing.assert_array_equal(ab, aa[perm])
    # sampled generation fed back in (the uniform depends on the row index,
    # so c, whose rows keep their indices, repeats a's sampled ids)
    for k in range(gen):
        la, aa, sa = _readout(a, cfg, step=k)
        lc, ac, sc = _readout(c, cfg, step=k)
        np.testing.assert_array_equal(lc, la)
        np.testing.assert_array_equal(sc, sa)
        for st, ids in ((a, sa), (c, sc)):
            st.encode(ids.reshape(B, 1).astype(np.int32))
            st.step()
    la, _, _ = _readout(a, cfg)
    lc, _, _ = _readout(c, cfg)
    np.testing.assert_array_equal(lc, la)
    np.testing.assert_array_equal(c.read(sd.PART_S), a.read(sd.PART_S))
    for st in (a, b, c):
        st.check()
        st.close()
    model.close()


def test_fresh_snapshot_restores_h0(sd):
    """A snapshot of a row with nothing encoded (H_0 = (s_star, empty))
    returns a used row to the start: the same results as a reset row."""
    cfg = ri.CONFIGS["tiny_fp32"]
    B, T = 2, 12
    model = _model(sd, cfg)
    toks = ri.make_tokens(cfg, B, T)
    fresh = sd.State(model, 1, T).save(0)
    assert sd.snapshot_info(fresh)[1:] == (0, 0)
    st = sd.State(model, B, T)
    st.encode(toks)
    st.prefill(T)
    ref, _, _ = _readout(st, cfg)
    st.load(0, fresh)
    st.load(1, fresh)
    assert [list(p) for p in st.positions()] == [[0, 0], [0, 0]]
    st.encode(toks)
    st.prefill(T)
    again, _, _ = _readout(st, cfg)
    np.testing.assert_array_equal(again, ref)
    st.close()
    model.close()


def test_snapshot_errors(sd):
    cfg = ri.CONFIGS["parity_bf16"]
    B, P = 2, 9
    model = _model(sd, cfg)
    st = sd.State(model, B, 16)
    st.encode(ri.make_tokens(cfg, B, P))
    st.prefill(P)
    snap = st.save(1)
    # another model with the same config but other weights
    other = _model(sd, cfg, seed=ri.WEIGHT_SEED + 1)
    st2 = sd.State(other, 1, 16)
    with pytest.raises(sd.RLTError) as e:
        st2.load(0, snap)
    assert e.value.code == sd.RLT_E_SNAPSHOT
    assert [list(p) for p in st2.positions()] == [[0], [0]]     # nothing written
    # a state too short for the snapshot's positions
    short = sd.State(model, 1, P - 1)
    with pytest.raises(sd.RLTError) as e:
        short.load(0, snap)
    assert e.value.code == sd.RLT_E_CAPACITY
    # truncated, corrupted, bad rows, wrong sizes
    with pytest.raises(sd.RLTError) as e:
        st.load(0, snap[:-2])
    assert e.value.code == sd.RLT_E_SNAPSHOT
    bad = snap.copy()
    bad[0] ^= 1
    with pytest.raises(sd.RLTError) as e:
        st.load(0, bad)
    assert e.value.code == sd.RLT_E_SNAPSHOT
    assert sd.rlt_state_load(st.handle, B, snap, snap.nbytes) == sd.RLT_E_ARG
    assert sd.rlt_state_load(st.handle, -1, snap, snap.nbytes) == sd.RLT_E_ARG
    code, n = sd.rlt_state_save(st.handle, 0)
    assert code == 0 and n == snap.nbytes
    buf = np.empty(n + 1, np.uint8)
    assert sd.rlt_state_save(st.handle, 0, buf, n + 1)[0] == sd.RLT_E_ARG
    assert sd.rlt_state_save(st.handle, B, buf, n)[0] == sd.RLT_E_ARG
    pe, pd = st.positions()
    assert list(pe) == [P, P] and list(pd) == [P, P]
    for s_ in (st, st2, short):
        s_.check()
        s_.close()
    other.close()
    model.close()

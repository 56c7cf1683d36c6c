"""The replayed transition graphs: the path the bench times.

rlt_prefill on a stream other than the legacy default captures 16 consecutive
transition blocks as one CUDA graph (one-position blocks hand the state to the
next block's merge input in one fused kernel) and replays it; with a null
stream the same blocks run launch by launch.  Rows never interact, so the
result must not depend on the schedule: bit for bit the same logits, state s
and (RLT-2) register R.  RLT_ROW_GROUPS=g splits the rows of a captured run
into g groups whose kernel chains are concurrent branches of the graph; it is
read once per process, so each group count runs in a child process.
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

import rlt_inputs as ri

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def sd():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tests.conftest import build_library
    build_library()
    import stateful_decoding_b200 as sd
    return sd


def config(name):
    if name == "rlt0_parity":
        return ri.CONFIGS["parity_bf16"].replace(name="rlt0_parity", variant=0)
    if name == "large_slice":
        return ri.CONFIGS["large_bf16"].replace(name="large_slice", n_enc=2, n_dec=2)
    return ri.CONFIGS[name]


# (workload, rows, positions): every run is long enough for one replayed graph
# of 16 blocks plus a ragged rest run launch by launch
CASES = [("parity_bf16", 6, 40), ("rlt2_mod5_bf16", 5, 72), ("rlt0_parity", 3, 40),
         ("tiny_fp32", 3, 40), ("large_slice", 4, 20)]


def run_case(sd, name, B, T, use_stream):
    """Encode and prefill B rows of T positions; return (logits, state parts)."""
    import torch
    cfg = config(name)
    W = ri.generate_weights(cfg)
    model = sd.Model(ri.write_blob(cfg, W))
    st = sd.State(model, B, T)
    stream = torch.cuda.Stream() if use_stream else None
    st.encode(ri.make_tokens(cfg, B, T), stream=stream)
    st.prefill(T, stream=stream)
    lg = np.zeros((B, cfg.vocab), np.float32)
    am = np.zeros(B, np.int32)
    sp = np.zeros(B, np.int32)
    st.readout(lg, am, sp, seed=ri.SAMPLE_SEED, stream=stream)
    torch.cuda.synchronize()
    parts = {"s": st.read(sd.PART_S).copy()}
    if cfg.variant == 2:
        parts["R"] = st.read(sd.PART_R).copy()
    st.check()
    st.close()
    model.close()
    return lg, parts


CHILD = r"""
import sys, numpy as np
sys.path.insert(0, {root!r})
import stateful_decoding_b200 as sd
from tests.test_graphs_gpu import run_case
lg, parts = run_case(sd, {name!r}, {B}, {T}, True)
np.savez({out!r}, lg=lg, **parts)
"""


@pytest.mark.parametrize("name,B,T", CASES)
def test_graph_replay_matches_launch_by_launch(sd, name, B, T):
    lg_d, parts_d = run_case(sd, name, B, T, use_stream=False)
    lg_g, parts_g = run_case(sd, name, B, T, use_stream=True)
    bad = [int(b) for b in np.nonzero(np.any(lg_g != lg_d, axis=1))[0]]
    assert not bad, (f"rows {bad} differ, max |dlogit| per row "
                     f"{np.abs(lg_g - lg_d).max(axis=1)[bad]}")
    for k in parts_d:
        np.testing.assert_array_equal(parts_g[k], parts_d[k])


@pytest.mark.parametrize("name,B,T", [("parity_bf16", 6, 40), ("rlt2_mod5_bf16", 5, 72),
                                      ("large_slice", 4, 20)])
@pytest.mark.parametrize("groups", [2, 3])
def test_row_groups_as_graph_branches(sd, tmp_path, name, B, T, groups):
    lg_1, parts_1 = run_case(sd, name, B, T, use_stream=True)
    out = str(tmp_path / f"g{groups}.npz")
    env = dict(os.environ, RLT_ROW_GROUPS=str(groups))
    code = CHILD.format(root=ROOT, name=name, B=B, T=T, out=out)
    r = subprocess.run([sys.executable, "-c", code], env=env, cwd=ROOT, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    got = np.load(out)
    np.testing.assert_array_equal(got["lg"], lg_1)
    for k in parts_1:
        np.testing.assert_array_equal(got[k], parts_1[k])

"""The library's schedule switches select other correct schedules: each one,
set in a child process (the library reads them once), still matches the
oracle on a small run through the replayed graphs.

RLT_SQ=0 (one-position attention on the register-batch kernel),
RLT_SQ_STAGES=2|4 (key tiles in flight), RLT_MQ=0 (chunk blocks on the
CUDA-core kernels), RLT_XSPLIT_SWA=0 (the wide-head window attention on one
warp per item), RLT_GRAPH_CHAIN=1 (the fused state hand-off inside captured
runs), RLT_GEMM_PERSIST=0 (no persistent GEMM).
"""
import os
import subprocess
import sys

import numpy as np
import pytest

import rlt_inputs as ri
from oracle import RLTOracle
from tests.rlt_testlib import Tally, check_argmax, oracle_mode, tol_for
from tests.test_graphs_gpu import ROOT, config

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def built():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tests.conftest import build_library
    build_library()


CHILD = r"""
import sys, numpy as np
sys.path.insert(0, {root!r})
import stateful_decoding_b200 as sd
from tests.test_graphs_gpu import run_case
lg, parts = run_case(sd, {name!r}, {B}, {T}, True)
np.savez({out!r}, lg=lg)
"""


@pytest.mark.parametrize("env,name,B,T", [
    ({"RLT_SQ": "0"}, "parity_bf16", 3, 40),
    ({"RLT_SQ_STAGES": "2"}, "parity_bf16", 3, 40),
    ({"RLT_SQ_STAGES": "4"}, "parity_bf16", 3, 40),
    ({"RLT_MQ": "0"}, "rlt2_mod5_bf16", 3, 40),
    ({"RLT_XSPLIT_SWA": "0"}, "large_slice", 2, 20),
    ({"RLT_GRAPH_CHAIN": "1"}, "parity_bf16", 3, 40),
    ({"RLT_GEMM_PERSIST": "0"}, "parity_bf16", 8, 256),
])
def test_switch_matches_oracle(built, tmp_path, env, name, B, T):
    out = str(tmp_path / "lg.npz")
    r = subprocess.run([sys.executable, "-c",
                        CHILD.format(root=ROOT, name=name, B=B, T=T, out=out)],
                       env=dict(os.environ, **env), cwd=ROOT, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    lg = np.load(out)["lg"]
    cfg = config(name)
    W = ri.generate_weights(cfg)
    orc = RLTOracle(cfg, W, oracle_mode(cfg))
    toks = ri.make_tokens(cfg, B, T)
    tol = tol_for(cfg)
    tally = Tally()
    for b in (0, B - 1):
        st = orc.new_state()
        orc.encode(st, toks[b])
        orc.prefill(st, T, chunked=cfg.variant == 2)
        ol = orc.readout(st)
        err = float(np.max(np.abs(lg[b] - ol)))
        assert err <= tol, f"{env} {name} row {b}: |dlogit| {err} > {tol}"
        check_argmax(int(np.argmax(lg[b])), ol, tol, tally, f"row {b}")

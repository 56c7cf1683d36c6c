"""The RLT_DEBUG build (librlt_debug.so): the same kernels with bounds checks
of positions, ring slots and key indices compiled in, reporting through the
state's error word instead of trapping.

CPU: both libraries build and export the same functions; the build flags
tell them apart; the release build refuses the debug-only entry point.
GPU (each run in a child process, since a process loads one of the two
libraries): the debug build computes bit for bit what the release build
computes; device position counters that disagree with the encoded tokens
(a row about to consume a position never encoded) or with the capacity are
reported by rlt_state_check as RLT_E_ORDER / RLT_E_CAPACITY, and every
access stays inside the buffers.
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _builder():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "rlt_build", os.path.join(ROOT, "stateful_decoding_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _child(code: str, debug: bool, timeout=600) -> dict:
    env = dict(os.environ)
    if debug:
        env["RLT_LIB"] = "debug"
    else:
        env.pop("RLT_LIB", None)
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=timeout)
    assert r.returncode == 0, r.stderr[-3000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


FLAGS = """
import json, stateful_decoding_b200 as sd
print(json.dumps({"flags": sd.rlt_build_flags(), "lib": sd.LIB_PATH,
                  "exports": sd.header_functions()}))
"""


def test_debug_library_builds_and_reports_its_flag():
    b = _builder()
    b.build()
    b.build(debug=True)
    rel = _child(FLAGS, debug=False)
    dbg = _child(FLAGS, debug=True)
    assert rel["flags"] == 0 and rel["lib"].endswith("librlt.so")
    assert dbg["flags"] == 1 and dbg["lib"].endswith("librlt_debug.so")
    import ctypes
    lib_d = ctypes.CDLL(dbg["lib"])
    for name in rel["exports"]:
        getattr(lib_d, name)            # every declared function is exported by both


RUN = """
import json, numpy as np, torch
import rlt_inputs as ri, stateful_decoding_b200 as sd
cfg = ri.CONFIGS["parity_bf16"]
B, T = 3, 24
model = sd.Model(ri.write_blob(cfg, ri.generate_weights(cfg)))
st = sd.State(model, B, T)
toks = ri.make_tokens(cfg, B, T)
st.encode(toks)
st.prefill(T)
lg = np.zeros((B, cfg.vocab), np.float32)
st.readout(lg)
st.check()
out = {"logits": lg.tolist(), "flags": sd.rlt_build_flags()}
# a row whose device counters say it may consume a position that was never
# encoded (pos_dec = pos_enc on the device, the host still at 4 of 6): every
# index the step forms stays inside the buffers (capacity 24)
st2 = sd.State(model, 2, T)
st2.encode(np.ascontiguousarray(toks[:2, :6]))
st2.prefill(4)
st2.check()
out["set"] = sd.rlt_debug_set_positions(st2.handle, 1, 6, 6)
if out["set"] == sd.RLT_OK:
    st2.step()
    out["order"] = sd.rlt_state_check(st2.handle)
    out["after"] = sd.rlt_state_check(st2.handle)
    # encoded positions beyond the capacity on the device: only a step
    # follows (it reads no encoder counter but the check's)
    st3 = sd.State(model, 2, 8)
    st3.encode(np.ascontiguousarray(toks[:2, :4]))
    st3.prefill(2)
    st3.check()
    sd.rlt_debug_set_positions(st3.handle, 0, 8 + 5, 2)
    st3.step()
    out["capacity"] = sd.rlt_state_check(st3.handle)
print(json.dumps(out))
"""


@pytest.mark.gpu
def test_debug_build_matches_release_and_reports_bad_positions():
    pytest.importorskip("torch")
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    b = _builder()
    b.build()
    b.build(debug=True)
    rel = _child(RUN, debug=False)
    dbg = _child(RUN, debug=True)
    assert rel["flags"] == 0 and dbg["flags"] == 1
    np.testing.assert_array_equal(np.array(dbg["logits"], np.float32),
                                  np.array(rel["logits"], np.float32))
    import stateful_decoding_b200 as sd
    assert rel["set"] == sd.RLT_E_UNSUPPORTED
    assert dbg["set"] == sd.RLT_OK
    assert dbg["order"] == sd.RLT_E_ORDER
    assert dbg["after"] == sd.RLT_OK
    assert dbg["capacity"] == sd.RLT_E_CAPACITY

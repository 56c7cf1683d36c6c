"""C ABI checks that need no GPU: the library loads, exports every function
include/rlt.h declares, and rejects bad input on the host before any CUDA work."""
import ctypes
import os
import subprocess
import sys

import numpy as np
import pytest

import rlt_inputs as ri

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from tests.conftest import build_library
    build_library()
    import stateful_decoding_b200 as sd
    return sd


def test_exports_every_declared_function(lib):
    declared = lib.header_functions()
    assert "rlt_create" in declared and "rlt_prefill" in declared
    raw = ctypes.CDLL(lib.LIB_PATH)
    for name in declared:
        assert hasattr(raw, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", lib.LIB_PATH], capture_output=True,
                         text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l and l.split()[-1].startswith("rlt_")}
    assert set(declared) <= exported


def test_strerror_covers_codes(lib):
    for code in range(0, -10, -1):
        assert lib.rlt_strerror(code) != "unknown error"
    assert lib.rlt_strerror(-99) == "unknown error"


def _blob(name="tiny_fp32", **kw):
    cfg = ri.CONFIGS[name].replace(**kw) if kw else ri.CONFIGS[name]
    return cfg, ri.write_blob(cfg, ri.generate_weights(cfg))


def test_bad_blobs_rejected_before_device(lib):
    cfg, blob = _blob()
    assert lib.rlt_create(b"XXXX" + blob[4:])[0] == lib.RLT_E_BLOB
    assert lib.rlt_create(blob[:100])[0] == lib.RLT_E_BLOB
    bad = bytearray(blob)
    bad[300] ^= 0x40                                  # payload byte: checksum mismatch
    assert lib.rlt_create(bytes(bad))[0] == lib.RLT_E_BLOB
    bad = bytearray(blob)
    bad[4] = 2                                        # version
    assert lib.rlt_create(bytes(bad))[0] == lib.RLT_E_BLOB
    # a config whose manifest differs from the records (vocab changed in the header)
    cfg2 = cfg.replace(vocab=33)
    hdr = ri.write_blob(cfg2, ri.generate_weights(cfg2))[:256]
    assert lib.rlt_create(hdr + blob[256:])[0] == lib.RLT_E_BLOB


def test_valid_blob_without_gpu_reports_device(lib):
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    _, blob = _blob()
    assert lib.rlt_create(blob)[0] == lib.RLT_E_DEVICE


def test_null_arguments(lib):
    assert lib._lib.rlt_create(None, 0, 0, None) == lib.RLT_E_ARG
    assert lib._lib.rlt_state_create(None, 1, 1, None) == lib.RLT_E_ARG
    assert lib._lib.rlt_encode(None, None, 1, None) == lib.RLT_E_ARG
    assert lib._lib.rlt_step(None, None) == lib.RLT_E_ARG
    assert lib._lib.rlt_prefill(None, 1, None) == lib.RLT_E_ARG
    assert lib._lib.rlt_readout(None, None, None, None, 0, 0, 1.0, None) == lib.RLT_E_ARG
    assert lib._lib.rlt_state_check(None, None) == lib.RLT_E_ARG
    assert lib._lib.rlt_state_save(None, 0, None, 0, None, None) == lib.RLT_E_ARG
    assert lib._lib.rlt_state_load(None, 0, None, 0, None) == lib.RLT_E_ARG
    assert lib._lib.rlt_snapshot_info(None, 0, None, None, None) == lib.RLT_E_ARG
    assert lib._lib.rlt_prefill_packed(None, None, None, 1, None) == lib.RLT_E_ARG
    assert lib._lib.rlt_replay_logprobs(None, None, 1, None, 1.0, None) == lib.RLT_E_ARG
    assert lib.rlt_kernel_launches() >= 0


def test_package_fails_loudly_without_library(tmp_path):
    """The product path has no CPU fallback: without librlt.so the import raises."""
    pkg = tmp_path / "stateful_decoding_b200"
    pkg.mkdir()
    src = open(os.path.join(ROOT, "stateful_decoding_b200", "__init__.py")).read()
    (pkg / "__init__.py").write_text(src)
    r = subprocess.run([sys.executable, "-c", "import stateful_decoding_b200"], cwd=tmp_path,
                       capture_output=True, text=True)
    assert r.returncode != 0 and "librlt.so not built" in r.stderr


def test_product_package_never_imports_oracle():
    pkg = os.path.join(ROOT, "stateful_decoding_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in txt.replace("no fallback", ""), f


def test_readout_rows_scratch_limit_matches_header():
    """The binding's copy of the static scratch size and its size rule agree
    with the header (and its worked example: vocab 32000, d 2048, bf16, host
    logits -> at most 127 rows)."""
    import re
    hdr = open(os.path.join(ROOT, "include", "rlt.h")).read()
    m = re.search(r"#define RLT_READOUT_ROWS_SCRATCH_BYTES \((\d+)u << (\d+)\)", hdr)
    assert m, "scratch size define not found"
    import importlib
    sd = importlib.import_module("stateful_decoding_b200")
    assert sd.READOUT_ROWS_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))
    fits = [r for r in range(1, 200)
            if sd.readout_rows_scratch_bytes(r, 2048, 32000, True, True)
            <= sd.READOUT_ROWS_SCRATCH_BYTES]
    assert max(fits) == 127 and "at most 127 rows" in hdr


# ---------------------------------------------------------------- snapshots
def _snapshot_bytes(cfg, pos_enc, pos_dec, checksum=0x0123456789ABCDEF):
    """A snapshot laid out as include/rlt.h states it (header fields, then
    zero-filled sections of the stated sizes), written independently of the
    library."""
    import struct
    h, dh = cfg.heads, cfg.d // cfg.heads
    e = 2 if cfg.dtype == ri.DT_BF16 else 4
    g_ = cfg.groups if cfg.n_dec > 0 else 0
    hdr = b"RLTS" + struct.pack("<IQii", 1, checksum, pos_enc, pos_dec)
    hdr += struct.pack("<12i", cfg.vocab, cfg.d, cfg.heads, cfg.n_enc, cfg.n_dec, cfg.ffn,
                       cfg.window, cfg.groups, cfg.chunk, cfg.variant, int(cfg.tied), cfg.dtype)
    hdr += struct.pack("<3d", cfg.alpha, cfg.eps, cfg.rope_base)
    assert len(hdr) == 96
    hdr += bytes(128 - 96)
    body = (8 * cfg.d + 4 * pos_enc * cfg.d + (2 * h * cfg.n_enc + 2 * h * g_) * pos_enc * dh * e
            + 2 * h * cfg.n_dec * (cfg.window - 1) * dh * e)
    return bytearray(hdr + bytes(body))


@pytest.mark.parametrize("name", ["tiny_fp32", "parity_bf16", "s5_bf16", "rlt2_mod5_bf16"])
def test_snapshot_info_reads_the_documented_layout(lib, name):
    cfg = ri.CONFIGS[name]
    snap = _snapshot_bytes(cfg, 7, 5)
    c, pe, pd = lib.snapshot_info(bytes(snap))
    assert (pe, pd) == (7, 5)
    for f in ("vocab", "d", "heads", "n_enc", "n_dec", "ffn", "window", "groups", "chunk",
              "variant", "dtype"):
        assert getattr(c, f) == getattr(cfg, f), f
    assert (c.alpha, c.eps, c.rope_base) == (cfg.alpha, cfg.eps, cfg.rope_base)
    # a fresh row (nothing encoded) has only s, R and the rings
    c0, pe0, pd0 = lib.snapshot_info(bytes(_snapshot_bytes(cfg, 0, 0)))
    assert (pe0, pd0) == (0, 0)


def test_snapshot_info_rejects_malformed(lib):
    cfg = ri.CONFIGS["parity_bf16"]
    good = _snapshot_bytes(cfg, 6, 6)
    info = lambda b: lib.rlt_snapshot_info(np.frombuffer(bytes(b), np.uint8).copy(), len(b))[0]  # noqa: E731
    assert info(good) == lib.RLT_OK
    bad = bytearray(good); bad[0:4] = b"RLTB"                      # magic
    assert info(bad) == lib.RLT_E_SNAPSHOT
    bad = bytearray(good); bad[4] = 2                              # version
    assert info(bad) == lib.RLT_E_SNAPSHOT
    bad = bytearray(good); bad[100] = 1                            # reserved bytes
    assert info(bad) == lib.RLT_E_SNAPSHOT
    assert info(good[:-1]) == lib.RLT_E_SNAPSHOT                   # truncated
    assert info(good + b"\0") == lib.RLT_E_SNAPSHOT               # trailing byte
    assert info(good[:100]) == lib.RLT_E_SNAPSHOT                  # shorter than a header
    assert info(_snapshot_bytes(cfg, 3, 4)) == lib.RLT_E_SNAPSHOT  # pos_dec > pos_enc
    bad = _snapshot_bytes(cfg, 0, 0); bad[16:20] = (-1).to_bytes(4, "little", signed=True)
    assert info(bad) == lib.RLT_E_SNAPSHOT                         # negative pos_enc
    # the size follows pos_enc: a snapshot relabelled with another pos_enc no longer fits
    bad = bytearray(good); bad[16] = 7
    assert info(bad) == lib.RLT_E_SNAPSHOT
    # heads not dividing d
    bad = bytearray(good); bad[32:36] = (7).to_bytes(4, "little")
    assert info(bad) == lib.RLT_E_SNAPSHOT


# ---------------------------------------------------------------- blob parser
def _no_gpu():
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("a GPU is present: a valid blob would create a model")


def test_every_config_blob_parses(lib):
    """Each workload's blob (the large one at full width and vocabulary on a
    2+2-layer slice; zero weights, which the parser does not look at) gets
    past the parser: without a device the call ends at RLT_E_DEVICE."""
    _no_gpu()
    for name, cfg in ri.CONFIGS.items():
        if name == "large_bf16":
            cfg = cfg.replace(n_enc=2, n_dec=2)
        W = {n: np.zeros(shape, np.float32) for n, shape in ri.manifest(cfg)}
        assert lib.rlt_create(ri.write_blob(cfg, W))[0] == lib.RLT_E_DEVICE, name


def _fix_checksum(blob: bytearray) -> bytearray:
    import struct
    struct.pack_into("<Q", blob, 104, ri.blob_checksum(bytes(blob[256:])))
    return blob


_TINY_BLOB = None


def _tiny_blob() -> bytes:
    global _TINY_BLOB
    if _TINY_BLOB is None:
        _TINY_BLOB = _blob()[1]
    return _TINY_BLOB


def test_malformed_headers_fail_cleanly(lib):
    """Random header fields (with a matching payload checksum, so every check
    of the config and the manifest is reached) are rejected with an error
    code: no crash, no overflow, no huge manifest."""
    import struct
    from hypothesis import HealthCheck, given, settings
    from hypothesis import strategies as st
    _no_gpu()
    edge = st.sampled_from([-(2 ** 31), -1, 0, 1, 2, 3, 4, 8, 64, 4096, 4097, 1 << 16,
                            (1 << 16) + 1, 1 << 20, (1 << 20) + 1, 1 << 24, (1 << 24) + 1,
                            2 ** 31 - 1])
    i32 = st.one_of(st.integers(-(2 ** 31), 2 ** 31 - 1), edge)

    @settings(max_examples=400, deadline=None, derandomize=True,
              suppress_health_check=list(HealthCheck))
    @given(fields=st.lists(i32, min_size=12, max_size=12),
           keep=st.lists(st.booleans(), min_size=12, max_size=12),
           nt=st.one_of(st.just(None), st.integers(0, 2 ** 64 - 1)))
    def run(fields, keep, nt):
        blob = bytearray(_tiny_blob())
        orig = struct.unpack_from("<12i", blob, 8)
        struct.pack_into("<12i", blob, 8, *[o if k else f for o, k, f in zip(orig, keep, fields)])
        if nt is not None:
            struct.pack_into("<Q", blob, 88, nt)
        code = lib.rlt_create(bytes(blob))[0]
        assert code in (lib.RLT_E_BLOB, lib.RLT_E_UNSUPPORTED, lib.RLT_E_DEVICE), code

    run()


def test_malformed_records_fail_cleanly(lib):
    """Random bytes written over the tensor records (checksum fixed up) are
    rejected, or -- where they only hit weight values -- still parse."""
    from hypothesis import HealthCheck, given, settings
    from hypothesis import strategies as st
    _no_gpu()
    base = _tiny_blob()

    @settings(max_examples=300, deadline=None, derandomize=True,
              suppress_health_check=list(HealthCheck))
    @given(at=st.integers(256, min(len(base) - 1, 256 + 8192)),
           data=st.binary(min_size=1, max_size=16))
    def run(at, data):
        blob = bytearray(base)
        blob[at:at + len(data)] = data
        blob = _fix_checksum(blob[:len(base)] if len(blob) > len(base) else blob)
        code = lib.rlt_create(bytes(blob))[0]
        assert code in (lib.RLT_E_BLOB, lib.RLT_E_DEVICE), code

    run()


# ---------------------------------------------------------------- binding guards
def test_owner_methods_reject_wrong_buffers_before_the_library(lib):
    """The owners check element types and sizes of caller buffers before any
    library call (the library reads raw memory): checked here on a State
    shell whose handle would fail any real call."""
    cfg = ri.CONFIGS["tiny_fp32"]
    model = lib.Model.__new__(lib.Model)
    model.handle, model.config, model.device = None, lib.rlt_config(vocab=cfg.vocab, d=cfg.d), 0
    st = lib.State.__new__(lib.State)
    st.model, st.batch, st.max_len, st.handle = model, 2, 8, None
    with pytest.raises(TypeError, match="int32"):
        st.encode(np.zeros((2, 3), np.int64))          # numpy's default integer
    with pytest.raises(ValueError, match="shape"):
        st.encode(np.zeros((3, 3), np.int32))          # rows != batch
    with pytest.raises(ValueError, match="shape"):
        st.encode(np.zeros(6, np.int32))
    with pytest.raises(TypeError, match="float32"):
        st.readout(logits=np.zeros((2, cfg.vocab), np.float64))
    with pytest.raises(ValueError, match="elements"):
        st.readout(logits=np.zeros((2, cfg.vocab - 1), np.float32))
    with pytest.raises(TypeError, match="int32"):
        st.readout(argmax=np.zeros(2, np.int64))
    with pytest.raises(ValueError, match="elements"):
        st.readout(sampled=np.zeros(3, np.int32))
    with pytest.raises(TypeError, match="int32"):
        st.replay_logprobs(np.zeros((2, 4), np.int64))
    with pytest.raises(ValueError, match="elements"):
        st.replay_logprobs(np.zeros((2, 4), np.int32), logprobs=np.zeros((2, 3), np.float32))
    with pytest.raises(TypeError, match="uint8"):
        st.load(0, np.zeros(200, np.float32))
    with pytest.raises(TypeError, match="float32"):
        model.readout_rows(np.zeros((2, cfg.d), np.float64))
    with pytest.raises(ValueError, match="elements"):
        model.readout_rows(np.zeros((2, cfg.d), np.float32), logits=np.zeros(5, np.float32))
    torch = pytest.importorskip("torch")
    with pytest.raises(TypeError, match="int32"):
        st.encode(torch.zeros(2, 3, dtype=torch.int64))
    lib._check_buf(torch.zeros(2, 3, dtype=torch.int32), "int32", "t", 6, rows=2)
    lib._check_buf(np.zeros((2, 3), np.int32), "int32", "t", 6, rows=2)


def test_header_is_plain_c_and_links(lib, tmp_path):
    """include/rlt.h compiles as C99 with warnings as errors, and a C program
    links against librlt.so and calls functions that need no device."""
    src = tmp_path / "abi.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "rlt.h"
int main(void) {
    rlt_config c;
    int32_t pe = -1, pd = -1;
    unsigned char junk[RLT_SNAPSHOT_HEADER_BYTES];
    memset(junk, 0, sizeof junk);
    if (rlt_snapshot_info(junk, sizeof junk, &c, &pe, &pd) != RLT_E_SNAPSHOT) return 1;
    if (rlt_snapshot_info(NULL, 0, NULL, NULL, NULL) != RLT_E_ARG) return 2;
    if (rlt_step(NULL, NULL) != RLT_E_ARG) return 3;
    if (strcmp(rlt_strerror(RLT_OK), "ok") != 0) return 4;
    printf("%s|%s\n", rlt_strerror(RLT_E_SNAPSHOT), rlt_strerror(RLT_E_UNSUPPORTED));
    return 0;
}
''')
    exe = tmp_path / "abi"
    libdir = os.path.dirname(lib.LIB_PATH)
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                        "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                        "-L", libdir, "-lrlt", f"-Wl,-rpath,{libdir}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, (r.returncode, r.stderr)
    assert r.stdout.strip() == f"{lib.rlt_strerror(-9)}|{lib.rlt_strerror(-8)}"

"""Python binding of librlt.so: argument marshalling only.

Every function named ``rlt_*`` here forwards to the C function of the same
name in ``include/rlt.h``; buffers may be torch tensors (host or CUDA),
numpy arrays or raw integer addresses, and streams torch.cuda.Stream objects,
raw handles or None (legacy default stream).  All computation runs in the
library's CUDA kernels; there is no fallback: if librlt.so is missing or does
not load, importing this package raises.

``Model`` and ``State`` are small owners that call the same functions; they
also check the element types and sizes of the buffers they are given (the
library reads raw memory), which the ``rlt_*`` functions leave to the caller.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
# RLT_LIB=debug loads the bounds-checking build (librlt_debug.so) instead
LIB_PATH = os.path.join(_HERE, "librlt_debug.so" if os.environ.get("RLT_LIB") == "debug"
                        else "librlt.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "rlt.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{os.path.basename(LIB_PATH)} not built at {LIB_PATH}; run "
                      f"`python stateful_decoding_b200/build.py`"
                      f"{' --debug' if LIB_PATH.endswith('_debug.so') else ''}")
_lib = ctypes.CDLL(LIB_PATH)

RLT_OK, RLT_E_ARG, RLT_E_OOM, RLT_E_CAPACITY, RLT_E_ORDER = 0, -1, -2, -3, -4
RLT_E_BLOB, RLT_E_DEVICE, RLT_E_TIMEOUT, RLT_E_UNSUPPORTED = -5, -6, -7, -8
RLT_E_SNAPSHOT = -9
RLT_BUILD_DEBUG = 1
SNAPSHOT_HEADER_BYTES = 128                # RLT_SNAPSHOT_HEADER_BYTES
PART_S, PART_R, PART_E, PART_MEM, PART_RING, PART_ENC = range(6)
PROF_XATTN, PROF_SWA, PROF_STEP, PROF_ENC, PROF_ENC1 = range(5)
PROF_NCLS = 5          # cls + PROF_NCLS * (layer + 1): one decoder layer's launches
READOUT_ROWS_SCRATCH_BYTES = 16 << 20      # RLT_READOUT_ROWS_SCRATCH_BYTES


class rlt_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("vocab", "d", "heads", "n_enc", "n_dec", "ffn",
                                               "window", "groups", "chunk", "variant", "tied",
                                               "dtype")] + \
               [("alpha", ctypes.c_double), ("eps", ctypes.c_double), ("rope_base", ctypes.c_double)]


_vp, _i, _sz, _u64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint64
_SIGS = {
    "rlt_create": (_i, [_vp, _sz, _i, ctypes.POINTER(_vp)]),
    "rlt_destroy": (None, [_vp]),
    "rlt_model_config": (_i, [_vp, ctypes.POINTER(rlt_config)]),
    "rlt_state_create": (_i, [_vp, _i, _i, ctypes.POINTER(_vp)]),
    "rlt_state_destroy": (None, [_vp]),
    "rlt_state_bytes": (_i, [_vp, ctypes.POINTER(_sz), ctypes.POINTER(_sz)]),
    "rlt_state_reset": (_i, [_vp, _vp, _i, _vp]),
    "rlt_encode": (_i, [_vp, _vp, _i, _vp]),
    "rlt_step": (_i, [_vp, _vp]),
    "rlt_prefill": (_i, [_vp, _i, _vp]),
    "rlt_readout": (_i, [_vp, _vp, _vp, _vp, _u64, _u64, ctypes.c_float, _vp]),
    "rlt_readout_rows": (_i, [_vp, _vp, _i, _vp, _vp, _vp, _u64, _u64, ctypes.c_float, _vp]),
    "rlt_replay_logprobs": (_i, [_vp, _vp, _i, _vp, ctypes.c_float, _vp]),
    "rlt_prefill_packed": (_i, [_vp, _vp, _vp, _i, _vp]),
    "rlt_state_positions": (_i, [_vp, _vp, _vp]),
    "rlt_state_read": (_i, [_vp, _i, _vp, _sz, ctypes.POINTER(_sz), _vp]),
    "rlt_state_check": (_i, [_vp, _vp]),
    "rlt_selftest_wait": (_i, [_vp, _i, ctypes.c_uint32, _vp]),
    "rlt_state_save": (_i, [_vp, _i, _vp, _sz, ctypes.POINTER(_sz), _vp]),
    "rlt_state_load": (_i, [_vp, _i, _vp, _sz, _vp]),
    "rlt_snapshot_info": (_i, [_vp, _sz, ctypes.POINTER(rlt_config), ctypes.POINTER(ctypes.c_int32),
                               ctypes.POINTER(ctypes.c_int32)]),
    "rlt_kernel_launches": (_u64, []),
    "rlt_build_flags": (ctypes.c_uint32, []),
    "rlt_debug_set_positions": (_i, [_vp, _i, ctypes.c_int32, ctypes.c_int32, _vp]),
    "rlt_strerror": (ctypes.c_char_p, [_i]),
    "rlt_profile_enable": (_i, [_vp, _i]),
    "rlt_profile_query": (_i, [_vp, _i, ctypes.POINTER(_u64), ctypes.POINTER(ctypes.c_double),
                               ctypes.POINTER(ctypes.c_double), _vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype, _f.argtypes = _res, _args


def header_functions() -> list:
    """Names of the functions include/rlt.h declares."""
    src = open(HEADER_PATH).read()
    return sorted(set(re.findall(r"\b(rlt_[a-z_]+)\s*\(", src)))


class RLTError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {rlt_strerror(code)} ({code})")
        self.code = code


def _check(code: int, what: str) -> int:
    if code != RLT_OK:
        raise RLTError(code, what)
    return code


def _ptr(x) -> Optional[int]:
    """Address of a buffer: torch tensor, numpy array, int, or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        if not x.is_contiguous():
            raise ValueError("buffer must be contiguous")
        return x.data_ptr()
    if hasattr(x, "ctypes"):
        if not x.flags["C_CONTIGUOUS"]:
            raise ValueError("buffer must be C-contiguous")
        return x.ctypes.data
    raise TypeError(f"cannot take the address of {type(x)}")


def _numel(x) -> int:
    return int(x.numel()) if hasattr(x, "numel") else int(x.size)


def _check_buf(x, dtype: str, what: str, numel: Optional[int] = None,
               rows: Optional[int] = None) -> None:
    """The owners' guard on caller buffers (numpy arrays or torch tensors):
    element type `dtype` ('int32', 'float32' or 'uint8'), and `numel`
    elements in all or a 2-D shape with `rows` rows, when given.  The library
    reads raw memory: an int64 token array would be read as pairs of int32."""
    if x is None:
        return
    dt = getattr(x, "dtype", None)
    name = str(dt).replace("torch.", "") if dt is not None else None
    if name != dtype:
        raise TypeError(f"{what}: element type {dt}, expected {dtype}")
    if rows is not None and (len(x.shape) != 2 or int(x.shape[0]) != rows):
        raise ValueError(f"{what}: shape {tuple(x.shape)}, expected ({rows}, n)")
    if numel is not None and _numel(x) != numel:
        raise ValueError(f"{what}: {_numel(x)} elements, expected {numel}")


def _stream(s) -> Optional[int]:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


# ---------------------------------------------------------------- C names
def rlt_strerror(code: int) -> str:
    return _lib.rlt_strerror(code).decode()


def rlt_kernel_launches() -> int:
    return int(_lib.rlt_kernel_launches())


def rlt_create(blob: bytes, device: int = 0):
    h = _vp()
    buf = ctypes.create_string_buffer(blob, len(blob))
    code = _lib.rlt_create(buf, len(blob), device, ctypes.byref(h))
    return code, h.value


def rlt_destroy(model) -> None:
    _lib.rlt_destroy(model)


def rlt_model_config(model):
    c = rlt_config()
    return _lib.rlt_model_config(model, ctypes.byref(c)), c


def rlt_state_create(model, batch: int, max_len: int):
    h = _vp()
    code = _lib.rlt_state_create(model, batch, max_len, ctypes.byref(h))
    return code, h.value


def rlt_state_destroy(state) -> None:
    _lib.rlt_state_destroy(state)


def rlt_state_bytes(state):
    a, b = _sz(), _sz()
    return _lib.rlt_state_bytes(state, ctypes.byref(a), ctypes.byref(b)), a.value, b.value


def rlt_state_reset(state, rows=None, n: int = 0, stream=None) -> int:
    return _lib.rlt_state_reset(state, _ptr(rows), n, _stream(stream))


def rlt_encode(state, tokens, n: int, stream=None) -> int:
    return _lib.rlt_encode(state, _ptr(tokens), n, _stream(stream))


def rlt_step(state, stream=None) -> int:
    return _lib.rlt_step(state, _stream(stream))


def rlt_prefill(state, T: int, stream=None) -> int:
    return _lib.rlt_prefill(state, T, _stream(stream))


def rlt_readout(state, logits=None, argmax=None, sampled=None, rng_seed: int = 0,
                rng_step: int = 0, temperature: float = 1.0, stream=None) -> int:
    return _lib.rlt_readout(state, _ptr(logits), _ptr(argmax), _ptr(sampled), rng_seed, rng_step,
                            temperature, _stream(stream))


def rlt_readout_rows(model, s_rows, rows: int, logits=None, argmax=None, sampled=None,
                     rng_seed: int = 0, rng_step: int = 0, temperature: float = 1.0,
                     stream=None) -> int:
    return _lib.rlt_readout_rows(model, _ptr(s_rows), rows, _ptr(logits), _ptr(argmax),
                                 _ptr(sampled), rng_seed, rng_step, temperature, _stream(stream))


def rlt_replay_logprobs(state, tokens, n: int, logprobs, temperature: float = 1.0,
                        stream=None) -> int:
    return _lib.rlt_replay_logprobs(state, _ptr(tokens), n, _ptr(logprobs), temperature,
                                    _stream(stream))


def rlt_prefill_packed(state, tokens, doc_start, n: int, stream=None) -> int:
    return _lib.rlt_prefill_packed(state, _ptr(tokens), _ptr(doc_start), n, _stream(stream))


def readout_rows_scratch_bytes(rows: int, d: int, vocab: int, bf16: bool,
                               host_logits: bool) -> int:
    """Static scratch a rlt_readout_rows call needs (its limit is
    READOUT_ROWS_SCRATCH_BYTES)."""
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    return (up(rows * d * (2 if bf16 else 4)) + (up(rows * vocab * 4) if host_logits else 0)
            + up(rows * 8))


def rlt_state_positions(state, pos_enc=None, pos_dec=None) -> int:
    return _lib.rlt_state_positions(state, _ptr(pos_enc), _ptr(pos_dec))


def rlt_state_read(state, part: int, dst=None, nbytes: int = 0, stream=None):
    out = _sz()
    code = _lib.rlt_state_read(state, part, _ptr(dst), nbytes, ctypes.byref(out), _stream(stream))
    return code, out.value


def rlt_state_check(state, stream=None) -> int:
    return _lib.rlt_state_check(state, _stream(stream))


def rlt_build_flags() -> int:
    return _lib.rlt_build_flags()


def rlt_debug_set_positions(state, row: int, pos_enc: int, pos_dec: int, stream=None) -> int:
    return _lib.rlt_debug_set_positions(state, row, pos_enc, pos_dec, _stream(stream))


def rlt_selftest_wait(state, kind: int, polls: int, stream=None) -> int:
    return _lib.rlt_selftest_wait(state, kind, polls, _stream(stream))


def rlt_state_save(state, row: int, dst=None, nbytes: int = 0, stream=None):
    out = _sz()
    code = _lib.rlt_state_save(state, row, _ptr(dst), nbytes, ctypes.byref(out), _stream(stream))
    return code, out.value


def rlt_state_load(state, row: int, src, nbytes: int, stream=None) -> int:
    return _lib.rlt_state_load(state, row, _ptr(src), nbytes, _stream(stream))


def rlt_snapshot_info(snap, nbytes: int):
    """(code, rlt_config, pos_enc, pos_dec) of a snapshot in host memory."""
    c, pe, pd = rlt_config(), ctypes.c_int32(), ctypes.c_int32()
    code = _lib.rlt_snapshot_info(_ptr(snap), nbytes, ctypes.byref(c), ctypes.byref(pe),
                                  ctypes.byref(pd))
    return code, c, pe.value, pd.value


def _as_bytes_array(snap):
    """A host snapshot as a contiguous numpy uint8 array (bytes are copied)."""
    import numpy as np
    if isinstance(snap, (bytes, bytearray, memoryview)):
        return np.frombuffer(bytes(snap), np.uint8).copy()
    return snap


def snapshot_info(snap):
    """Config and positions of a snapshot held in host memory."""
    a = _as_bytes_array(snap)
    code, c, pe, pd = rlt_snapshot_info(a, a.nbytes)
    _check(code, "rlt_snapshot_info")
    return c, pe, pd


def rlt_profile_enable(state, on: bool) -> int:
    return _lib.rlt_profile_enable(state, int(on))


def rlt_profile_query(state, cls: int, stream=None):
    n, ms, by = _u64(), ctypes.c_double(), ctypes.c_double()
    code = _lib.rlt_profile_query(state, cls, ctypes.byref(n), ctypes.byref(ms), ctypes.byref(by),
                                  _stream(stream))
    return code, n.value, ms.value, by.value


# ---------------------------------------------------------------- owners
class Model:
    def __init__(self, blob: bytes, device: int = 0):
        code, self.handle = rlt_create(blob, device)
        _check(code, "rlt_create")
        code, self.config = rlt_model_config(self.handle)
        _check(code, "rlt_model_config")
        self.device = device

    def readout_rows(self, s_rows, logits=None, argmax=None, sampled=None, seed=0, step=0,
                     temperature=1.0, stream=None):
        """Readout of caller-supplied state vectors (device fp32 [rows][d])
        with no allocation: the scratch is a static device array."""
        rows = int(s_rows.shape[0])
        c = self.config
        _check_buf(s_rows, "float32", "s_rows", rows * c.d)
        _check_buf(logits, "float32", "logits", rows * c.vocab)
        _check_buf(argmax, "int32", "argmax", rows)
        _check_buf(sampled, "int32", "sampled", rows)
        code = rlt_readout_rows(self.handle, s_rows, rows, logits, argmax, sampled, seed, step,
                                temperature, stream)
        if code == RLT_E_ARG:
            c = self.config
            host_logits = logits is not None and not getattr(logits, "is_cuda", False)
            need = readout_rows_scratch_bytes(rows, c.d, c.vocab, c.dtype == 1, host_logits)
            if need > READOUT_ROWS_SCRATCH_BYTES:
                raise ValueError(
                    f"rlt_readout_rows: {rows} rows need {need} bytes of static scratch, more "
                    f"than its {READOUT_ROWS_SCRATCH_BYTES} bytes; split the rows over calls")
        return _check(code, "rlt_readout_rows")

    def close(self):
        if self.handle:
            rlt_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class State:
    def __init__(self, model: Model, batch: int, max_len: int):
        self.model = model
        self.batch, self.max_len = batch, max_len
        code, self.handle = rlt_state_create(model.handle, batch, max_len)
        _check(code, "rlt_state_create")

    def close(self):
        if self.handle:
            rlt_state_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def reset(self, rows: Optional[Sequence[int]] = None, stream=None):
        if rows is None:
            return _check(rlt_state_reset(self.handle, None, 0, stream), "rlt_state_reset")
        import numpy as np
        r = np.ascontiguousarray(rows, dtype=np.int32)
        return _check(rlt_state_reset(self.handle, r, len(r), stream), "rlt_state_reset")

    def encode(self, tokens, stream=None):
        """Append int32 [batch][n] tokens (host numpy / torch, or CUDA)."""
        _check_buf(tokens, "int32", "tokens", rows=self.batch)
        n = int(tokens.shape[1])
        return _check(rlt_encode(self.handle, tokens, n, stream), "rlt_encode")

    def step(self, stream=None):
        return _check(rlt_step(self.handle, stream), "rlt_step")

    def prefill(self, T: int, stream=None):
        return _check(rlt_prefill(self.handle, T, stream), "rlt_prefill")

    def readout(self, logits=None, argmax=None, sampled=None, seed=0, step=0, temperature=1.0,
                stream=None):
        """Outputs (each optional, host or CUDA): logits fp32 [batch][vocab],
        argmax and sampled int32 [batch]."""
        _check_buf(logits, "float32", "logits", self.batch * self.model.config.vocab)
        _check_buf(argmax, "int32", "argmax", self.batch)
        _check_buf(sampled, "int32", "sampled", self.batch)
        return _check(rlt_readout(self.handle, logits, argmax, sampled, seed, step, temperature,
                                  stream), "rlt_readout")

    def replay_logprobs(self, tokens, logprobs=None, temperature=1.0, stream=None):
        """log p of each given token (int32 [batch][n]) read before it is
        consumed; returns `logprobs` (fp32 [batch][n], host numpy by default)."""
        import numpy as np
        _check_buf(tokens, "int32", "tokens", rows=self.batch)
        n = int(tokens.shape[1])
        if logprobs is None:
            logprobs = np.empty((self.batch, n), np.float32)
        _check_buf(logprobs, "float32", "logprobs", self.batch * n)
        _check(rlt_replay_logprobs(self.handle, tokens, n, logprobs, temperature, stream),
               "rlt_replay_logprobs")
        return logprobs

    def prefill_packed(self, tokens, doc_start, stream=None):
        """Encode and consume int32 [batch][n] tokens holding packed documents;
        doc_start (host, bool or uint8 [batch][n]) marks where each starts."""
        import numpy as np
        _check_buf(tokens, "int32", "tokens", rows=self.batch)
        n = int(tokens.shape[1])
        starts = np.ascontiguousarray(doc_start, dtype=np.uint8)
        if starts.shape != (self.batch, n):
            raise ValueError(f"doc_start: shape {starts.shape}, expected ({self.batch}, {n})")
        return _check(rlt_prefill_packed(self.handle, tokens, starts, n, stream),
                      "rlt_prefill_packed")

    def positions(self):
        import numpy as np
        pe = np.zeros(self.batch, np.int32)
        pd = np.zeros(self.batch, np.int32)
        _check(rlt_state_positions(self.handle, pe, pd), "rlt_state_positions")
        return pe, pd

    def read(self, part: int, stream=None):
        """Copy a state component to a new host numpy array (raw element type)."""
        import numpy as np
        code, nbytes = rlt_state_read(self.handle, part)
        _check(code, "rlt_state_read")
        buf = np.empty(nbytes, np.uint8)
        _check(rlt_state_read(self.handle, part, buf, nbytes, stream)[0], "rlt_state_read")
        return buf

    def check(self, stream=None):
        return _check(rlt_state_check(self.handle, stream), "rlt_state_check")

    def save(self, row: int, dst=None, stream=None):
        """Snapshot of one row: into a new host numpy uint8 array, or into
        `dst` (a host or CUDA buffer of exactly the snapshot's size)."""
        import numpy as np
        code, nbytes = rlt_state_save(self.handle, row)
        _check(code, "rlt_state_save")
        if dst is None:
            dst = np.empty(nbytes, np.uint8)
        _check_buf(dst, "uint8", "snapshot buffer", nbytes)
        _check(rlt_state_save(self.handle, row, dst, nbytes, stream)[0], "rlt_state_save")
        return dst

    def load(self, row: int, snap, stream=None):
        """Replace one row with a snapshot (host bytes / numpy, or a CUDA tensor)."""
        a = _as_bytes_array(snap)
        _check_buf(a, "uint8", "snapshot")
        nbytes = _numel(a)
        return _check(rlt_state_load(self.handle, row, a, nbytes, stream), "rlt_state_load")

    def profile(self, on: int):
        """0: off; 1: time kernel classes (graph-replayed transition blocks
        as whole blocks); 2: also every attention launch inside the graphs."""
        return _check(rlt_profile_enable(self.handle, int(on)), "rlt_profile_enable")

    def profile_query(self, cls: int, stream=None):
        """(launches, total_ms, algorithmic_bytes) of a kernel class since enable."""
        code, n, ms, by = rlt_profile_query(self.handle, cls, stream)
        _check(code, "rlt_profile_query")
        return n, ms, by

    def bytes(self):
        code, per_row, total = rlt_state_bytes(self.handle)
        _check(code, "rlt_state_bytes")
        return per_row, total

"""Seeded synthetic inputs shared by the CPU oracle and the CUDA library.

This module holds the workload definitions (model shapes and input recipes),
the counter-based random generator, the weight manifest and the weight-blob
file format.  It contains none of the model's arithmetic: no norm, attention,
gate or readout.  Both implementations read the same blob and the same token
arrays, and each computes everything else on its own.

Random numbers
--------------
SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
generators", OOPSLA 2014): the k-th output of a stream seeded with ``s`` is
``mix64(s + k * GOLDEN)`` for k = 1, 2, ...  Normals use the Box-Muller
transform (Box and Muller, 1958), cosine branch only: one normal per pair of
uniforms.  Both are written out here from their published definitions.

Workloads
---------
The five workloads mirror the shapes of the tasks the pages train on
(greeksharifa summary "Recurrent Looped Transformer 요약 설명", §3.1 and App. J;
jiphyeonjeon.kr review "Recurrent Looped Transformer", §2): width 512, FFN
1365 (= floor(8*512/3)), window 64, plus a tiny fp32 model (the tistory
smoke-test shape, ch4u.tistory.com "Recurrent Looped Transformer란?", §4-§5)
and a large tied model.  Weights are N(0, 0.02) with gains 1 and gate bias 0.
"""
from __future__ import annotations

import dataclasses
import struct
from dataclasses import dataclass
from typing import Dict, List, Tuple

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
MASK64 = (1 << 64) - 1

WEIGHT_SEED = 42          # first initialisation seed on the pages (greeksharifa §3.1)
TOKEN_SEED = 20260916     # the pages' test-data seed (greeksharifa App. J.5)
SAMPLE_SEED = 42

# ----------------------------------------------------------------------------
# SplitMix64
# ----------------------------------------------------------------------------


def mix64_int(z: int) -> int:
    """SplitMix64 finaliser on a Python int (scalar reference)."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def splitmix64_stream_int(seed: int, n: int) -> List[int]:
    """First n outputs of SplitMix64 seeded with ``seed`` (scalar reference)."""
    out, s = [], seed & MASK64
    for _ in range(n):
        s = (s + 0x9E3779B97F4A7C15) & MASK64
        out.append(mix64_int(s))
    return out


def mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 finaliser, vectorised over uint64 arrays (wrapping arithmetic)."""
    z = z.astype(np.uint64, copy=True)
    with np.errstate(over="ignore"):
        z ^= z >> np.uint64(30)
        z *= _M1
        z ^= z >> np.uint64(27)
        z *= _M2
        z ^= z >> np.uint64(31)
    return z


def splitmix64_stream(seed: int, start: int, n: int) -> np.ndarray:
    """Outputs start+1 .. start+n of the SplitMix64 stream seeded with ``seed``."""
    k = np.arange(start + 1, start + n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return mix64(np.uint64(seed & MASK64) + k * GOLDEN)


def u53(x: np.ndarray) -> np.ndarray:
    """Map uint64 to a double in [0, 1) using its top 53 bits."""
    return (x >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


def substream_key(seed: int, *labels: int) -> int:
    """Derive an independent stream key from a seed and integer labels."""
    key = seed & MASK64
    for lab in labels:
        key = mix64_int((key ^ mix64_int((lab + 1) * 0x9E3779B97F4A7C15)) & MASK64)
    return key


def normal(seed: int, n: int, std: float, start: int = 0) -> np.ndarray:
    """Draws start .. start+n-1 of N(0, std^2) by Box-Muller (cosine branch)
    from one SplitMix64 stream: draw i uses stream outputs 2i+1 and 2i+2, so
    any range of draws can be produced on its own."""
    raw = splitmix64_stream(seed, 2 * start, 2 * n)
    u1 = (raw[0::2] >> np.uint64(11)).astype(np.float64) + 1.0
    u1 *= 1.0 / 9007199254740992.0          # (0, 1]: log never sees 0
    u2 = u53(raw[1::2])
    return std * np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


def sample_uniform(seed: int, row: int, step: int) -> float:
    """The sampler's uniform for (row, step): u53(mix64(key(seed,row) + (step+1)*GOLDEN)).

    The readout's inverse-CDF sampler consumes this value.  Both the CUDA
    library and the oracle tests implement the same definition.
    """
    key = substream_key(seed, row)
    return (mix64_int((key + (step + 1) * 0x9E3779B97F4A7C15) & MASK64) >> 11) / 9007199254740992.0


# ----------------------------------------------------------------------------
# bf16 storage rounding (round to nearest even), used to store bf16 weights
# ----------------------------------------------------------------------------


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest, ties to even (finite inputs)."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    with np.errstate(over="ignore"):
        r = (b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (h.astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------------------
# Configurations
# ----------------------------------------------------------------------------

DT_F32 = 0
DT_BF16 = 1


@dataclass(frozen=True)
class RLTConfig:
    name: str
    vocab: int
    d: int
    heads: int
    n_enc: int            # L_E
    n_dec: int            # L_D
    ffn: int              # f, SwiGLU hidden width
    window: int           # W (current token included)
    groups: int           # G: 1 (shared memory) or n_dec (per-layer projections)
    chunk: int = 1        # B_c: feedback interval (1 = RLT-1)
    variant: int = 1      # 0 = RLT-0 (no feedback), 1 = RLT-1, 2 = RLT-2
    tied: bool = False    # encoder layer l shares attention and FFN with decoder layer l
    dtype: int = DT_BF16
    alpha: float = 0.1
    eps: float = 1e-6
    rope_base: float = 10000.0
    # workload
    batch: int = 1
    prompt: int = 16
    decode: int = 0
    token_recipe: str = "uniform"

    @property
    def head_dim(self) -> int:
        return self.d // self.heads

    def replace(self, **kw) -> "RLTConfig":
        return dataclasses.replace(self, **kw)

    def validate(self) -> None:
        assert self.d % self.heads == 0 and self.head_dim % 2 == 0
        assert self.window >= 1 and self.chunk >= 1
        assert self.variant in (0, 1, 2)
        assert self.groups in (1, max(1, self.n_dec))
        if self.variant != 2:
            assert self.chunk == 1
        if self.tied:
            assert self.n_enc == self.n_dec


CONFIGS: Dict[str, RLTConfig] = {
    # Tiny RLT-1 fp32: vocab 32, d=64, 2+2 layers, 4 heads x 16, FFN 4d, W=4, G=1,
    # batch 2 x 16 uniform tokens, 6 sampled continuation tokens.
    "tiny_fp32": RLTConfig("tiny_fp32", vocab=32, d=64, heads=4, n_enc=2, n_dec=2, ffn=256,
                           window=4, groups=1, dtype=DT_F32, batch=2, prompt=16, decode=6,
                           token_recipe="uniform"),
    # Parity-shaped RLT-1 bf16: vocab {0,1,BOS,SEP}, d=512, 8 heads, 5+3, W=64, G=1,
    # batch 256 x 256 = [BOS, 254 Bernoulli(0.5) bits, SEP].
    "parity_bf16": RLTConfig("parity_bf16", vocab=4, d=512, heads=8, n_enc=5, n_dec=3, ffn=1365,
                             window=64, groups=1, batch=256, prompt=256, token_recipe="parity"),
    # S5-tracking-shaped RLT-1 bf16: vocab 12 (identity, 10 transpositions, BOS),
    # d=512, 8 heads, 4+4, W=64, G=L_D, batch 512 x 256 = [BOS, 255 uniform ops].
    "s5_bf16": RLTConfig("s5_bf16", vocab=12, d=512, heads=8, n_enc=4, n_dec=4, ffn=1365,
                         window=64, groups=4, batch=512, prompt=256, token_recipe="s5"),
    # RLT-2 chunked feedback (B_c=4) bf16: d=512, 4+4, W=64, batch 1024 x 64 mod-5
    # expression tokens (digits 0-4, + - * =, BOS).
    "rlt2_mod5_bf16": RLTConfig("rlt2_mod5_bf16", vocab=10, d=512, heads=8, n_enc=4, n_dec=4,
                                ffn=1365, window=64, groups=1, chunk=4, variant=2, batch=1024,
                                prompt=64, token_recipe="mod5"),
    # Large RLT-1 bf16: vocab 32000, d=2048, 16 heads x 128, 24+24 tied, W=256, G=1,
    # batch 64, 4096-token prompt + 512 decoded, Zipf(1.1) tokens.
    "large_bf16": RLTConfig("large_bf16", vocab=32000, d=2048, heads=16, n_enc=24, n_dec=24,
                            ffn=5461, window=256, groups=1, tied=True, batch=64, prompt=4096,
                            decode=512, token_recipe="zipf"),
}
CONFIG_ORDER = ["tiny_fp32", "parity_bf16", "s5_bf16", "rlt2_mod5_bf16", "large_bf16"]


# ----------------------------------------------------------------------------
# Weight manifest
# ----------------------------------------------------------------------------


def manifest(cfg: RLTConfig) -> List[Tuple[str, Tuple[int, ...]]]:
    """Names and shapes of every stored tensor, in blob order.

    Matrices follow the y = W x convention: shape [out, in].  With ``tied``
    the encoder layers store only their norms; their attention and FFN
    matrices are the decoder layer's of the same index.
    """
    d, f, V = cfg.d, cfg.ffn, cfg.vocab
    out: List[Tuple[str, Tuple[int, ...]]] = [("embed", (V, d))]
    if cfg.variant != 0:
        out.append(("s_star", (d,)))
    for l in range(cfg.n_enc):
        p = f"enc.{l}."
        out.append((p + "attn_norm", (d,)))
        if not cfg.tied:
            out += [(p + "wq", (d, d)), (p + "wk", (d, d)), (p + "wv", (d, d)), (p + "wo", (d, d))]
        out.append((p + "ffn_norm", (d,)))
        if not cfg.tied:
            out += [(p + "w1", (f, d)), (p + "w3", (f, d)), (p + "w2", (d, f))]
    if cfg.n_dec > 0:
        out.append(("mem_norm", (d,)))
        for g in range(cfg.groups):
            out += [(f"mem.{g}.wk", (d, d)), (f"mem.{g}.wv", (d, d))]
    if cfg.variant != 0:
        out += [("merge.norm", (d,)), ("merge.wg", (d, 2 * d)), ("merge.bg", (d,)),
                ("merge.ws", (d, d))]
    for l in range(cfg.n_dec):
        p = f"dec.{l}."
        out += [(p + "swa_norm", (d,)), (p + "wq", (d, d)), (p + "wk", (d, d)),
                (p + "wv", (d, d)), (p + "wo", (d, d)),
                (p + "x_norm", (d,)), (p + "xq", (d, d)), (p + "xo", (d, d)),
                (p + "ffn_norm", (d,)), (p + "w1", (f, d)), (p + "w3", (f, d)), (p + "w2", (d, f))]
    out += [("out_norm", (d,)), ("out", (V, d))]
    return out


def param_count(cfg: RLTConfig) -> int:
    return int(sum(int(np.prod(s)) for _, s in manifest(cfg)))


def _init_kind(name: str) -> str:
    if name.endswith("norm"):
        return "ones"
    if name == "merge.bg":
        return "zeros"
    return "normal"


_GEN_CHUNK = 1 << 22        # draws per piece when a tensor is generated in pieces


def generate_weights(cfg: RLTConfig, seed: int = WEIGHT_SEED, std: float = 0.02,
                     threads: int | None = None) -> Dict[str, np.ndarray]:
    """Seeded weights as float32 arrays (already bf16-valued for bf16 configs).

    Tensor k of the manifest draws from its own SplitMix64 substream, so any
    tensor can be regenerated alone.  Large tensors are produced in pieces of
    consecutive draws on a thread pool (numpy releases the GIL inside its
    array operations); the values do not depend on the number of threads.
    """
    cfg.validate()
    import concurrent.futures as cf
    import os
    W: Dict[str, np.ndarray] = {}
    jobs = []
    for k, (name, shape) in enumerate(manifest(cfg)):
        n = int(np.prod(shape))
        kind = _init_kind(name)
        if kind == "ones":
            W[name] = np.ones(shape, np.float32)
        elif kind == "zeros":
            W[name] = np.zeros(shape, np.float32)
        else:
            a = np.empty(n, np.float32)
            W[name] = a
            key = substream_key(seed, k)
            for i0 in range(0, n, _GEN_CHUNK):
                jobs.append((a, key, i0, min(n, i0 + _GEN_CHUNK)))

    def fill(job):
        a, key, i0, i1 = job
        v = normal(key, i1 - i0, std, start=i0).astype(np.float32)
        if cfg.dtype == DT_BF16:
            v = bf16_bits_to_f32(to_bf16_bits(v))
        a[i0:i1] = v

    nthr = threads if threads is not None else min(16, os.cpu_count() or 1)
    if nthr <= 1 or len(jobs) <= 1:
        for j in jobs:
            fill(j)
    else:
        with cf.ThreadPoolExecutor(nthr) as ex:
            list(ex.map(fill, jobs))
    for name, shape in manifest(cfg):
        W[name] = W[name].reshape(shape)
    return W


# ----------------------------------------------------------------------------
# Blob format
# ----------------------------------------------------------------------------
#
# Header (256 bytes, little endian):
#   0  char[4] magic "RLTB"        4  u32 version (=1)
#   8  u32 vocab, d, heads, n_enc, n_dec, ffn, window, groups, chunk, variant,
#          tied, dtype                                    (12 x u32, ends at 56)
#   56 f64 alpha, eps, rope_base                          (ends at 80)
#   80 u64 seed   88 u64 n_tensors   96 u64 payload_bytes   104 u64 checksum
#   112..255 zero
# Payload: n_tensors records, each a 64-byte record header
#   char[48] name (NUL padded), u32 ndim, u32 dtype, u32 dim0, u32 dim1
# followed by the tensor data (fp32 or bf16, row major), zero padded to a
# multiple of 64 bytes.  checksum = sum_i (w_i * (2 i + 1)) mod 2^64 over the
# payload read as little-endian u64 words w_i.

BLOB_MAGIC = b"RLTB"
BLOB_VERSION = 1
HEADER_BYTES = 256
RECORD_BYTES = 64


def blob_checksum(payload: bytes) -> int:
    n = len(payload) // 8 * 8
    w = np.frombuffer(payload[:n], dtype="<u8")
    idx = np.arange(w.size, dtype=np.uint64)
    with np.errstate(over="ignore"):
        s = np.sum(w * (np.uint64(2) * idx + np.uint64(1)), dtype=np.uint64)
    return int(s)


def write_blob(cfg: RLTConfig, W: Dict[str, np.ndarray], seed: int = WEIGHT_SEED) -> bytes:
    parts = []
    for name, shape in manifest(cfg):
        a = W[name]
        assert tuple(a.shape) == tuple(shape), (name, a.shape, shape)
        if cfg.dtype == DT_BF16:
            data = to_bf16_bits(a.reshape(-1)).tobytes()
        else:
            data = np.ascontiguousarray(a, np.float32).tobytes()
        dims = list(shape) + [1] * (2 - len(shape))
        rec = struct.pack("<48sIIII", name.encode(), len(shape), cfg.dtype, dims[0], dims[1])
        pad = (-len(data)) % 64
        parts += [rec, data, b"\0" * pad]
    payload = b"".join(parts)
    hdr = struct.pack("<4sI12I3d4Q", BLOB_MAGIC, BLOB_VERSION, cfg.vocab, cfg.d, cfg.heads,
                      cfg.n_enc, cfg.n_dec, cfg.ffn, cfg.window, cfg.groups, cfg.chunk,
                      cfg.variant, int(cfg.tied), cfg.dtype, cfg.alpha, cfg.eps, cfg.rope_base,
                      seed, len(manifest(cfg)), len(payload), blob_checksum(payload))
    hdr += b"\0" * (HEADER_BYTES - len(hdr))
    return hdr + payload


def read_blob(blob: bytes) -> Tuple[RLTConfig, Dict[str, np.ndarray]]:
    """Parse a blob back into a config and float32 weights (for round-trip tests)."""
    (magic, ver, V, d, h, le, ld, f, w, g, c, var, tied, dt, alpha, eps, base, seed, nt, nb,
     ck) = struct.unpack_from("<4sI12I3d4Q", blob, 0)
    assert magic == BLOB_MAGIC and ver == BLOB_VERSION
    payload = blob[HEADER_BYTES:HEADER_BYTES + nb]
    assert len(payload) == nb and blob_checksum(payload) == ck
    cfg = RLTConfig("blob", vocab=V, d=d, heads=h, n_enc=le, n_dec=ld, ffn=f, window=w, groups=g,
                    chunk=c, variant=var, tied=bool(tied), dtype=dt, alpha=alpha, eps=eps,
                    rope_base=base)
    W, off = {}, 0
    for _ in range(nt):
        name, nd, tdt, d0, d1 = struct.unpack_from("<48sIIII", payload, off)
        off += RECORD_BYTES
        n = d0 * d1
        nbytes = n * (2 if tdt == DT_BF16 else 4)
        raw = payload[off:off + nbytes]
        if tdt == DT_BF16:
            a = bf16_bits_to_f32(np.frombuffer(raw, np.uint16))
        else:
            a = np.frombuffer(raw, np.float32).copy()
        W[name.rstrip(b"\0").decode()] = a.reshape((d0, d1) if nd == 2 else (d0,))
        off += nbytes + ((-nbytes) % 64)
    return cfg, W


# ----------------------------------------------------------------------------
# Token streams
# ----------------------------------------------------------------------------


def _uniform_int(key: int, n: int, lo: int, hi: int) -> np.ndarray:
    return lo + np.floor(u53(splitmix64_stream(key, 0, n)) * (hi - lo)).astype(np.int64)


def make_tokens(cfg: RLTConfig, batch: int | None = None, length: int | None = None,
                seed: int = TOKEN_SEED, row0: int = 0) -> np.ndarray:
    """int32 [batch, length] prompt tokens for ``cfg.token_recipe``.

    Row r draws from substream (seed, recipe, row0 + r), so a row's tokens do
    not depend on the batch size it is generated in.
    """
    B = cfg.batch if batch is None else batch
    T = cfg.prompt if length is None else length
    rid = {"uniform": 0, "parity": 1, "s5": 2, "mod5": 3, "zipf": 4}[cfg.token_recipe]
    out = np.zeros((B, T), np.int32)
    for r in range(B):
        key = substream_key(seed, rid, row0 + r)
        if cfg.token_recipe == "uniform":
            row = _uniform_int(key, T, 0, cfg.vocab)
        elif cfg.token_recipe == "parity":        # 0/1 bits, BOS=2, SEP=3
            row = _uniform_int(key, T, 0, 2)
            row[0] = 2
            if T > 1:
                row[-1] = 3
        elif cfg.token_recipe == "s5":            # ops 0..10, BOS=11
            row = _uniform_int(key, T, 0, 11)
            row[0] = 11
        elif cfg.token_recipe == "mod5":          # digits 0-4, + - * = as 5 6 7 8, BOS=9
            dig = _uniform_int(key, T, 0, 5)
            ops = _uniform_int(substream_key(key, 1), T, 5, 8)
            row = np.where(np.arange(T) % 2 == 1, dig, ops)   # t=2,4,.. digits; 3,5,.. ops
            row[0] = 9
            if T >= 3:
                row[-2] = 8                       # '=' then an answer digit
                row[-1] = dig[-1]
        elif cfg.token_recipe == "zipf":          # BOS=0, then Zipf(1.1) over 1..V-1
            k = np.arange(1, cfg.vocab, dtype=np.float64)
            cdf = np.cumsum(k ** -1.1)
            cdf /= cdf[-1]
            u = u53(splitmix64_stream(key, 0, T))
            row = 1 + np.minimum(np.searchsorted(cdf, u, side="right"), cfg.vocab - 2)
            row[0] = 0
        else:
            raise ValueError(cfg.token_recipe)
        out[r] = row
    return out

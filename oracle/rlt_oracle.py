"""Plain CPU oracle of the Recurrent Looped Transformer transition.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module.  The
product path (``stateful_decoding_b200``) never imports, links or runs it, and
it never imports the product path.  The two share only the seeded inputs of
``rlt_inputs``.

What it computes, one sequence ("row") at a time, in float64:

* causal encoder e_{1:T} = E(x_{1:T}), runnable over any split of the tokens
  (parallel over a block, or one token at a time with the encoder cache C^E)
  -- jiphyeonjeon.kr review "Recurrent Looped Transformer", §3.2 (paper §2.4);
* encoder memory k^g_t = RoPE_t(W^g_K RMSNorm_E(e_t)), v^g_t = W^g_V RMSNorm_E(e_t)
  -- same review, §2 (paper eq. 2.1-2.2);
* the merge r = RMSNorm_s(s_{t-1}), g = sigmoid(W_g [e_t; r] + b_g),
  u_t = e_t + alpha * g (.) W_s r
  -- greeksharifa summary "Recurrent Looped Transformer 요약 설명", §2.5;
* L_D decoder blocks, each: causal sliding-window self-attention over the
  layer's cache (window W counts the current token; the current K/V come from
  the layer input before attention; after the update positions
  max(1, t-W+2)..t are kept), cross-attention to the memory prefix M_{<=t},
  and an FFN, with a residual around each sub-layer
  -- greeksharifa §2.5; jiphyeonjeon review §3.3 (paper eq. 2.12-2.16);
* the transition F_t and its composition from H_0 = (s_star, empty), the same
  for prompt and response tokens -- jiphyeonjeon review §3.1 (paper eq. 2.7);
* RLT-2 (register held inside B-token chunks counted from BOS, replaced by s
  at a complete chunk's end) and RLT-0 (u_t = e_t) -- greeksharifa §2.7, App. I;
* the readout: RMSNorm, linear map, softmax -- greeksharifa §2.3;
* the replay log-probabilities log p(y_i | c, y_<i), each read from the state
  that precedes the token -- jiphyeonjeon review §6.2 (paper eq. 5.3-5.5),
  greeksharifa App. D.3, F.4;
* packed documents, each restarting from H_0 -- jiphyeonjeon review §6.1,
  greeksharifa App. F.

Where the pages leave a step open (the block equations are missing from the
extracted text) this follows these readings: pre-norm RMSNorm (eps 1e-6,
learnable gain) before every sub-layer; rotate-half RoPE (base 10000, 1-based
positions) on every query and key; d_KV = d with h heads of d/h; scale
1/sqrt(d_h); SwiGLU FFN W_2(SiLU(W_1 y) * W_3 y); no biases except b_g; no
final encoder norm; the merge reads the raw encoder output e_t; untied readout.

Precision modes.  ``mode="fp64"`` computes everything in float64 on the
stored weights.  ``mode="bf16"`` rounds, in addition, at exactly the points
where the bf16 CUDA path stores bf16: every matrix-product input activation
-- the projections' inputs, and in the encoder's causal attention the query
and the probabilities, which enter the products q K^T and P V (the
normaliser then sums the rounded probabilities): at head size 64 with
prefixes of at most 256 keys always, otherwise in calls of at least
ENC_TC_MIN_POSITIONS tokens -- and every stored
key/value (encoder cache, memory, window cache; the current position's
key/value are used rounded too).  The decoder's attention of one position
is a matrix-vector computation on the CUDA path and keeps q and p
unrounded; a decoder block of DEC_MQ_MIN_POSITIONS .. DEC_MQ_MAX_POSITIONS
positions at head size 64 (an RLT-2 chunk, a short RLT-0 block) scores its
queries against each key tile as one small matrix product, so there q and p
are bf16 values as in the encoder (the window's only when W exceeds the
block).  Everything else stays float64.

Pinning: every function here is checked by ``tests/test_oracle_pins.py``
against identities the pages state (serving-split invariance, causality,
B=1 RLT-2 = RLT-1, encoder schedules), closed forms (one-key attention,
W=1 window, W >= T window = full causal attention, alpha = 0 = RLT-0,
saturated gates), independent parallel formulations (RLT-0 teacher-forced
pass; full-history windowed decoder), parameter counts printed on the pages,
and the random-init loss ~ ln V; the replay against closed forms of the
log-softmax, scipy's log_softmax, and the chain rule (the probabilities of all
continuations of a fixed length sum to one).  Absolute logit values have no worked
example on the pages: beyond those identities they are parity unpinned.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence

import numpy as np


# Encode calls of at least this many tokens form the encoder attention's
# products from bf16 q and probabilities in mode "bf16" at any head size and
# prefix length (see RLTOracle.encode).
ENC_TC_MIN_POSITIONS = 16
# decoder blocks of this many positions (head size 64, bf16) multiply q and
# the probabilities as bf16 values (the multi-query tile products)
DEC_MQ_MIN_POSITIONS = 2
DEC_MQ_MAX_POSITIONS = 16

# ----------------------------------------------------------------------------
# Scalar helpers (float64)
# ----------------------------------------------------------------------------


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 -> float32 -> bfloat16 (nearest, ties to even), as float64.

    The CUDA path holds fp32 values before it stores bf16, hence the fp32 step.
    """
    f = np.asarray(x, dtype=np.float32)
    b = f.view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def rmsnorm(x: np.ndarray, gain: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * gain over the last axis."""
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * gain


def rope(x: np.ndarray, pos: np.ndarray, base: float) -> np.ndarray:
    """Rotate-half rotary embedding of x[..., n, h, dh] at 1-based positions pos[n].

    Pair (i, i + dh/2) turns by the angle pos * base^(-2i/dh).
    """
    dh = x.shape[-1]
    half = dh // 2
    inv = base ** (-2.0 * np.arange(half, dtype=np.float64) / dh)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv[None, :]     # [n, half]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, rounded: bool = False) -> np.ndarray:
    """Per-head softmax attention of one query q[h,dh] over keys K[m,h,dh].

    With ``rounded`` the query and the probabilities exp(s - max s) are bf16
    values -- they are the inputs of the two matrix products q K^T and P V --
    and the normaliser is the sum of the rounded probabilities."""
    scale = 1.0 / np.sqrt(q.shape[-1])
    if rounded:
        q = round_bf16(q)
    s = np.einsum("hd,mhd->hm", q, K) * scale
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    if rounded:
        p = round_bf16(p)
    p = p / p.sum(axis=1, keepdims=True)
    return np.einsum("hm,mhd->hd", p, V)


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def sigmoid(x: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-x))


# ----------------------------------------------------------------------------
# State
# ----------------------------------------------------------------------------


@dataclass
class RowState:
    """Everything one sequence carries: H_t = (s_t, C^D_t), plus C^E, M and e.

    jiphyeonjeon review §2 (state, memory, encoder cache); greeksharifa §2.1.
    """
    pos_enc: int = 0                       # tokens encoded so far
    pos_dec: int = 0                       # transitions applied so far (t)
    e: List[np.ndarray] = field(default_factory=list)          # e_1..e_{pos_enc}
    enc_k: List[np.ndarray] = field(default_factory=list)      # per layer [t, h, dh]
    enc_v: List[np.ndarray] = field(default_factory=list)
    mem_k: List[np.ndarray] = field(default_factory=list)      # per group [t, h, dh]
    mem_v: List[np.ndarray] = field(default_factory=list)
    swa: List[Dict[int, tuple]] = field(default_factory=list)  # per layer {pos: (k, v)}
    s: Optional[np.ndarray] = None
    R: Optional[np.ndarray] = None         # RLT-2 feedback register

    def copy(self) -> "RowState":
        return RowState(self.pos_enc, self.pos_dec, list(self.e),
                        [a.copy() for a in self.enc_k], [a.copy() for a in self.enc_v],
                        [a.copy() for a in self.mem_k], [a.copy() for a in self.mem_v],
                        [dict(c) for c in self.swa],
                        None if self.s is None else self.s.copy(),
                        None if self.R is None else self.R.copy())


# ----------------------------------------------------------------------------
# The model
# ----------------------------------------------------------------------------


class RLTOracle:
    def __init__(self, cfg, weights: Dict[str, np.ndarray], mode: str = "fp64"):
        assert mode in ("fp64", "bf16")
        self.cfg = cfg
        self.mode = mode
        self.W = {k: np.asarray(v, dtype=np.float64) for k, v in weights.items()}
        self.h = cfg.heads
        self.dh = cfg.d // cfg.heads

    # -- precision points -------------------------------------------------
    def _store(self, x: np.ndarray) -> np.ndarray:
        return round_bf16(x) if self.mode == "bf16" else x

    def _lin(self, x: np.ndarray, name: str) -> np.ndarray:
        """y = W x for rows of x (W stored [out, in]); the input is a storage point."""
        return self._store(x) @ self.W[name].T

    def _enc(self, l: int, name: str) -> str:
        """Encoder layer l's matrix; tied models reuse decoder layer l's
        (greeksharifa App. A.1; jiphyeonjeon review §3.4)."""
        return f"dec.{l}.{name}" if self.cfg.tied else f"enc.{l}.{name}"

    def _heads(self, x: np.ndarray) -> np.ndarray:
        return x.reshape(x.shape[0], self.h, self.dh)

    def _ffn(self, x: np.ndarray, w1: str, w3: str, w2: str) -> np.ndarray:
        return self._lin(silu(self._lin(x, w1)) * self._lin(x, w3), w2)

    # -- state -------------------------------------------------------------
    def new_state(self) -> RowState:
        """H_0 = (s_star, empty): all caches empty, t = 0 (jiphyeonjeon §3.1)."""
        c = self.cfg
        st = RowState()
        st.enc_k = [np.zeros((0, self.h, self.dh)) for _ in range(c.n_enc)]
        st.enc_v = [np.zeros((0, self.h, self.dh)) for _ in range(c.n_enc)]
        ng = c.groups if c.n_dec > 0 else 0
        st.mem_k = [np.zeros((0, self.h, self.dh)) for _ in range(ng)]
        st.mem_v = [np.zeros((0, self.h, self.dh)) for _ in range(ng)]
        st.swa = [dict() for _ in range(c.n_dec)]
        s0 = self.W["s_star"].copy() if c.variant != 0 else np.zeros(c.d)
        st.s, st.R = s0.copy(), s0.copy()
        return st

    # -- encoder -----------------------------------------------------------
    def encode(self, st: RowState, tokens: Sequence[int]) -> np.ndarray:
        """Append tokens to the encoder: e, C^E and the memory for their positions.

        All new positions of a layer are processed together under the causal
        mask, over the cached keys of earlier calls; calling it once with T
        tokens or T times with one token is the same computation
        (jiphyeonjeon §3.2: parallel encoding and incremental stepping are two
        schedules of one causal computation).
        """
        c, W = self.cfg, self.W
        tok = np.asarray(tokens, dtype=np.int64)
        n = len(tok)
        if n == 0:
            return np.zeros((0, c.d))
        p0 = st.pos_enc
        pos = p0 + 1 + np.arange(n)
        # bf16 mode: q and the attention probabilities are bf16 values where
        # the bf16 path multiplies them on the tensor cores -- every call at
        # head size 64 with prefixes of at most 256 keys, and calls of at
        # least ENC_TC_MIN_POSITIONS tokens otherwise; elsewhere they stay
        # unrounded, as its key-streaming kernel keeps them
        rounded_attn = self.mode == "bf16" and (
            n >= ENC_TC_MIN_POSITIONS or (self.dh == 64 and p0 + n <= 256))
        x = W["embed"][tok].copy()
        for l in range(c.n_enc):
            y = rmsnorm(x, W[f"enc.{l}.attn_norm"], c.eps)
            q = rope(self._heads(self._lin(y, self._enc(l, "wq"))), pos, c.rope_base)
            k = self._store(rope(self._heads(self._lin(y, self._enc(l, "wk"))), pos, c.rope_base))
            v = self._store(self._heads(self._lin(y, self._enc(l, "wv"))))
            st.enc_k[l] = np.concatenate([st.enc_k[l], k])
            st.enc_v[l] = np.concatenate([st.enc_v[l], v])
            a = np.stack([attend(q[i], st.enc_k[l][:p0 + i + 1], st.enc_v[l][:p0 + i + 1],
                                 rounded=rounded_attn)
                          for i in range(n)])
            x = x + self._lin(a.reshape(n, c.d), self._enc(l, "wo"))
            y = rmsnorm(x, W[f"enc.{l}.ffn_norm"], c.eps)
            x = x + self._ffn(y, self._enc(l, "w1"), self._enc(l, "w3"), self._enc(l, "w2"))
        st.e.extend(list(x))
        if c.n_dec > 0:
            nu = rmsnorm(x, W["mem_norm"], c.eps)
            for g in range(c.groups):
                mk = self._store(rope(self._heads(self._lin(nu, f"mem.{g}.wk")), pos, c.rope_base))
                mv = self._store(self._heads(self._lin(nu, f"mem.{g}.wv")))
                st.mem_k[g] = np.concatenate([st.mem_k[g], mk])
                st.mem_v[g] = np.concatenate([st.mem_v[g], mv])
        st.pos_enc += n
        return x

    # -- merge ---------------------------------------------------------------
    def merge(self, e: np.ndarray, fb: np.ndarray) -> np.ndarray:
        """u = e + alpha * sigmoid(W_g [e; r] + b_g) * (W_s r), r = RMSNorm_s(fb).

        greeksharifa §2.5 (merge equations); RLT-0 passes e through (§2.7).
        e may hold several positions (rows); fb is one vector.
        """
        c, W = self.cfg, self.W
        e = np.atleast_2d(e)
        if c.variant == 0:
            return e.copy()
        r = rmsnorm(fb, W["merge.norm"], c.eps)[None, :].repeat(e.shape[0], 0)
        g = sigmoid(self._lin(np.concatenate([e, r], axis=1), "merge.wg") + W["merge.bg"])
        return e + c.alpha * g * self._lin(r, "merge.ws")

    # -- decoder -------------------------------------------------------------
    def _dec_layer(self, st: RowState, l: int, z: np.ndarray, pos: np.ndarray) -> np.ndarray:
        """One decoder block over consecutive positions pos (one, or one chunk).

        Sliding-window self-attention: position t attends to t-W+1..t, taking
        positions before the block from the layer's cache and positions in
        the block from this pass; then the cache keeps max(1, t-W+2)..t.
        Cross-attention: position t reads memory keys 1..t of group g(l).
        """
        c, W = self.cfg, self.W
        p = f"dec.{l}."
        n = z.shape[0]
        y = rmsnorm(z, W[p + "swa_norm"], c.eps)
        q = rope(self._heads(self._lin(y, p + "wq")), pos, c.rope_base)
        k = self._store(rope(self._heads(self._lin(y, p + "wk")), pos, c.rope_base))
        v = self._store(self._heads(self._lin(y, p + "wv")))
        cache = st.swa[l]
        # bf16 mode: a block of several positions at head size 64 enters the
        # attention products with bf16 q and probabilities
        mq = (self.mode == "bf16" and self.dh == 64
              and DEC_MQ_MIN_POSITIONS <= n <= DEC_MQ_MAX_POSITIONS)
        a = np.zeros((n, self.h, self.dh))
        for i in range(n):
            t = int(pos[i])
            lo = t - c.window + 1
            ks = [cache[j][0] for j in sorted(cache) if j >= lo] + [k[m] for m in range(i + 1)
                                                                     if pos[m] >= lo]
            vs = [cache[j][1] for j in sorted(cache) if j >= lo] + [v[m] for m in range(i + 1)
                                                                     if pos[m] >= lo]
            a[i] = attend(q[i], np.stack(ks), np.stack(vs), rounded=mq and c.window > n)
        z = z + self._lin(a.reshape(n, c.d), p + "wo")
        for m in range(n):
            cache[int(pos[m])] = (k[m], v[m])
        keep_from = int(pos[-1]) - c.window + 2
        for j in [j for j in cache if j < keep_from]:
            del cache[j]
        y = rmsnorm(z, W[p + "x_norm"], c.eps)
        qx = rope(self._heads(self._lin(y, p + "xq")), pos, c.rope_base)
        g = l if c.groups > 1 else 0
        ax = np.stack([attend(qx[i], st.mem_k[g][:int(pos[i])], st.mem_v[g][:int(pos[i])],
                              rounded=mq) for i in range(n)])
        z = z + self._lin(ax.reshape(n, c.d), p + "xo")
        y = rmsnorm(z, W[p + "ffn_norm"], c.eps)
        return z + self._ffn(y, p + "w1", p + "w3", p + "w2")

    def transition(self, st: RowState) -> np.ndarray:
        """H_t = F_t(H_{t-1}) for the next position t (one token).

        RLT-1 merges with s_{t-1}; RLT-2 with the register R, which becomes s_t
        when t closes a chunk (t mod B_c = 0, BOS = position 1); RLT-0 uses
        e_t directly (greeksharifa §2.7, App. I).
        """
        c = self.cfg
        t = st.pos_dec + 1
        if t > st.pos_enc:
            raise ValueError("transition needs an encoded token at position t")
        fb = st.R if c.variant == 2 else st.s
        z = self.merge(st.e[t - 1], fb)
        pos = np.array([t])
        for l in range(c.n_dec):
            z = self._dec_layer(st, l, z, pos)
        st.s = z[0].copy()
        st.pos_dec = t
        if c.variant == 2 and t % c.chunk == 0:
            st.R = st.s.copy()
        return st.s

    def transition_chunk(self, st: RowState, n: int) -> np.ndarray:
        """n positions at once, layer by layer, for schedules where no position
        of the block feeds another's merge: an RLT-2 chunk (all positions read
        the held register) or any block under RLT-0 (greeksharifa App. I.2).
        Returns s for every position of the block."""
        c = self.cfg
        t0 = st.pos_dec
        if c.variant == 1 and n != 1:
            raise ValueError("RLT-1 feeds s_t to position t+1; use transition()")
        if c.variant == 2 and (t0 // c.chunk) != ((t0 + n - 1) // c.chunk):
            raise ValueError("an RLT-2 block must lie inside one chunk")
        if t0 + n > st.pos_enc:
            raise ValueError("transition needs encoded tokens")
        pos = t0 + 1 + np.arange(n)
        fb = st.R if c.variant == 2 else st.s
        z = self.merge(np.stack(st.e[t0:t0 + n]), fb)
        for l in range(c.n_dec):
            z = self._dec_layer(st, l, z, pos)
        st.s = z[-1].copy()
        st.pos_dec = t0 + n
        if c.variant == 2 and st.pos_dec % c.chunk == 0:
            st.R = st.s.copy()
        return z

    def prefill(self, st: RowState, T: int, chunked: bool = False) -> List[np.ndarray]:
        """T sequential transitions (jiphyeonjeon §3.2, greeksharifa App. F.1).
        With ``chunked`` an RLT-2 model runs the positions of each chunk, or of
        the part of a chunk that lies in range, as one block."""
        c = self.cfg
        out: List[np.ndarray] = []
        end = st.pos_dec + T
        while st.pos_dec < end:
            t0 = st.pos_dec
            if chunked and c.variant == 2:
                n = min(end - t0, c.chunk - t0 % c.chunk)
                out.extend(list(self.transition_chunk(st, n)))
            else:
                out.append(self.transition(st).copy())
        return out

    # -- readout -------------------------------------------------------------
    def logits(self, s: np.ndarray) -> np.ndarray:
        """logits = W_out RMSNorm_out(s) (greeksharifa §2.3)."""
        c = self.cfg
        y = rmsnorm(np.atleast_2d(s), self.W["out_norm"], c.eps)
        return self._lin(y, "out")[0] if np.ndim(s) == 1 else self._lin(y, "out")

    def readout(self, st: RowState) -> np.ndarray:
        return self.logits(st.s)


# ----------------------------------------------------------------------------
# Sampling rule (shared definition, written independently on each side)
# ----------------------------------------------------------------------------


def softmax(logits: np.ndarray, temperature: float = 1.0) -> np.ndarray:
    z = np.asarray(logits, dtype=np.float64) / temperature
    z = z - z.max()
    p = np.exp(z)
    return p / p.sum()


def argmax_lowest(logits: np.ndarray) -> int:
    """Index of the maximum; the lowest index among equal maxima."""
    return int(np.argmax(np.asarray(logits)))


def sample_inverse_cdf(logits: np.ndarray, u: float, temperature: float = 1.0) -> int:
    """First index i with sum_{j<=i} p_j > u, summed in index order.  Untruncated
    softmax (no top-k / top-p): jiphyeonjeon §6.2 on truncated supports."""
    p = softmax(logits, temperature)
    cdf = np.cumsum(p)
    i = int(np.searchsorted(cdf, u, side="right"))
    if i >= len(p):                   # u above the rounded total: last index with p > 0
        i = int(np.nonzero(p > 0)[0][-1])
    return i


def run_sequence(model: RLTOracle, tokens: Sequence[int]) -> List[np.ndarray]:
    """Encode a whole row in parallel, prefill it, and return the logits after
    every position (the logits after position t predict token t+1)."""
    st = model.new_state()
    model.encode(st, tokens)
    out = []
    for _ in range(len(tokens)):
        model.transition(st)
        out.append(model.readout(st))
    return out


# ----------------------------------------------------------------------------
# Replay: the policy's per-token log-probabilities
# ----------------------------------------------------------------------------


def log_softmax_at(logits: np.ndarray, index: int, temperature: float = 1.0) -> float:
    """log p_index with p = softmax(logits / temperature), from its definition:
    z_index - log sum_j exp(z_j), the sum taken after subtracting max z."""
    z = np.asarray(logits, dtype=np.float64) / temperature
    m = z.max()
    return float((z[index] - m) - np.log(np.sum(np.exp(z - m))))


def replay_logprobs(model: RLTOracle, st: RowState, tokens: Sequence[int],
                    temperature: float = 1.0) -> np.ndarray:
    """The trainer's side of the replay contract (jiphyeonjeon review §6.2,
    eq. 5.3-5.5; greeksharifa App. D.3, F.4): for each given token in order,
    read log p(token | everything consumed so far) from the current state,
    then consume the token -- encode it onto the cache and take one transition.
    ``st`` must have consumed every token it encoded.  Returns the log-
    probabilities; ``st`` ends having consumed all the tokens."""
    assert st.pos_dec == st.pos_enc, "replay starts from a state with nothing pending"
    out = np.empty(len(tokens), np.float64)
    for j, tok in enumerate(tokens):
        out[j] = log_softmax_at(model.readout(st), int(tok), temperature)
        model.encode(st, [int(tok)])
        model.transition(st)
    return out


# ----------------------------------------------------------------------------
# Packed documents
# ----------------------------------------------------------------------------


def prefill_packed(model: RLTOracle, tokens: Sequence[int], starts: Sequence[bool],
                   st: Optional[RowState] = None) -> RowState:
    """One row holding independent documents one after another: where a
    document starts the row restarts from H_0 -- recurrent output, window
    cache, encoder cache and positions all reset -- then every token is
    encoded and consumed in order (jiphyeonjeon review §6.1; greeksharifa
    App. F).  Returns the state of the last document."""
    st = model.new_state() if st is None else st
    for tok, start in zip(tokens, starts):
        if start:
            st = model.new_state()
        model.encode(st, [int(tok)])
        model.transition(st)
    return st

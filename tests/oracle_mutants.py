"""Planted mistakes in the CPU oracle, to show that its pins catch them.

Test infrastructure only.  Loaded as a pytest plugin (``-p tests.oracle_mutants``)
with the environment variable RLT_ORACLE_MUTANT=<name>, it builds a copy of
``oracle/rlt_oracle.py`` with that one expression replaced -- in memory; no
file is written -- and installs it as ``oracle`` and ``oracle.rlt_oracle``
before the pins are collected.  Each mistake is one a careful reader could
make from the pages: an off-by-one in the window or the memory prefix, a sign
or frequency error in RoPE, a swapped or dropped term, a wrong norm, scale or
rounding, and in the replay a token read after it is consumed.
"""
import os
import sys
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE_SRC = os.path.join(ROOT, "oracle", "rlt_oracle.py")

# name -> (expression in the oracle, the mistaken expression)
MUTANTS = {
    # window of W positions including the current one, and what the ring keeps
    "window_off_by_one": ("lo = t - c.window + 1", "lo = t - c.window"),
    "ring_keeps_one_more": ("keep_from = int(pos[-1]) - c.window + 2",
                            "keep_from = int(pos[-1]) - c.window + 1"),
    "window_too_short": ("lo = t - c.window + 1", "lo = t - c.window + 2"),
    "ring_keeps_one_fewer": ("keep_from = int(pos[-1]) - c.window + 2",
                             "keep_from = int(pos[-1]) - c.window + 3"),
    # rotate-half RoPE: sign of the second half, frequency exponent
    "rope_sign": ("x2 * c + x1 * s", "x2 * c - x1 * s"),
    "rope_frequency": ("inv = base ** (-2.0 * np.arange(half, dtype=np.float64) / dh)",
                       "inv = base ** (-1.0 * np.arange(half, dtype=np.float64) / dh)"),
    "rope_pairs_interleaved": (
        "x1, x2 = x[..., :half], x[..., half:]\n"
        "    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)",
        "x1, x2 = x[..., 0::2], x[..., 1::2]\n    out = np.empty_like(x)\n"
        "    out[..., 0::2] = x1 * c - x2 * s\n    out[..., 1::2] = x2 * c + x1 * s\n"
        "    return out"),
    "memory_keys_rotated_one_back": (
        'mk = self._store(rope(self._heads(self._lin(nu, f"mem.{g}.wk")), pos, c.rope_base))',
        'mk = self._store(rope(self._heads(self._lin(nu, f"mem.{g}.wk")), pos - 1, c.rope_base))'),
    # heads split with the wrong layout; the state normalised before it is carried
    "heads_layout_transposed": ("return x.reshape(x.shape[0], self.h, self.dh)",
                                "return x.reshape(x.shape[0], self.dh, self.h).transpose(0, 2, 1)"),
    "state_normalised": ("st.s = z[0].copy()", 'st.s = rmsnorm(z[0], self.W["out_norm"], c.eps)'),
    # cross-attention reads the memory prefix 1..t, not t+1
    "memory_prefix_leak": ("st.mem_k[g][:int(pos[i])], st.mem_v[g][:int(pos[i])]",
                           "st.mem_k[g][:int(pos[i]) + 1], st.mem_v[g][:int(pos[i]) + 1]"),
    # the merge gate: inverted, alpha dropped, operands of W_g swapped
    "merge_gate_inverted": ('return e + c.alpha * g * self._lin(r, "merge.ws")',
                            'return e + c.alpha * (1 - g) * self._lin(r, "merge.ws")'),
    "merge_alpha_dropped": ('return e + c.alpha * g * self._lin(r, "merge.ws")',
                            'return e + g * self._lin(r, "merge.ws")'),
    "merge_operands_swapped": ("np.concatenate([e, r], axis=1)", "np.concatenate([r, e], axis=1)"),
    "merge_gate_silu": (
        'g = sigmoid(self._lin(np.concatenate([e, r], axis=1), "merge.wg") + W["merge.bg"])',
        'g = silu(self._lin(np.concatenate([e, r], axis=1), "merge.wg") + W["merge.bg"])'),
    "merge_gate_bias_dropped": (
        'g = sigmoid(self._lin(np.concatenate([e, r], axis=1), "merge.wg") + W["merge.bg"])',
        'g = sigmoid(self._lin(np.concatenate([e, r], axis=1), "merge.wg"))'),
    # the merge reads a normalised encoder output instead of the raw e_t
    "merge_input_normalised": ("st.e.extend(list(x))",
                               'st.e.extend(list(rmsnorm(x, W["mem_norm"], c.eps)))'),
    # tied encoder layer l borrowing decoder layer l+1
    "tied_layer_shifted": (
        'return f"dec.{l}.{name}" if self.cfg.tied else f"enc.{l}.{name}"',
        'return f"dec.{(l + 1) % self.cfg.n_dec}.{name}" if self.cfg.tied else f"enc.{l}.{name}"'),
    # attention weights not normalised by their sum
    "attention_unnormalised": ("p = p / p.sum(axis=1, keepdims=True)", "p = p / p.shape[1]"),
    # RLT-2 register replaced one position early
    "register_timing": ("if c.variant == 2 and t % c.chunk == 0:",
                        "if c.variant == 2 and (t - 1) % c.chunk == 0:"),
    # block structure: residual, the norm in front of the cross-attention
    "ffn_residual_scaled": ('return z + self._ffn(y, p + "w1", p + "w3", p + "w2")',
                            'return self._ffn(y, p + "w1", p + "w3", p + "w2") + z * 0.999'),
    "cross_uses_window_norm": ('y = rmsnorm(z, W[p + "x_norm"], c.eps)',
                               'y = rmsnorm(z, W[p + "swa_norm"], c.eps)'),
    # the causal encoder sees one position ahead
    "encoder_causality_leak": ("st.enc_k[l][:p0 + i + 1], st.enc_v[l][:p0 + i + 1]",
                               "st.enc_k[l][:p0 + i + 2], st.enc_v[l][:p0 + i + 2]"),
    # attention scale 1/d_h instead of 1/sqrt(d_h); SiLU sign
    "attention_scale": ("scale = 1.0 / np.sqrt(q.shape[-1])", "scale = 1.0 / q.shape[-1]"),
    "silu_sign": ("return x / (1.0 + np.exp(-x))", "return x / (1.0 + np.exp(x))"),
    # bf16 rounding by truncation instead of nearest-even
    "bf16_truncates": ("b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16", "b = b >> 16"),
    # bf16 mode: a value cache or the product inputs left unrounded
    "bf16_encoder_values_unrounded": (
        'v = self._store(self._heads(self._lin(y, self._enc(l, "wv"))))',
        'v = self._heads(self._lin(y, self._enc(l, "wv")))'),
    "bf16_memory_values_unrounded": (
        'mv = self._store(self._heads(self._lin(nu, f"mem.{g}.wv")))',
        'mv = self._heads(self._lin(nu, f"mem.{g}.wv"))'),
    "bf16_ring_values_unrounded": ('v = self._store(self._heads(self._lin(y, p + "wv")))',
                                   'v = self._heads(self._lin(y, p + "wv"))'),
    "bf16_product_inputs_unrounded": ("return self._store(x) @ self.W[name].T",
                                      "return x @ self.W[name].T"),
    # SwiGLU gate and up projections swapped; norms dropped; projections mixed
    "swiglu_gate_up_swapped": ("silu(self._lin(x, w1)) * self._lin(x, w3)",
                               "silu(self._lin(x, w3)) * self._lin(x, w1)"),
    "memory_norm_dropped": ('nu = rmsnorm(x, W["mem_norm"], c.eps)', "nu = x"),
    "memory_v_from_wk": ('mv = self._store(self._heads(self._lin(nu, f"mem.{g}.wv")))',
                         'mv = self._store(self._heads(self._lin(nu, f"mem.{g}.wk")))'),
    "readout_norm_dropped": ('y = rmsnorm(np.atleast_2d(s), self.W["out_norm"], c.eps)',
                             "y = np.atleast_2d(s)"),
    "rmsnorm_gain_dropped": ("x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * gain",
                             "x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)"),
    "encoder_ffn_uses_attn_norm": ('y = rmsnorm(x, W[f"enc.{l}.ffn_norm"], c.eps)',
                                   'y = rmsnorm(x, W[f"enc.{l}.attn_norm"], c.eps)'),
    "decoder_ffn_uses_window_norm": ('y = rmsnorm(z, W[p + "ffn_norm"], c.eps)',
                                     'y = rmsnorm(z, W[p + "swa_norm"], c.eps)'),
    "cross_output_uses_wo": ('z = z + self._lin(ax.reshape(n, c.d), p + "xo")',
                             'z = z + self._lin(ax.reshape(n, c.d), p + "wo")'),
    # decoder keys from the un-normalised input; cross query without RoPE
    "window_keys_unnormalised": (
        'k = self._store(rope(self._heads(self._lin(y, p + "wk")), pos, c.rope_base))',
        'k = self._store(rope(self._heads(self._lin(z, p + "wk")), pos, c.rope_base))'),
    "cross_query_unrotated": ('qx = rope(self._heads(self._lin(y, p + "xq")), pos, c.rope_base)',
                              'qx = self._heads(self._lin(y, p + "xq"))'),
    # per-layer memory groups collapsed to group 0; embedding scaled by sqrt(d)
    "memory_group_ignored": ("g = l if c.groups > 1 else 0", "g = 0"),
    "embedding_scaled": ('x = W["embed"][tok].copy()', 'x = W["embed"][tok] * np.sqrt(c.d)'),
    # the window leaves out the current position's own key
    "window_drops_current_key": ("+ [k[m] for m in range(i + 1)", "+ [k[m] for m in range(i)"),
    # sampling: the temperature dropped from the sampled distribution
    "sampler_temperature_dropped": (
        "    z = np.asarray(logits, dtype=np.float64) / temperature\n    z = z - z.max()",
        "    z = np.asarray(logits, dtype=np.float64)\n    z = z - z.max()"),
    # packed documents: the reset at a document start left out
    "packed_reset_dropped": ("        if start:\n            st = model.new_state()\n",
                             "        if start and st is None:\n            st = model.new_state()\n"),
    # replay: temperature dropped, normaliser dropped, token read after it is consumed
    "logprob_temperature_dropped": (
        "    z = np.asarray(logits, dtype=np.float64) / temperature\n    m = z.max()",
        "    z = np.asarray(logits, dtype=np.float64)\n    m = z.max()"),
    "logprob_unnormalised": ("return float((z[index] - m) - np.log(np.sum(np.exp(z - m))))",
                             "return float(z[index] - m)"),
    "replay_reads_after_consuming": (
        "        out[j] = log_softmax_at(model.readout(st), int(tok), temperature)\n"
        "        model.encode(st, [int(tok)])\n"
        "        model.transition(st)\n",
        "        model.encode(st, [int(tok)])\n"
        "        model.transition(st)\n"
        "        out[j] = log_softmax_at(model.readout(st), int(tok), temperature)\n"),
}


def mutant_module(name: str) -> types.ModuleType:
    """A copy of the oracle module with mutant `name` planted."""
    old, new = MUTANTS[name]
    src = open(ORACLE_SRC).read()
    if src.count(old) != 1:
        raise RuntimeError(f"mutant {name}: the expression is not in the oracle exactly once")
    mod = types.ModuleType("oracle.rlt_oracle")
    mod.__file__ = ORACLE_SRC
    sys.modules["oracle.rlt_oracle"] = mod        # dataclasses look their module up
    exec(compile(src.replace(old, new), f"{ORACLE_SRC} [{name}]", "exec"), mod.__dict__)
    return mod


def pytest_configure(config):
    name = os.environ.get("RLT_ORACLE_MUTANT")
    if not name:
        return
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    mod = mutant_module(name)
    pkg = types.ModuleType("oracle")
    pkg.__path__ = []
    for k, v in vars(mod).items():
        if not k.startswith("__"):
            setattr(pkg, k, v)
    pkg.rlt_oracle = mod
    sys.modules["oracle"] = pkg

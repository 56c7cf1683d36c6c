"""Shared helpers of the parity tests: run the CUDA library and the oracle on
the same seeded weights and tokens, and compare under the stated tolerances.

Tolerances (|delta logit|): 1e-4 for the fp32 path against the fp64 oracle,
3e-2 for the bf16 path against the bf16-mirrored oracle.  Argmax and sampled
ids must match exactly, except where the oracle itself puts the GPU's choice
within the tolerance of a tie (argmax) or the uniform within the tolerance of
a CDF edge (sampling); such cases are counted and reported.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List

import numpy as np

import rlt_inputs as ri

TOL_F32 = 1e-4
TOL_BF16 = 3e-2


def tol_for(cfg) -> float:
    return TOL_F32 if cfg.dtype == ri.DT_F32 else TOL_BF16


def oracle_mode(cfg) -> str:
    return "fp64" if cfg.dtype == ri.DT_F32 else "bf16"


@dataclass
class Tally:
    max_err: float = 0.0
    max_err_exact: float = 0.0
    argmax_ties: int = 0
    sample_ties: int = 0
    compared: int = 0
    notes: List[str] = field(default_factory=list)


def check_argmax(gpu_id: int, oracle_logits: np.ndarray, tol: float, tally: Tally, where=""):
    o = int(np.argmax(oracle_logits))
    if gpu_id == o:
        return
    assert oracle_logits[gpu_id] >= oracle_logits[o] - tol, \
        f"argmax {gpu_id} vs oracle {o} ({where}): gap {oracle_logits[o] - oracle_logits[gpu_id]}"
    tally.argmax_ties += 1


def check_sample(gpu_id: int, oracle_logits: np.ndarray, u: float, temperature: float, tol: float,
                 tally: Tally, where=""):
    z = (oracle_logits - oracle_logits.max()) / temperature
    p = np.exp(z)
    p /= p.sum()
    cdf = np.cumsum(p)
    o = min(int(np.searchsorted(cdf, u, side="right")), len(p) - 1)
    if gpu_id == o:
        return
    # a logit error of tol moves each probability by at most ~2 tol / temperature relative
    slack = 2.0 * tol / temperature + 1e-6
    edges = [cdf[i] for i in range(min(gpu_id, o), max(gpu_id, o))]
    assert all(abs(u - e) <= slack for e in edges), \
        f"sampled {gpu_id} vs oracle {o} ({where}): u={u} edges={edges}"
    tally.sample_ties += 1


def logits_of(state_logits_host: np.ndarray, cfg) -> np.ndarray:
    return state_logits_host.reshape(-1, cfg.vocab)

"""Seeded synthetic inputs for the StagQ GEMV workloads.

This module only draws random numbers; it holds none of the format's
arithmetic (no grid, no encoding, no decoding). Both the CUDA path and the
CPU oracle take their inputs from here, so a test can feed them the same
weights and activations.

Weight recipe (the workloads of the StagQ GEMV timing, synthetic weights):
``W`` is drawn from N(0, sigma) with sigma = 0.02; a fraction ``tail_frac``
(0.5 %) of the entries, chosen uniformly at random, is replaced by
``sigma * tail_scale * t`` with ``t`` ~ Student-t(nu = 3) and tail_scale = 5,
and the matrix is rounded to fp16. Activations ``x`` are fp16 N(0, 1).
Shapes are ``out x in`` (row = output channel, K = in).
"""
from __future__ import annotations

import numpy as np

SIGMA = 0.02
TAIL_FRAC = 0.005
TAIL_SCALE = 5.0
TAIL_NU = 3.0

# out x in shapes of the single-layer linears the benchmarks use.
LLAMA31_8B_LINEARS = {
    "q_proj": (4096, 4096),
    "k_proj": (1024, 4096),
    "v_proj": (1024, 4096),
    "o_proj": (4096, 4096),
    "gate_proj": (14336, 4096),
    "up_proj": (14336, 4096),
    "down_proj": (4096, 14336),
}
PHI4_LINEARS = {
    "qo": (5120, 5120),
    "kv": (1280, 5120),
    "gate_up": (17920, 5120),
    "down": (5120, 17920),
}
OLMO2_7B_LINEARS = {
    "qkvo": (4096, 4096),
    "gate_up": (11008, 4096),
    "down": (4096, 11008),
}


def weights(out: int, inp: int, seed: int, tail_frac: float = TAIL_FRAC,
            sigma: float = SIGMA, tail_scale: float = TAIL_SCALE) -> np.ndarray:
    """fp16 weight matrix [out, inp]: Gaussian body plus heavy Student-t tails."""
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((out, inp), dtype=np.float32) * np.float32(sigma)
    n_tail = int(np.floor(tail_frac * out * inp + 0.5))
    if n_tail > 0:
        flat = rng.choice(out * inp, size=n_tail, replace=False)
        t = rng.standard_t(TAIL_NU, size=n_tail).astype(np.float32)
        w.reshape(-1)[flat] = np.float32(sigma * tail_scale) * t
    return w.astype(np.float16)


def activations(n: int, inp: int, seed: int) -> np.ndarray:
    """fp16 activations [n, inp] drawn from N(0, 1)."""
    rng = np.random.default_rng(seed)
    return rng.standard_normal((n, inp), dtype=np.float32).astype(np.float16)

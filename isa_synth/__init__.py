"""Seeded synthetic inputs shaped like in-context (ICL) video-editing attention.

This module only draws numbers. It holds none of the attention method's
arithmetic, so both the CUDA path (through its tests and ``bench.py``) and the
CPU oracle can take their inputs from it without sharing any of the method.

Shape of the data (Lightning Unified Video Editing via In-Context Sparse
Attention, papernotes.org notes, "Overall framework"): Q, K, V are [B, H, N, D]
and the N = L_src + L_ctx tokens are the source video followed by the context.
The pages give no statistics for the tokens, so the recipe below is a reading:

* each (batch, head) slice gets its own stream,
  ``SeedSequence([seed, batch, head, attempt])`` into PCG64;
* one sigma per block of b tokens, drawn from U[sigma_lo, sigma_hi] and shared
  by Q, K and V;
* for Q, K, V in that order: one centroid per block drawn from N(0, I_D),
  independent across Q/K/V, and each token = its block's centroid +
  sigma * N(0, I_D);
* context rows (t >= L_src) of Q, K and V are multiplied by ``s_ctx``, so that
  source-source scores dominate, as the pages observe for ICL attention;
* the values are rounded to bfloat16 (round-to-nearest-even) unless the
  workload is fp32.

``attempt`` lets a caller redraw a single slice. The test suite uses it to skip
slices whose top-k or routing decision sits within a relative 1e-3 of a tie.
The accepted attempt of every slice is stored in ``tests/golden/attempts.json``.
"""
from __future__ import annotations

import dataclasses
import json
import os
from typing import Dict, Iterable, List, Optional, Tuple

import numpy as np

__all__ = [
    "Workload",
    "WORKLOADS",
    "RAGGED",
    "SWEEP_51K",
    "sweep_workloads",
    "make_slice",
    "make_inputs",
    "round_to_bf16_bits",
    "bf16_bits_to_f32",
    "load_attempts",
    "attempts_for",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic ICL attention workload (sizes, ratios and generator knobs)."""

    name: str
    B: int
    H: int
    D: int
    L_src: int
    L_ctx: int
    b: int
    alpha_s: float
    alpha_f: float
    sigma_lo: float
    sigma_hi: float
    s_ctx: float
    dtype: str  # "bf16" or "f32"

    @property
    def N(self) -> int:
        return self.L_src + self.L_ctx

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workload families: a tiny fp32 case the oracle finishes in seconds,
# 8K / 16K / 32K-token bf16 cases and the 51K-token sweep. 32K is the headline.
WORKLOADS: Dict[str, Workload] = {
    "tiny_f32_n1024": Workload("tiny_f32_n1024", 1, 2, 64, 512, 512, 64, 0.5, 0.5, 0.1, 1.0, 0.5, "f32"),
    "bf16_n8192_b64": Workload("bf16_n8192_b64", 1, 40, 128, 4096, 4096, 64, 0.25, 0.5, 0.1, 1.0, 0.5, "bf16"),
    "bf16_n16384_b64": Workload("bf16_n16384_b64", 1, 40, 128, 8192, 8192, 64, 0.25, 0.5, 0.05, 1.5, 0.5, "bf16"),
    "bf16_n32768_b128": Workload("bf16_n32768_b128", 1, 40, 128, 16384, 16384, 128, 0.25, 0.6, 0.1, 1.0, 0.5, "bf16"),
}

HEADLINE = "bf16_n32768_b128"

# The headline shape with lengths that b = 128 divides in neither part (a short last block in the
# source part, 44 tokens, and in the context part, 116 tokens): a benchmark of ragged lengths.
RAGGED: Dict[str, Workload] = {
    "bf16_n32800_b128_ragged": Workload("bf16_n32800_b128_ragged", 1, 40, 128, 16300, 16500, 128, 0.25, 0.6, 0.1,
                                        1.0, 0.5, "bf16"),
}

_SWEEP_BASE = Workload("bf16_n51200_b128", 1, 40, 128, 25600, 25600, 128, 0.25, 0.5, 0.1, 1.0, 0.5, "bf16")
SWEEP_51K_ALPHA_S = (0.1, 0.25, 0.5)
SWEEP_51K_ALPHA_F = (0.3, 0.5, 0.7)
SWEEP_51K_S_CTX = (0.3, 0.5, 1.0)


def _sweep_name(a_s: float, a_f: float, s_ctx: float) -> str:
    return f"bf16_n51200_b128_as{a_s:g}_af{a_f:g}_sc{s_ctx:g}"


def sweep_workloads() -> List[Workload]:
    """The 51K-token sweep: alpha_s x alpha_f x s_ctx, plus the dense-equivalent point."""
    out = []
    for s_ctx in SWEEP_51K_S_CTX:
        for a_s in SWEEP_51K_ALPHA_S:
            for a_f in SWEEP_51K_ALPHA_F:
                out.append(_SWEEP_BASE.with_(name=_sweep_name(a_s, a_f, s_ctx), alpha_s=a_s, alpha_f=a_f, s_ctx=s_ctx))
    out.append(_SWEEP_BASE.with_(name=_sweep_name(1.0, 0.0, 0.5), alpha_s=1.0, alpha_f=0.0, s_ctx=0.5))
    return out


SWEEP_51K: Dict[str, Workload] = {w.name: w for w in sweep_workloads()}


def all_workloads() -> Dict[str, Workload]:
    d = dict(WORKLOADS)
    d.update(SWEEP_51K)
    return d


def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round finite values to bfloat16, nearest-even, via float32; returns the uint16 bit patterns."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _slice_rng(seed: int, batch: int, head: int, attempt: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, batch, head, attempt])))


def make_slice(w: Workload, seed: int, batch: int, head: int, attempt: int = 0,
               sigma_override: Optional[Tuple[float, float, float]] = None) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Draw Q, K, V for one (batch, head) slice as float32 [N, D] arrays.

    For bf16 workloads every value is exactly representable in bfloat16.
    ``sigma_override`` (Q, K, V multipliers on the per-block sigma) lets tests
    build special cases, e.g. keys that are constant inside every block.
    """
    rng = _slice_rng(seed, batch, head, attempt)
    N, D, b = w.N, w.D, w.b
    # token -> block: source blocks of b tokens from 0, context blocks from L_src (the last
    # block of either part is short when b does not divide its length)
    n_src = -(-w.L_src // b)
    tok = np.arange(N)
    blk = np.where(tok < w.L_src, tok // b, n_src + (tok - w.L_src) // b)
    n_q = int(blk[-1]) + 1
    sigma = rng.uniform(w.sigma_lo, w.sigma_hi, size=n_q)
    blk_sigma = sigma[blk][:, None]
    mult = sigma_override if sigma_override is not None else (1.0, 1.0, 1.0)
    outs = []
    for t in range(3):
        cent = rng.standard_normal((n_q, D))
        eps = rng.standard_normal((N, D))
        x = cent[blk] + (mult[t] * blk_sigma) * eps
        x[w.L_src:] *= w.s_ctx
        if w.dtype == "bf16":
            x = bf16_bits_to_f32(round_to_bf16_bits(x))
        else:
            x = x.astype(np.float32)
        outs.append(x)
    return outs[0], outs[1], outs[2]


def make_inputs(w: Workload, seed: int = 0, attempts: Optional[np.ndarray] = None,
                heads: Optional[Iterable[Tuple[int, int]]] = None):
    """Draw the whole [B, H, N, D] Q, K, V (float32 arrays holding the exact input values).

    ``attempts`` is an int array [B, H] of per-slice attempts (default all 0).
    ``heads`` restricts the draw to some (batch, head) slices; the other slices
    are left as zeros (used for bounded CPU samples).
    """
    q = np.zeros((w.B, w.H, w.N, w.D), np.float32)
    k = np.zeros_like(q)
    v = np.zeros_like(q)
    sl = list(heads) if heads is not None else [(bi, h) for bi in range(w.B) for h in range(w.H)]
    for bi, h in sl:
        a = 0 if attempts is None else int(attempts[bi, h])
        q[bi, h], k[bi, h], v[bi, h] = make_slice(w, seed, bi, h, a)
    return q, k, v


_ATTEMPTS_PATH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "tests", "golden", "attempts.json")


def load_attempts(path: str = _ATTEMPTS_PATH) -> Dict[str, dict]:
    if not os.path.exists(path):
        return {}
    with open(path) as f:
        return json.load(f)


def attempts_for(w: Workload, seed: int = 0, table: Optional[Dict[str, dict]] = None) -> Optional[np.ndarray]:
    """Accepted per-slice attempts for workload ``w`` and ``seed`` from the stored table, or None."""
    table = load_attempts() if table is None else table
    ent = table.get(w.name)
    if ent is None or int(ent.get("seed", -1)) != seed:
        return None
    a = np.asarray(ent["attempts"], dtype=np.int64)
    if a.shape != (w.B, w.H):
        return None
    return a

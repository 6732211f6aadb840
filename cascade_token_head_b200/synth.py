"""Seeded synthetic workloads for the cascade-pruned attention path.

This module only *draws* inputs and lists workload constants; it holds none of the method's
arithmetic (no attention, no quantization, no selection).  It is the single place both the CUDA
path's tests/bench and the float64 oracle get their inputs from, so both see the same arrays.

Every tensor comes from one ``numpy.random.Generator(PCG64(SeedSequence(seed)))`` in a fixed,
documented order (float64 draws; callers cast to the workload dtype).  The shapes stand in for the
BERT-base, GPT-2-medium and long-context models that the SpAtten evaluation uses (SpAtten §V
"Evaluation Setup"); no dataset or trained weight is involved.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from fractions import Fraction

import numpy as np


def rng_for(seed: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed)))


# --------------------------------------------------------------------------------------------
# keep schedules (integers, exact rational arithmetic)
# --------------------------------------------------------------------------------------------
def geometric_keep(T: int, ratio: Fraction, L: int) -> list[int]:
    """k_l = ceil(T * ratio**l): tokens entering layer l, cumulative keep ratio per layer."""
    out = []
    for l in range(L):
        v = Fraction(T) * ratio ** l
        out.append(int(math.ceil(v)))
    return out


def linear_decode_keep(n: int, L: int) -> list[int]:
    """k_l(n) = n - floor(l * (n - ceil(n/2)) / (L-1)): 50 % of n kept by the last layer."""
    half = -(-n // 2)
    return [n - (l * (n - half)) // (L - 1) for l in range(L)]


def bert_head_keep(H: int, L: int, every: int, floor_heads: int) -> list[int]:
    """H_l = H - floor((l+1)/every), never below floor_heads (one head dropped every `every`)."""
    return [max(floor_heads, H - (l + 1) // every) for l in range(L)]


# --------------------------------------------------------------------------------------------
# workloads
# --------------------------------------------------------------------------------------------
@dataclass
class PrefillWorkload:
    name: str
    B: int
    T: int
    D: int
    H: int
    d_h: int
    L: int
    dtype: str                      # "f32" | "bf16"
    token_keep: list[int]
    head_keep: list[int]
    quant: bool
    theta: float
    boost: tuple | None = None      # ("uniform", count, gain) | ("spans", n_spans, span_len, gain)
    seed: int = 0

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.d_h)


@dataclass
class DecodeWorkload:
    name: str
    B: int
    T0: int
    steps: int
    D: int
    H: int
    d_h: int
    L: int
    theta: float
    seed: int = 0

    @property
    def cap(self) -> int:
        return self.T0 + self.steps

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.d_h)


@dataclass
class TopkWorkload:
    name: str
    R: int
    Ns: list[int] = field(default_factory=lambda: [1024, 16384, 262144, 1048576])
    fracs: list[float] = field(default_factory=lambda: [0.1, 0.5])
    dists: list[str] = field(default_factory=lambda: ["uniform", "lognormal"])
    dup_frac: float = 0.01
    seed: int = 0


def tiny_fp32() -> PrefillWorkload:
    return PrefillWorkload("tiny_cascade_fp32", B=1, T=128, D=256, H=4, d_h=64, L=4, dtype="f32",
                           token_keep=geometric_keep(128, Fraction(4, 5), 4), head_keep=[4] * 4,
                           quant=False, theta=0.0)


def bert_base_prefill() -> PrefillWorkload:
    return PrefillWorkload("bert_base_prefill_bf16", B=32, T=512, D=768, H=12, d_h=64, L=12,
                           dtype="bf16", token_keep=geometric_keep(512, Fraction(9, 10), 12),
                           head_keep=bert_head_keep(12, 12, 3, 8), quant=True, theta=0.1,
                           boost=("uniform", 26, 4.0))


def long_prefill() -> PrefillWorkload:
    return PrefillWorkload("long_context_prefill_bf16", B=1, T=16384, D=4096, H=32, d_h=128, L=4,
                           dtype="bf16", token_keep=geometric_keep(16384, Fraction(1, 2), 4),
                           head_keep=[32, 32, 24, 24], quant=True, theta=0.1,
                           boost=("spans", 8, 41, 4.0))


def gpt2m_decode() -> DecodeWorkload:
    return DecodeWorkload("gpt2_medium_decode", B=16, T0=1024, steps=128, D=1024, H=16, d_h=64,
                          L=24, theta=0.2)


def topk_sweep() -> TopkWorkload:
    return TopkWorkload("topk_sweep_fp32", R=64)


def scaled_prefill(base: PrefillWorkload, **over) -> PrefillWorkload:
    """A copy of a workload with some sizes replaced (used for small parity cases)."""
    d = dict(base.__dict__)
    d.update(over)
    return PrefillWorkload(**d)


# --------------------------------------------------------------------------------------------
# draws
# --------------------------------------------------------------------------------------------
def draw_prefill(w: PrefillWorkload) -> dict:
    """Draw order: X, then per layer W_q, W_k, W_v, W_o, then the boosted-token choice.

    X ~ N(0,1) [B,T,D]; W ~ N(0, 1/D).  W_q/W_k/W_v are [D, H*d_h] (x @ W), W_o is [H*d_h, D].
    Returned float64; ``w_qkv[l]`` is the column concatenation [W_q | W_k | W_v] (a layout, not
    arithmetic).  ``key_gain`` [B,T] is 1 except for boosted tokens, whose K rows are scaled by the
    gain after projection in every layer.
    """
    g = rng_for(w.seed)
    HD = w.H * w.d_h
    X = g.standard_normal((w.B, w.T, w.D))
    sd = 1.0 / math.sqrt(w.D)
    w_qkv, w_o = [], []
    for _ in range(w.L):
        wq = g.standard_normal((w.D, HD)) * sd
        wk = g.standard_normal((w.D, HD)) * sd
        wv = g.standard_normal((w.D, HD)) * sd
        wo = g.standard_normal((HD, w.D)) * sd
        w_qkv.append(np.concatenate([wq, wk, wv], axis=1))
        w_o.append(wo)
    gain = None
    if w.boost is not None:
        gain = np.ones((w.B, w.T))
        if w.boost[0] == "uniform":
            _, count, gval = w.boost
            for b in range(w.B):
                pos = g.choice(w.T, size=count, replace=False)
                gain[b, pos] = gval
        elif w.boost[0] == "spans":
            _, n_spans, span_len, gval = w.boost
            # non-overlapping starts: place spans in n_spans equal slots at seeded offsets
            slot = w.T // n_spans
            for b in range(w.B):
                for s in range(n_spans):
                    off = int(g.integers(0, slot - span_len + 1))
                    gain[b, s * slot + off: s * slot + off + span_len] = gval
        else:
            raise ValueError(w.boost)
    return dict(X=X, w_qkv=w_qkv, w_o=w_o, key_gain=gain)


def draw_decode(w: DecodeWorkload, steps: int | None = None, layers: int | None = None) -> dict:
    """Draw order: per layer W_q, W_k, W_v, W_o; per layer prompt K then V [B,H,T0,d_h]; x_t per step.

    The prompt cache entries are drawn directly as N(0,1): that is the distribution of A @ W_k for
    A ~ N(0,1) and W_k ~ N(0,1/D), without forming the [B*T0, D] activations.
    """
    g = rng_for(w.seed)
    L = w.L if layers is None else layers
    S = w.steps if steps is None else steps
    HD = w.H * w.d_h
    sd = 1.0 / math.sqrt(w.D)
    w_qkv, w_o = [], []
    for _ in range(L):
        wq = g.standard_normal((w.D, HD)) * sd
        wk = g.standard_normal((w.D, HD)) * sd
        wv = g.standard_normal((w.D, HD)) * sd
        wo = g.standard_normal((HD, w.D)) * sd
        w_qkv.append(np.concatenate([wq, wk, wv], axis=1))
        w_o.append(wo)
    k_prompt, v_prompt = [], []
    for _ in range(L):
        k_prompt.append(g.standard_normal((w.B, w.H, w.T0, w.d_h), dtype=np.float32))
        v_prompt.append(g.standard_normal((w.B, w.H, w.T0, w.d_h), dtype=np.float32))
    xs = g.standard_normal((S, w.B, w.D))
    return dict(w_qkv=w_qkv, w_o=w_o, k_prompt=k_prompt, v_prompt=v_prompt, x_steps=xs)


def draw_topk_row_block(R: int, N: int, dist: str, dup_frac: float, seed: int) -> np.ndarray:
    """[R, N] float32 scores: uniform(0,1) or lognormal(0,2), then dup_frac of the positions of
    each row overwritten with copies of other randomly chosen positions' values (exact ties)."""
    g = rng_for(seed)
    if dist == "uniform":
        x = g.random((R, N)).astype(np.float32)
    elif dist == "lognormal":
        x = g.lognormal(0.0, 2.0, size=(R, N)).astype(np.float32)
    else:
        raise ValueError(dist)
    n_dup = int(round(dup_frac * N))
    if n_dup:
        for r in range(R):
            dst = g.choice(N, size=n_dup, replace=False)
            src = g.integers(0, N, size=n_dup)
            x[r, dst] = x[r, src]
    return x


def to_bf16_f64(a: np.ndarray) -> np.ndarray:
    """Round float64/float32 values to bfloat16 (nearest-even) and return them as float64.

    Used to give the oracle exactly the values a bf16 device tensor holds.
    """
    f = np.asarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    # round to nearest even on the upper 16 bits (finite inputs only)
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).astype(np.float64)

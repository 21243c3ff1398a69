"""Seeded input generator for the FlashLoop attention-sublayer workloads.

Recipe (every number below is a choice of this generator, shared verbatim by
the CPU oracle and the CUDA path, which receive the same bytes):

* Weights come from ``numpy.random.default_rng([seed, 0])``: W_q, W_k, W_v,
  W_o in that order, each ``[d_model, d_model]`` (torch ``Linear`` layout,
  ``y = x @ W.T``), drawn N(0, 1) in fp32 and scaled by ``1/sqrt(d_model)``
  (variance ``1/d_model``), then rounded to bf16 (round to nearest even).
* Sequence ``b`` of a prefill workload comes from ``default_rng([seed, 1, b])``:
  ``H0 ~ N(0, 1)`` of shape ``[S, d_model]``, then a permutation ``pi`` of
  ``[0, S)``, then one perturbation ``delta_r`` per loop r = 2..R.  The
  loop-r active set is ``pi[:n_r]`` (so the sets nest); ``delta_r`` has
  standard deviation 0.05 on those rows and 1e-4 on all others.  The fp32
  master is ``X_1 = H0`` and ``X_r = X_{r-1} + delta_r``; each X_r is handed
  over rounded to bf16.
* Decode token ``b`` comes from ``default_rng([seed, 2, b])``: ``h0 ~ N(0, 1)``
  of shape ``[d_model]``, then one ``delta_r ~ N(0, 0.05^2)`` per loop r >= 2
  (the decode token is active at every loop).

Sizes round half up: ``n_r = floor(f_r * S + 1/2)``, ``k = floor(f_k * S + 1/2)``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np


def round_half_up(x: float) -> int:
    """floor(x + 1/2): the rounding used for every budget (n_r and k)."""
    return int(math.floor(x + 0.5))


def f32_to_bf16_bits(x) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns uint16 bits."""
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = a.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(bits) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float32."""
    b = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16))
    return (b.astype(np.uint32) << 16).view(np.float32)


@dataclass(frozen=True)
class Config:
    """One synthetic workload of the loop-r attention sublayer.

    ``active_fracs[r-2]`` is the fraction of tokens active at loop r (r >= 2);
    ``bits[r-1]`` is the KV code width at loop r (loop 1 = the INT8 base).
    For a decode workload ``seq`` is the context length S_ctx, ``batch``
    the number of sequences, and each sequence appends one token at
    position ``seq``.
    """

    name: str
    d_model: int
    n_heads: int
    head_dim: int
    seq: int
    n_loops: int
    tau: float
    topk_frac: float
    active_fracs: tuple
    bits: tuple
    batch: int = 1
    decode: bool = False
    rope_theta: float = 1.0e4
    seed: int = 0
    description: str = field(default="", compare=False)

    def __post_init__(self):
        assert self.d_model == self.n_heads * self.head_dim
        assert len(self.active_fracs) == self.n_loops - 1
        assert len(self.bits) == self.n_loops

    @property
    def k(self) -> int:
        """Selected key columns per head (constant over loops r >= 2)."""
        return round_half_up(self.topk_frac * self.seq)

    def n_active(self, r: int) -> int:
        """Active-token budget at loop r of a prefill sequence."""
        if r == 1:
            return self.seq
        return round_half_up(self.active_fracs[r - 2] * self.seq)

    def k_per_loop(self):
        """Column budget per loop, index r-1 (loop 1 is dense: k = S)."""
        return [self.seq] + [self.k] * (self.n_loops - 1)

    def with_(self, **kw) -> "Config":
        d = {f: getattr(self, f) for f in self.__dataclass_fields__}
        d.update(kw)
        return Config(**d)


CONFIGS = {
    "tiny": Config(
        "tiny", 256, 4, 64, 256, 4, 0.01, 0.10, (0.75, 0.40, 0.20), (8, 4, 2, 2),
        description="d 256, 4x64 heads, S 256, R 4, k 26"),
    "ouro14_4k": Config(
        "ouro14_4k", 2048, 16, 128, 4096, 4, 0.01, 0.10, (0.75, 0.40, 0.20), (8, 4, 2, 2),
        description="Ouro-1.4B-like attention shape, S 4096, R 4, k 410"),
    "prefill_32k": Config(
        "prefill_32k", 2048, 16, 128, 32768, 4, 0.01, 0.10, (0.75, 0.40, 0.20), (8, 4, 2, 2),
        description="32K prefill, d 2048, 16x128, R 4, k 3277"),
    "decode_32k": Config(
        "decode_32k", 2048, 16, 128, 32768, 4, 0.01, 0.10, (0.75, 0.40, 0.20), (8, 4, 2, 2),
        batch=8, decode=True,
        description="decode: 8 sequences x 1 token against a 32768-token context, R 4"),
    "depth_8k_r8": Config(
        "depth_8k_r8", 2048, 16, 128, 8192, 8, 0.01, 0.05,
        (0.80, 0.40, 0.20, 0.10, 0.05, 0.025, 0.0125), (8, 4, 2, 2, 2, 2, 2, 2),
        description="depth sweep: S 8192, R 8, k 410, INT2 residuals from loop 3"),
}


def make_weights(cfg: Config, seed: int | None = None):
    """bf16 bit arrays W_q, W_k, W_v, W_o (each [d, d]) and W_qkv = [W_q; W_k; W_v]."""
    seed = cfg.seed if seed is None else seed
    rng = np.random.default_rng([seed, 0])
    d = cfg.d_model
    scale = np.float32(1.0 / math.sqrt(d))
    out = {}
    for name in ("wq", "wk", "wv", "wo"):
        w = rng.standard_normal((d, d), dtype=np.float32) * scale
        out[name] = f32_to_bf16_bits(w)
    out["wqkv"] = np.concatenate([out["wq"], out["wk"], out["wv"]], axis=0)
    return out


def make_hidden_states(cfg: Config, b: int = 0, seed: int | None = None, seq: int | None = None):
    """Hidden states X_1..X_R (bf16 bits, [S, d]) and the planted nested active sets.

    Returns ``(X, planted)`` with ``X[r-1]`` the loop-r input and ``planted[r-1]``
    the ascending token set whose rows were perturbed strongly at loop r
    (``planted[0]`` is every token).
    """
    seed = cfg.seed if seed is None else seed
    S = cfg.seq if seq is None else seq
    d = cfg.d_model
    rng = np.random.default_rng([seed, 1, b])
    master = rng.standard_normal((S, d), dtype=np.float32)
    perm = rng.permutation(S)
    X = [f32_to_bf16_bits(master)]
    planted = [np.arange(S, dtype=np.int64)]
    for r in range(2, cfg.n_loops + 1):
        n = round_half_up(cfg.active_fracs[r - 2] * S)
        strong = np.zeros(S, dtype=bool)
        strong[perm[:n]] = True
        delta = rng.standard_normal((S, d), dtype=np.float32)
        delta *= np.where(strong, np.float32(0.05), np.float32(1e-4)).astype(np.float32)[:, None]
        master = master + delta
        del delta
        X.append(f32_to_bf16_bits(master))
        planted.append(np.sort(perm[:n]).astype(np.int64))
    return X, planted


def make_decode_tokens(cfg: Config, b: int, seed: int | None = None):
    """Hidden states of decode token b at loops 1..R (bf16 bits, each [d])."""
    seed = cfg.seed if seed is None else seed
    rng = np.random.default_rng([seed, 2, b])
    d = cfg.d_model
    master = rng.standard_normal(d, dtype=np.float32)
    out = [f32_to_bf16_bits(master)]
    for _ in range(2, cfg.n_loops + 1):
        master = master + rng.standard_normal(d, dtype=np.float32) * np.float32(0.05)
        out.append(f32_to_bf16_bits(master))
    return out

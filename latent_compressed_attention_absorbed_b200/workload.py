"""Seeded synthetic workloads for absorbed-MLA decode.

This module only draws random numbers and rounds them to the storage dtype.
It holds none of the attention arithmetic, so both the CPU oracle tests and
the CUDA parity tests can take their inputs from here without sharing any of
the method's code.

Shapes follow the DeepSeek-V3 MLA configuration table (128 heads, KV latent
rank 512, per-head no-position width 128, RoPE width 64, value width 128) and
the five decode workloads this library is measured on:

  tiny      fp32, B=1, H=4, d_c=32, d_r=8, d_n=16, d_v=16, T=64, q_len=1
  v3_b1     bf16, B=1, T=4096, q_len=1
  v3_b64    bf16, B=64, T=4096, q_len=1
  v3_long   bf16, B=8, T=131072, q_len=1
  v3_ragged bf16, B=128, T_b uniform in [2048, 16384], q_len=2

Value distributions: c_KV, k_R, q_nope, q_R ~ N(0, 1); W_UK, W_UV ~ N(0, s)
with s = 1/sqrt(d_c) for the tiny case and s = 0.02 for the V3 shapes (the
second parameter is read as a standard deviation).

Random streams.  Every tensor has its own counter-free stream,
``numpy.random.default_rng([seed, tag, index])``, so that any one sequence's
cache can be generated without drawing the others (the oracle checks sampled
sequences at the full sizes).  Values are drawn in float64 and rounded once to
the storage dtype; the oracle consumes the rounded values, so input
quantisation is not counted as kernel error.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import numpy as np

# Stream tags: one per tensor kind.
_TAG_W_UK, _TAG_W_UV, _TAG_Q_NOPE, _TAG_Q_ROPE, _TAG_C_KV, _TAG_K_ROPE, _TAG_NEW = range(7)
_TAG_X, _TAG_W_A, _TAG_GAMMA, _TAG_W_O = range(7, 11)


@dataclasses.dataclass(frozen=True)
class MLAConfig:
    name: str
    B: int
    H: int
    d_c: int
    d_r: int
    d_n: int
    d_v: int
    q_len: int
    seqlens: tuple  # per-sequence cached length, including the q_len new tokens
    dtype: str  # "f32" or "bf16"
    w_std: float
    seed: int
    rope_base: float = 10000.0
    # 0: W_UK ~ N(0, w_std).  Otherwise W_UK[h][d][c] = w_uk_select when
    # d == c % d_n and 0 elsewhere: every folded query component is then a
    # query component times w_uk_select, exactly representable in the storage
    # dtype when w_uk_select is a power of two (sharp-score test inputs).
    w_uk_select: float = 0.0
    d_model: int = 7168  # hidden size of the block (the projections around the decode)

    @property
    def T_max(self) -> int:
        return int(max(self.seqlens)) if self.seqlens else 0

    @property
    def row(self) -> int:
        """Cache row width: latent then RoPE key."""
        return self.d_c + self.d_r

    @property
    def softmax_scale(self) -> float:
        return 1.0 / float(np.sqrt(self.d_n + self.d_r))

    def with_(self, **kw) -> "MLAConfig":
        return dataclasses.replace(self, **kw)


def _ragged_seqlens(n: int, lo: int, hi: int, seed: int) -> tuple:
    return tuple(int(x) for x in np.random.default_rng(seed).integers(lo, hi + 1, size=n))


CONFIGS = {
    "tiny": MLAConfig("tiny", B=1, H=4, d_c=32, d_r=8, d_n=16, d_v=16, q_len=1,
                      seqlens=(64,), dtype="f32", w_std=1.0 / np.sqrt(32.0), seed=0),
    "v3_b1": MLAConfig("v3_b1", B=1, H=128, d_c=512, d_r=64, d_n=128, d_v=128, q_len=1,
                       seqlens=(4096,), dtype="bf16", w_std=0.02, seed=1),
    "v3_b64": MLAConfig("v3_b64", B=64, H=128, d_c=512, d_r=64, d_n=128, d_v=128, q_len=1,
                        seqlens=(4096,) * 64, dtype="bf16", w_std=0.02, seed=2),
    "v3_long": MLAConfig("v3_long", B=8, H=128, d_c=512, d_r=64, d_n=128, d_v=128, q_len=1,
                         seqlens=(131072,) * 8, dtype="bf16", w_std=0.02, seed=3),
    "v3_ragged": MLAConfig("v3_ragged", B=128, H=128, d_c=512, d_r=64, d_n=128, d_v=128, q_len=2,
                           seqlens=_ragged_seqlens(128, 2048, 16384, 0), dtype="bf16",
                           w_std=0.02, seed=4),
}
CONFIG_ORDER = ["tiny", "v3_b1", "v3_b64", "v3_long", "v3_ragged"]


# ---------------------------------------------------------------- rounding

def round_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round to the nearest bfloat16 (ties to even); returns the uint16 bit patterns."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


class Stored:
    """One tensor: ``values`` (float64, already rounded) and ``raw`` (the bytes to upload)."""

    __slots__ = ("values", "raw", "dtype")

    def __init__(self, x: np.ndarray, dtype: str):
        self.dtype = dtype
        if dtype == "bf16":
            self.raw = round_bf16_bits(x)
            self.values = bf16_bits_to_f64(self.raw)
        elif dtype == "f32":
            self.raw = np.ascontiguousarray(x, dtype=np.float32)
            self.values = self.raw.astype(np.float64)
        else:
            raise ValueError(dtype)


def _normal(seed: int, tag: int, index: int, shape, std: float = 1.0) -> np.ndarray:
    rng = np.random.default_rng([seed, tag, index])
    return rng.standard_normal(size=shape) * std


# ---------------------------------------------------------------- tensors

def weights(cfg: MLAConfig):
    """W_UK, W_UV as [H, d_n, d_c] and [H, d_v, d_c] (k_C = W_UK[h] @ c, v = W_UV[h] @ c)."""
    if cfg.w_uk_select:
        sel = np.zeros((cfg.H, cfg.d_n, cfg.d_c))
        c = np.arange(cfg.d_c)
        sel[:, c % cfg.d_n, c] = cfg.w_uk_select
        w_uk = Stored(sel, cfg.dtype)
    else:
        w_uk = Stored(_normal(cfg.seed, _TAG_W_UK, 0, (cfg.H, cfg.d_n, cfg.d_c), cfg.w_std), cfg.dtype)
    w_uv = Stored(_normal(cfg.seed, _TAG_W_UV, 0, (cfg.H, cfg.d_v, cfg.d_c), cfg.w_std), cfg.dtype)
    return w_uk, w_uv


def queries(cfg: MLAConfig):
    """q_nope [B, q_len, H, d_n] and un-rotated q_R [B, q_len, H, d_r]."""
    qn = Stored(_normal(cfg.seed, _TAG_Q_NOPE, 0, (cfg.B, cfg.q_len, cfg.H, cfg.d_n)), cfg.dtype)
    qr = Stored(_normal(cfg.seed, _TAG_Q_ROPE, 0, (cfg.B, cfg.q_len, cfg.H, cfg.d_r)), cfg.dtype)
    return qn, qr


def sequence_history(cfg: MLAConfig, b: int):
    """Token inputs of sequence b for positions 0..T_b-1: c_KV [T_b, d_c] and un-rotated k_R [T_b, d_r].

    These are what the cache-append call receives; the append rotates k_R by
    its position before storing it.
    """
    T = int(cfg.seqlens[b])
    c = Stored(_normal(cfg.seed, _TAG_C_KV, b, (T, cfg.d_c)), cfg.dtype)
    k = Stored(_normal(cfg.seed, _TAG_K_ROPE, b, (T, cfg.d_r)), cfg.dtype)
    return c, k


def new_tokens(cfg: MLAConfig, n_tok: int, index: int = 0):
    """Fresh per-step token inputs for an append: c_KV [B, n_tok, d_c], k_R [B, n_tok, d_r]."""
    c = Stored(_normal(cfg.seed, _TAG_NEW, 2 * index, (cfg.B, n_tok, cfg.d_c)), cfg.dtype)
    k = Stored(_normal(cfg.seed, _TAG_NEW, 2 * index + 1, (cfg.B, n_tok, cfg.d_r)), cfg.dtype)
    return c, k


def block_input(cfg: MLAConfig, n_tok: int, index: int = 0):
    """The attention block's input x [B, n_tok, d_model] ~ N(0, 1) (unit rms, as after the block's pre-norm)."""
    return Stored(_normal(cfg.seed, _TAG_X, index, (cfg.B, n_tok, cfg.d_model)), cfg.dtype)


def append_weights(cfg: MLAConfig):
    """W_A = [W_DKV; W_KR] as [d_c + d_r, d_model] ~ N(0, w_std), and the latent's RMSNorm gain
    gamma [d_c] ~ N(1, 0.1)."""
    w_a = Stored(_normal(cfg.seed, _TAG_W_A, 0, (cfg.d_c + cfg.d_r, cfg.d_model), cfg.w_std), cfg.dtype)
    gamma = Stored(1.0 + _normal(cfg.seed, _TAG_GAMMA, 0, (cfg.d_c,), 0.1), cfg.dtype)
    return w_a, gamma


def output_weights(cfg: MLAConfig):
    """W_O [d_model, H * d_v] ~ N(0, w_std)."""
    return Stored(_normal(cfg.seed, _TAG_W_O, 0, (cfg.d_model, cfg.H * cfg.d_v), cfg.w_std), cfg.dtype)


def small_variant(cfg: MLAConfig, B: Optional[int] = None, seqlens: Optional[Sequence[int]] = None,
                  q_len: Optional[int] = None, seed: Optional[int] = None) -> MLAConfig:
    """Same head geometry and value distributions, other batch / lengths (parity cases)."""
    kw = {}
    if seqlens is not None:
        kw["seqlens"] = tuple(int(s) for s in seqlens)
        kw["B"] = len(kw["seqlens"])
    elif B is not None:
        kw["B"] = B
        kw["seqlens"] = tuple(cfg.seqlens[:B]) if len(cfg.seqlens) >= B else (cfg.seqlens[0],) * B
    if q_len is not None:
        kw["q_len"] = q_len
    if seed is not None:
        kw["seed"] = seed
    kw["name"] = cfg.name + "_var"
    return cfg.with_(**kw)

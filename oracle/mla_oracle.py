"""CPU fp64 oracle for absorbed Multi-head Latent Attention (MLA) decode.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use it.  It shares no code with the CUDA library.

What it computes, and where the pages define it
-----------------------------------------------
Sources (web write-ups of the DeepSeek-V3 Technical Report):

[P1] wq-win.github.io/llm/092-deepseekv3.html, "092｜DeepSeek-V3：让模型、
     数值精度与通信共同接受成本约束", section 二, paragraphs "MLA：缓存压缩后的
     历史" (per token and layer the cache holds a 512-d KV latent plus a 64-d
     decoupled RoPE key, 576 numbers) and "缓存压缩也可以做一个代数检查" (the
     identity q^T (U c) = (U^T q)^T c with U in R^{d_h x d_c}; the RoPE key
     branch is computed separately and is not absorbed).
[P3] ailearn.mscapital.top/deepseek-v3.html, the MLA "状态传导图" panel and
     the MLA paragraphs after the configuration table: only c_KV in R^512 and
     a RoPE-rotated k_R in R^64 are cached; the query's content part is
     multiplied by W_UK first and dotted with every cached c_KV, the RoPE part
     is scored separately and added; the softmax weights aggregate
     sum_j p_j c_KV,j first and W_UV is applied afterwards; the configuration
     table gives 128 heads, KV rank 512, no-position width 128, RoPE width 64,
     value width 128; the cache-count paragraph gives 128*(128+128) = 32,768
     (MHA) and 128*(192+128) = 40,960 (naive MLA branch) against 576.
[P5] m.lsln.cn/news/222502, sections 2.1 (decode attention at step t is
     softmax(Q_t K_{1:t}^T) V_{1:t}; MHA caches 2 n_h d_h per token),
     2.2 (c^KV = W^DKV h; W^UK is absorbed into the query side, W^UV into the
     output side) and 2.3 (decoupled RoPE: queries and keys are the
     concatenation of a content part and a small RoPE part; q^R per head, k^R
     shared by all heads; RoPE does not commute with a linear map).

The oracle's definition is the *expanded* one, which the absorbed method
reaches exactly in exact arithmetic: for sequence b, query i and head h,

    m        = T_b - q_len + i                    (position of query i)
    k_j      = [ W_UK[h] c_j  ||  RoPE(kR_j, j) ]   j = 0..m    (192-d)
    v_j      =   W_UV[h] c_j                                    (128-d)
    q        = [ q_nope[b,i,h] || RoPE(qR[b,i,h], m) ]
    s_j      = q . k_j / sqrt(d_n + d_r)
    p        = softmax(s)
    out      = sum_j p_j v_j

Readings where the pages are silent (each is listed in the design notes):
  * softmax scale 1/sqrt(d_n + d_r) (no YaRN factor; YaRN is named on the
    pages without a formula);
  * RoPE rotates consecutive pairs (2k, 2k+1) by pos * base^(-2k/d_r),
    base 10000, positions counted from 0;
  * the cache stores k_R already rotated at its own position; the query RoPE
    part is rotated at the query's position;
  * seqlens include the q_len new tokens; query i sees keys 0..T_b-q_len+i
    (causal between the draft tokens of a speculative verify step);
  * W_UK and W_UV are stored [H, 128, 512]: k_C = W_UK[h] @ c, v = W_UV[h] @ c.

Pins: every function here is checked in ``tests/test_oracle.py`` against
facts that do not come from this file (closed forms, invariants, the pages'
cache counts and a hand-derived example).  None is "parity unpinned".
"""
from __future__ import annotations

import math
from typing import Iterable, List, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "rope",
    "rms_norm",
    "cache_rows",
    "cache_rows_from_hidden",
    "decode_expanded",
    "decode_absorbed",
    "cache_elements_per_token",
    "output_projection",
]


def rope(x: np.ndarray, pos, base: float = 10000.0) -> np.ndarray:
    """Rotary position embedding of the last axis at position(s) ``pos``.

    [P5] section 2.3 applies RoPE to the small position part q^R / k^R only.
    Pair (2k, 2k+1) is rotated by the angle pos * base**(-2k/d_r).
    ``pos`` broadcasts against ``x.shape[:-1]``.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    if d % 2:
        raise ValueError("RoPE width must be even")
    k = np.arange(d // 2, dtype=np.float64)
    inv_freq = base ** (-2.0 * k / d)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * inv_freq  # [..., d/2]
    c, s = np.cos(ang), np.sin(ang)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    out = np.empty(np.broadcast_shapes(x.shape, ang.shape[:-1] + (d,)), dtype=np.float64)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


def cache_rows(c_kv: np.ndarray, k_rope: np.ndarray, positions, base: float = 10000.0) -> np.ndarray:
    """Cache rows written for new tokens: [c_KV || RoPE(k_R, position)].

    [P1] section 二 "MLA：缓存压缩后的历史" and [P3]'s MLA paragraph: per
    token and layer only the latent and the rotated RoPE key are stored.
    c_kv [..., d_c], k_rope [..., d_r], positions broadcast to c_kv.shape[:-1].
    """
    c_kv = np.asarray(c_kv, dtype=np.float64)
    return np.concatenate([c_kv, rope(k_rope, positions, base)], axis=-1)


def rms_norm(v: np.ndarray, gamma: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """RMSNorm over the last axis: v / sqrt(mean(v^2) + eps) * gamma.

    [P5] section 1 names RMSNorm as the normalisation of the V3 block
    (Pre-Norm), and its configuration block gives rms_norm_eps = 1e-6.
    """
    v = np.asarray(v, dtype=np.float64)
    return v / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + eps) * np.asarray(gamma, dtype=np.float64)


def cache_rows_from_hidden(x: np.ndarray, W_DKV: np.ndarray, W_KR: np.ndarray, gamma: np.ndarray, positions,
                           base: float = 10000.0, eps: float = 1e-6) -> np.ndarray:
    """Cache rows computed from the attention block's input x (hidden size d):
    [ RMSNorm_gamma(W_DKV x) || RoPE(W_KR x, position) ].

    [P5] section 2.2 and [P1] section 二: the latent is a down-projection of
    the hidden state, c^KV = W^DKV h (d_c = 512 of hidden 7168); [P3]'s MLA
    panel: the hidden state is projected to c_KV and to the decoupled RoPE key
    k_R, which is stored rotated.  The RMSNorm of the latent (gain gamma) is
    the reading that gives the cached latent its unit scale; x is the block's
    input after its own pre-norm.
    x [..., d]; W_DKV [d_c, d]; W_KR [d_r, d]; gamma [d_c]; positions broadcast to x.shape[:-1].
    """
    x = np.asarray(x, dtype=np.float64)
    c = x @ np.asarray(W_DKV, dtype=np.float64).T
    k = x @ np.asarray(W_KR, dtype=np.float64).T
    return np.concatenate([rms_norm(c, gamma, eps), rope(k, positions, base)], axis=-1)


def _softmax(s: np.ndarray) -> np.ndarray:
    e = np.exp(s - s.max())
    return e / e.sum()


def decode_expanded(q_nope: np.ndarray, q_rope: np.ndarray, W_UK: np.ndarray, W_UV: np.ndarray,
                    histories: Sequence[Tuple[np.ndarray, np.ndarray]], q_len: int,
                    base: float = 10000.0, seqs: Optional[Iterable[int]] = None,
                    heads: Optional[Iterable[int]] = None) -> np.ndarray:
    """Textbook decode attention with K and V expanded per head.

    [P5] section 2.1 (softmax(Q_t K_{1:t}^T) V_{1:t}) with the keys and values
    of [P5] section 2.3 / [P3]'s naive branch: K_h = [W_UK[h] c || k_R],
    V_h = W_UV[h] c.

    q_nope [B, q_len, H, d_n]; q_rope [B, q_len, H, d_r] (un-rotated);
    W_UK [H, d_n, d_c]; W_UV [H, d_v, d_c];
    histories[b] = (c_KV [T_b, d_c], k_R [T_b, d_r] un-rotated) for positions 0..T_b-1.
    Returns out [B, q_len, H, d_v]; entries not selected by ``seqs``/``heads`` are NaN.
    """
    B, QL, H, d_n = q_nope.shape
    assert QL == q_len
    d_r = q_rope.shape[-1]
    d_v = W_UV.shape[1]
    scale = 1.0 / math.sqrt(d_n + d_r)
    out = np.full((B, q_len, H, d_v), np.nan)
    seqs = range(B) if seqs is None else list(seqs)
    heads = range(H) if heads is None else list(heads)
    for b in seqs:
        c, k_raw = histories[b]
        c = np.asarray(c, dtype=np.float64)
        T = c.shape[0]
        if T < q_len:
            raise ValueError("a sequence must already hold its q_len new tokens")
        k_rot = rope(k_raw, np.arange(T), base)  # key j rotated at its own position j
        for h in heads:
            K = np.concatenate([c @ W_UK[h].T, k_rot], axis=1)  # [T, d_n + d_r]
            V = c @ W_UV[h].T  # [T, d_v]
            for i in range(q_len):
                m = T - q_len + i
                q = np.concatenate([q_nope[b, i, h], rope(q_rope[b, i, h], m, base)])
                s = (K[: m + 1] @ q) * scale
                p = _softmax(s)
                out[b, i, h] = p @ V[: m + 1]
    return out


def decode_absorbed(q_nope: np.ndarray, q_rope: np.ndarray, W_UK: np.ndarray, W_UV: np.ndarray,
                    histories: Sequence[Tuple[np.ndarray, np.ndarray]], q_len: int,
                    base: float = 10000.0, seqs: Optional[Iterable[int]] = None,
                    return_latent: bool = False):
    """The same decode in absorbed order, on the CPU in fp64.

    [P1] section 二's identity q^T (U c) = (U^T q)^T c for the content
    branch, with the RoPE score added separately; [P3]'s MLA panel: aggregate
    sum_j p_j c_j in latent space, then apply W_UV.  Used to cover all heads at
    sizes where the expanded form is too slow; it is itself pinned to the
    expanded form by the identity tests.
    Returns out [B, q_len, H, d_v] (and the latent o_lat [B, q_len, H, d_c]).
    """
    B, QL, H, d_n = q_nope.shape
    d_r = q_rope.shape[-1]
    d_c = W_UK.shape[2]
    d_v = W_UV.shape[1]
    scale = 1.0 / math.sqrt(d_n + d_r)
    out = np.full((B, q_len, H, d_v), np.nan)
    olat = np.full((B, q_len, H, d_c), np.nan)
    seqs = range(B) if seqs is None else list(seqs)
    for b in seqs:
        c, k_raw = histories[b]
        c = np.asarray(c, dtype=np.float64)
        T = c.shape[0]
        k_rot = rope(k_raw, np.arange(T), base)
        for i in range(q_len):
            m = T - q_len + i
            q_lat = np.einsum("hdc,hd->hc", W_UK, q_nope[b, i])  # W_UK[h]^T q_nope, [H, d_c]
            q_rot = rope(q_rope[b, i], m, base)  # [H, d_r]
            S = (c[: m + 1] @ q_lat.T + k_rot[: m + 1] @ q_rot.T) * scale  # [m+1, H]
            S = S - S.max(axis=0, keepdims=True)
            P = np.exp(S)
            P /= P.sum(axis=0, keepdims=True)
            o = P.T @ c[: m + 1]  # [H, d_c]
            olat[b, i] = o
            out[b, i] = np.einsum("hvc,hc->hv", W_UV, o)
    return (out, olat) if return_latent else out


def output_projection(out: np.ndarray, W_O: np.ndarray) -> np.ndarray:
    """The block's output projection after W_UV: y = W_O concat_h(out_h).

    [P3]'s MLA panel: aggregate sum_j p_j c_KV,j, then W_UV and the output
    projection; the MLA steps of the taojin168.com forum page (section 2.1,
    last step): the attention output is mapped back to the model width.
    out [..., H, d_v]; W_O [d, H * d_v] (head-major columns).  Returns [..., d].
    """
    out = np.asarray(out, dtype=np.float64)
    flat = out.reshape(out.shape[:-2] + (out.shape[-2] * out.shape[-1],))
    return flat @ np.asarray(W_O, dtype=np.float64).T


def cache_elements_per_token(H: int, d_c: int, d_r: int, d_n: int, d_v: int):
    """Elements cached per token per layer: (absorbed MLA, standard MHA, naive MLA).

    [P3] cache-count paragraph: MLA keeps d_c + d_r; MHA keeps H*(d_n + d_v)
    (its [P5] section 2.1 form 2 n_h d_h with d_h = d_n = d_v); the naive MLA
    branch caches expanded keys H*(d_n + d_r) and values H*d_v.
    """
    return d_c + d_r, H * (d_n + d_v), H * (d_n + d_r + d_v)

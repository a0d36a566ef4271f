"""Pins for the CPU fp64 oracle: facts that do not come from the oracle itself.

Each test fixes one part of the oracle against a closed form, an invariant of
the mathematics, a hand-derived example, or the figures the pages print, so
that a dropped term, a wrong sign, a wrong position or a transposed operand in
the oracle fails at least one of them.
"""
import math
import os

import numpy as np
import pytest

from oracle import (cache_elements_per_token, cache_rows, cache_rows_from_hidden, decode_absorbed, decode_expanded,
                    output_projection, rms_norm, rope)
from latent_compressed_attention_absorbed_b200 import workload as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                k, v = line.split()
                vals[k] = float(v)
    return vals


def _rand_problem(rng, B=2, H=3, d_c=12, d_r=4, d_n=6, d_v=5, T=(9, 5), q_len=1, w=0.4):
    qn = rng.standard_normal((B, q_len, H, d_n))
    qr = rng.standard_normal((B, q_len, H, d_r))
    W_UK = rng.standard_normal((H, d_n, d_c)) * w
    W_UV = rng.standard_normal((H, d_v, d_c)) * w
    hist = [(rng.standard_normal((t, d_c)), rng.standard_normal((t, d_r))) for t in T]
    return qn, qr, W_UK, W_UV, hist


# ------------------------------------------------------------------ page figures

def test_cache_counts_match_the_pages():
    g = _golden("v3_mla_cache_counts.txt")
    H, d_c, d_r = int(g["heads"]), int(g["kv_latent_rank"]), int(g["qk_rope_head_dim"])
    d_n, d_v = int(g["qk_nope_head_dim"]), int(g["v_head_dim"])
    mla, mha, naive = cache_elements_per_token(H, d_c, d_r, d_n, d_v)
    assert mla == g["mla_cached_elements_per_token_per_layer"]
    assert mha == g["mha_cached_elements_per_token_per_layer"]
    assert naive == g["naive_mla_cached_elements_per_token_per_layer"]
    assert round(100.0 * (1.0 - mla / mha), 2) == g["mla_reduction_vs_mha_percent"]


def test_v3_workload_shapes_follow_the_page_table():
    g = _golden("v3_mla_cache_counts.txt")
    for name in ("v3_b1", "v3_b64", "v3_long", "v3_ragged"):
        c = wl.CONFIGS[name]
        assert (c.H, c.d_c, c.d_n, c.d_r, c.d_v) == (
            g["heads"], g["kv_latent_rank"], g["qk_nope_head_dim"], g["qk_rope_head_dim"], g["v_head_dim"])
        assert c.row == g["mla_cached_elements_per_token_per_layer"]


# ------------------------------------------------------------------ RoPE

def test_rope_position_zero_is_identity():
    x = np.random.default_rng(1).standard_normal((7, 64))
    np.testing.assert_array_equal(rope(x, 0), x)


def test_rope_closed_form_pairs_and_frequencies():
    # d_r = 4: pair (0,1) turns by pos * 1, pair (2,3) by pos * base**(-1/2).
    base, pos = 10000.0, 3.0
    a0, a1 = pos, pos * base ** -0.5
    np.testing.assert_allclose(rope(np.array([1.0, 0, 0, 0]), pos), [math.cos(a0), math.sin(a0), 0, 0], atol=1e-15)
    np.testing.assert_allclose(rope(np.array([0, 1.0, 0, 0]), pos), [-math.sin(a0), math.cos(a0), 0, 0], atol=1e-15)
    np.testing.assert_allclose(rope(np.array([0, 0, 1.0, 0]), pos), [0, 0, math.cos(a1), math.sin(a1)], atol=1e-15)
    np.testing.assert_allclose(rope(np.array([0, 0, 0, 1.0]), pos), [0, 0, -math.sin(a1), math.cos(a1)], atol=1e-15)


def test_rope_preserves_norm_and_is_relative():
    rng = np.random.default_rng(2)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    for m, n in [(5, 2), (4095, 17), (131071, 131000)]:
        qm, kn = rope(q, m), rope(k, n)
        assert abs(np.linalg.norm(qm) - np.linalg.norm(q)) < 1e-12
        # <R_m q, R_n k> depends on m - n only
        assert abs(qm @ kn - rope(q, m - n) @ k) < 1e-9


def test_cache_rows_layout():
    rng = np.random.default_rng(3)
    c, k = rng.standard_normal((3, 10)), rng.standard_normal((3, 4))
    rows = cache_rows(c, k, np.array([0, 5, 9]))
    np.testing.assert_array_equal(rows[:, :10], c)
    np.testing.assert_array_equal(rows[0, 10:], k[0])
    np.testing.assert_allclose(rows[2, 10:], rope(k[2], 9), atol=1e-15)


# ------------------------------------------------------------------ cache rows from the hidden state

def test_rms_norm_hand_example_and_invariants():
    # v = (3, 4): mean of squares 12.5, so v / sqrt(12.5 + eps) * gamma.
    eps = 1e-6
    got = rms_norm(np.array([3.0, 4.0]), np.array([2.0, -1.0]), eps)
    d = math.sqrt(12.5 + eps)
    np.testing.assert_allclose(got, [6.0 / d, -4.0 / d], rtol=1e-15)
    rng = np.random.default_rng(15)
    v = rng.standard_normal((5, 512))
    # scale invariance (eps = 0) and unit rms with gamma = 1
    np.testing.assert_allclose(rms_norm(v * 37.0, np.ones(512), 0.0), rms_norm(v, np.ones(512), 0.0), rtol=1e-13)
    np.testing.assert_allclose(np.sqrt(np.mean(rms_norm(v, np.ones(512), 0.0) ** 2, axis=-1)), 1.0, rtol=1e-13)


def test_cache_rows_from_hidden_hand_example():
    # d = 2, d_c = 2, d_r = 2: x = (1, 2); W_DKV = I -> c = (1, 2), mean square 2.5;
    # W_KR = [[1, 1], [0, 1]] -> k = (3, 2), rotated at position p by angle p (pair 0).
    x = np.array([[1.0, 2.0]])
    W_DKV = np.eye(2)
    W_KR = np.array([[1.0, 1.0], [0.0, 1.0]])
    gamma = np.array([0.5, 3.0])
    p, eps = 5, 1e-6
    rows = cache_rows_from_hidden(x, W_DKV, W_KR, gamma, np.array([p]), eps=eps)
    d = math.sqrt(2.5 + eps)
    np.testing.assert_allclose(rows[0], [0.5 / d, 6.0 / d, 3 * math.cos(p) - 2 * math.sin(p),
                                         3 * math.sin(p) + 2 * math.cos(p)], rtol=1e-14, atol=1e-15)


def test_cache_rows_from_hidden_properties():
    rng = np.random.default_rng(16)
    x = rng.standard_normal((3, 40))
    W_DKV, W_KR = rng.standard_normal((12, 40)), rng.standard_normal((4, 40))
    gamma = rng.standard_normal(12)
    pos = np.array([0, 7, 300])
    rows = cache_rows_from_hidden(x, W_DKV, W_KR, gamma, pos, eps=0.0)
    # the latent part does not change when x is scaled (RMSNorm after a linear map)
    rows2 = cache_rows_from_hidden(4.5 * x, W_DKV, W_KR, gamma, pos, eps=0.0)
    np.testing.assert_allclose(rows2[:, :12], rows[:, :12], rtol=1e-12)
    # the RoPE part is linear in x and keeps the norm of W_KR x
    np.testing.assert_allclose(rows2[:, 12:], 4.5 * rows[:, 12:], rtol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(rows[:, 12:], axis=1), np.linalg.norm(x @ W_KR.T, axis=1), rtol=1e-12)
    # position 0 leaves the key unrotated
    np.testing.assert_allclose(rows[0, 12:], W_KR @ x[0], rtol=1e-12)


def test_output_projection_hand_example():
    # H = 2, d_v = 2, d = 1: out = [[1, 2], [3, 4]] (head-major) and W_O = [[10, 20, 30, 40]]
    # give y = 10 + 40 + 90 + 160 = 300.
    y = output_projection(np.array([[1.0, 2.0], [3.0, 4.0]]), np.array([[10.0, 20.0, 30.0, 40.0]]))
    assert y.shape == (1,) and y[0] == 300.0


def test_output_projection_folds_with_W_UV():
    # W_O (W_UV o) = (W_O W_UV) o per head: projecting the decode's per-head
    # outputs equals applying the folded per-head maps W_O[:, h] W_UV[h] to the
    # latent aggregates o_h (associativity; the order the pages describe).
    rng = np.random.default_rng(17)
    qn, qr, W_UK, W_UV, hist = _rand_problem(rng)
    W_O = rng.standard_normal((7, 3 * 5))
    out, olat = decode_absorbed(qn, qr, W_UK, W_UV, hist, q_len=1, return_latent=True)
    y = output_projection(out, W_O)
    folded = sum(olat[..., h, :] @ (W_O[:, 5 * h:5 * h + 5] @ W_UV[h]).T for h in range(3))
    np.testing.assert_allclose(y, folded, rtol=1e-12)


# ------------------------------------------------------------------ decode: closed forms

def test_softmax_hand_example_and_invariants():
    # The softmax the decode applies per score row: weights proportional to
    # e^s that sum to one, unchanged by a constant shift, and [0, ln 2] gives
    # [1/3, 2/3] by hand.
    from oracle.mla_oracle import _softmax

    np.testing.assert_allclose(_softmax(np.array([0.0, math.log(2.0)])), [1.0 / 3.0, 2.0 / 3.0], rtol=1e-15)
    rng = np.random.default_rng(8)
    for n in (1, 7, 4096):
        s = rng.standard_normal(n) * 10.0
        p = _softmax(s)
        assert abs(p.sum() - 1.0) < 1e-12 and (p >= 0).all()
        np.testing.assert_allclose(_softmax(s + 123.25), p, rtol=1e-12, atol=1e-300)
        np.testing.assert_allclose(p[1:] / p[:-1] if n > 1 else p, np.exp(np.diff(s)) if n > 1 else [1.0],
                                   rtol=1e-9)
    # a score of -inf (a key the query may not see) gets weight zero
    p = _softmax(np.array([0.5, -np.inf, 0.5]))
    np.testing.assert_array_equal(p, [0.5, 0.0, 0.5])


def test_single_token_history_returns_W_UV_c():
    # T = 1: the softmax over one key is 1, so out_h = W_UV[h] c_0 whatever the query.
    qn, qr, W_UK, W_UV, hist = _rand_problem(np.random.default_rng(4), T=(1, 1))
    out = decode_expanded(qn, qr, W_UK, W_UV, hist, q_len=1)
    for b in range(2):
        for h in range(3):
            np.testing.assert_allclose(out[b, 0, h], W_UV[h] @ hist[b][0][0], rtol=1e-14)


def test_zero_query_gives_uniform_average():
    # q = 0: every score is 0, p is uniform, out_h = W_UV[h] mean_j c_j.
    qn, qr, W_UK, W_UV, hist = _rand_problem(np.random.default_rng(5))
    qn[:] = 0
    qr[:] = 0
    out = decode_expanded(qn, qr, W_UK, W_UV, hist, q_len=1)
    for b in range(2):
        for h in range(3):
            np.testing.assert_allclose(out[b, 0, h], W_UV[h] @ hist[b][0].mean(axis=0), rtol=1e-12)


def test_equal_latents_give_that_value_whatever_the_weights():
    # All c_j equal: every V row is W_UV c, so out = W_UV c exactly when sum p = 1,
    # even though the RoPE scores make p non-uniform.
    qn, qr, W_UK, W_UV, hist = _rand_problem(np.random.default_rng(6), T=(9, 9))
    hist = [(np.tile(c[:1], (c.shape[0], 1)), k) for c, k in hist]
    out = decode_expanded(qn, qr, W_UK, W_UV, hist, q_len=1)
    for b in range(2):
        for h in range(3):
            np.testing.assert_allclose(out[b, 0, h], W_UV[h] @ hist[b][0][0], rtol=1e-12)


def test_hand_derived_two_key_example():
    # H=1, d_c=d_n=d_v=1, d_r=2, T=2, q_len=1 (query at position 1).
    # Content: W_UK=a, W_UV=1, c=(1, 2), q_nope=x   -> content scores a*x*c_j.
    # RoPE: k_R=(1,0) at positions 0 and 1, q_R=(1,0) at position 1, theta_0 = 1 rad:
    #   key 0 rotated by 0 -> (1,0); key 1 -> (cos1, sin1); query -> (cos1, sin1)
    #   RoPE scores: cos(1) and 1.
    # s_j = (a x c_j + r_j)/sqrt(3); out = (1*e^{s0} + 2*e^{s1}) / (e^{s0} + e^{s1}).
    a, x = 0.7, -1.3
    W_UK = np.array([[[a]]])
    W_UV = np.array([[[1.0]]])
    hist = [(np.array([[1.0], [2.0]]), np.array([[1.0, 0.0], [1.0, 0.0]]))]
    qn = np.array([[[[x]]]])
    qr = np.array([[[[1.0, 0.0]]]])
    s0 = (a * x * 1.0 + math.cos(1.0)) / math.sqrt(3.0)
    s1 = (a * x * 2.0 + 1.0) / math.sqrt(3.0)
    expect = (1.0 * math.exp(s0) + 2.0 * math.exp(s1)) / (math.exp(s0) + math.exp(s1))
    out_e = decode_expanded(qn, qr, W_UK, W_UV, hist, q_len=1)
    out_a = decode_absorbed(qn, qr, W_UK, W_UV, hist, q_len=1)
    assert abs(out_e[0, 0, 0, 0] - expect) < 1e-14
    assert abs(out_a[0, 0, 0, 0] - expect) < 1e-14


def test_hand_derived_rope_base_applies_to_keys_and_queries():
    # Decoupled RoPE rotates q^R and k^R alike (m.lsln.cn/news/222502 section 2.3),
    # so a non-default base must turn the keys too.  H=1, d_c=d_n=d_v=1, d_r=4,
    # T=2, q_len=1 (query at position 1), content branch off (W_UK = 0).
    # Only RoPE pair 1 is used; it turns by pos * base**(-1/2) (pair 0 by pos,
    # whatever the base).  k_R = (0,0,1,0) at positions 0 and 1 -> (0,0,1,0) and
    # (0,0,cos a,sin a); q_R = (0,0,1,0) at position 1 -> (0,0,cos a,sin a), with
    # a = base**-0.5.  RoPE scores: cos a and 1.  Scale 1/sqrt(d_n + d_r) = 1/sqrt(5).
    base = 500.0
    a = base ** -0.5
    W_UK = np.zeros((1, 1, 1))
    W_UV = np.ones((1, 1, 1))
    hist = [(np.array([[1.0], [2.0]]), np.array([[0.0, 0.0, 1.0, 0.0], [0.0, 0.0, 1.0, 0.0]]))]
    qn = np.zeros((1, 1, 1, 1))
    qr = np.array([[[[0.0, 0.0, 1.0, 0.0]]]])
    s0, s1 = math.cos(a) / math.sqrt(5.0), 1.0 / math.sqrt(5.0)
    expect = (1.0 * math.exp(s0) + 2.0 * math.exp(s1)) / (math.exp(s0) + math.exp(s1))
    out_e = decode_expanded(qn, qr, W_UK, W_UV, hist, q_len=1, base=base)
    out_a = decode_absorbed(qn, qr, W_UK, W_UV, hist, q_len=1, base=base)
    assert abs(out_e[0, 0, 0, 0] - expect) < 1e-14
    assert abs(out_a[0, 0, 0, 0] - expect) < 1e-14
    # the cached key rows written for those tokens carry the same rotation
    rows = cache_rows(hist[0][0], hist[0][1], np.arange(2), base)
    np.testing.assert_allclose(rows[1, 1:], [0.0, 0.0, math.cos(a), math.sin(a)], atol=1e-15)


def test_scores_depend_on_relative_position_only_at_any_base():
    # The RoPE score of a query at m and a key at n, at a non-default base, equals
    # the closed form of turning each pair by (m - n) theta_k, theta_k = base**(-2k/d):
    #   (q0 k0 + q1 k1) cos((m-n) theta_k) + (q0 k1 - q1 k0) sin((m-n) theta_k).
    base = 777.0
    rng = np.random.default_rng(14)
    q, k = rng.standard_normal(8), rng.standard_normal(8)
    for m, n in [(9, 4), (1000, 3)]:
        lhs = rope(q, m, base) @ rope(k, n, base)
        inv = base ** (-2.0 * np.arange(4) / 8.0)
        ang = (m - n) * inv
        # closed form of the pairwise rotation by (m - n) theta_k
        rhs = sum((q[2 * i] * k[2 * i] + q[2 * i + 1] * k[2 * i + 1]) * math.cos(ang[i])
                  + (q[2 * i] * k[2 * i + 1] - q[2 * i + 1] * k[2 * i]) * math.sin(ang[i]) for i in range(4))
        assert abs(lhs - rhs) < 1e-9


def test_hand_derived_causal_pair():
    # q_len = 2, T = 2, same one-dimensional set-up with q_R = 0: query 0 sits at
    # position 0 and sees key 0 only, so out = c_0 = 1; query 1 sees both keys.
    a, x = 0.5, 2.0
    W_UK = np.array([[[a]]])
    W_UV = np.array([[[1.0]]])
    hist = [(np.array([[1.0], [3.0]]), np.zeros((2, 2)))]
    qn = np.full((1, 2, 1, 1), x)
    qr = np.zeros((1, 2, 1, 2))
    out = decode_expanded(qn, qr, W_UK, W_UV, hist, q_len=2)
    s0, s1 = a * x * 1.0 / math.sqrt(3.0), a * x * 3.0 / math.sqrt(3.0)
    assert abs(out[0, 0, 0, 0] - 1.0) < 1e-15
    expect1 = (math.exp(s0) + 3.0 * math.exp(s1)) / (math.exp(s0) + math.exp(s1))
    assert abs(out[0, 1, 0, 0] - expect1) < 1e-14


# ------------------------------------------------------------------ decode: invariants

@pytest.mark.parametrize("q_len", [1, 2])
def test_absorbed_equals_expanded(q_len):
    # The identity q^T (U c) = (U^T q)^T c: both orders agree to fp64 rounding.
    rng = np.random.default_rng(7 + q_len)
    for dims in [dict(), dict(H=4, d_c=32, d_r=8, d_n=16, d_v=16, T=(64, 33)),
                 dict(H=2, d_c=64, d_r=16, d_n=24, d_v=8, T=(70, 3))]:
        qn, qr, W_UK, W_UV, hist = _rand_problem(rng, q_len=q_len, **dims)
        e = decode_expanded(qn, qr, W_UK, W_UV, hist, q_len=q_len)
        a = decode_absorbed(qn, qr, W_UK, W_UV, hist, q_len=q_len)
        assert np.linalg.norm(e - a) <= 1e-12 * np.linalg.norm(e)


def test_causality_of_the_draft_token():
    qn, qr, W_UK, W_UV, hist = _rand_problem(np.random.default_rng(10), q_len=2, T=(12, 6))
    base = decode_expanded(qn, qr, W_UK, W_UV, hist, q_len=2)
    c, k = hist[0]
    c2, k2 = c.copy(), k.copy()
    c2[-1] += 1.0
    k2[-1] -= 1.0
    pert = decode_expanded(qn, qr, W_UK, W_UV, [(c2, k2), hist[1]], q_len=2)
    np.testing.assert_array_equal(pert[0, 0], base[0, 0])  # query 0 never sees the last key
    assert np.abs(pert[0, 1] - base[0, 1]).max() > 1e-6  # query 1 does
    np.testing.assert_array_equal(pert[1], base[1])


def test_rope_branch_is_not_absorbable():
    # Rotating the expanded content key by its position (the garbled ordering that
    # puts RoPE on the up-projected key) is not the same operator: the oracle's
    # decoupled branch must differ from it on generic inputs.
    rng = np.random.default_rng(11)
    qn, qr, W_UK, W_UV, hist = _rand_problem(rng, B=1, H=1, d_c=8, d_r=4, d_n=4, d_v=3, T=(6,))
    out = decode_expanded(qn, qr, W_UK, W_UV, hist, q_len=1)
    c, k = hist[0]
    T = c.shape[0]
    K_alt = np.concatenate([rope(c @ W_UK[0].T, np.arange(T)), rope(k, np.arange(T))], 1)
    q_alt = np.concatenate([rope(qn[0, 0, 0], T - 1), rope(qr[0, 0, 0], T - 1)])
    s = K_alt @ q_alt / math.sqrt(8.0)
    p = np.exp(s - s.max())
    p /= p.sum()
    alt = p @ (c @ W_UV[0].T)
    assert np.abs(alt - out[0, 0, 0]).max() > 1e-3


def test_zero_rope_reduces_to_content_only_attention():
    # q_R = 0 and k_R = 0: the RoPE branch contributes nothing and the result is
    # plain softmax attention over the expanded content keys (scale unchanged).
    qn, qr, W_UK, W_UV, hist = _rand_problem(np.random.default_rng(12))
    qr[:] = 0
    hist0 = [(c, np.zeros_like(k)) for c, k in hist]
    full = decode_expanded(qn, qr, W_UK, W_UV, hist0, q_len=1)
    # content-only expanded attention with the same scale 1/sqrt(d_n + d_r)
    d_n, d_r = qn.shape[-1], 4
    for b in range(2):
        c = hist[b][0]
        for h in range(3):
            s = (c @ W_UK[h].T) @ qn[b, 0, h] / math.sqrt(d_n + d_r)
            p = np.exp(s - s.max())
            p /= p.sum()
            np.testing.assert_allclose(full[b, 0, h], p @ (c @ W_UV[h].T), rtol=1e-12)


# ------------------------------------------------------------------ workload generator

def test_bf16_rounding_matches_torch():
    torch = pytest.importorskip("torch")
    x = np.random.default_rng(13).standard_normal(100000) * 3.0
    x[:4] = [0.0, -0.0, 1.00390625, 1.01171875]  # exact ties: round to even
    mine = wl.round_bf16_bits(x)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(mine, ref)


def test_ragged_seqlens_recipe():
    s = np.array(wl.CONFIGS["v3_ragged"].seqlens)
    assert len(s) == 128 and s.min() >= 2048 and s.max() <= 16384
    assert (s.min(), s.max(), int(s.sum())) == (2087, 16344, 1199369)


def test_streams_are_per_sequence():
    cfg = wl.CONFIGS["v3_ragged"].with_(seqlens=(5, 7, 9), B=3)
    c1, _ = wl.sequence_history(cfg, 1)
    cfg2 = cfg.with_(seqlens=(50, 7, 1), B=3)
    c1b, _ = wl.sequence_history(cfg2, 1)
    np.testing.assert_array_equal(c1.raw, c1b.raw)

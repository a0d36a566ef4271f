"""GPU parity: the CUDA library (through its C ABI) against the CPU fp64 oracle.

Small cases compare every output element; the full-size workloads compare
sampled sequences (all heads through the fp64 absorbed form, a few heads
through the fp64 expanded form, which is the definition).
"""
import numpy as np
import pytest
import torch

from oracle import cache_rows, decode_absorbed, decode_expanded
from latent_compressed_attention_absorbed_b200 import workload as wl
from mla_testutil import Problem, as_f64, check_close, dims_of, to_device, torch_dtype

pytestmark = pytest.mark.gpu

V3 = wl.CONFIGS["v3_b1"]


def _v3(seqlens, q_len=1, seed=11):
    return V3.with_(name="v3_case", B=len(seqlens), seqlens=tuple(seqlens), q_len=q_len, seed=seed)


# ------------------------------------------------------------------ the tiny fp32 workload

def test_tiny_fp32_workload(lib):
    cfg = wl.CONFIGS["tiny"]
    P = Problem(lib, cfg)
    out = P.decode()
    assert lib.last_path() == "generic"
    ref = P.oracle_expanded(range(cfg.B))
    check_close(as_f64(out), ref, "f32", "tiny")


# ------------------------------------------------------------------ append (a1)

@pytest.mark.parametrize("path_cfg", ["v3", "tiny"])
def test_append_rows(lib, path_cfg):
    base = V3 if path_cfg == "v3" else wl.CONFIGS["tiny"]
    cfg = base.with_(B=3, seqlens=(40, 40, 40), seed=5)
    dims = dims_of(lib, cfg)
    T_max, n_tok = 40, 3
    cache = torch.zeros((cfg.B, T_max, cfg.row), dtype=torch_dtype(cfg), device="cuda")
    c, k = wl.new_tokens(cfg, n_tok)
    pos = np.array([0, 17, T_max - n_tok], dtype=np.int32)
    lib.append_cache(dims, cache, to_device(c), to_device(k), torch.from_numpy(pos).cuda())
    assert lib.device_status() == 0
    got = as_f64(cache)
    for b in range(cfg.B):
        rows = cache_rows(c.values[b], k.values[b], pos[b] + np.arange(n_tok), cfg.rope_base)
        want = wl.bf16_bits_to_f64(wl.round_bf16_bits(rows)) if cfg.dtype == "bf16" else rows.astype(np.float32)
        g = got[b, pos[b]:pos[b] + n_tok]
        np.testing.assert_array_equal(g[:, :cfg.d_c], want[:, :cfg.d_c])  # latent copied bit-exactly
        # RoPE key: the kernel rounds once from an fp64 rotation, like the reference rounding
        tol = 2.0 ** -8 if cfg.dtype == "bf16" else 1e-6
        np.testing.assert_allclose(g[:, cfg.d_c:], want[:, cfg.d_c:], rtol=tol, atol=tol)
        untouched = np.ones(T_max, bool)
        untouched[pos[b]:pos[b] + n_tok] = False
        assert not got[b, untouched].any()


def test_append_rejects_out_of_range_positions(lib):
    cfg = V3.with_(B=2, seqlens=(8, 8))
    dims = dims_of(lib, cfg)
    cache = torch.zeros((2, 8, cfg.row), dtype=torch.bfloat16, device="cuda")
    c, k = wl.new_tokens(cfg, 2)
    pos = torch.tensor([7, -1], dtype=torch.int32, device="cuda")  # 7 + 2 > 8, -1 < 0
    lib.append_cache(dims, cache, to_device(c), to_device(k), pos)
    assert lib.device_status() & 1
    assert not cache.float().abs().sum().item()


# ------------------------------------------------------------------ whole decode, small V3 cases

SMALL_CASES = [
    ((1,), 1, 0),          # one key: out = W_UV c_0
    ((64,), 1, 0),         # exactly one tile
    ((65,), 1, 0),         # ragged tail of one key
    ((130, 1, 7, 64), 1, 0),
    ((300, 17), 2, 0),     # speculative verify, causal pair
    ((2, 129), 2, 0),
    ((700, 333, 64), 1, 1),    # one cluster does everything
    ((700, 333, 64), 1, 3),    # sequences cut across clusters
    ((1000, 999), 2, 16),
    ((513, 2000, 5), 3, 7),
    ((257, 1024), 4, 5),
    ((4096,), 1, 64),          # long sequence cut in many pieces
    ((4000,) + (5,) * 24, 1, 0),  # one long sequence among short ones: many pieces in a large batch
    ((3000, 2, 900) * 3, 2, 0),   # ragged verify batch
    ((1500, 9, 260), 8, 0),       # long verify window: 8 query tokens per sequence
    ((16, 700), 16, 5),           # the largest q_len; the first sequence holds only its new tokens
    ((640,) * 7, 1, 8),           # equal lengths: one whole sequence per cluster, one cluster idle
    ((256,) * 7, 2, 8),           # equal lengths: two whole sequences per cluster group
]


@pytest.mark.parametrize("seqlens,q_len,pairs", SMALL_CASES)
def test_decode_small_v3_against_expanded_oracle(lib, seqlens, q_len, pairs):
    cfg = _v3(seqlens, q_len)
    P = Problem(lib, cfg)
    out = P.decode(opts=lib.opts(num_pairs=pairs))
    assert lib.last_path() == "sm100"
    assert lib.device_status() == 0
    ref = P.oracle_expanded(range(cfg.B))
    check_close(as_f64(out), ref, "bf16", f"{seqlens} q_len={q_len} pairs={pairs}")


def test_generic_path_against_expanded_oracle(lib):
    cfg = _v3((130, 7), 2)
    P = Problem(lib, cfg)
    out = P.decode(opts=lib.opts(path=2))
    assert lib.last_path() == "generic"
    check_close(as_f64(out), P.oracle_expanded(range(cfg.B)), "bf16", "generic v3")


def test_single_key_closed_form(lib):
    # T = 1: out_h = W_UV[h] c_0 exactly, whatever the query (softmax of one score is 1).
    cfg = _v3((1, 1), 1, seed=3)
    P = Problem(lib, cfg)
    out = as_f64(P.decode())
    for b in range(2):
        ref = np.einsum("hvc,c->hv", P.w_uv.values, P.history[b][0][0])
        check_close(out[b, 0], ref, "bf16", "T=1")


def test_nan_rows_beyond_length_are_ignored(lib):
    # Rows past seqlens[b] may hold anything (here NaN); masked keys must not leak.
    cfg = _v3((70, 5, 129), 1)
    P = Problem(lib, cfg, T_max=256)
    with torch.no_grad():
        for b, T in enumerate(cfg.seqlens):
            P.cache[b, T:] = float("nan")
    out = P.decode(opts=lib.opts(num_pairs=2))
    assert torch.isfinite(out.float()).all()
    check_close(as_f64(out), P.oracle_expanded(range(cfg.B)), "bf16", "nan tail")


def test_bad_seqlens_are_flagged_and_zeroed(lib):
    cfg = _v3((100, 60), 1)
    P = Problem(lib, cfg)
    P.seqlens = torch.tensor([100, 10 ** 6], dtype=torch.int32, device="cuda")
    out = P.decode()
    assert lib.device_status() & 2
    assert torch.isfinite(out.float()).all()
    assert out[1].float().abs().max().item() == 0.0
    check_close(as_f64(out[:1]), P.oracle_expanded([0])[:1], "bf16", "valid sequence")


# Sharp softmax.  W_UK = 8 x a selection matrix makes every folded query
# component a query component times 8, exactly representable in bf16, so the
# folded query carries no rounding and the score error comes only from the
# kernel's own score arithmetic (the pair's exchange of partial scores).
# Scores then span about +-80 log2 units (std ~19), and the softmax still
# spreads its weight over several keys.  (Scaling a random query instead
# mostly measures the bf16 rounding of the folded query, which grows with the
# scores and is inherent to a bf16 absorbed path.)
SHARP_CASES = [
    ((4096,), 1, 0),
    ((3000, 700), 2, 8),      # split pieces, causal pair
    ((4096, 5, 64), 1, 40),   # many pieces merged by the projection kernel
    ((2000,) * 9, 1, 3),      # more than eight query rows: tensor-core GEMMs and the combine kernel
]


@pytest.mark.parametrize("seqlens,q_len,pairs", SHARP_CASES)
def test_sharp_scores_against_expanded_oracle(lib, seqlens, q_len, pairs):
    cfg = _v3(seqlens, q_len, seed=13).with_(w_uk_select=8.0)
    P = Problem(lib, cfg)
    out = P.decode(opts=lib.opts(num_pairs=pairs))
    assert lib.last_path() == "sm100"
    assert lib.device_status() == 0
    check_close(as_f64(out), P.oracle_expanded(range(cfg.B)), "bf16", f"sharp {seqlens} q_len={q_len}")


@pytest.mark.parametrize("base", [500.0, 1.0e6])
def test_rope_base_through_append_and_decode(lib, base):
    # The cache append rotates k_R and the absorb step rotates q_R with the
    # caller's base; the oracle rotates both with the same base.
    cfg = _v3((700, 333, 65), 2, seed=17).with_(rope_base=base)
    P = Problem(lib, cfg)
    out = P.decode(opts=lib.opts(num_pairs=4))
    assert lib.last_path() == "sm100"
    check_close(as_f64(out), P.oracle_expanded(range(cfg.B)), "bf16", f"rope_base={base}")


@pytest.mark.parametrize("layout", ["padded_rows", "every_other_sequence"])
def test_strided_cache_matches_contiguous_and_oracle(lib, layout):
    # The cache as a view of a larger buffer (rows padded to 640 values, or every
    # other sequence of a batch twice as large), NaN everywhere the view does not
    # cover: the same output, bit for bit, as the contiguous cache.
    cfg = _v3((300, 17, 129), 2)
    P = Problem(lib, cfg)
    ref_out = P.decode(opts=lib.opts(num_pairs=5)).clone()
    T_max = P.cache.shape[1]
    if layout == "padded_rows":
        big = torch.full((cfg.B, T_max, 640), float("nan"), dtype=torch.bfloat16, device="cuda")
        view = big[:, :, :cfg.row]
    else:
        big = torch.full((2 * cfg.B, T_max, cfg.row), float("nan"), dtype=torch.bfloat16, device="cuda")
        view = big[::2]
    view.copy_(P.cache)
    out = lib.decode(P.dims, P.qn, P.qr, P.W_UK, P.W_UV, view, P.seqlens, opts=lib.opts(num_pairs=5))
    assert lib.device_status() == 0
    assert torch.equal(out, ref_out)
    check_close(as_f64(out), P.oracle_expanded(range(cfg.B)), "bf16", f"cache layout {layout}")


def test_repeat_runs_are_bitwise_equal(lib):
    cfg = _v3((900, 77), 2)
    P = Problem(lib, cfg)
    a = P.decode(opts=lib.opts(num_pairs=5)).clone()
    b = P.decode(opts=lib.opts(num_pairs=5))
    assert torch.equal(a, b)


# ------------------------------------------------------------------ the three steps one by one

def test_steps_match_oracle_intermediates(lib):
    cfg = _v3((200, 77), 2, seed=21)
    P = Problem(lib, cfg)
    q_hat = lib.absorb_query(P.dims, P.qn, P.qr, P.W_UK, P.seqlens)
    qh = as_f64(q_hat)
    q_lat_ref = np.einsum("hdc,bihd->bihc", P.w_uk.values, P.q_nope.values)
    check_close(qh[..., :cfg.d_c], q_lat_ref, "bf16", "q_lat")
    from oracle import rope
    m = np.array(cfg.seqlens)[:, None] - cfg.q_len + np.arange(cfg.q_len)[None, :]
    q_rot_ref = rope(P.q_rope.values, m[:, :, None])
    check_close(qh[..., cfg.d_c:], q_rot_ref, "bf16", "q_rot")
    o_lat = lib.attend_latent(P.dims, q_hat, P.cache, P.seqlens, opts=lib.opts(num_pairs=3))
    _, o_ref = P.oracle_absorbed(range(cfg.B), return_latent=True)
    check_close(as_f64(o_lat), o_ref, "bf16", "o_lat")
    out = lib.project_out(P.dims, o_lat, P.W_UV)
    ref = np.einsum("hvc,bihc->bihv", P.w_uv.values, as_f64(o_lat))
    check_close(as_f64(out), ref, "bf16", "W_UV projection")


# ------------------------------------------------------------------ the V3-shaped workloads at full size

def test_workload_v3_b1_full(lib):
    cfg = wl.CONFIGS["v3_b1"]
    P = Problem(lib, cfg)
    out = P.decode()
    assert lib.last_path() == "sm100"
    check_close(as_f64(out), P.oracle_expanded([0]), "bf16", "v3_b1")


def _sampled(lib, name, seqs, heads):
    cfg = wl.CONFIGS[name]
    P = Problem(lib, cfg, keep_history=seqs)
    out = as_f64(P.decode())
    assert lib.last_path() == "sm100"
    assert lib.device_status() == 0
    assert np.all(np.isfinite(out))
    check_close(out[seqs], P.oracle_absorbed(seqs)[seqs], "bf16", f"{name} absorbed-oracle")
    ref = P.oracle_expanded(seqs[:2], heads=heads)
    check_close(out[seqs[:2]][:, :, heads], ref[seqs[:2]][:, :, heads], "bf16", f"{name} expanded-oracle")


def test_workload_v3_b64_sampled(lib):
    _sampled(lib, "v3_b64", [0, 31, 63], [0, 77, 127])


def test_workload_v3_long_every_sequence(lib):
    # All 8 sequences of 128K tokens: every head through the fp64 absorbed form
    # and 4 heads (one per TMEM lane quarter) through the fp64 expanded
    # definition.  Histories are regenerated one sequence at a time.
    cfg = wl.CONFIGS["v3_long"]
    P = Problem(lib, cfg, keep_history=[])
    out = as_f64(P.decode())
    assert lib.last_path() == "sm100"
    assert lib.device_status() == 0
    assert np.all(np.isfinite(out))
    heads = [0, 37, 70, 127]
    for b in range(cfg.B):
        c, k = wl.sequence_history(cfg, b)
        hist = [(None, None)] * cfg.B
        hist[b] = (c.values, k.values)
        del c, k
        args = (P.q_nope.values, P.q_rope.values, P.w_uk.values, P.w_uv.values, hist, cfg.q_len, cfg.rope_base)
        check_close(out[b], decode_absorbed(*args, seqs=[b])[b], "bf16", f"v3_long seq {b} absorbed-oracle")
        ref = decode_expanded(*args, seqs=[b], heads=heads)[b]
        check_close(out[b][:, heads], ref[:, heads], "bf16", f"v3_long seq {b} expanded-oracle")


def test_workload_v3_ragged_sampled(lib):
    s = np.array(wl.CONFIGS["v3_ragged"].seqlens)
    seqs = [int(s.argmin()), int(s.argmax()), 0, 64, 127]
    _sampled(lib, "v3_ragged", seqs, [0, 100])

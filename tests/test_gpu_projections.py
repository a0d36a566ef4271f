"""GPU parity of the projections around the decode (through the C ABI):

* mla_append_from_hidden: cache rows [RMSNorm_gamma(W_DKV x) || RoPE(W_KR x, pos)]
  from the block input x, against the oracle's cache_rows_from_hidden;
* mla_output_projection: y = W_O out, against the oracle's output_projection,
  alone and chained after a decode.

The kernels accumulate bf16 products in fp32 and round the result to bf16
once, so each output element may differ from the fp64 oracle by half a bf16
unit in the last place plus the fp32 accumulation error; the tests allow
one unit (2^-8 relative) plus 1e-3 of the row's rms.
"""
import numpy as np
import pytest
import torch

from oracle import cache_rows_from_hidden, decode_expanded, output_projection
from latent_compressed_attention_absorbed_b200 import workload as wl
from mla_testutil import Problem, as_f64, check_close, dims_of, to_device

pytestmark = pytest.mark.gpu

V3 = wl.CONFIGS["v3_b1"]


def _close_bf16(got, want, what):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    rms = np.sqrt(np.mean(want ** 2, axis=-1, keepdims=True))
    bad = np.abs(got - want) > 2.0 ** -8 * np.abs(want) + 1e-3 * rms
    assert not bad.any(), f"{what}: {bad.sum()} elements off, worst {np.abs(got - want).max():.3e}"


@pytest.mark.parametrize("B,n_tok,d_model", [(3, 2, 7168), (70, 2, 7168), (2, 1, 1024), (1, 3, 4160)])
def test_append_from_hidden_against_oracle(lib, B, n_tok, d_model):
    cfg = V3.with_(B=B, seqlens=(40,) * B, seed=23, d_model=d_model)
    dims = dims_of(lib, cfg)
    T_max = 40
    cache = torch.zeros((B, T_max, cfg.row), dtype=torch.bfloat16, device="cuda")
    x = wl.block_input(cfg, n_tok)
    w_a, gamma = wl.append_weights(cfg)
    pos = np.array([(17 * b) % (T_max - n_tok + 1) for b in range(B)], dtype=np.int32)
    lib.append_from_hidden(dims, cache, to_device(x), to_device(w_a), to_device(gamma), torch.from_numpy(pos).cuda())
    assert lib.device_status() == 0
    got = as_f64(cache)
    W = w_a.values
    for b in range(B):
        want = cache_rows_from_hidden(x.values[b], W[:cfg.d_c], W[cfg.d_c:], gamma.values, pos[b] + np.arange(n_tok),
                                      cfg.rope_base)
        rows = got[b, pos[b]:pos[b] + n_tok]
        _close_bf16(rows[:, :cfg.d_c], want[:, :cfg.d_c], f"latent b={b}")
        _close_bf16(rows[:, cfg.d_c:], want[:, cfg.d_c:], f"RoPE key b={b}")
        untouched = np.ones(T_max, bool)
        untouched[pos[b]:pos[b] + n_tok] = False
        assert not got[b, untouched].any()


def test_append_from_hidden_rejects_out_of_range_positions(lib):
    cfg = V3.with_(B=2, seqlens=(8, 8), seed=24, d_model=1024)
    dims = dims_of(lib, cfg)
    cache = torch.zeros((2, 8, cfg.row), dtype=torch.bfloat16, device="cuda")
    x = wl.block_input(cfg, 2)
    w_a, gamma = wl.append_weights(cfg)
    pos = torch.tensor([7, -1], dtype=torch.int32, device="cuda")
    lib.append_from_hidden(dims, cache, to_device(x), to_device(w_a), to_device(gamma), pos)
    assert lib.device_status() & 1
    assert not cache.float().abs().sum().item()


@pytest.mark.parametrize("rows,d_model", [(3, 7168), (200, 7168), (1, 1024), (256, 4096)])
def test_output_projection_against_oracle(lib, rows, d_model):
    cfg = V3.with_(seed=25, d_model=d_model)
    dims = dims_of(lib, cfg)
    a = wl.Stored(np.random.default_rng(26).standard_normal((rows, cfg.H, cfg.d_v)) * 0.05, "bf16")
    w_o = wl.output_weights(cfg)
    y = lib.output_projection(dims, to_device(a), to_device(w_o))
    assert lib.device_status() == 0
    _close_bf16(as_f64(y), output_projection(a.values, w_o.values), f"W_O rows={rows}")


def test_decode_then_output_projection_against_oracle(lib):
    # The whole attention block from the cache to the block output.
    cfg = V3.with_(name="block", B=3, seqlens=(700, 65, 1300), q_len=2, seed=27)
    P = Problem(lib, cfg)
    out = P.decode(opts=lib.opts(num_pairs=5))
    w_o = wl.output_weights(cfg)
    y = lib.output_projection(P.dims, out, to_device(w_o))
    ref = output_projection(decode_expanded(P.q_nope.values, P.q_rope.values, P.w_uk.values, P.w_uv.values,
                                            P.histories(), cfg.q_len, cfg.rope_base), w_o.values)
    check_close(as_f64(y).reshape(ref.shape[:-1] + (1, -1)), ref[..., None, :], "bf16", "decode + W_O")

"""Shared helpers of the GPU parity tests: upload seeded inputs, fill the
cache through the library's append entry point, run the oracle on a chosen
subset, and compare with the tolerances of the numerics contract.

Tolerances (floating point):
  bf16 storage, fp32 accumulation: relative L2 <= 5e-3 over the array and
      max|gpu - ref| / rms(ref of the same query token) <= 2e-2
  fp32 storage (tiny case):        relative L2 <= 1e-5
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import decode_absorbed, decode_expanded
from latent_compressed_attention_absorbed_b200 import workload as wl

TOL_BF16_REL_L2 = 5e-3
TOL_BF16_MAX_OVER_RMS = 2e-2
TOL_F32_REL_L2 = 1e-5


def to_device(st: wl.Stored, device="cuda") -> torch.Tensor:
    if st.dtype == "bf16":
        return torch.from_numpy(st.raw.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(st.raw).to(device)


def torch_dtype(cfg) -> torch.dtype:
    return torch.bfloat16 if cfg.dtype == "bf16" else torch.float32


def dims_of(lib, cfg):
    return lib.dims(cfg.H, cfg.d_c, cfg.d_r, cfg.d_n, cfg.d_v, torch_dtype(cfg), cfg.rope_base)


class Problem:
    """Device-resident inputs of one workload plus the host values the oracle needs."""

    def __init__(self, lib, cfg, keep_history=None, T_max=None, device="cuda"):
        self.lib, self.cfg = lib, cfg
        self.dims = dims_of(lib, cfg)
        self.w_uk, self.w_uv = wl.weights(cfg)
        self.q_nope, self.q_rope = wl.queries(cfg)
        self.W_UK = to_device(self.w_uk)
        self.W_UV = to_device(self.w_uv)
        self.qn = to_device(self.q_nope)
        self.qr = to_device(self.q_rope)
        self.seqlens = torch.tensor(cfg.seqlens, dtype=torch.int32, device=device)
        T_max = T_max or cfg.T_max
        self.cache = torch.zeros((cfg.B, T_max, cfg.row), dtype=torch_dtype(cfg), device=device)
        keep = set(range(cfg.B)) if keep_history is None else set(keep_history)
        self.history = {}
        zero = torch.zeros(1, dtype=torch.int32, device=device)
        for b in range(cfg.B):
            c, k = wl.sequence_history(cfg, b)
            cd = to_device(c)[None]
            kd = to_device(k)[None]
            lib.append_cache(self.dims, self.cache[b:b + 1], cd, kd, zero)
            if b in keep:
                self.history[b] = (c.values, k.values)
            del cd, kd
        assert lib.device_status() == 0

    def histories(self):
        return [self.history.get(b, (None, None)) for b in range(self.cfg.B)]

    def decode(self, opts=None):
        return self.lib.decode(self.dims, self.qn, self.qr, self.W_UK, self.W_UV, self.cache, self.seqlens,
                               opts=opts)

    def oracle_absorbed(self, seqs, return_latent=False):
        return decode_absorbed(self.q_nope.values, self.q_rope.values, self.w_uk.values, self.w_uv.values,
                               self.histories(), self.cfg.q_len, self.cfg.rope_base, seqs=seqs,
                               return_latent=return_latent)

    def oracle_expanded(self, seqs, heads=None):
        return decode_expanded(self.q_nope.values, self.q_rope.values, self.w_uk.values, self.w_uv.values,
                               self.histories(), self.cfg.q_len, self.cfg.rope_base, seqs=seqs, heads=heads)


def as_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (8 significant bits): 2^(e-7) for |x| in [2^e, 2^(e+1))."""
    _, E = np.frexp(np.abs(x))
    return np.where(x == 0, 0.0, np.ldexp(1.0, E - 8))


def check_close(gpu: np.ndarray, ref: np.ndarray, dtype: str, what: str = ""):
    """Compare GPU output with the oracle (NaN in ``ref`` = not computed).

    The last two axes (heads, features) belong to one query token; every
    leading axis indexes tokens.  "Max abs error on unit-scale outputs" is
    taken per token: each token's errors are divided by the rms of that
    token's reference output, because the natural scale of an attention
    output depends on its history length (an average over T latents shrinks
    like 1/sqrt(T)).  For bf16 results the half-unit-in-the-last-place
    rounding of the bf16 format itself is not charged (the exact reference,
    merely rounded to bf16, already shows up to ~1.4e-2 on this measure),
    just as input quantisation is not charged.  The relative L2 error is
    taken over the whole array with nothing excused.
    """
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    mask = ~np.isnan(ref)
    g, r = gpu[mask], ref[mask]
    assert g.size > 0
    assert np.all(np.isfinite(g)), f"{what}: non-finite GPU values"
    err = g - r
    rel_l2 = float(np.linalg.norm(err) / max(np.linalg.norm(r), 1e-300))
    if dtype != "bf16":
        assert rel_l2 <= TOL_F32_REL_L2, f"{what}: rel L2 {rel_l2:.3e} > {TOL_F32_REL_L2}"
        return rel_l2, None
    assert rel_l2 <= TOL_BF16_REL_L2, f"{what}: rel L2 {rel_l2:.3e} > {TOL_BF16_REL_L2}"
    R = ref.reshape((-1,) + ref.shape[-2:]) if ref.ndim >= 2 else ref[None, None]
    G = gpu.reshape(R.shape)
    worst = 0.0
    for t in range(R.shape[0]):
        m = ~np.isnan(R[t])
        if not m.any():
            continue
        rms = float(np.sqrt(np.mean(R[t][m] ** 2)))
        e = np.maximum(np.abs(G[t][m] - R[t][m]) - 0.5 * bf16_ulp(R[t][m]), 0.0)
        worst = max(worst, float(e.max()) / max(rms, 1e-300))
    assert worst <= TOL_BF16_MAX_OVER_RMS, (
        f"{what}: max|err| / rms(token) {worst:.3e} > {TOL_BF16_MAX_OVER_RMS} (rel L2 {rel_l2:.2e})")
    return rel_l2, worst

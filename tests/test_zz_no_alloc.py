"""The no-allocation decode entry point (mla_decode_no_alloc).

Some callers cannot hand the library a workspace: their device memory is
owned by another allocator, or they must not allocate after start-up because
allocation can synchronise the device.  This entry point takes its scratch
from a fixed array inside the library instead.  The test calls it through the
C ABI twice in a row, on different problems.  Both entry points run the same
deterministic kernels, so each result must equal the ordinary
workspace-taking entry point's bit for bit; each is also checked against the
CPU fp64 oracle within the numerics tolerance of the other GPU tests.  The
file is named so that pytest collects it last.
"""
import pytest
import torch

from latent_compressed_attention_absorbed_b200 import binding
from latent_compressed_attention_absorbed_b200 import workload as wl
from mla_testutil import Problem, as_f64, check_close

pytestmark = pytest.mark.gpu


def test_no_alloc_decode_matches_workspace_decode_twice(lib):
    cases = [((700, 65, 4096), 1, 31), ((1000, 333, 17), 2, 32)]
    for seqlens, q_len, seed in cases:
        cfg = wl.CONFIGS["v3_b1"].with_(name="no_alloc", B=len(seqlens), seqlens=seqlens, q_len=q_len, seed=seed)
        P = Problem(lib, cfg)
        ref = P.decode()
        got = lib.decode_no_alloc(P.dims, P.qn, P.qr, P.W_UK, P.W_UV, P.cache, P.seqlens)
        torch.cuda.synchronize()
        assert lib.last_path() == "sm100"
        assert lib.device_status() == 0
        assert torch.equal(got, ref), f"no-alloc decode differs from the workspace decode {seqlens}"
        check_close(as_f64(got), P.oracle_expanded(range(cfg.B)), "bf16", f"no-alloc vs fp64 oracle {seqlens}")


def test_no_alloc_decode_rejects_batches_beyond_its_scratch(lib):
    cfg = wl.CONFIGS["v3_b1"]
    dims = lib.dims(cfg.H, cfg.d_c, cfg.d_r, cfg.d_n, cfg.d_v, torch.bfloat16)
    B = 256
    assert lib.workspace_bytes(dims, B, 1) > (64 << 20)
    t = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    cache = torch.zeros((B, 1, cfg.row), dtype=torch.bfloat16, device="cuda")
    seq = torch.ones(B, dtype=torch.int32, device="cuda")
    qn = torch.zeros((B, 1, cfg.H, cfg.d_n), dtype=torch.bfloat16, device="cuda")
    qr = torch.zeros((B, 1, cfg.H, cfg.d_r), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(binding.MLAError) as e:
        lib.decode_no_alloc(dims, qn, qr, t, t, cache, seq)
    assert e.value.code == -7 and "static scratch" in str(e.value)

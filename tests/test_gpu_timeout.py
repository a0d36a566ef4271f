"""Failure path of the attention kernel's bounded waits, on the GPU.

Every barrier wait of the attention kernel has a time limit.  The test makes
one wait run out without faulting anything: the test hook `withhold_tile`
stops the kernel's loader before one tile, so the score issuer's wait for
that tile expires (after a 50 ms limit).  The kernel must then flag
MLA_STATUS_TIMEOUT, drain what it has in flight and exit; the CUDA context
stays usable, which the test checks with a normal decode against the CPU
fp64 oracle.
"""
import pytest

from latent_compressed_attention_absorbed_b200 import binding
from latent_compressed_attention_absorbed_b200 import workload as wl
from mla_testutil import Problem, as_f64, check_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("seqlens,q_len,pairs", [((700, 333, 64), 1, 2), ((900, 77), 2, 4)])
def test_expired_wait_reports_timeout_and_context_stays_usable(lib, seqlens, q_len, pairs):
    cfg = wl.CONFIGS["v3_b1"].with_(name="timeout", B=len(seqlens), seqlens=seqlens, q_len=q_len, seed=19)
    P = Problem(lib, cfg)
    P.decode(opts=lib.opts(num_pairs=pairs, wait_limit_ns=50_000_000, withhold_tile=3))
    status = lib.device_status()
    assert status & binding.STATUS_TIMEOUT, f"device status {status}"
    out = P.decode(opts=lib.opts(num_pairs=pairs))
    assert lib.device_status() == 0
    check_close(as_f64(out), P.oracle_expanded(range(cfg.B)), "bf16", f"decode after a timeout {seqlens}")

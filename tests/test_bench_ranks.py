"""The bench's multi-rank path on CPU: replicas only, so the one collective
is the timing reduction (maximum over ranks), checked here with two gloo
ranks; and each rank decodes its own seeded sequences."""
import json
import os
import socket
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from latent_compressed_attention_absorbed_b200 import workload as wl  # noqa: E402

_RANK_SCRIPT = """
import json, os, sys
import torch
sys.path.insert(0, {root!r})
import bench
torch.distributed.init_process_group("gloo", init_method="env://")
rank = torch.distributed.get_rank()
world = torch.distributed.get_world_size()
got = bench.max_over_ranks([1.0 + rank, 5.0 - rank, 0.25 * rank], world, torch.device("cpu"))
torch.distributed.barrier()
torch.distributed.destroy_process_group()
print(json.dumps({{"rank": rank, "got": got}}))
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_timings_are_the_maximum_over_two_gloo_ranks():
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE="2")
        procs.append(subprocess.Popen([sys.executable, "-c", _RANK_SCRIPT.format(root=ROOT)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=120)
        assert p.returncode == 0, err[-2000:]
        outs.append(json.loads(out.strip().splitlines()[-1]))
    for o in outs:
        assert o["got"] == [2.0, 5.0, 0.25], o


def test_single_rank_reduction_is_the_identity():
    assert bench.max_over_ranks([3.5, 1.0], 1, None) == [3.5, 1.0]


def test_replicas_decode_distinct_sequences_of_the_same_shape():
    base = wl.CONFIGS["v3_b64"]
    cfgs = [bench.replica_config(base, r) for r in range(3)]
    assert len({c.seed for c in cfgs}) == 3
    assert all(c.seqlens == base.seqlens and c.B == base.B and c.q_len == base.q_len for c in cfgs)
    small = [c.with_(B=1, seqlens=(16,)) for c in cfgs]
    hist = [wl.sequence_history(c, 0)[0].values for c in small]
    assert not np.array_equal(hist[0], hist[1]) and not np.array_equal(hist[1], hist[2])

"""The bench's reference arm (the fp64 oracle timed on host cores) runs
without a GPU: its JSON line keeps the contract the driver reads, and under
torchrun only rank 0 prints it."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(extra_env=None, *args):
    env = dict(os.environ)
    env.update(extra_env or {})
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--ref-budget", "0.1", *args],
                       capture_output=True, text=True, env=env, cwd=ROOT, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    return [l for l in r.stdout.splitlines() if l.strip()]


def test_reference_arm_prints_one_contract_line():
    lines = _run()
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["unit"] == "us/step" and d["higher_is_better"] is False
    assert d["value"] > 0 and d["steps"] == 1 and d["warmup"] >= 3
    assert d["config"]["workload"].startswith("v3_ragged")
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert cb["absorbed"]["value"] > 0 and cb["absorbed"]["unit"] == "us/step" and cb["absorbed"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "us/step", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_prints_nothing_on_other_ranks():
    assert _run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}) == []


class _FakeNvml:
    """Host GPUs 0..2 (NVML numbering); CUDA sees only the one with bus 0x3B."""

    def __init__(self, fail_uuid=False):
        self.fail_uuid = fail_uuid

    def nvmlDeviceGetHandleByUUID(self, u):
        if self.fail_uuid or u != "GPU-0000-feed":
            raise RuntimeError("not found")
        return "gpu1"

    def nvmlDeviceGetHandleByPciBusId(self, bus):
        if bus != "00000000:3B:00.0":
            raise RuntimeError("not found")
        return "gpu1"

    def nvmlDeviceGetHandleByIndex(self, i):
        return f"gpu{i}"


class _Props:
    uuid = "0000-feed"
    pci_domain_id, pci_bus_id, pci_device_id = 0, 0x3B, 0


def test_clock_sampler_watches_the_gpu_cuda_runs_on():
    sys.path.insert(0, ROOT)
    import bench

    # CUDA device 0 is host GPU 1: matched by UUID, else by PCI address, never by index 0
    assert bench.nvml_handle(_FakeNvml(), _Props(), 0) == ("gpu1", "uuid")
    assert bench.nvml_handle(_FakeNvml(fail_uuid=True), _Props(), 0) == ("gpu1", "pci")
    assert bench.nvml_handle(_FakeNvml(), None, 0) == ("gpu0", "index")

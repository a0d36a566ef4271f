#!/usr/bin/env python
"""Benchmark of one absorbed-MLA decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload v3_b1] [--impl ours|reference]

The timed step is one mla_decode call on one batch: absorb the query through
W_UK, attend over the compressed cache in latent space, merge split
partials, project through W_UV.  The append of the step's q_len new tokens
per sequence (mla_append_cache) is timed on its own and reported beside it.
The cache and the weights are resident in HBM; the timed region covers the
device work of K steps (CUDA-graph replays, CUDA events on the launching
stream), with L2 flushed by a 256 MiB write before every step, untimed; a
second pass without the flush gives the warm-L2 figure.  One JSON line is
printed by rank 0.

Multi-GPU (torchrun): every rank runs an independent replica of the workload
on its own sequences (sequences are independent; nothing is exchanged on the
data path), so scaling is weak; the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from latent_compressed_attention_absorbed_b200 import workload as wl  # noqa: E402

DEFAULT_WORKLOAD = "v3_ragged"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.json")
CSRC = os.path.join(ROOT, "latent_compressed_attention_absorbed_b200", "csrc")
L2_FLUSH_BYTES = 256 << 20


# ------------------------------------------------------------------ work accounting

def work(cfg):
    """Algorithmic bytes / flops of one decode step, per kernel (absorbed MLA does this much, no more)."""
    U = cfg.B * cfg.q_len
    H, dc, dr, dn, dv = cfg.H, cfg.d_c, cfg.d_r, cfg.d_n, cfg.d_v
    es = 2 if cfg.dtype == "bf16" else 4
    keys = sum(T - cfg.q_len + 1 + i for T in cfg.seqlens for i in range(cfg.q_len))
    cache = sum(cfg.seqlens) * (dc + dr) * es
    qhat = U * H * (dc + dr) * es
    olat = U * H * dc * es
    k = {
        "absorb": {"bytes": H * dn * dc * es + U * H * (dn + dr) * es + qhat, "flops": 2 * U * H * dn * dc},
        "attend": {"bytes": cache + qhat + olat, "flops": 2 * H * keys * (dc + dr + dc)},
        "project": {"bytes": H * dv * dc * es + olat + U * H * dv * es, "flops": 2 * U * H * dc * dv},
        "append": {"bytes": 2 * U * (dc + dr) * es, "flops": 0},
    }
    step = {  # one mla_decode call (the append is timed on its own)
        "bytes": cache + 2 * H * dn * dc * es + U * H * (dn + dr) * es + U * H * dv * es,
        "flops": k["absorb"]["flops"] + k["attend"]["flops"] + k["project"]["flops"],
        "cache_bytes": cache,
    }
    return k, step


def peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# The sources that define the attention kernel and its launch (grid, plan,
# workspace): a DRAM capture stays valid while none of them changes.
ATTEND_SOURCES = ("mla_api.cu", "mla_internal.h", "mla_rope.cuh", "mla_sm100.cu", "sm100_attend.cuh", "sm100_host.h",
                  "sm100_ptx.cuh")


def replica_config(base, rank):
    """The workload one rank decodes: same shape, its own seeded sequences."""
    return base.with_(seed=base.seed + 1000 * rank)


def max_over_ranks(values, world, device):
    """Element-wise maximum of per-rank timings over all ranks (unchanged for one rank)."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t]


def csrc_hash():
    h = hashlib.sha256()
    for f in ATTEND_SOURCES:
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def traffic_for(workload, kernel):
    """DRAM bytes per launch from a committed ncu capture, if it was taken on the current sources."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
        e = t[workload][kernel]
        return float(e["dram_bytes_per_launch"]) if e.get("csrc_sha") == csrc_hash() else None
    except Exception:
        return None


# ------------------------------------------------------------------ clocks

def nvml_handle(nv, props, index):
    """NVML handle of the CUDA device `index` described by `props`, and how it
    was matched.  NVML numbers the GPUs of the host, ignoring
    CUDA_VISIBLE_DEVICES, so the device is matched by UUID, then by PCI
    address, and by index only as a last resort."""
    uuid = str(getattr(props, "uuid", "") or "") if props is not None else ""
    if uuid:
        try:
            return nv.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid), "uuid"
        except Exception:
            pass
    if props is not None and hasattr(props, "pci_bus_id"):
        bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
        try:
            return nv.nvmlDeviceGetHandleByPciBusId(bus), "pci"
        except Exception:
            pass
    return nv.nvmlDeviceGetHandleByIndex(index), "index"


class ClockSampler:
    """Samples SM clock and throttle reasons with NVML during the timed region."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index, props=None, period=0.01):
        self.samples, self.reasons, self.period = [], set(), period
        self._stop = threading.Event()
        self.match = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h, self.match = nvml_handle(pynvml, props, index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None
            self.max_mhz = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.nv:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples),
                "nvml_match": self.match}


# ------------------------------------------------------------------ our arm

def upload(torch, st, device):
    if st.dtype == "bf16":
        return torch.from_numpy(st.raw.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(st.raw).to(device)


def run_ours(args, rank, world, local_rank):
    import torch
    from latent_compressed_attention_absorbed_b200 import binding

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    lib = binding.load()
    base = wl.CONFIGS[args.workload]
    cfg = replica_config(base, rank)  # each replica decodes its own sequences
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    dims = lib.dims(cfg.H, cfg.d_c, cfg.d_r, cfg.d_n, cfg.d_v, dt, cfg.rope_base)

    # ---- resident state: weights and the cache of every sequence (filled through the library)
    w_uk, w_uv = wl.weights(cfg)
    W_UK, W_UV = upload(torch, w_uk, device), upload(torch, w_uv, device)
    del w_uk, w_uv
    cache = torch.zeros((cfg.B, cfg.T_max, cfg.row), dtype=dt, device=device)
    zero = torch.zeros(1, dtype=torch.int32, device=device)
    for b in range(cfg.B):
        c, k = wl.sequence_history(cfg, b)
        lib.append_cache(dims, cache[b:b + 1], upload(torch, c, device)[None], upload(torch, k, device)[None], zero)
        del c, k
    seqlens = torch.tensor(cfg.seqlens, dtype=torch.int32, device=device)
    pos = seqlens - cfg.q_len  # the step re-appends the q_len newest tokens at their own positions
    qn_h, qr_h = wl.queries(cfg)
    c_new_h, k_new_h = wl.new_tokens(cfg, cfg.q_len)
    q_nope, q_rope = upload(torch, qn_h, device), upload(torch, qr_h, device)
    c_new, k_new = upload(torch, c_new_h, device), upload(torch, k_new_h, device)
    out = torch.empty((cfg.B, cfg.q_len, cfg.H, cfg.d_v), dtype=dt, device=device)
    ws = torch.empty(lib.workspace_bytes(dims, cfg.B, cfg.q_len), dtype=torch.uint8, device=device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    torch.cuda.synchronize()
    assert lib.device_status() == 0

    def append(stream=None):
        lib.append_cache(dims, cache, c_new, k_new, pos, stream=stream)

    def step(stream=None, opts=None):
        lib.decode(dims, q_nope, q_rope, W_UK, W_UV, cache, seqlens, out=out, workspace=ws, opts=opts, stream=stream)

    # ---- capture the decode step, and the append on its own, in CUDA graphs
    s = torch.cuda.Stream(device)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        append(stream=s)
        step(stream=s)
    torch.cuda.current_stream().wait_stream(s)
    status = lib.device_status()
    if status:
        raise RuntimeError(f"the first decode step reported device status {status}; not timing it")
    with torch.cuda.stream(s):
        step(stream=s)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    path = lib.last_path()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step(stream=s)
    g_app = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_app, stream=s):
        append(stream=s)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    def busy(cycles=200000):
        # keep the GPU busy while the host enqueues, so no host gap lands inside a timed step
        torch.cuda._sleep(cycles)
        flush.zero_()

    # ---- warm-up
    for _ in range(args.warmup):
        busy()
        g.replay()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()

    # ---- timed: K graph replays, each bracketed by events, L2 flushed before each
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    with ClockSampler(local_rank, torch.cuda.get_device_properties(device)) as clk:
        torch.cuda.synchronize()
        for i in range(args.steps):
            busy()
            starts[i].record(stream)
            g.replay()
            ends[i].record(stream)
        torch.cuda.synchronize()
    times_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]

    def timed_loop(graph, flush_between):
        st = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        en = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        torch.cuda.synchronize()
        for i in range(args.steps):
            if flush_between:
                busy()
            st[i].record(stream)
            graph.replay()
            en[i].record(stream)
        torch.cuda.synchronize()
        return float(np.mean([a.elapsed_time(b) for a, b in zip(st, en)]))

    # ---- the same decode with L2 warm (no flush between replays), and the append alone (flushed)
    for _ in range(3):
        g.replay()
    ms_warm = timed_loop(g, flush_between=False)
    for _ in range(3):
        g_app.replay()
    ms_append = timed_loop(g_app, flush_between=True)
    if world > 1:
        torch.distributed.barrier()
    ms_step = float(np.mean(times_ms))
    ms_med = float(np.median(times_ms))
    ms_step, ms_med, ms_warm, ms_append = max_over_ranks([ms_step, ms_med, ms_warm, ms_append], world, device)

    # ---- per-kernel stage times (same kernels, launched directly with stage events)
    n_ev = binding.NUM_EVENTS
    kinds = ["absorb", "plan", "attend", "combine", "project"]
    stage = {k: [] for k in kinds}
    prof_steps = max(3, min(args.steps, 50))
    for _ in range(prof_steps):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
        for e in evs:
            e.record(stream)  # materialise the handles
        busy(4000000)
        step(opts=lib.opts(events=evs))
        torch.cuda.synchronize()
        for j, k in enumerate(kinds):
            stage[k].append(evs[j].elapsed_time(evs[j + 1]))
    stage_ms = {k: float(np.mean(v)) for k, v in stage.items()}
    assert lib.device_status() == 0

    # ---- end to end through the public API: pinned host inputs in, result out
    e2e = None
    if not args.no_e2e:
        pin = lambda st: torch.from_numpy(st.raw.view(np.int16) if st.dtype == "bf16" else st.raw).pin_memory()
        h_qn, h_qr = pin(qn_h), pin(qr_h)
        h_out = torch.empty(out.shape, dtype=torch.int16 if cfg.dtype == "bf16" else torch.float32).pin_memory()
        d_qn, d_qr = torch.empty_like(h_qn, device=device), torch.empty_like(h_qr, device=device)
        view = (lambda t: t.view(torch.bfloat16)) if cfg.dtype == "bf16" else (lambda t: t)

        def e2e_step():
            d_qn.copy_(h_qn, non_blocking=True)
            d_qr.copy_(h_qr, non_blocking=True)
            o = lib.decode(dims, view(d_qn), view(d_qr), W_UK, W_UV, cache, seqlens, out=out, workspace=ws)
            h_out.copy_(o.view(torch.int16) if cfg.dtype == "bf16" else o, non_blocking=True)
            torch.cuda.current_stream().synchronize()

        for _ in range(max(3, args.warmup)):
            e2e_step()
        wall = []
        for _ in range(args.steps):
            flush.zero_()
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            e2e_step()
            wall.append((time.perf_counter() - t0) * 1e3)
        e2e_ms = float(np.mean(wall))
        e2e_ms = max_over_ranks([e2e_ms], world, device)[0]
        h2d = sum(x.numel() * x.element_size() for x in (h_qn, h_qr))
        d2h = h_out.numel() * h_out.element_size()
        e2e = {"value": round(e2e_ms * 1e3, 3), "unit": "us/step", "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "timing": "host wall clock per step incl. synchronize"}
    times = {"ms_step": ms_step, "ms_med": ms_med, "ms_warm": ms_warm, "ms_append": ms_append}
    proj = None if args.no_projections or path != "sm100" else time_projections(
        torch, lib, dims, cfg, device, out, flush, args.steps)
    return cfg, path, times, stage_ms, clk.summary(), e2e, proj


def time_projections(torch, lib, dims, cfg, device, attn_out, flush, steps):
    """The projections around the decode at this step's rows (B * q_len tokens):
    the cache append from the block input x and the output projection W_O,
    each a CUDA graph replayed with L2 flushed between replays."""
    rows = cfg.B * cfg.q_len
    x = upload(torch, wl.block_input(cfg, cfg.q_len), device)
    w_a, gamma = wl.append_weights(cfg)
    W_A, g = upload(torch, w_a, device), upload(torch, gamma, device)
    W_O = upload(torch, wl.output_weights(cfg), device)
    del w_a, gamma
    scratch = torch.zeros((cfg.B, cfg.q_len, cfg.row), dtype=W_A.dtype, device=device)
    pos0 = torch.zeros(cfg.B, dtype=torch.int32, device=device)
    y = torch.empty((rows, cfg.d_model), dtype=W_O.dtype, device=device)
    ws_a = torch.empty(lib.lib.mla_append_from_hidden_workspace_bytes(dims, cfg.B, cfg.q_len, cfg.d_model),
                       dtype=torch.uint8, device=device)
    ws_o = torch.empty(lib.lib.mla_output_projection_workspace_bytes(dims, rows, cfg.d_model), dtype=torch.uint8,
                       device=device)
    calls = {
        "append_from_hidden": lambda st: lib.append_from_hidden(dims, scratch, x, W_A, g, pos0, workspace=ws_a,
                                                                stream=st),
        "output_projection": lambda st: lib.output_projection(dims, attn_out, W_O, y=y, workspace=ws_o, stream=st),
    }
    es = 2
    nbytes = {
        "append_from_hidden": (cfg.row * cfg.d_model + rows * cfg.d_model + rows * cfg.row + cfg.d_c) * es,
        "output_projection": (cfg.d_model * cfg.H * cfg.d_v + rows * cfg.H * cfg.d_v + rows * cfg.d_model) * es,
    }
    pk, _ = peaks()
    res = {}
    stream = torch.cuda.current_stream()
    for name, call in calls.items():
        s = torch.cuda.Stream(device)
        s.wait_stream(stream)
        with torch.cuda.stream(s):
            call(s)
        stream.wait_stream(s)
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=s):
            call(s)
        torch.cuda.synchronize()
        ev = []
        for _ in range(max(20, min(steps, 200))):
            torch.cuda._sleep(100000)
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            gr.replay()
            b.record(stream)
            ev.append((a, b))
        torch.cuda.synchronize()
        us = float(np.mean([a.elapsed_time(b) for a, b in ev])) * 1e3
        gbps = nbytes[name] / (us * 1e-6) / 1e9
        res[name] = {"us": round(us, 3), "algorithmic_bytes": int(nbytes[name]), "gbps": round(gbps, 1),
                     "frac_of_hbm": round(gbps / pk["hbm_gbs"], 4), "rows": rows, "d_model": cfg.d_model}
        del gr
    assert lib.device_status() == 0
    return res


class OracleSample:
    """The fp64 expanded oracle on this host, on a bounded sample of (sequence 0, heads),
    and beside it the fp64 absorbed CPU form (all heads of sequence 0)."""

    def __init__(self, cfg):
        self.cfg = cfg
        w_uk, w_uv = wl.weights(cfg)
        qn, qr = wl.queries(cfg)
        c, k = wl.sequence_history(cfg, 0)
        self.args = (qn.values, qr.values, w_uk.values, w_uv.values,
                     [(c.values, k.values)] + [(None, None)] * (cfg.B - 1), cfg.q_len, cfg.rope_base)
        try:
            from threadpoolctl import threadpool_info
            self.cores = max([p.get("num_threads", 1) for p in threadpool_info()] or [1])
        except Exception:
            self.cores = len(os.sched_getaffinity(0))
        t0 = time.perf_counter()
        self._run(1)
        self.one_head_s = max(time.perf_counter() - t0, 1e-6)

    def _run(self, n_heads):
        from oracle import decode_expanded
        decode_expanded(*self.args, seqs=[0], heads=range(n_heads))

    def measure(self, budget_s):
        cfg = self.cfg
        n_heads = int(max(1, min(cfg.H, budget_s / self.one_head_s)))
        t0 = time.perf_counter()
        self._run(n_heads)
        dt = time.perf_counter() - t0
        # the cost of one (sequence, head) unit is linear in that sequence's history length
        full_s = dt / (n_heads * cfg.seqlens[0]) * cfg.H * sum(cfg.seqlens)
        sample = (f"sequence 0 (T={cfg.seqlens[0]}) x {n_heads} of {cfg.H} heads x {cfg.q_len} query token(s), "
                  f"fp64 expanded K/V; per-step time extrapolated linearly in heads x history length")
        return {"value": round(full_s * 1e6, 1), "unit": "us/step", "cores": int(self.cores), "kind": "oracle",
                "sample": sample, "sample_seconds": round(dt, 3), "absorbed": self.measure_absorbed()}

    def measure_absorbed(self):
        from oracle import decode_absorbed
        cfg = self.cfg
        t0 = time.perf_counter()
        decode_absorbed(*self.args, seqs=[0])
        dt = time.perf_counter() - t0
        return {"value": round(dt / cfg.seqlens[0] * sum(cfg.seqlens) * 1e6, 1), "unit": "us/step",
                "sample": f"sequence 0 (T={cfg.seqlens[0]}) x all {cfg.H} heads x {cfg.q_len} query token(s), fp64 "
                          f"absorbed CPU form; per-step time extrapolated linearly in history length",
                "sample_seconds": round(dt, 3)}


def cpu_baseline(cfg, budget_s):
    return OracleSample(cfg).measure(budget_s)


def run_reference(args):
    cfg = wl.CONFIGS[args.workload]
    sampler = OracleSample(cfg)
    budget = min(args.ref_budget, max(0.05, 150.0 / (args.steps + args.warmup)))
    per, last = [], None
    for i in range(args.warmup + args.steps):
        last = sampler.measure(budget)
        if i >= args.warmup:
            per.append(last["value"])
    v = float(np.mean(per))
    cb = dict(last)
    cb["value"] = round(v, 1)
    line = {"impl": "reference", "metric": metric_name(), "value": round(v, 1), "unit": "us/step", "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(v / 1e3, 3), "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded; c_KV, k_R, q ~ N(0,1), "
            "W ~ N(0,0.02))", "config": config_of(cfg, args), "cpu_baseline": cb,
            "e2e": {"value": round(v, 1), "unit": "us/step", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def metric_name():
    return "MLA decode us/step, cache GB/s & TFLOP/s as % of B200 roofline (1 GPU)"


def config_of(cfg, args):
    return {"workload": f"{cfg.name}: B={cfg.B}, T={'ragged' if len(set(cfg.seqlens)) > 1 else cfg.seqlens[0]}, "
                        f"q_len={cfg.q_len}, H={cfg.H}, d_c={cfg.d_c}, d_r={cfg.d_r}, d_n={cfg.d_n}, d_v={cfg.d_v}, "
                        f"{cfg.dtype}",
            "B": cfg.B, "seq_len": int(max(cfg.seqlens)), "sum_seqlens": int(sum(cfg.seqlens)), "q_len": cfg.q_len,
            "step": "one mla_decode call (absorb, attend, combine, W_UV); the q_len-token append is timed apart",
            "l2": "flushed before every step (256 MiB write, untimed); warm_l2_us_per_step without the flush",
            "parallelism": f"replicas x{args.gpus} (sequences are independent; no collective on the data path)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(wl.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-projections", action="store_true", help="skip timing the projections around the decode")
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--ref-budget", type=float, default=5.0, help="seconds of oracle work per reference step")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            run_reference(args)
        return

    if world > 1:
        import datetime
        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    cfg, path, times, stage_ms, clocks, e2e, proj = run_ours(args, rank, world, local_rank)
    ms_step, ms_med = times["ms_step"], times["ms_med"]
    if world > 1:
        import torch
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return

    pk, pk_kind = peaks()
    kern, step_work = work(cfg)
    bw = pk["hbm_gbs"] * 1e9
    fl = pk["bf16_tflops"] * 1e12
    # dominant kernel: largest share of the step.  Kernel names follow the
    # library's dispatch: matrix-vector absorb up to 2 query rows and
    # matrix-vector project (with the split merge) up to 8 rows, tensor-core
    # GEMMs (and a separate combine kernel) above.
    rows = cfg.B * cfg.q_len
    dom = max(("absorb", "attend", "project"), key=lambda k: stage_ms[k])
    kt = stage_ms[dom] * 1e-3
    kb, kf = kern[dom]["bytes"], kern[dom]["flops"]
    hbm_bound = kb / bw >= kf / fl
    kname = {"absorb": "absorb_gemv_kernel" if rows <= 2 else "head_gemm_kernel (W_UK absorb)",
             "attend": "mla_attend_kernel",
             "project": "project_gemv_kernel" if rows <= 8 else "head_gemm_kernel (W_UV project)"}[dom]
    traffic = traffic_for(cfg.name, kname)
    # The library prefetches W_UV into L2 from inside the attention kernel when
    # the cache read is small (at most 64 MiB over B x T_max rows), for the
    # projection that follows; those bytes are the projection's, not attention's.
    prefetch = (cfg.H * cfg.d_v * cfg.d_c * 2 if dom == "attend" and
                cfg.B * cfg.T_max * cfg.row * 2 <= (64 << 20) else 0)
    roof = {"kernel": kname, "bound": "hbm" if hbm_bound else "tensor",
            "achieved": round((kb / kt / 1e9) if hbm_bound else (kf / kt / 1e12), 2),
            "peak": pk["hbm_gbs"] if hbm_bound else pk["bf16_tflops"],
            "unit": "GB/s" if hbm_bound else "TFLOP/s",
            "traffic": traffic,
            "algorithmic_bytes": int(kb), "algorithmic_flops": int(kf),
            "kernel_us": round(kt * 1e6, 3),
            "l2_prefetch_bytes_in_traffic": int(prefetch),
            "peak_source": f"{pk_kind} (MEASURED_PEAKS.json burst figure)" if pk_kind == "measured" else "fallback"}
    roof["frac"] = round(roof["achieved"] / roof["peak"], 4)
    t_step = ms_step * 1e-3
    step_roof_s = max(step_work["bytes"] / bw, step_work["flops"] / fl)
    line = {
        "metric": metric_name(),
        "value": round(ms_step * 1e3, 3),
        "unit": "us/step",
        "n_gpus": args.gpus,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 6),
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": cfg.dtype,
        "data": "synthetic (seeded; c_KV, k_R, q ~ N(0,1), W ~ N(0,0.02)); cache and weights resident in HBM",
        "config": config_of(cfg, args),
        "path": path,
        "median_us_per_step": round(ms_med * 1e3, 3),
        "cache_gbps": round(step_work["cache_bytes"] / t_step / 1e9, 1),
        "step_gbps": round(step_work["bytes"] / t_step / 1e9, 1),
        "tflops": round(step_work["flops"] / t_step / 1e12, 2),
        "step_roofline_us": round(step_roof_s * 1e6, 3),
        "step_roofline_frac": round(step_roof_s / t_step, 4),
        "warm_l2_us_per_step": round(times["ms_warm"] * 1e3, 3),
        "append_us": round(times["ms_append"] * 1e3, 3),
        "step_with_append_us": round((ms_step + times["ms_append"]) * 1e3, 3),
        "stage_us": {k: round(v * 1e3, 3) for k, v in stage_ms.items()},
        "roofline": roof,
        # absorb + attend (+ combine above 8 query rows) + project per timed step
        "gpu_launches": ((3 if rows <= 8 else 4) if path == "sm100" else 3) * args.steps * args.gpus,
        "clocks": clocks,
        "e2e": e2e,
    }
    if proj:
        line["projections"] = proj
    if args.gpus == 1 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, args.cpu_budget)
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Benchmark of the GDN hot path on B200: prefill tokens/s and % of roofline.

One step = one pass of every hot-path call:
  gdn_ba_gates + gdn_chunk_prefill on the 48-head, 4576-token workload
  (x [4576, 5120] -> gates -> prefill, d = 128, H_k = 16, H_v = 48, h0 = 0), then
  gdn_flag_clear + gdn_verify_woa + gdn_fold on the speculative-verify batch
  (64 sequences x 4 rows, states reached through a pointer table).
value = prefill tokens per second of device time (4576 tokens per step, all
ranks summed; inputs resident in HBM; the per-step working set, ~560 MB, is
larger than L2, so no flush is needed between steps).

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]

Prints one JSON line on rank 0.  Under torchrun every rank runs an independent
replica of the step (the method has no cross-rank exchange: weak scaling).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "GDN prefill tokens/s (1xB200) and % of roofline (bf16 TC peak vs HBM)"
UNIT = "tokens/s"
WORKLOAD = "gdn-prefill-ba: M=4576 K=5120 H_k=16 H_v=48 d=128 C=64, h0=0; " \
           "+ verify/fold batch=64 K=4 H_k=16 H_v=48 d=128"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# --------------------------------------------------------------------------
# Algorithmic work of one prefill launch (bytes that must move; flops that must
# be done), chunk C = 64:
#   bytes/token = 2 H_k d_k 2 (q, k bf16) + 2 H_v d_v 2 (v in, o out) + 2 H_v 4 (g, beta)
#   bytes/seq   = 2 H_v d_k d_v 4 (h0 read, hT write)
#   flops/(token, v-head) = (C-1) d_k + 2 C (d_k + d_v) + 6 d_k d_v
# --------------------------------------------------------------------------

def prefill_alg_bytes(T, N, H_k, H_v, d_k, d_v):
    return T * (4 * H_k * d_k + 4 * H_v * d_v + 8 * H_v) + N * 8 * H_v * d_k * d_v


def prefill_alg_flops(T, H_v, d_k, d_v, C=64):
    return T * H_v * ((C - 1) * d_k + 2 * C * (d_k + d_v) + 6 * d_k * d_v)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            m = json.load(f)
        return float(m["hbm_gbs"]), float(m["bf16_tflops"]), float(m.get(
            "bf16_tflops_sustained", m["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS, "fallback"


def profiled_traffic():
    """dram read+write bytes per prefill launch from the committed ncu summary,
    or None once gdn_prefill.cu no longer matches the source that was profiled."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "prefill_dram_traffic.txt")
    src = os.path.join(ROOT, "linear_attention_ssm_gdn_b200", "csrc", "gdn_prefill.cu")
    try:
        vals = {}
        with open(path) as f:
            for line in f:
                if "=" in line and not line.startswith("#"):
                    k, v = line.split("=", 1)
                    vals[k.strip()] = v.split()[0]
        with open(src, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
        if vals.get("source_sha256") != sha:
            return None
        return float(vals["bytes_per_launch_full_workload"])
    except Exception:
        return None


# --------------------------------------------------------------------------
# Clock sampling during the timed region (NVML, a few ms period)
# --------------------------------------------------------------------------

class ClockSampler:
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.002):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            return self
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self._h))
            except Exception:
                pass
            time.sleep(self.period)

    def stop(self):
        self._stop.set()
        if self._t is not None:
            self._t.join()
        if not self.ok:
            return None
        names = [n for b, n in self.REASONS.items() if self.reasons & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# --------------------------------------------------------------------------
# Our arm
# --------------------------------------------------------------------------

def max_over_ranks(ms: float, dist, device) -> float:
    """The slowest rank's time (every rank calls this; identity for one rank)."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, steps: int, tokens_per_step: int, max_ms: float) -> float:
    """Whole-job tokens/s: every rank runs `steps` steps of `tokens_per_step`."""
    return world * steps * tokens_per_step / (max_ms / 1e3)


def make_inputs(dev):
    import torch

    from linear_attention_ssm_gdn_b200 import (gdn_chunk_prefill_workspace_bytes,
                                               gdn_stash_seq_floats)
    from linear_attention_ssm_gdn_b200 import inputs as I

    w2 = I.workload(2)
    w4 = I.workload(4)
    p, ba, vi = w2.prefill, w2.ba, w4.verify
    host = {"x": ba.x, "q": p.q, "k": p.k, "v": p.v, "vq": vi.q, "vk": vi.k, "vv": vi.v,
            "vg": vi.g, "vb": vi.beta, "na": vi.na}
    d = {k: t.to(dev) for k, t in host.items()}
    d.update(w=ba.w.to(dev), a_log=ba.a_log.to(dev), dt_bias=ba.dt_bias.to(dev),
             cu=p.cu_seqlens.to(dev), h0=p.h0.to(dev), pool=vi.pool.to(dev))
    T, H_v, dv = p.total_tokens, p.H_v, p.d_v
    d["gates"] = torch.empty(T, 2 * ba.nv, device=dev)
    d["o"] = torch.empty(T, H_v, dv, dtype=torch.bfloat16, device=dev)
    d["hT"] = torch.empty_like(d["h0"])
    per = d["pool"][0].numel() * 4
    d["table"] = torch.tensor([d["pool"].data_ptr() + int(s) * per for s in vi.slots],
                              dtype=torch.int64, device=dev)
    d["flag"] = torch.zeros(1, dtype=torch.int32, device=dev)
    d["vo"] = torch.empty(vi.batch * 4, vi.H_v, vi.d_v, dtype=torch.bfloat16, device=dev)
    d["stash"] = torch.empty(vi.batch, gdn_stash_seq_floats(vi.H_v, vi.d_k, vi.d_v), device=dev)
    ws = gdn_chunk_prefill_workspace_bytes(T, p.num_seqs, p.H_k, H_v, p.d_k, dv)
    d["ws"] = torch.empty(max(ws, 1), dtype=torch.uint8, device=dev)
    meta = dict(T=T, N=p.num_seqs, H_k=p.H_k, H_v=H_v, d_k=p.d_k, d_v=dv, nv=ba.nv,
                vpg=ba.vheads_per_group, vbatch=vi.batch)
    return host, d, meta


def step_calls(d, meta, ev=None):
    """Queue one step on the current stream.  ev: optional list of 6 events
    (None entries are skipped) recorded before BA, prefill, flag clear,
    verify, fold and after fold."""
    from linear_attention_ssm_gdn_b200 import (gdn_ba_gates, gdn_chunk_prefill, gdn_flag_clear,
                                               gdn_fold, gdn_verify_woa)
    nv = meta["nv"]
    if ev and ev[0] is not None:
        ev[0].record()
    gdn_ba_gates(d["x"], d["w"], d["a_log"], d["dt_bias"], meta["vpg"], gate_out=d["gates"])
    if ev and ev[1] is not None:
        ev[1].record()
    gdn_chunk_prefill(d["q"], d["k"], d["v"], d["gates"][:, :nv], d["gates"][:, nv:], d["cu"],
                      h0=d["h0"], hT=d["hT"], o=d["o"], workspace=d["ws"])
    if ev and ev[2] is not None:
        ev[2].record()
    gdn_flag_clear(d["flag"])
    if ev and ev[3] is not None:
        ev[3].record()
    gdn_verify_woa(d["table"], d["vq"], d["vk"], d["vv"], d["vg"], d["vb"], d["flag"], o=d["vo"],
                   stash=d["stash"])
    if ev and ev[4] is not None:
        ev[4].record()
    gdn_fold(d["table"], d["stash"], d["na"], d["vk"], d["flag"], meta["H_v"])
    if ev and ev[5] is not None:
        ev[5].record()


LAUNCHES_PER_STEP = 5  # ba_gates, prefill, flag_clear, verify, fold


def run_ours(args, rank, world, dist):
    import torch

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    host, d, meta = make_inputs(dev)
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        step_calls(d, meta)
    torch.cuda.synchronize()

    # ---- timed region: exactly K steps.  Only the prefill kernel (the
    # roofline kernel) is bracketed by events here: every event record costs
    # the stream about 2.7 us, so the split of the other kernels comes from a
    # separate, untimed pass below.
    K = args.steps
    evs = [[None, torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
            None, None, None] for _ in range(K)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev.index).start()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t_start.record(stream)
    for i in range(K):
        step_calls(d, meta, evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clk = clocks.stop()
    total_ms = t_start.elapsed_time(t_end)
    t_prefill_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    total_ms = max_over_ranks(total_ms, dist, dev)

    # ---- untimed split: per-kernel events on every kernel of a few steps
    ks = max(1, min(K, 50))
    evs2 = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(ks)]
    for i in range(ks):
        step_calls(d, meta, evs2[i])
    torch.cuda.synchronize()
    per = {name: statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs2)
           for j, name in enumerate(["ba_gates", "prefill", "flag_clear", "verify", "fold"])}

    # ---- end to end through the public API: H2D inputs, the calls, D2H results
    pinned = {k: v.pin_memory() for k, v in host.items()}
    outs = {k: torch.empty(d[k].shape, dtype=d[k].dtype, pin_memory=True)
            for k in ("o", "hT", "vo")}
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = sum(v.numel() * v.element_size() for v in outs.values())
    e_s = torch.cuda.Event(enable_timing=True)
    e_e = torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e_s.record(stream)
    for _ in range(K):
        for k_, v_ in pinned.items():
            d[k_].copy_(v_, non_blocking=True)
        step_calls(d, meta)
        for k_, v_ in outs.items():
            v_.copy_(d[k_], non_blocking=True)
    e_e.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e_s.elapsed_time(e_e)
    e2e_ms = max_over_ranks(e2e_ms, dist, dev)
    if dist:
        dist.barrier()

    if rank != 0:
        return None
    T = meta["T"]
    value = job_value(world, K, T, total_ms)
    e2e_value = job_value(world, K, T, e2e_ms)
    hbm, tf_burst, tf_sust, src = peaks()
    B = prefill_alg_bytes(T, meta["N"], meta["H_k"], meta["H_v"], meta["d_k"], meta["d_v"])
    F = prefill_alg_flops(T, meta["H_v"], meta["d_k"], meta["d_v"])
    t_pf = t_prefill_ms / 1e3
    achieved = B / t_pf / 1e9
    t_roof = max(B / (hbm * 1e9), F / (tf_burst * 1e12))
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "tokens_per_step": T, "l2": "inputs larger than L2 "
                   "(~560 MB per step), no flush", "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": profiled_traffic(),
                     "peak_source": src, "kernel": "prefill_kernel",
                     "alg_bytes_per_launch": B, "alg_flops_per_launch": F,
                     "tflops_achieved": F / t_pf / 1e12,
                     "roofline_time_us": t_roof * 1e6,
                     "frac_of_roofline_time": t_roof / t_pf},
        "kernels_us": {k: v * 1e3 for k, v in per.items()},
        "kernels_us_note": "separate untimed pass with events around every kernel "
                           "(each event record adds about 2.7 us to its interval)",
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": LAUNCHES_PER_STEP * K,
        "clocks": clk,
    }
    return line


# --------------------------------------------------------------------------
# The oracle on the host cores (cpu_baseline leg and the reference arm)
# --------------------------------------------------------------------------

def oracle_step_seconds(budget_s: float):
    """Time the oracle on a bounded sample of one step and scale it to the full
    step.  Returns (seconds per full step, threads, sample description)."""
    import numpy as np

    import oracle
    from linear_attention_ssm_gdn_b200 import inputs as I

    def f64(t):
        return t.to(dtype=__import__("torch").float64).numpy()

    nt = oracle.default_threads()
    w2 = I.workload(2)
    p, ba = w2.prefill, w2.ba
    vi = I.workload(4).verify
    T, H_v, H_k, nv = p.total_tokens, p.H_v, p.H_k, ba.nv
    vpg = H_v // H_k
    # BA gates on a row sample
    m_s = min(T, max(32, int(64 * nt)))
    x, w = f64(ba.x[:m_s]), f64(ba.w)
    t0 = time.perf_counter()
    g = oracle.ba_gates(x, w, f64(ba.a_log), f64(ba.dt_bias), ba.vheads_per_group, nthreads=nt)
    t_ba = (time.perf_counter() - t0) * T / m_s
    # prefill (token recurrence, the definition) on a head sample, full length
    heads = list(range(min(H_v, max(1, nt))))
    kh = [h // vpg for h in heads]
    # The oracle's cost does not depend on the gate values, so the sampled heads
    # use drawn gates instead of running the BA oracle over all rows first.
    rng = np.random.default_rng(0)
    gs = -np.abs(rng.standard_normal((T, len(heads)))) * 0.1
    bs = rng.uniform(0.1, 0.9, (T, len(heads)))
    args = (f64(p.q)[:, kh], f64(p.k)[:, kh], f64(p.v)[:, heads], gs, bs, [0, T], None)
    t0 = time.perf_counter()
    oracle.gdn_token(*args, nthreads=nt)
    t_pf = (time.perf_counter() - t0) * H_v / len(heads)
    # verify + fold on a batch sample
    b_s = min(vi.batch, max(1, nt))
    sl = slice(0, 4 * b_s)
    t0 = time.perf_counter()
    oracle.gdn_verify_fold(f64(vi.pool[vi.slots[:b_s]]), f64(vi.q[sl]), f64(vi.k[sl]),
                           f64(vi.v[sl]), f64(vi.g[sl]), f64(vi.beta[sl]), vi.na[:b_s].numpy(),
                           nthreads=nt)
    t_vf = (time.perf_counter() - t0) * vi.batch / b_s
    del g
    sample = (f"oracle (f64 C, {nt} threads): BA gates on {m_s}/{T} rows, token recurrence on "
              f"{len(heads)}/{H_v} v-heads x {T} tokens, verify+fold on {b_s}/{vi.batch} "
              f"sequences; each scaled to the full step")
    return t_ba + t_pf + t_vf, nt, sample


def run_reference(args):
    steps = []
    for i in range(args.warmup + args.steps):
        s, nt, sample = oracle_step_seconds(budget_s=5.0)
        if i >= args.warmup:
            steps.append(s)
    T = 4576
    sec = sum(steps)
    value = len(steps) * T / sec
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec / len(steps) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": WORKLOAD, "tokens_per_step": T},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": nt, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0

    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    try:
        line = run_ours(args, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            s, nt, sample = oracle_step_seconds(budget_s=20.0)
            line["cpu_baseline"] = {"value": 4576 / s, "unit": UNIT, "cores": nt,
                                    "kind": "oracle", "sample": sample}
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())

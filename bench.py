#!/usr/bin/env python
"""Benchmark of the GDN hot path on B200: prefill tokens/s and % of roofline.

One step = one pass of every hot-path call:
  gdn_ba_gates + gdn_chunk_prefill on the 48-head, 4576-token workload
  (x [4576, 5120] -> gates -> prefill, d = 128, H_k = 16, H_v = 48, h0 = 0), then
  gdn_flag_clear + gdn_verify_woa + gdn_fold on the speculative-verify batch
  (64 sequences x 4 rows, states reached through a pointer table).
value = prefill tokens per second: 4576 tokens over the prefill launch's own
device time (CUDA events around it inside the timed steps; all ranks summed).
The whole step's rate is reported beside it (step_tokens_per_s).  Inputs are
resident in HBM; the per-step working set (~560 MB) is larger than L2, so no
flush is needed between steps.  The single-sequence (4096 tokens, 32 heads)
and varlen (8 sequences, 24,674 tokens) prefill workloads are timed after the
steps, each launch on its own (an L2 flush between launches of the first,
whose working set fits in L2).

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
    """SM clocks and clock-event reasons of this GPU, sampled by nvidia-smi in
    a child process (read-only queries) while the GPU works; the device is
    named by its UUID, which stays right under CUDA_VISIBLE_DEVICES."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}
    QUERY = "clocks.sm,clocks.max.sm,clocks_event_reasons.active"

    def __init__(self, device, period_ms: int = 50):
        self.device, self.period_ms = device, period_ms
        self._p = None
        self.ok = False

    def start(self):
        import shutil
        import subprocess
        try:
            import torch
            exe = shutil.which("nvidia-smi")
            if exe is None:
                return self
            uuid = "GPU-" + str(torch.cuda.get_device_properties(self.device).uuid)
            self._p = subprocess.Popen(
                [exe, "-i", uuid, f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", str(self.period_ms)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.ok = True
        except Exception:
            self._p = None
        return self

    def stop(self):
        if self._p is None:
            return None
        self._p.terminate()
        try:
            out, _ = self._p.communicate(timeout=10)
        except Exception:
            self._p.kill()
            out, _ = self._p.communicate()
        mhz, mx, reasons = [], None, 0
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 3:
                continue
            try:
                mhz.append(float(f[0]))
                mx = float(f[1])
                reasons |= int(f[2], 16)
            except ValueError:
                continue
        names = [n for b, n in self.REASONS.items() if reasons & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": mx,
                "reasons": names, "samples": len(mhz)}


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


def progress(msg: str) -> None:
    """One line on stderr per bench phase (stdout carries only the JSON line)."""
    print(f"[bench] {time.strftime('%H:%M:%S')} {msg}", file=sys.stderr, flush=True)


def roofline_entry(T, N, H_k, H_v, d, us):
    """Roofline of one prefill launch of T tokens (N sequences) taking `us`."""
    hbm, tf_burst, _, src = peaks()
    B = prefill_alg_bytes(T, N, H_k, H_v, d, d)
    F = prefill_alg_flops(T, H_v, d, d)
    t = us / 1e6
    t_roof = max(B / (hbm * 1e9), F / (tf_burst * 1e12))
    return {"us": us, "tokens_per_s": T / t, "achieved_gbs": B / t / 1e9,
            "frac": B / t / 1e9 / hbm, "roofline_us": t_roof * 1e6,
            "frac_of_roofline_time": t_roof / t, "alg_bytes": B, "alg_flops": F,
            "peak_source": src}


def time_prefill(p, dev, reps, flush=None, **kw):
    """Mean device time (us) of `reps` launches of gdn_chunk_prefill on inputs
    p (resident in HBM), CUDA events around each launch; `flush` (a tensor
    larger than L2) is overwritten between launches when given."""
    import torch

    from linear_attention_ssm_gdn_b200 import gdn_chunk_prefill
    d = {k: getattr(p, k).to(dev) for k in ("q", "k", "v", "g", "beta", "cu_seqlens", "h0")}
    o = torch.empty(p.total_tokens, p.H_v, p.d_v, dtype=torch.bfloat16, device=dev)
    hT = torch.empty_like(d["h0"])

    def call():
        gdn_chunk_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], h0=d["h0"],
                          hT=hT, o=o, **kw)
    for _ in range(3):
        call()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(reps)]
    for e0, e1 in evs:
        if flush is not None:
            flush.zero_()
        e0.record()
        call()
        e1.record()
    torch.cuda.synchronize()
    return statistics.mean(a.elapsed_time(b) for a, b in evs) * 1e3


def run_ours(args, rank, world, dist):
    import torch

    from linear_attention_ssm_gdn_b200 import inputs as I

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    host, d, meta = make_inputs(dev)
    stream = torch.cuda.current_stream()
    progress("inputs ready")

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
    clocks = ClockSampler(dev).start()
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
    total_ms = t_start.elapsed_time(t_end)
    prefill_ms = sum(e[1].elapsed_time(e[2]) for e in evs)  # K prefill launches
    total_ms = max_over_ranks(total_ms, dist, dev)
    prefill_ms = max_over_ranks(prefill_ms, dist, dev)

    progress("timed steps done")
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

    progress("end-to-end steps done")
    # ---- the other prefill workloads, one launch at a time (every rank runs
    # the same calls; rank 0 reports its own device times)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # > L2 (126 MB)
    p1 = I.workload(1).prefill
    p3 = I.workload(3).prefill
    p2 = I.prefill_inputs([4576], 16, 48, 128, 128, seed=2, h0_std=None)  # drawn gates
    tp = I.prefill_inputs([16384], 2, 6, 128, 128, seed=2, h0_std=None)
    others = {
        "single_sequence": (p1, time_prefill(p1, dev, 10, flush=flush),
                            "T=4096 H_k=16 H_v=32 d=128, h0~N(0,0.02); L2 flushed per launch"),
        "varlen": (p3, time_prefill(p3, dev, 5),
                   f"8 seqs {sum(I.varlen_lengths(3))} tokens H_k=16 H_v=48 d=128; "
                   "inputs > L2"),
    }
    variants = {
        "prefill_x2_us": time_prefill(p2, dev, 10, limbs=2),
        "prefill_x1_drawn_gates_us": time_prefill(p2, dev, 10),
        "tp_shard_single_level_us": time_prefill(tp, dev, 10, flush=flush, segments=1),
        "tp_shard_two_level_us": time_prefill(tp, dev, 10, flush=flush),
        "note": "us per launch. x2/x1: the 4576-token 48-head prefill with drawn gates, "
                "two-limb vs one-limb state operand.  tp_shard: 16384 tokens, H_k=2, "
                "H_v=6 (the same geometry over 8 GPUs), single-level scan vs the "
                "library's choice (two-level, segment-parallel)",
    }
    del flush
    clk = clocks.stop()
    if clk is not None:
        clk["window"] = ("sampled every 50 ms from the start of the timed steps to the end of "
                         "the other workloads (the GPU is busy throughout)")
    progress("other workloads done")

    if rank != 0:
        return None
    T = meta["T"]
    value = world * K * T / (prefill_ms / 1e3)
    step_value = job_value(world, K, T, total_ms)
    e2e_value = job_value(world, K, T, e2e_ms)
    hbm, tf_burst, tf_sust, src = peaks()
    t_prefill_us = prefill_ms / K * 1e3
    rf = roofline_entry(T, meta["N"], meta["H_k"], meta["H_v"], meta["d_k"], t_prefill_us)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "tokens_per_step": T, "l2": "inputs larger than L2 "
                   "(~560 MB per step), no flush", "parallelism": f"replicas x{world}"},
        "value_note": "prefill tokens/s: tokens over the prefill launch's device time "
                      "(CUDA events around it in the timed steps)",
        "step_tokens_per_s": step_value,
        "roofline": {"bound": "hbm", "achieved": rf["achieved_gbs"], "peak": hbm, "unit": "GB/s",
                     "frac": rf["frac"], "traffic": profiled_traffic(),
                     "peak_source": src, "kernel": "prefill_kernel",
                     "alg_bytes_per_launch": rf["alg_bytes"],
                     "alg_flops_per_launch": rf["alg_flops"],
                     "tflops_achieved": rf["alg_flops"] / (t_prefill_us / 1e6) / 1e12,
                     "roofline_time_us": rf["roofline_us"],
                     "frac_of_roofline_time": rf["frac_of_roofline_time"]},
        "workloads": {name: dict(roofline_entry(pp.total_tokens, pp.num_seqs, pp.H_k, pp.H_v,
                                                pp.d_k, us), config=desc)
                      for name, (pp, us, desc) in others.items()},
        "variants": variants,
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

def _f64(t):
    import torch
    return t.to(dtype=torch.float64).numpy()


def oracle_prefill_rate(p, form, threads, heads, seqs=None, max_tokens=None):
    """Oracle tokens/s for the whole prefill workload p, from a timed sample:
    `heads` v-heads (each with its own k-head) over the sequences `seqs` (all
    by default), each cut to its first `max_tokens` tokens, scaled by the
    heads and tokens left out (the oracle's cost is linear in both).  The
    oracle's cost does not depend on the gate values."""
    import numpy as np
    import torch

    import oracle
    vpg = p.H_v // p.H_k
    hs = list(range(heads))
    kh = [h // vpg for h in hs]
    cu = p.cu_seqlens.numpy()
    seqs = list(range(p.num_seqs)) if seqs is None else seqs
    cap = (lambda n: int(cu[n + 1] - cu[n])) if max_tokens is None else \
        (lambda n: min(int(cu[n + 1] - cu[n]), max_tokens))
    rows = torch.from_numpy(np.concatenate([np.arange(cu[n], cu[n] + cap(n)) for n in seqs]))
    lens = [cap(n) for n in seqs]
    cu_s = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    # select the sample before widening to f64 (the full varlen tensors would
    # take gigabytes of host memory in f64)
    ht, kt = torch.tensor(hs), torch.tensor(kh)
    rng = np.random.default_rng(0)
    gs = (_f64(p.g[rows][:, ht]) if p.g is not None
          else -np.abs(rng.standard_normal((len(rows), heads))) * 0.1)
    bs = (_f64(p.beta[rows][:, ht]) if p.beta is not None
          else rng.uniform(0.1, 0.9, (len(rows), heads)))
    h0 = _f64(p.h0[torch.tensor(seqs)][:, ht])
    args = (_f64(p.q[rows][:, kt]), _f64(p.k[rows][:, kt]), _f64(p.v[rows][:, ht]), gs, bs,
            cu_s, h0)
    fn = oracle.gdn_token if form == "token" else oracle.gdn_chunked
    t0 = time.perf_counter()
    fn(*args, nthreads=threads)
    dt = time.perf_counter() - t0
    scale = (p.H_v / heads) * (p.total_tokens / max(1, len(rows)))
    return p.total_tokens / (dt * scale)


def cpu_baseline(detail=True):
    """The oracle on this host's cores, on bounded samples of the workloads.
    Returns (step seconds, threads, sample text, detail dict or None): a step
    is BA gates + token-form prefill (4576 tokens, 48 heads) + verify/fold of
    the speculative batch, all cores; the detail adds both prefill forms on
    all cores and on one core for the three prefill workloads."""
    import oracle
    from linear_attention_ssm_gdn_b200 import inputs as I

    nt = oracle.default_threads()
    w2 = I.workload(2)
    p2, ba = w2.prefill, w2.ba
    vi = I.workload(4).verify
    T = p2.total_tokens
    # BA gates on a row sample
    m_s = min(T, max(32, int(64 * nt)))
    t0 = time.perf_counter()
    oracle.ba_gates(_f64(ba.x[:m_s]), _f64(ba.w), _f64(ba.a_log), _f64(ba.dt_bias),
                    ba.vheads_per_group, nthreads=nt)
    t_ba = (time.perf_counter() - t0) * T / m_s
    # verify + fold on a batch sample
    b_s = min(vi.batch, max(1, nt))
    sl = slice(0, 4 * b_s)
    t0 = time.perf_counter()
    oracle.gdn_verify_fold(_f64(vi.pool[vi.slots[:b_s]]), _f64(vi.q[sl]), _f64(vi.k[sl]),
                           _f64(vi.v[sl]), _f64(vi.g[sl]), _f64(vi.beta[sl]),
                           vi.na[:b_s].numpy(), nthreads=nt)
    t_vf = (time.perf_counter() - t0) * vi.batch / b_s
    heads_all = min(p2.H_v, max(1, nt))
    rate2 = oracle_prefill_rate(p2, "token", nt, heads_all)
    step_s = t_ba + T / rate2 + t_vf
    sample = (f"oracle (f64 C, {nt} threads): BA gates on {m_s}/{T} rows, token recurrence on "
              f"{heads_all}/{p2.H_v} v-heads x {T} tokens, verify+fold on {b_s}/{vi.batch} "
              f"sequences; each scaled to the full step")
    if not detail:
        return step_s, nt, sample, None
    det = {"ba_gates_us": t_ba * 1e6, "verify_fold_us": t_vf * 1e6, "cores": nt,
           "prefill_tokens_per_s": {}}
    p1 = I.workload(1).prefill
    p3 = I.workload(3).prefill
    for name, pp, seqs in (("single_sequence", p1, None), ("ba_geometry", p2, None),
                           ("varlen", p3, [0])):
        r = {}
        for form, cap in (("token", None), ("chunked", 1024)):
            r[f"{form}_all_cores"] = oracle_prefill_rate(pp, form, nt, min(pp.H_v, nt), seqs,
                                                         cap)
            r[f"{form}_1_core"] = oracle_prefill_rate(pp, form, 1, 1, seqs, cap)
        det["prefill_tokens_per_s"][name] = r
    det["sample"] = ("each prefill rate from a timed sample scaled to the whole workload: "
                     f"min(H_v, {nt}) heads on all cores or 1 head on one core, over all "
                     "sequences (varlen: its first sequence); the chunked form over the "
                     "first 1024 tokens of each")
    return step_s, nt, sample, det


def run_reference(args):
    steps = []
    for i in range(args.warmup + args.steps):
        s, nt, sample, _ = cpu_baseline(detail=False)
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
    import faulthandler
    faulthandler.enable()  # a crash in native code prints every thread's Python stack
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
            progress("cpu baseline")
            s, nt, sample, det = cpu_baseline(detail=True)
            line["cpu_baseline"] = {"value": 4576 / s, "unit": UNIT, "cores": nt,
                                    "kind": "oracle", "sample": sample, "detail": det}
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())

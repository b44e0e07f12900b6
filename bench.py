"""Benchmark of the TriAttention KV-cache prune step on B200.

One step = one tria_prune over the whole synthetic workload (score every key,
z-score + GQA max, select the top budget, compact K/V/pos in place).  Before
every timed step the pruned rows are restored from a pristine copy and L2 is
flushed: a 512 MiB buffer is written, then another 512 MiB buffer is read, so the
cache holds only clean lines of unrelated data (the write-backs of the first
buffer's dirty lines would otherwise land in the timed span).  Neither is timed;
the figures with the write alone are reported beside the main ones.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload I] [--impl ours|reference]

Prints one JSON line (rank 0).  Multi-GPU (torchrun): every rank prunes its
own copy of the workload (weak scaling, no collective on the data path); the
step times are reduced with MAX over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from kv_cache_eviction_trig_b200 import tria, workloads  # noqa: E402

METRIC = "fused prune keys/s and HBM GB/s (score+top-k+compact), 8B-shape 32K cache"
UNIT = "keys/s"
PEAKS = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")


def _rank_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def _peaks():
    try:
        with open(PEAKS) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        props = torch.cuda.get_device_properties(device_index)
        uuid = str(getattr(props, "uuid", "") or "")
        self.gpu = (uuid if uuid.startswith("GPU-") else f"GPU-{uuid}") if uuid else str(device_index)
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        time.sleep(0.1)
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        for line in (self.out or "").splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v == "Active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": rows[0][1],
                "reasons": reasons, "samples": len(rows)}


def rank_workload(index: int, rank: int):
    """The workload a rank prunes: the same shapes on every rank, its own draw
    (seed + 1000 * rank) so that ranks never share inputs."""
    wl = workloads.workload(index)
    return workloads.workload(index, seed=wl.seed + 1000 * rank) if rank else wl


def max_over_ranks(values, device=None):
    """Element-wise maximum of a list of floats over all ranks (identity with one
    process); every rank receives the result."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


class OracleSample:
    """The oracle, as it stands, on the host cores, over a bounded sample of the
    workload: every query head of every KV head of layer 0, sequence 0, on the
    first n keys (budget scaled by n/T), n sized for about `seconds` of wall time."""

    def __init__(self, wl, seconds):
        import oracle
        from tests import common  # the oracle's numpy marshalling helpers

        self.oracle = oracle
        T = wl.seq_lens[0]
        per_key_cos = wl.group * len(wl.offsets) * (wl.head_dim // 2)
        self.threads = oracle.num_threads()
        # about 20 ns per cosine term per thread
        n = int(seconds * self.threads / (per_key_cos * 20e-9 * wl.n_kv_heads))
        n = max(64, min(T, n))
        sub = workloads.custom("cpu-sample", L=1, B=1, Hq=wl.n_q_heads, Hkv=wl.n_kv_heads,
                               D=wl.head_dim, theta=wl.rope_theta,
                               budget=max(1, wl.budget * n // T), offsets=wl.offsets,
                               seq_lens=[n], seed=wl.seed, nu=wl.kv_noise,
                               position_mode=wl.position_mode, rope_layout=wl.rope_layout,
                               n_calib=wl.n_calib)
        sub.position_span = lambda t, _T=T: wl.position_span(_T)
        data = workloads.generate(sub)
        stats = common.stats_fp32(data["q_calib"], wl.rope_layout)
        self.prob = common.problem(sub, data, stats)
        self.v = common.bf16_bits(data["v"])
        self.keys = n * wl.n_kv_heads
        self.desc = (f"layer 0, all {wl.n_kv_heads} KV heads x {wl.group} query heads, "
                     f"first {n} of {T} keys, budget {sub.budget}")

    def run(self):
        """Seconds of one oracle prune of the sample."""
        t0 = time.perf_counter()
        self.oracle.prune(self.prob, self.v)
        return time.perf_counter() - t0


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def _host_problem(wl, host, stats, seq_index, n_keys):
    """The oracle's problem over layer 0 and sequences [0, seq_index) of the pristine
    cache held in host memory, keeping the first n_keys keys of each sequence (all of
    them when n_keys is None); the budget scales with the kept fraction."""
    import numpy as np
    from tests import common

    import oracle
    starts = wl.seq_start
    lens = [wl.seq_lens[b] if n_keys is None else min(n_keys, wl.seq_lens[b])
            for b in range(seq_index)]
    k, v, pos = [], [], []
    new_starts = [0]
    for b in range(seq_index):
        s0 = starts[b]
        k.append(host["k"][0:1, :, s0:s0 + lens[b]])
        v.append(host["v"][0:1, :, s0:s0 + lens[b]])
        pos.append(host["pos"][0:1, :, s0:s0 + lens[b]])
        new_starts.append(new_starts[-1] + lens[b])
    import torch
    kk, vv, pp = (torch.cat(x, dim=2) for x in (k, v, pos))
    full = n_keys is None or all(wl.seq_lens[b] <= n_keys for b in range(seq_index))
    budget = wl.budget if full else max(1, wl.budget * lens[0] // wl.seq_lens[0])
    c, m, r = (x[0:1].double().numpy() for x in stats)
    prob = oracle.Problem(k=common.bf16_bits(kk), pos=pp.numpy(), seq_start=new_starts,
                          seq_len=lens, cur_pos=host["cur_pos"][:seq_index].numpy(),
                          centre=c, mean_norm=m, mrl=r, theta=wl.rope_theta, budget=budget,
                          offsets=wl.offsets, n_q_heads=wl.n_q_heads, layout=wl.rope_layout)
    keys = wl.n_kv_heads * sum(t for t in lens if t > budget)
    return prob, common.bf16_bits(vv), keys, budget, np.sum(lens)


def _cpu_baseline(wl, host, stats, seconds_target=12.0):
    """The oracle as it stands on this host's cores.  All cores: the term-by-term
    prune over the whole workload when that fits about `seconds_target` (else a
    labelled, extrapolated sample: layer 0, leading sequences, leading keys); one
    core: a smaller sample of the same kind, extrapolated; and the oracle's folded
    scoring path (one weight per head and pair, no per-key trigonometry) on the
    same sample as the all-cores figure."""
    import oracle
    threads = oracle.num_threads()
    out = {"unit": UNIT, "cores": threads, "kind": "oracle", "cpu_model": _cpu_model()}
    # cost per key (cosine terms) sets the sample: measured once on a small sample
    probe, probe_v, probe_keys, _, _ = _host_problem(wl, host, stats, 1, 256)
    t0 = time.perf_counter()
    oracle.prune(probe, probe_v)
    rate = probe_keys / max(time.perf_counter() - t0, 1e-6)
    want = rate * seconds_target
    if wl.keys_scored <= want:   # layer 0, every sequence, every key
        prob, v, keys, _, _ = _host_problem(wl, host, stats, wl.batch, None)
    else:
        seqs = max(1, min(wl.batch, int(want // (wl.n_kv_heads * max(wl.seq_lens)))))
        n = int(max(256, min(max(wl.seq_lens), want // (wl.n_kv_heads * seqs))))
        prob, v, keys, _, _ = _host_problem(wl, host, stats, seqs, n)
    full = keys == wl.keys_scored  # the whole workload (one layer, nothing cut)
    t0 = time.perf_counter()
    oracle.prune(prob, v)
    dt = time.perf_counter() - t0
    out["value"] = keys / dt
    out["extrapolated"] = not full
    out["sample"] = ("full workload" if full else
                     f"extrapolated from layer 0, {prob.B} sequence(s) x {prob.Hkv} KV heads, "
                     f"first {int(max(prob.seq_len))} keys each, budget {prob.budget}") + \
        f"; term by term; {dt:.1f} s wall"
    t0 = time.perf_counter()
    oracle.prune_folded(prob, v)
    dtf = time.perf_counter() - t0
    out["value_folded"] = keys / dtf
    out["sample_folded"] = "same sample, folded scoring path" + ("" if full else " (extrapolated)")
    # one core: a smaller sample, about a third of the target time
    n1 = int(max(128, min(max(wl.seq_lens), rate / threads * seconds_target / 3 / wl.n_kv_heads)))
    p1, v1, k1, _, _ = _host_problem(wl, host, stats, 1, n1)
    oracle.set_num_threads(1)
    try:
        t0 = time.perf_counter()
        oracle.prune(p1, v1)
        dt1 = time.perf_counter() - t0
    finally:
        oracle.set_num_threads(threads)
    k1 = p1.Hkv * sum(int(t) for t in p1.seq_len if t > p1.budget)
    out["value_1core"] = k1 / dt1
    out["sample_1core"] = (f"extrapolated from layer 0, sequence 0 x {p1.Hkv} KV heads, first "
                           f"{int(p1.seq_len[0])} keys, budget {p1.budget}; {dt1:.1f} s wall")
    return out


def run_reference(args):
    rank, world, _ = _rank_env()
    if rank != 0:
        return  # the oracle runs once, on rank 0's host
    wl = workloads.workload(args.workload)
    # each step is a bounded sample, sized so that the whole run takes a few minutes
    per_step = max(0.2, min(args.ref_seconds, 150.0 / (args.steps + args.warmup)))
    sample = OracleSample(wl, per_step)
    times = []
    for i in range(args.warmup + args.steps):
        dt = sample.run()
        if i >= args.warmup:
            times.append(dt)
    value = sample.keys / statistics.median(times)
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.median(times) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; the oracle on a bounded sample of the workload)",
        "config": dict(wl.describe(), l2="n/a (host)"),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": sample.threads, "kind": "oracle",
                         "sample": f"{sample.desc}; median of {args.steps} runs"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# Flops per key of the scoring arithmetic: per RoPE pair and query head two FMAs of
# the trigonometric term and one of the norm term (2 flops each), per pair |k|^2
# (3 flops) and its square root (1): F * (6 G + 4) = 3 G D + 2 D.
def flops_per_key(wl):
    return (wl.head_dim // 2) * (6 * wl.group + 4)


def fp32_peak_tflops(sm_mhz):
    """FP32 peak of a B200 at the given SM clock: 148 SMs x 128 FP32 lanes x 2 flops
    (one FMA) per lane per clock."""
    return 148 * 128 * 2 * sm_mhz * 1e6 / 1e12


def _kernel_hash(names):
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(ROOT, "kv_cache_eviction_trig_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


KERNEL_SOURCES = {"prune_kernel": ("prune.cu", "score_math.cuh", "tria_internal.cuh"),
                  "score_kernel": ("score.cu", "mma_sync.cuh", "tria_internal.cuh"),
                  "unit_kernel": ("unit.cu", "tria_internal.cuh")}


def _traffic(kernel, key):
    """DRAM bytes per launch of `kernel` on workload `key` from the committed ncu
    summary, or None if there is none or the kernel source changed since."""
    try:
        with open(TRAFFIC) as f:
            t = json.load(f)
        e = t.get(f"{kernel}:{key}")
        if e and e.get("source_hash") == _kernel_hash(KERNEL_SOURCES[kernel]):
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


L2_NOTE = ("flushed before every step: 512 MiB written, then another 512 MiB read "
           "(L2 left holding clean lines of unrelated data)")


class L2Flush:
    """Evicts every line of L2 (126 MB on a B200): a 512 MiB buffer is written, then
    (unless write_only) a second 512 MiB buffer is read, so that the dirty lines of the
    first are written back here rather than inside the next timed span."""

    def __init__(self, dev):
        self.buf = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
        self.other = torch.ones(64 << 20, dtype=torch.int64, device=dev)
        self.sink = torch.empty(1, dtype=torch.int64, device=dev)

    def __call__(self, write_only=False):
        self.buf.fill_(1)
        if not write_only:
            torch.amax(self.other, dim=0, keepdim=True, out=self.sink)


class Bench:
    """One workload resident on the device, ready to be pruned again and again:
    before every step the rows a prune overwrites are restored from a pristine
    copy and L2 is flushed (L2Flush); neither is timed."""

    def __init__(self, wl, dev, flags=0):
        self.wl, self.dev = wl, dev
        data = workloads.generate(wl, device=dev)
        self.cfg = tria.Config.from_workload(wl, flags=flags)
        self.stats = tria.calibrate(self.cfg, data["q_calib"])
        del data["q_calib"]
        self.data = data
        self.cache = tria.Cache.from_data(data)
        self.ws = tria.workspace(self.cfg, self.cache)
        starts, budget = data["seq_start"], wl.budget
        # rows a prune overwrites: [seg, seg + budget) of each sequence longer than budget
        self.restore = [(starts[b], budget) for b in range(wl.batch) if wl.seq_lens[b] > budget]
        self.backup = {n: [data[n][:, :, s:s + c].clone() for s, c in self.restore]
                       for n in ("k", "v", "pos")}
        self.seq_len0 = data["seq_len"].clone()
        self.flush = L2Flush(dev)
        self.stream = torch.cuda.current_stream()

    def reset(self, write_only=False):
        for n in ("k", "v", "pos"):
            for (s, c), t in zip(self.restore, self.backup[n]):
                self.data[n][:, :, s:s + c].copy_(t)
        self.data["seq_len"].copy_(self.seq_len0)
        self.flush(write_only)

    def prune(self):
        tria.tria_prune(self.cfg, self.stats, self.cache, self.ws, stream=self.stream)

    def warm(self, n):
        for _ in range(n):
            self.reset()
            self.prune()
        torch.cuda.synchronize()
        if tria.tria_get_device_error(self.ws) != 0:
            raise RuntimeError(f"device error flag set on {self.wl.name}")
        want = [min(t, self.wl.budget) for t in self.wl.seq_lens]
        if self.data["seq_len"].tolist() != want:
            raise RuntimeError(f"pruned lengths differ on {self.wl.name}")

    def timed(self, steps, write_only=False):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        for i in range(steps):
            self.reset(write_only)
            ev[i][0].record(self.stream)
            self.prune()
            ev[i][1].record(self.stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in ev]

    def kernels(self, steps):
        """Per-kernel event times (a separate pass: events between the prune's kernels)."""
        nst = tria.PRUNE_MAX_STAGES + 1
        kev = [[torch.cuda.Event(enable_timing=True) for _ in range(nst)] for _ in range(steps)]
        names = []
        for i in range(steps):
            self.reset()
            names = tria.tria_prune_profiled(self.cfg, self.stats, self.cache, self.ws, kev[i],
                                             stream=self.stream)
        torch.cuda.synchronize()
        per = [[kev[i][s].elapsed_time(kev[i][s + 1]) for s in range(len(names))]
               for i in range(steps)]
        return names, [statistics.mean(k[s] for k in per) for s in range(len(names))]

    def summary(self, step_ms, names, kern_ms, peak, sm_mhz):
        """Throughput and roofline figures of one workload (device-timed)."""
        wl = self.wl
        step = statistics.mean(step_ms)
        keys = wl.keys_scored
        algo = wl.algorithmic_bytes()
        out = {"workload": wl.name, "value": keys / (step / 1e3), "unit": UNIT,
               "ms_per_step": step, "us_per_layer": step * 1e3 / wl.num_layers,
               "hbm_gbs_path": algo / (step / 1e3) / 1e9,
               "frac_path": algo / (step / 1e3) / 1e9 / peak,
               "kernel_ms": dict(zip(names, kern_ms))}
        if "prune_kernel" in names:
            kt = kern_ms[names.index("prune_kernel")]
            out["prune_kernel_frac"] = algo / (kt / 1e3) / 1e9 / peak
            busy_ms = kt
        else:
            ut = kern_ms[names.index("unit_kernel")]
            out["unit_kernel_frac"] = (algo - keys * 2 * wl.head_dim) / (ut / 1e3) / 1e9 / peak
            kt = kern_ms[names.index("score_kernel")]
            out["score_kernel_frac"] = keys * 2 * wl.head_dim / (kt / 1e3) / 1e9 / peak
            busy_ms = kt
        tflops = keys * flops_per_key(wl) / (busy_ms / 1e3) / 1e12
        out["fp32_tflops"] = tflops
        if sm_mhz:
            out["frac_fp32"] = tflops / fp32_peak_tflops(sm_mhz)
        return out

    def free(self):
        del self.data, self.cache, self.ws, self.backup, self.flush, self.stats
        torch.cuda.empty_cache()


def attention_figures(dev, B, T, steps, peak):
    """tria_decode_attention on one 8B-shaped layer (8 KV heads x 4 query heads, D = 128)
    with B sequences of T live keys, L2 flushed before every call: mean device time and
    HBM rate (K and V of the live slots read once); also the time with the flush's write
    alone."""
    H, Hq, D = 8, 32, 128
    gen = torch.Generator(device=dev).manual_seed(B * 100003 + T)
    k = torch.randn(1, H, B * T, D, device=dev, generator=gen).to(torch.bfloat16)
    v = torch.randn(1, H, B * T, D, device=dev, generator=gen).to(torch.bfloat16)
    pos = torch.zeros(1, H, B * T, dtype=torch.int32, device=dev)
    sl = torch.full((B,), T, dtype=torch.int32, device=dev)
    cfg = tria.Config(num_layers=1, batch=B, n_q_heads=Hq, n_kv_heads=H, head_dim=D,
                      rope_theta=1e6, budget=T, offsets=[1])
    cache = tria.Cache(k, v, pos, sl, sl.clone(), [b * T for b in range(B + 1)])
    ws = tria.workspace(cfg, cache)
    q = torch.randn(B, Hq, D, device=dev, generator=gen).to(torch.bfloat16)
    out = torch.empty(B, Hq, D, device=dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()
    for _ in range(3):
        tria.tria_decode_attention(cfg, cache, 0, q, out, ws, stream=stream)

    def run(write_only):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        for a, b in ev:
            flush(write_only)
            a.record(stream)
            tria.tria_decode_attention(cfg, cache, 0, q, out, ws, stream=stream)
            b.record(stream)
        torch.cuda.synchronize()
        return statistics.mean(a.elapsed_time(b) for a, b in ev)

    ms, ms_w = run(False), run(True)
    if tria.tria_get_device_error(ws) != 0:
        raise RuntimeError("device error flag set in decode attention")
    algo = B * H * T * 4 * D
    return {"batch": B, "live_keys": T, "us": ms * 1e3, "gbs": algo / (ms / 1e3) / 1e9,
            "frac": algo / (ms / 1e3) / 1e9 / peak, "algorithmic_bytes": algo, "steps": steps,
            "us_write_only_flush": ms_w * 1e3,
            "frac_write_only_flush": algo / (ms_w / 1e3) / 1e9 / peak}


def run_ours(args):
    rank, world, local = _rank_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", device_id=dev, timeout=timedelta(seconds=120))
    wl = rank_workload(args.workload, rank)
    peak, peak_kind = _peaks()
    bench = Bench(wl, dev)
    bench.warm(args.warmup)

    # ---- timed region: K steps, each bracketed by events on the launching stream
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        step_ms = bench.timed(args.steps)
    if world > 1:
        dist.barrier()
    clocks = clk.summary()
    sm_mhz = clocks["sm_mhz"] if clocks else None
    names, kern_ms = bench.kernels(args.steps)
    # the same steps with the flush's write alone (its dirty lines written back in the span)
    wo_ms = bench.timed(args.steps, write_only=True)

    # ---- end to end through the C ABI with host buffers (pinned), copies timed
    data, restore, backup = bench.data, bench.restore, bench.backup
    host = {n: data[n].cpu().pin_memory() for n in ("k", "v", "pos", "seq_len", "cur_pos")}
    for n in ("k", "v", "pos"):
        for (s, c), t in zip(restore, backup[n]):
            host[n][:, :, s:s + c].copy_(t.cpu())
    host["seq_len"].copy_(bench.seq_len0.cpu())
    budget = wl.budget
    out_k = torch.empty(wl.num_layers, wl.n_kv_heads, len(restore), budget, wl.head_dim,
                        dtype=torch.bfloat16).pin_memory()
    out_v = torch.empty_like(out_k).pin_memory()
    out_p = torch.empty(wl.num_layers, wl.n_kv_heads, len(restore), budget,
                        dtype=torch.int32).pin_memory()
    out_len = torch.empty(wl.batch, dtype=torch.int32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in (out_k, out_v, out_p, out_len))
    e2e_steps = max(3, min(args.steps, 20))
    eev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(e2e_steps)]
    stream = bench.stream
    for i in range(e2e_steps):
        bench.flush()
        eev[i][0].record(stream)
        for n in ("k", "v", "pos", "seq_len", "cur_pos"):
            data[n].copy_(host[n], non_blocking=True)
        bench.prune()
        for j, (s, c) in enumerate(restore):
            out_k[:, :, j].copy_(data["k"][:, :, s:s + c], non_blocking=True)
            out_v[:, :, j].copy_(data["v"][:, :, s:s + c], non_blocking=True)
            out_p[:, :, j].copy_(data["pos"][:, :, s:s + c], non_blocking=True)
        out_len.copy_(data["seq_len"], non_blocking=True)
        eev[i][1].record(stream)
    torch.cuda.synchronize()
    e2e_ms = statistics.mean(a.elapsed_time(b) for a, b in eev)
    if tria.tria_get_device_error(bench.ws) != 0:
        raise RuntimeError("device error flag set during the timed runs")

    total_ms = sum(step_ms)
    red = max_over_ranks([total_ms, e2e_ms, sum(wo_ms)] + kern_ms, device=dev)
    total_ms, e2e_ms, wo_total, kern_ms = red[0], red[1], red[2], red[3:]
    step = total_ms / args.steps
    head = bench.summary([step], names, kern_ms, peak, sm_mhz)
    keys = wl.keys_scored
    dom = max(range(len(names)), key=lambda s: kern_ms[s])
    kern = names[dom]
    if kern == "prune_kernel":
        algo_launch = wl.algorithmic_bytes()  # the whole step: keys read, kept rows moved
    elif kern == "unit_kernel":
        algo_launch = wl.algorithmic_bytes() - keys * 2 * wl.head_dim  # kept rows moved
    else:
        algo_launch = keys * 2 * wl.head_dim  # the score kernel reads every key once
    achieved = algo_launch / (kern_ms[dom] / 1e3) / 1e9
    out = {
        "metric": METRIC, "value": keys * world / (step / 1e3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded; pages' shapes and value distributions)",
        "config": dict(wl.describe(), l2=L2_NOTE,
                       parallelism=f"dp{world} (independent caches per GPU)"),
        "hbm_gbs_path": head["hbm_gbs_path"],
        "frac_path": head["frac_path"],
        "us_per_layer": head["us_per_layer"],
        "roofline": {"bound": "hbm", "kernel": kern, "achieved": achieved,
                     "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_source": peak_kind, "traffic": _traffic(kern, args.workload),
                     "algorithmic_bytes_per_launch": algo_launch,
                     "dominant_kernel": kern},
        "kernel_ms": dict(zip(names, kern_ms)),
        "fp32_tflops": head["fp32_tflops"], "frac_fp32": head.get("frac_fp32"),
        "clocks": clocks,
        "e2e": {"value": keys * world / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": len(names) * args.steps,
        "l2_write_only_flush": {"ms_per_step": wo_total / args.steps,
                                "value": keys * world / (wo_total / args.steps / 1e3)},
    }
    host_stats = [t.cpu() for t in bench.stats.tensors]
    bench.free()
    del data

    # ---- the other workloads and the pages' geometric offsets, same protocol, fewer steps
    if not args.no_extras:
        extras = {}
        geo = [2 ** i for i in range(17)]
        specs = [("workload2", workloads.workload(2)), ("workload3", workloads.workload(3)),
                 ("workload4", workloads.workload(4)),
                 ("workload1_geometric", workloads.workload(1, offsets=geo,
                                                            name=workloads.workload(1).name + " geometric offsets 1..65536")),
                 ("workload2_geometric", workloads.workload(2, offsets=geo,
                                                            name=workloads.workload(2).name + " geometric offsets 1..65536")),
                 # the same prune as one persistent launch (TRIA_FUSED_PRUNE)
                 ("workload1_fused", workloads.workload(1)),
                 ("workload2_fused", workloads.workload(2))]
        for key, xwl in specs:
            if rank:
                xwl = workloads.workload(int(key[8]), seed=xwl.seed + 1000 * rank,
                                         offsets=xwl.offsets, name=xwl.name)
            try:
                xb = Bench(xwl, dev, flags=tria.FUSED_PRUNE if key.endswith("_fused") else 0)
                xb.warm(3)
                with ClockSampler(local) as xclk:
                    xms = xb.timed(args.extra_steps)
                xnames, xkern = xb.kernels(args.extra_steps)
                xsum = max_over_ranks([sum(xms)] + xkern, device=dev)
                xc = xclk.summary()
                entry = xb.summary([xsum[0] / args.extra_steps], xnames, xsum[1:], peak,
                                   xc["sm_mhz"] if xc else None)
                entry["value"] *= world
                entry["steps"] = args.extra_steps
                entry["clocks"] = xc
                if tria.tria_get_device_error(xb.ws) != 0:
                    entry["error"] = "device error flag set"
                xb.free()
                del xb
            except Exception as e:  # a workload that does not fit is reported, not fatal
                entry = {"workload": xwl.name, "error": f"{type(e).__name__}: {e}"}
                torch.cuda.empty_cache()
            extras[key] = entry
        # decode attention over a pruned (2048) and an unpruned (32768) layer
        for B, T in ((1, 2048), (1, 32768), (16, 2048), (16, 32768)):
            try:
                extras[f"attention_b{B}_t{T}"] = attention_figures(dev, B, T, args.extra_steps, peak)
            except Exception as e:
                extras[f"attention_b{B}_t{T}"] = {"error": f"{type(e).__name__}: {e}"}
            torch.cuda.empty_cache()
        out["extra_workloads"] = extras

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = _cpu_baseline(wl, host, host_stats)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=1)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="time only the headline workload (not workloads 2-4 and the geometric offsets)")
    ap.add_argument("--extra-steps", type=int, default=10)
    ap.add_argument("--ref-seconds", type=float, default=8.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

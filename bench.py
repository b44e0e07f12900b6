"""Benchmark of the TriAttention KV-cache prune step on B200.

One step = one tria_prune over the whole synthetic workload (score every key,
z-score + GQA max, select the top budget, compact K/V/pos in place).  Before
every timed step the pruned rows are restored from a pristine copy and L2 is
flushed by writing a 512 MiB buffer; neither is inside the timed spans.

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


def _score_source_hash():
    h = hashlib.sha256()
    for name in ("score.cu", "tria_internal.cuh"):
        with open(os.path.join(ROOT, "kv_cache_eviction_trig_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _traffic_per_launch(workload_index):
    """DRAM bytes per score-kernel launch from the committed ncu summary, or None
    if there is none for this workload or the kernel source changed since."""
    try:
        with open(TRAFFIC) as f:
            t = json.load(f)
        e = t.get(str(workload_index))
        if e and e.get("source_hash") == _score_source_hash():
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


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


def run_ours(args):
    rank, world, local = _rank_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", device_id=dev, timeout=timedelta(seconds=120))
    wl = rank_workload(args.workload, rank)

    data = workloads.generate(wl, device=dev)
    cfg = tria.Config.from_workload(wl)
    stats = tria.calibrate(cfg, data["q_calib"])
    del data["q_calib"]
    cache = tria.Cache.from_data(data)
    ws = tria.workspace(cfg, cache)
    B, budget = wl.batch, wl.budget
    starts = data["seq_start"]
    # rows a prune overwrites: [seg, seg + budget) of each sequence longer than budget
    restore = [(starts[b], budget) for b in range(B) if wl.seq_lens[b] > budget]
    backup = {n: [data[n][:, :, s:s + c].clone() for s, c in restore] for n in ("k", "v", "pos")}
    seq_len0 = data["seq_len"].clone()
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)

    def reset():
        for n in ("k", "v", "pos"):
            for (s, c), t in zip(restore, backup[n]):
                data[n][:, :, s:s + c].copy_(t)
        data["seq_len"].copy_(seq_len0)
        flush.fill_(1)

    stream = torch.cuda.current_stream()
    sel = torch.empty(wl.num_layers, wl.n_kv_heads, B, budget, dtype=torch.int32, device=dev)

    # ---- warm-up and a correctness guard (the pruned lengths)
    for _ in range(args.warmup):
        reset()
        tria.tria_prune(cfg, stats, cache, ws, stream=stream)
    torch.cuda.synchronize()
    if tria.tria_get_device_error(ws) != 0:
        raise RuntimeError("device error flag set during warm-up")
    assert data["seq_len"].tolist() == [min(t, budget) for t in wl.seq_lens]

    # ---- timed region: K steps, each bracketed by events on the launching stream
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            reset()
            ev[i][0].record(stream)
            tria.tria_prune(cfg, stats, cache, ws, stream=stream)
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = sum(step_ms)
    clocks = clk.summary()

    # ---- per-kernel times (separate pass: events between the prune's kernels)
    nst = tria.PRUNE_MAX_STAGES + 1
    kern_ms = None
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(nst)] for _ in range(args.steps)]
    n_stages = 0
    for i in range(args.steps):
        reset()
        n_stages = tria.tria_prune_profiled(cfg, stats, cache, ws, kev[i], stream=stream)
    torch.cuda.synchronize()
    kern_ms = [[kev[i][s].elapsed_time(kev[i][s + 1]) for s in range(n_stages)]
               for i in range(args.steps)]
    avg_kern = [statistics.mean(k[s] for k in kern_ms) for s in range(n_stages)]
    names = [tria.tria_prune_stage_name(s) for s in range(n_stages)]

    # ---- end to end through the C ABI with host buffers (pinned), copies timed
    host = {n: data[n].cpu().pin_memory() for n in ("k", "v", "pos", "seq_len", "cur_pos")}
    for (s, c), t in zip(restore, backup["k"]):
        host["k"][:, :, s:s + c].copy_(t.cpu())
    for (s, c), t in zip(restore, backup["v"]):
        host["v"][:, :, s:s + c].copy_(t.cpu())
    for (s, c), t in zip(restore, backup["pos"]):
        host["pos"][:, :, s:s + c].copy_(t.cpu())
    host["seq_len"].copy_(seq_len0.cpu())
    out_k = torch.empty(wl.num_layers, wl.n_kv_heads, len(restore), budget, wl.head_dim,
                        dtype=torch.bfloat16).pin_memory()
    out_v = torch.empty_like(out_k).pin_memory()
    out_p = torch.empty(wl.num_layers, wl.n_kv_heads, len(restore), budget,
                        dtype=torch.int32).pin_memory()
    out_len = torch.empty(B, dtype=torch.int32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in (out_k, out_v, out_p, out_len))
    e2e_steps = max(3, min(args.steps, 20))
    eev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(e2e_steps)]
    for i in range(e2e_steps):
        flush.fill_(1)
        eev[i][0].record(stream)
        for n in ("k", "v", "pos", "seq_len", "cur_pos"):
            data[n].copy_(host[n], non_blocking=True)
        tria.tria_prune(cfg, stats, cache, ws, stream=stream)
        for j, (s, c) in enumerate(restore):
            out_k[:, :, j].copy_(data["k"][:, :, s:s + c], non_blocking=True)
            out_v[:, :, j].copy_(data["v"][:, :, s:s + c], non_blocking=True)
            out_p[:, :, j].copy_(data["pos"][:, :, s:s + c], non_blocking=True)
        out_len.copy_(data["seq_len"], non_blocking=True)
        eev[i][1].record(stream)
    torch.cuda.synchronize()
    e2e_ms = statistics.mean(a.elapsed_time(b) for a, b in eev)

    red = max_over_ranks([total_ms, e2e_ms] + avg_kern, device=dev)
    total_ms, e2e_ms, avg_kern = red[0], red[1], red[2:]

    keys = wl.keys_scored
    value = keys * world / (total_ms / 1e3 / args.steps)
    step = total_ms / args.steps
    peak, peak_kind = _peaks()
    score_i = names.index("score_kernel")
    score_bytes = keys * 2 * wl.head_dim        # K read once (positions are not needed)
    achieved = score_bytes / (avg_kern[score_i] / 1e3) / 1e9
    traffic = _traffic_per_launch(args.workload)
    dom = max(range(n_stages), key=lambda s: avg_kern[s])
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded; pages' shapes and value distributions)",
        "config": dict(wl.describe(), l2="flushed: 512 MiB write before every step",
                       parallelism=f"dp{world} (independent caches per GPU)"),
        "hbm_gbs_path": wl.algorithmic_bytes() / (step / 1e3) / 1e9,
        "frac_path": wl.algorithmic_bytes() / (step / 1e3) / 1e9 / peak,
        "roofline": {"bound": "hbm", "kernel": names[score_i], "achieved": achieved,
                     "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_source": peak_kind, "traffic": traffic,
                     "algorithmic_bytes_per_launch": score_bytes,
                     "dominant_kernel": names[dom]},
        "kernel_ms": dict(zip(names, avg_kern)),
        "clocks": clocks,
        "e2e": {"value": keys * world / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": n_stages * args.steps,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = _cpu_baseline(wl, host, [t.cpu() for t in stats.tensors])
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

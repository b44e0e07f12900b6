"""Test helpers: move a drawn workload into the oracle's numpy form."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from kv_cache_eviction_trig_b200 import workloads


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bits_to_float(a: np.ndarray) -> np.ndarray:
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def stats_fp32(q_calib: torch.Tensor, layout: int):
    """Oracle calibration of the drawn queries, rounded to float32 (the stats
    both implementations then score with)."""
    c, m, r = oracle.calibrate(q_calib.detach().cpu().double().numpy(), layout)
    return (c.astype(np.float32), m.astype(np.float32), r.astype(np.float32))


def problem(wl: workloads.Workload, data: dict, stats, flags: int = 0,
            seq_len=None) -> oracle.Problem:
    c, m, r = stats
    return oracle.Problem(
        k=bf16_bits(data["k"]), pos=data["pos"].cpu().numpy(), seq_start=data["seq_start"],
        seq_len=(data["seq_len"].cpu().numpy() if seq_len is None else seq_len),
        cur_pos=data["cur_pos"].cpu().numpy(), centre=c.astype(np.float64),
        mean_norm=m.astype(np.float64), mrl=r.astype(np.float64), theta=wl.rope_theta,
        budget=wl.budget, offsets=wl.offsets, n_q_heads=wl.n_q_heads, layout=wl.rope_layout,
        flags=flags)

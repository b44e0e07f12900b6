"""Seeded synthetic KV caches for the TriAttention prune step.

This module only draws inputs.  It holds none of the prune arithmetic (no
scoring, folding, normalisation, selection or compaction); both the CUDA path
and the CPU oracle receive the tensors it produces.

What is drawn, per the pages' setting (pre-RoPE Q/K concentrate around fixed
non-zero centres: TriAttention review, romaanj.github.io, "Key idea"; the
dimensionstp.github.io review, section 3-2 (1) "Q/K concentration"):

* per (layer, KV head) a complex key centre with pair magnitudes
  LogNormal(mu=0, sigma=0.5) and phases U[0, 2*pi);
* pre-RoPE keys = centre + Gaussian noise whose vector norm is about
  ``nu`` times the centre norm (per-component std nu*||c||/sqrt(D));
* per (layer, query head) a query centre drawn the same way, and ``n_calib``
  pre-RoPE calibration queries around it with the noise level of the head's
  KV group;
* keys are rotated by their token position with RoPE in float64 and stored
  as bfloat16 (torch's round-to-nearest-even cast); V ~ N(0, 1) in bfloat16.

RoPE here is the model's positional encoding applied to synthetic keys (an
input property), written out independently of both implementations.

Layout produced (the library's cache layout):
  k, v    bf16  [L][Hkv][cap_total][D]
  pos     int32 [L][Hkv][cap_total]   (positions of each sequence ascend)
  seq_start int64 [B+1] (host list), seq_len int32 [B], cur_pos int32 [B]
  q_calib fp32  [L][N][Hq][D]
"""
from __future__ import annotations

import dataclasses
import math
from typing import Callable, List, Optional, Sequence

import torch

HALF_SPLIT = 0
INTERLEAVED = 1


@dataclasses.dataclass
class Workload:
    name: str
    num_layers: int
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    rope_theta: float
    budget: int
    offsets: List[int]
    seq_lens: List[int]                 # T_b per sequence
    position_mode: str                  # "contiguous" or "subset"
    position_span: Callable[[int], int]  # T_b -> span P; positions drawn from [0, P)
    kv_noise: Callable[[int], float]    # kv head g -> nu
    seed: int
    rope_layout: int = HALF_SPLIT
    n_calib: int = 1024
    slack: int = 0                      # spare capacity after each segment

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def seq_start(self) -> List[int]:
        out = [0]
        for t in self.seq_lens:
            out.append(out[-1] + t + self.slack)
        return out

    @property
    def cap_total(self) -> int:
        return self.seq_start[-1]

    @property
    def keys_scored(self) -> int:
        """Keys a prune scores: every key of every (layer, KV head, sequence)
        whose length exceeds the budget (shorter sequences are left alone)."""
        return self.num_layers * self.n_kv_heads * sum(t for t in self.seq_lens if t > self.budget)

    def algorithmic_bytes(self) -> int:
        """Bytes a prune must move: every key read once, and for each pruned
        (layer, KV head, sequence) the survivors' K and V rows read and
        written plus their positions read and written."""
        d = self.head_dim
        total = 0
        for t in self.seq_lens:
            if t > self.budget:
                total += t * 2 * d + self.budget * (8 * d + 8)
        return total * self.num_layers * self.n_kv_heads

    def describe(self) -> dict:
        return {
            "workload": self.name,
            "layers": self.num_layers, "batch": self.batch,
            "q_heads": self.n_q_heads, "kv_heads": self.n_kv_heads,
            "head_dim": self.head_dim, "rope_theta": self.rope_theta,
            "budget": self.budget,
            "offsets": (f"{self.offsets[0]}..{self.offsets[-1]}"
                        if self.offsets == list(range(self.offsets[0], self.offsets[-1] + 1))
                        else f"{len(self.offsets)} offsets"),
            "seq_len": (self.seq_lens[0] if len(set(self.seq_lens)) == 1
                        else f"{min(self.seq_lens)}..{max(self.seq_lens)}"),
        }


def _nu_cfg1(g: int) -> float:
    # a quarter of the KV heads (and their query heads) are weakly concentrated
    return 1.5 if g % 4 == 3 else 0.3


def workload(index: int, **overrides) -> Workload:
    """The five synthetic workloads: 0 tiny, 1 one 8B-shaped layer at 32K,
    2 that layer x 36, 3 ragged batch of 16, 4 long (131072) with G=8."""
    if index == 0:
        wl = Workload("tiny L1 B1 Hq4 Hkv2 D64 T2048 budget512", 1, 1, 4, 2, 64, 1.0e4, 512,
                      list(range(1, 129)), [2048], "contiguous", lambda t: t,
                      lambda g: 0.3, seed=0)
    elif index == 1:
        wl = Workload("8B-shape layer L1 B1 Hq32 Hkv8 D128 T32768 budget2048", 1, 1, 32, 8, 128,
                      1.0e6, 2048, list(range(1, 257)), [32768], "subset",
                      lambda t: 2 * t, _nu_cfg1, seed=1)
    elif index == 2:
        wl = Workload("8B-shape model L36 B1 Hq32 Hkv8 D128 T32768 budget2048", 36, 1, 32, 8, 128,
                      1.0e6, 2048, list(range(1, 257)), [32768], "subset",
                      lambda t: 2 * t, _nu_cfg1, seed=2)
    elif index == 3:
        g = torch.Generator().manual_seed(3)
        lens = torch.randint(8192, 32769, (16,), generator=g).tolist()
        wl = Workload("ragged serving L36 B16 Hq32 Hkv8 D128 T8192..32768 budget2048", 36, 16,
                      32, 8, 128, 1.0e6, 2048, list(range(1, 257)), lens, "subset",
                      lambda t: 2 * t, _nu_cfg1, seed=3)
    elif index == 4:
        wl = Workload("long L1 B4 Hq64 Hkv8 D128 T131072 budget4096", 1, 4, 64, 8, 128, 1.0e6,
                      4096, list(range(1, 1025)), [131072] * 4, "contiguous",
                      lambda t: t, lambda g: 0.1 if g < 4 else 2.0, seed=4)
    else:
        raise ValueError(f"no workload {index}")
    return dataclasses.replace(wl, **overrides) if overrides else wl


def custom(name: str, *, L: int, B: int, Hq: int, Hkv: int, D: int, theta: float,
           budget: int, offsets: Sequence[int], seq_lens: Sequence[int], seed: int,
           position_mode: str = "subset", nu: float | Callable[[int], float] = 0.3,
           rope_layout: int = HALF_SPLIT, n_calib: int = 256, slack: int = 0) -> Workload:
    """A small workload with the same value distributions, for tests."""
    nu_fn = nu if callable(nu) else (lambda g, _nu=nu: _nu)
    span = (lambda t: 2 * t) if position_mode == "subset" else (lambda t: t)
    return Workload(name, L, B, Hq, Hkv, D, theta, budget, list(offsets), list(seq_lens),
                    position_mode, span, nu_fn, seed, rope_layout, n_calib, slack)


# --------------------------------------------------------------------------------------
# drawing


def _pair_index(D: int, layout: int):
    F = D // 2
    f = torch.arange(F)
    if layout == HALF_SPLIT:
        return f, f + F
    return 2 * f, 2 * f + 1


def _centres(gen: torch.Generator, n: int, D: int, layout: int) -> torch.Tensor:
    """n complex centres as real D-vectors: magnitudes LogNormal(0, 0.5), phases U[0, 2pi)."""
    F = D // 2
    mag = torch.exp(0.5 * torch.randn(n, F, generator=gen, dtype=torch.float64))
    ph = 2.0 * math.pi * torch.rand(n, F, generator=gen, dtype=torch.float64)
    xi, yi = _pair_index(D, layout)
    out = torch.zeros(n, D, dtype=torch.float64)
    out[:, xi] = mag * torch.cos(ph)
    out[:, yi] = mag * torch.sin(ph)
    return out


def _rope_rotate(vec: torch.Tensor, pos: torch.Tensor, theta: float, layout: int) -> torch.Tensor:
    """Rotate each pair (x, y) of vec[..., D] by angle w_f * pos, w_f = theta**(-2f/D), in float64."""
    D = vec.shape[-1]
    F = D // 2
    xi, yi = _pair_index(D, layout)
    xi = xi.to(vec.device)
    yi = yi.to(vec.device)
    w = torch.pow(torch.tensor(theta, dtype=torch.float64),
                  -2.0 * torch.arange(F, dtype=torch.float64) / D).to(vec.device)
    ang = pos.to(torch.float64).unsqueeze(-1) * w           # [..., F]
    c, s = torch.cos(ang), torch.sin(ang)
    x, y = vec[..., xi], vec[..., yi]
    out = torch.empty_like(vec)
    out[..., xi] = x * c - y * s
    out[..., yi] = x * s + y * c
    return out


def generate(wl: Workload, device: str | torch.device = "cpu", with_calib: bool = True) -> dict:
    """Draw the cache, positions and calibration queries of a workload.

    Small per-head parameters come from a CPU generator seeded with wl.seed;
    the bulk draws use a generator on ``device`` seeded with wl.seed + 1.
    """
    device = torch.device(device)
    L, B, Hq, Hkv, D = wl.num_layers, wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim
    G = Hq // Hkv
    cpu = torch.Generator().manual_seed(wl.seed)
    bulk = torch.Generator(device=device).manual_seed(wl.seed + 1)

    kc = _centres(cpu, L * Hkv, D, wl.rope_layout).view(L, Hkv, D)
    qc = _centres(cpu, L * Hq, D, wl.rope_layout).view(L, Hq, D)
    nu_kv = torch.tensor([wl.kv_noise(g) for g in range(Hkv)], dtype=torch.float64)
    k_scale = nu_kv * kc.norm(dim=-1) / math.sqrt(D)               # [L, Hkv]
    q_scale = nu_kv.repeat_interleave(G) * qc.norm(dim=-1) / math.sqrt(D)  # [L, Hq]

    starts = wl.seq_start
    cap = wl.cap_total
    k = torch.zeros(L, Hkv, cap, D, dtype=torch.bfloat16, device=device)
    v = torch.zeros(L, Hkv, cap, D, dtype=torch.bfloat16, device=device)
    pos = torch.zeros(L, Hkv, cap, dtype=torch.int32, device=device)
    cur = []
    for b, T in enumerate(wl.seq_lens):
        span = wl.position_span(T)
        cur.append(span - 1)
        s0 = starts[b]
        if wl.position_mode == "contiguous":
            p = torch.arange(T, device=device, dtype=torch.int64).expand(L, Hkv, T)
        else:
            r = torch.rand(L * Hkv, span, generator=bulk, device=device)
            p = r.argsort(dim=1)[:, :T].sort(dim=1).values.view(L, Hkv, T)
        pos[:, :, s0:s0 + T] = p.to(torch.int32)
        for l in range(L):
            noise = torch.randn(Hkv, T, D, generator=bulk, device=device, dtype=torch.float64)
            pre = kc[l].to(device).unsqueeze(1) + k_scale[l].to(device).view(Hkv, 1, 1) * noise
            k[l, :, s0:s0 + T] = _rope_rotate(pre, p[l], wl.rope_theta, wl.rope_layout).to(torch.bfloat16)
            v[l, :, s0:s0 + T] = torch.randn(Hkv, T, D, generator=bulk, device=device,
                                             dtype=torch.float32).to(torch.bfloat16)
    out = {
        "k": k, "v": v, "pos": pos,
        "seq_start": list(starts),
        "seq_len": torch.tensor(wl.seq_lens, dtype=torch.int32, device=device),
        "cur_pos": torch.tensor(cur, dtype=torch.int32, device=device),
        "q_centre": qc, "k_centre": kc,
    }
    if with_calib:
        N = wl.n_calib
        q = torch.empty(L, N, Hq, D, dtype=torch.float32, device=device)
        for l in range(L):
            noise = torch.randn(N, Hq, D, generator=bulk, device=device, dtype=torch.float64)
            q[l] = (qc[l].to(device) + q_scale[l].to(device).view(1, Hq, 1) * noise).to(torch.float32)
        out["q_calib"] = q
    return out


def sample_units(wl: Workload, n: int, seed: int = 1234) -> List[tuple]:
    """A deterministic sample of (layer, kv_head, seq) units that always
    includes the weakest- and the strongest-concentrated KV head."""
    g = torch.Generator().manual_seed(seed)
    nus = [wl.kv_noise(h) for h in range(wl.n_kv_heads)]
    units = {(0, int(max(range(len(nus)), key=lambda h: nus[h])), 0),
             (wl.num_layers - 1, int(min(range(len(nus)), key=lambda h: nus[h])), wl.batch - 1)}
    while len(units) < min(n, wl.num_layers * wl.n_kv_heads * wl.batch):
        l = int(torch.randint(wl.num_layers, (1,), generator=g))
        h = int(torch.randint(wl.n_kv_heads, (1,), generator=g))
        b = int(torch.randint(wl.batch, (1,), generator=g))
        units.add((l, h, b))
    return sorted(units)

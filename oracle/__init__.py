"""CPU oracle for the TriAttention prune step -- TEST INFRASTRUCTURE ONLY.

Thin ctypes marshalling around ``oracle.c`` (plain float64 C, term by term).
Only the tests, the smoke check and the benchmark's CPU-baseline leg may
import this package; the product path never does.

All arrays are numpy, host memory.  Keys and values are bf16 bit patterns
(``uint16``).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

from . import build as _build

NO_TRIG = 1
NO_CONC_WEIGHT = 2

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        _lib = ctypes.CDLL(path)
        P = ctypes.POINTER
        _lib.orc_calibrate.argtypes = [P(ctypes.c_double), ctypes.c_int64, ctypes.c_int64,
                                       ctypes.c_int64, ctypes.c_int64, ctypes.c_int32,
                                       P(ctypes.c_double), P(ctypes.c_double), P(ctypes.c_double)]
        _lib.orc_key_score.argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32,
                                       ctypes.c_int32, ctypes.c_int64]
        _lib.orc_key_score.restype = ctypes.c_double
        _lib.orc_raw_scores.argtypes = [ctypes.c_void_p, P(ctypes.c_double)]
        _lib.orc_raw_scores_folded.argtypes = [ctypes.c_void_p, P(ctypes.c_double)]
        _lib.orc_set_num_threads.argtypes = [ctypes.c_int32]
        _lib.orc_zmax.argtypes = [ctypes.c_void_p, P(ctypes.c_double), P(ctypes.c_double),
                                  P(ctypes.c_double)]
        _lib.orc_select.argtypes = [ctypes.c_void_p, P(ctypes.c_double), P(ctypes.c_int32)]
        _lib.orc_compact.argtypes = [ctypes.c_void_p, P(ctypes.c_int32), P(ctypes.c_uint16),
                                     P(ctypes.c_uint16), P(ctypes.c_int32), P(ctypes.c_int32),
                                     P(ctypes.c_int32)]
        _lib.orc_num_threads.restype = ctypes.c_int32
    return _lib


class _Problem(ctypes.Structure):
    _fields_ = [
        ("L", ctypes.c_int32), ("B", ctypes.c_int32), ("Hq", ctypes.c_int32),
        ("Hkv", ctypes.c_int32), ("D", ctypes.c_int32), ("layout", ctypes.c_int32),
        ("theta", ctypes.c_double), ("budget", ctypes.c_int32), ("n_offsets", ctypes.c_int32),
        ("offsets", ctypes.c_void_p), ("flags", ctypes.c_uint32), ("cap", ctypes.c_int64),
        ("seq_start", ctypes.c_void_p), ("seq_len", ctypes.c_void_p),
        ("cur_pos", ctypes.c_void_p), ("k", ctypes.c_void_p), ("pos", ctypes.c_void_p),
        ("centre", ctypes.c_void_p), ("mean_norm", ctypes.c_void_p), ("mrl", ctypes.c_void_p),
        ("head_budget", ctypes.c_void_p), ("unit_len", ctypes.c_void_p),
    ]


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


class Problem:
    """One prune problem: cache (post-RoPE bf16 keys as uint16, positions,
    segments), calibration statistics and hyper-parameters.  With head-specific
    budgets, `budgets` [L][Hkv] gives each KV head's budget (each <= budget, the
    row length of the selection lists) and `unit_len` [L][Hkv][B] every unit's
    live length (seq_len is then only the fallback when unit_len is None)."""

    def __init__(self, *, k: np.ndarray, pos: np.ndarray, seq_start: Sequence[int],
                 seq_len: Sequence[int], cur_pos: Sequence[int], centre: np.ndarray,
                 mean_norm: np.ndarray, mrl: np.ndarray, theta: float, budget: int,
                 offsets: Sequence[int], n_q_heads: int, layout: int = 0, flags: int = 0,
                 budgets: Optional[np.ndarray] = None, unit_len: Optional[np.ndarray] = None):
        L, Hkv, cap, D = k.shape
        self.k = np.ascontiguousarray(k, dtype=np.uint16)
        self.pos = np.ascontiguousarray(pos, dtype=np.int32)
        self.seq_start = np.ascontiguousarray(seq_start, dtype=np.int64)
        self.seq_len = np.ascontiguousarray(seq_len, dtype=np.int32)
        self.cur_pos = np.ascontiguousarray(cur_pos, dtype=np.int32)
        self.centre = np.ascontiguousarray(centre, dtype=np.float64)
        self.mean_norm = np.ascontiguousarray(mean_norm, dtype=np.float64)
        self.mrl = np.ascontiguousarray(mrl, dtype=np.float64)
        self.offsets = np.ascontiguousarray(offsets, dtype=np.int32)
        self.L, self.Hkv, self.cap, self.D = L, Hkv, cap, D
        self.Hq, self.B, self.budget = n_q_heads, len(self.seq_len), budget
        F = D // 2
        assert self.centre.shape == (L, n_q_heads, F, 2)
        assert self.mean_norm.shape == (L, n_q_heads, F) and self.mrl.shape == (L, n_q_heads, F)
        assert self.pos.shape == (L, Hkv, cap) and len(self.seq_start) == self.B + 1
        self.budgets = (None if budgets is None
                        else np.ascontiguousarray(budgets, dtype=np.int32).reshape(L, Hkv))
        self.unit_len = (None if unit_len is None
                         else np.ascontiguousarray(unit_len, dtype=np.int32).reshape(L, Hkv, self.B))
        if self.budgets is not None:
            assert self.unit_len is not None, "head budgets need per-unit lengths"
            assert np.all((self.budgets >= 1) & (self.budgets <= budget))
        self._s = _Problem(L, self.B, n_q_heads, Hkv, D, layout, float(theta), budget,
                           len(self.offsets), self.offsets.ctypes.data, flags, cap,
                           self.seq_start.ctypes.data, self.seq_len.ctypes.data,
                           self.cur_pos.ctypes.data, self.k.ctypes.data, self.pos.ctypes.data,
                           self.centre.ctypes.data, self.mean_norm.ctypes.data,
                           self.mrl.ctypes.data,
                           None if self.budgets is None else self.budgets.ctypes.data,
                           None if self.unit_len is None else self.unit_len.ctypes.data)

    def unit_lengths(self) -> np.ndarray:
        """[L][Hkv][B] live length of every unit."""
        if self.unit_len is not None:
            return self.unit_len.copy()
        return np.broadcast_to(self.seq_len, (self.L, self.Hkv, self.B)).astype(np.int32).copy()

    def unit_budgets(self) -> np.ndarray:
        """[L][Hkv] budget of every KV head."""
        if self.budgets is not None:
            return self.budgets.copy()
        return np.full((self.L, self.Hkv), self.budget, dtype=np.int32)

    @property
    def ref(self):
        return ctypes.byref(self._s)


def calibrate(q: np.ndarray, layout: int = 0):
    """q: [L][N][Hq][D] pre-RoPE queries -> (centre [L,Hq,F,2], mean_norm, mrl [L,Hq,F])."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    L, N, Hq, D = q.shape
    F = D // 2
    centre = np.zeros((L, Hq, F, 2))
    mean_norm = np.zeros((L, Hq, F))
    mrl = np.zeros((L, Hq, F))
    lib().orc_calibrate(_ptr(q, ctypes.c_double), L, N, Hq, D, layout,
                        _ptr(centre, ctypes.c_double), _ptr(mean_norm, ctypes.c_double),
                        _ptr(mrl, ctypes.c_double))
    return centre, mean_norm, mrl


def key_score(p: Problem, l: int, h: int, b: int, t: int) -> float:
    """Raw score of slot t of sequence b for query head h of layer l."""
    return lib().orc_key_score(p.ref, l, h, b, t)


def raw_scores(p: Problem) -> np.ndarray:
    """[L][Hq][cap] raw scores; NaN outside the live part of each segment."""
    raw = np.full((p.L, p.Hq, p.cap), np.nan)
    lib().orc_raw_scores(p.ref, _ptr(raw, ctypes.c_double))
    return raw


def raw_scores_folded(p: Problem) -> np.ndarray:
    """raw_scores through the angle-addition fold (one weight per head and pair,
    then one pass per key); pinned to raw_scores, timed as a CPU baseline."""
    raw = np.full((p.L, p.Hq, p.cap), np.nan)
    lib().orc_raw_scores_folded(p.ref, _ptr(raw, ctypes.c_double))
    return raw


def prune_folded(p: Problem, v: np.ndarray):
    """prune with the folded raw scores."""
    raw = raw_scores_folded(p)
    z, score = zmax(p, raw)
    sel = select(p, score)
    k2, v2, pos2, sl, ul = compact_units(p, sel, v)
    return {"raw": raw, "z": z, "score": score, "sel": sel, "k": k2, "v": v2, "pos": pos2,
            "seq_len": sl, "unit_len": ul}


def set_num_threads(n: int):
    lib().orc_set_num_threads(int(n))


def zmax(p: Problem, raw: np.ndarray):
    """-> (z [L][Hq][cap], score [L][Hkv][cap]); NaN outside live slots."""
    raw = np.ascontiguousarray(raw, dtype=np.float64)
    z = np.full((p.L, p.Hq, p.cap), np.nan)
    score = np.full((p.L, p.Hkv, p.cap), np.nan)
    lib().orc_zmax(p.ref, _ptr(raw, ctypes.c_double), _ptr(z, ctypes.c_double),
                   _ptr(score, ctypes.c_double))
    return z, score


def select(p: Problem, score: np.ndarray) -> np.ndarray:
    """-> sel [L][Hkv][B][budget] ascending slots within each segment, -1 padded."""
    score = np.ascontiguousarray(score, dtype=np.float64)
    sel = np.empty((p.L, p.Hkv, p.B, p.budget), dtype=np.int32)
    lib().orc_select(p.ref, _ptr(score, ctypes.c_double), _ptr(sel, ctypes.c_int32))
    return sel


def compact_units(p: Problem, sel: np.ndarray, v: np.ndarray):
    """Compacted copies -> (k, v, pos, seq_len, unit_len [L][Hkv][B]); the problem's
    arrays are not modified."""
    sel = np.ascontiguousarray(sel, dtype=np.int32)
    k2 = p.k.copy()
    v2 = np.ascontiguousarray(v, dtype=np.uint16).copy()
    pos2 = p.pos.copy()
    sl = np.empty(p.B, dtype=np.int32)
    ul = np.empty((p.L, p.Hkv, p.B), dtype=np.int32)
    lib().orc_compact(p.ref, _ptr(sel, ctypes.c_int32), _ptr(k2, ctypes.c_uint16),
                      _ptr(v2, ctypes.c_uint16), _ptr(pos2, ctypes.c_int32), _ptr(sl, ctypes.c_int32),
                      _ptr(ul, ctypes.c_int32))
    return k2, v2, pos2, sl, ul


def compact(p: Problem, sel: np.ndarray, v: np.ndarray):
    """Compacted copies -> (k, v, pos, seq_len); the problem's arrays are not modified."""
    return compact_units(p, sel, v)[:4]


def prune(p: Problem, v: np.ndarray):
    """Whole prune step -> dict with raw, z, score, sel and the compacted cache."""
    raw = raw_scores(p)
    z, score = zmax(p, raw)
    sel = select(p, score)
    k2, v2, pos2, sl, ul = compact_units(p, sel, v)
    return {"raw": raw, "z": z, "score": score, "sel": sel, "k": k2, "v": v2, "pos": pos2,
            "seq_len": sl, "unit_len": ul}


def prune_window(p: Problem, v: np.ndarray, window: int):
    """Window-based pruning (dimensionstp.github.io review, section 3-2 (5); in the
    romaanj.github.io review, "Method", a prune round runs once per 128 decoded
    tokens and cuts the cache to the budget): a unit (layer, KV head, sequence) is
    pruned only once its live length reaches its budget + max(window, 1); every
    other unit keeps its cache as it is.  With a single budget all units of a
    sequence share length and budget, so this is decided per sequence.
    Units are independent, so a pruned unit's result is `prune`'s.
    -> `prune`'s dict; the sel rows of the units held back are -2 (not
    selected this call)."""
    out = prune(p, v)
    v0 = np.ascontiguousarray(v, dtype=np.uint16)
    lens, buds = p.unit_lengths(), p.unit_budgets()
    for l in range(p.L):
        for g in range(p.Hkv):
            bud = int(buds[l, g])
            thr = bud + max(int(window), 1)
            for b in range(p.B):
                T = int(lens[l, g, b])
                if T >= thr or T <= bud:
                    continue
                s0, e0 = int(p.seq_start[b]), int(p.seq_start[b + 1])
                out["k"][l, g, s0:e0] = p.k[l, g, s0:e0]
                out["v"][l, g, s0:e0] = v0[l, g, s0:e0]
                out["pos"][l, g, s0:e0] = p.pos[l, g, s0:e0]
                out["unit_len"][l, g, b] = T
                if p.unit_len is None:
                    out["seq_len"][b] = T
                out["sel"][l, g, b] = -2
    return out


def append(k: np.ndarray, v: np.ndarray, pos: np.ndarray, seq_start: Sequence[int],
           seq_len: Sequence[int], cur_pos: Sequence[int], k_new: np.ndarray,
           v_new: np.ndarray, unit_len: Optional[np.ndarray] = None):
    """One decoded token per sequence joins the cache (romaanj.github.io review,
    "Background"): in every (layer, KV head) row, the unit's next slot (its live
    length) in segment b takes the new key and value and the position
    cur_pos[b] + 1; then every unit's length and cur_pos[b] grow by one.  A
    sequence with a unit whose segment has no free slot, or whose length is out of
    range, is left as it is.  Lengths are seq_len[b], shared by the sequence's
    units, or unit_len [L][Hkv][B] when the units differ (head budgets).  k, v:
    uint16 [L][Hkv][cap][D]; k_new, v_new: uint16 [L][Hkv][B][D].  -> copies
    (k, v, pos, lengths, cur_pos) and the list of sequences that were skipped;
    lengths is seq_len, or unit_len when that was given."""
    k, v, pos = k.copy(), v.copy(), pos.copy()
    L, Hkv = k.shape[0], k.shape[1]
    cur_pos = np.array(cur_pos, dtype=np.int32)
    B = len(cur_pos)
    if unit_len is None:
        lens = np.broadcast_to(np.array(seq_len, dtype=np.int32), (L, Hkv, B)).copy()
    else:
        lens = np.array(unit_len, dtype=np.int32).reshape(L, Hkv, B).copy()
    skipped = []
    for b in range(B):
        Ts = lens[:, :, b]
        room = int(seq_start[b + 1]) - int(seq_start[b])
        if (Ts < 0).any() or (Ts >= room).any():
            skipped.append(b)
            continue
        for l in range(L):
            for g in range(Hkv):
                T = int(Ts[l, g])
                slot = int(seq_start[b]) + T
                k[l, g, slot] = k_new[l, g, b]
                v[l, g, slot] = v_new[l, g, b]
                pos[l, g, slot] = cur_pos[b] + 1
        lens[:, :, b] += 1
        cur_pos[b] += 1
    out_len = lens[0, 0].copy() if unit_len is None else lens
    return k, v, pos, out_len, cur_pos, skipped


def decode_attention(k: np.ndarray, v: np.ndarray, seq_start: Sequence[int],
                     seq_len: Sequence[int], layer: int, q: np.ndarray, scale: float,
                     unit_len: Optional[np.ndarray] = None):
    """Decode attention over the (pruned) cache, the step after the prune
    (romaanj.github.io review, "Results": decoding reads the budgeted cache).
    Plain definition in float64: for sequence b and query head h, whose KV head
    is h // G,
        out[b, h] = sum_t softmax_t(scale * q[b, h] . k_t) v_t
    over the live slots t of segment b (t < seq_len[b], or t < unit_len[layer][g][b]
    when units have their own lengths; post-RoPE keys, so positions do not enter).
    The softmax subtracts the largest logit first, which leaves its value
    unchanged.  k, v: uint16 bf16 bits [L][Hkv][cap][D]; q: uint16 [B][Hq][D].
    -> float64 [B][Hq][D]; zeros where a unit is empty."""
    def f64(bits):
        return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)
    B, Hq, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    qf = f64(q)
    out = np.zeros((B, Hq, D))
    if unit_len is None:
        lens = np.broadcast_to(np.array(seq_len, dtype=np.int64), (Hkv, B))
    else:
        lens = np.array(unit_len, dtype=np.int64).reshape(-1, Hkv, B)[layer]
    for b in range(B):
        s0 = int(seq_start[b])
        for h in range(Hq):
            g = h // G
            T = int(lens[g, b])
            if T == 0:
                continue
            K = f64(k[layer, g, s0:s0 + T])
            V = f64(v[layer, g, s0:s0 + T])
            logits = scale * (K @ qf[b, h])
            w = np.exp(logits - logits.max())
            out[b, h] = (w / w.sum()) @ V
    return out


def num_threads() -> int:
    return int(lib().orc_num_threads())

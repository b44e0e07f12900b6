"""ctypes binding of libtria (include/tria.h), same names as the C ABI.

Argument marshalling only: every step of the prune runs in the library's CUDA
kernels.  PyTorch supplies device memory and streams.  If the library is not
built, or no CUDA device is present, the calls raise; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtria.so")

OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED = 2
ERR_WORKSPACE = 3
ERR_CUDA = 4
ERR_DEVICE_FLAG = 5

ROPE_HALF_SPLIT = 0
ROPE_INTERLEAVED = 1
NO_TRIG = 1
NO_CONC_WEIGHT = 2
FUSED_PRUNE = 4
DTYPE_F32 = 0
DTYPE_BF16 = 1
MAX_BATCH = 256
MAX_OFFSETS = 4096
MAX_SEGMENT = 1 << 18
PRUNE_MAX_STAGES = 8
NOALLOC_SCRATCH_BYTES = 16 << 20

DEVERR_SEQ_LEN = 1
DEVERR_SELECTION = 2
DEVERR_TIMEOUT = 4
DEVERR_SEGMENT_BIG = 8
DEVERR_SEGMENT_FULL = 16
DEVERR_BUDGET = 32

EXPORTS = ["tria_workspace_size", "tria_workspace_init", "tria_calibrate", "tria_score",
           "tria_select", "tria_compact", "tria_prune", "tria_prune_profiled",
           "tria_prune_stage_name", "tria_get_device_error", "tria_status_string", "tria_version",
           "tria_prune_noalloc", "tria_append", "tria_decode_attention"]


class TriaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


class tria_config(ctypes.Structure):
    _fields_ = [("num_layers", ctypes.c_int32), ("batch", ctypes.c_int32),
                ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("rope_theta", ctypes.c_double),
                ("rope_layout", ctypes.c_int32), ("budget", ctypes.c_int32),
                ("offsets", ctypes.POINTER(ctypes.c_int32)), ("n_offsets", ctypes.c_int32),
                ("flags", ctypes.c_uint32), ("prune_window", ctypes.c_int32),
                ("head_budgets", ctypes.c_void_p)]


class tria_cache(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("pos", ctypes.c_void_p),
                ("seq_len", ctypes.c_void_p), ("cur_pos", ctypes.c_void_p),
                ("seq_start", ctypes.POINTER(ctypes.c_int64)), ("cap_total", ctypes.c_int64),
                ("unit_len", ctypes.c_void_p)]


class tria_stats(ctypes.Structure):
    _fields_ = [("centre", ctypes.c_void_p), ("mean_norm", ctypes.c_void_p),
                ("mrl", ctypes.c_void_p)]


_lib = None


def lib():
    """The loaded libtria; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with __graft_entry__.build() "
                               "(nvcc, sm_100a); there is no fallback path")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER
        vp = ctypes.c_void_p
        L.tria_workspace_size.argtypes = [P(tria_config), P(tria_cache), P(ctypes.c_size_t)]
        L.tria_workspace_init.argtypes = [vp, ctypes.c_size_t, vp]
        L.tria_calibrate.argtypes = [P(tria_config), vp, ctypes.c_int32, ctypes.c_int64, vp, vp,
                                     vp, vp]
        L.tria_score.argtypes = [P(tria_config), P(tria_stats), P(tria_cache), vp, vp, vp,
                                 ctypes.c_size_t, vp]
        L.tria_select.argtypes = [P(tria_config), P(tria_cache), vp, vp, vp, ctypes.c_size_t, vp]
        L.tria_compact.argtypes = [P(tria_config), P(tria_cache), vp, vp, ctypes.c_size_t, vp]
        L.tria_prune.argtypes = [P(tria_config), P(tria_stats), P(tria_cache), vp, vp,
                                 ctypes.c_size_t, vp]
        L.tria_prune_profiled.argtypes = [P(tria_config), P(tria_stats), P(tria_cache), vp, vp,
                                          ctypes.c_size_t, vp, P(vp), P(ctypes.c_int32),
                                          P(ctypes.c_int32)]
        L.tria_prune_noalloc.argtypes = [P(tria_config), P(tria_stats), P(tria_cache), vp, vp,
                                         vp]
        L.tria_append.argtypes = [P(tria_config), P(tria_cache), vp, vp, vp, ctypes.c_size_t, vp]
        L.tria_decode_attention.argtypes = [P(tria_config), P(tria_cache), ctypes.c_int32, vp,
                                            ctypes.c_float, vp, vp, ctypes.c_size_t, vp]
        L.tria_prune_stage_name.argtypes = [ctypes.c_int32]
        L.tria_prune_stage_name.restype = ctypes.c_char_p
        L.tria_get_device_error.argtypes = [vp, P(ctypes.c_int32), vp]
        L.tria_status_string.argtypes = [ctypes.c_int]
        L.tria_status_string.restype = ctypes.c_char_p
        L.tria_version.restype = ctypes.c_char_p
        for name in EXPORTS:
            if name not in ("tria_prune_stage_name", "tria_status_string", "tria_version"):
                getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().tria_status_string(status).decode()


def _check(status: int, where: str):
    if status != OK:
        raise TriaError(status, where)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libtria takes CUDA tensors for device arguments")
    if not t.is_contiguous():
        raise ValueError("libtria takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


class Config:
    """tria_config plus the host offsets array it points to."""

    def __init__(self, *, num_layers: int, batch: int, n_q_heads: int, n_kv_heads: int,
                 head_dim: int, rope_theta: float, budget: int, offsets: Sequence[int],
                 rope_layout: int = ROPE_HALF_SPLIT, flags: int = 0, prune_window: int = 0,
                 head_budgets: Optional[torch.Tensor] = None):
        """head_budgets: int32 [L][Hkv] device tensor of per-head budgets (each <= budget),
        or None for the single budget."""
        self._offsets = (ctypes.c_int32 * max(1, len(offsets)))(*offsets)
        self.head_budgets = head_budgets
        self.c = tria_config(num_layers, batch, n_q_heads, n_kv_heads, head_dim,
                             float(rope_theta), rope_layout, budget,
                             ctypes.cast(self._offsets, ctypes.POINTER(ctypes.c_int32)),
                             len(offsets), flags, prune_window, _ptr(head_budgets))

    @classmethod
    def from_workload(cls, wl, flags: int = 0, prune_window: int = 0,
                      head_budgets: Optional[torch.Tensor] = None) -> "Config":
        return cls(num_layers=wl.num_layers, batch=wl.batch, n_q_heads=wl.n_q_heads,
                   n_kv_heads=wl.n_kv_heads, head_dim=wl.head_dim, rope_theta=wl.rope_theta,
                   budget=wl.budget, offsets=wl.offsets, rope_layout=wl.rope_layout, flags=flags,
                   prune_window=prune_window, head_budgets=head_budgets)


class Cache:
    """tria_cache over torch tensors (k, v bf16 [L][Hkv][cap][D]; pos int32 [L][Hkv][cap];
    seq_len, cur_pos int32 [B] on the device; seq_start a host list of B+1 ints;
    optionally unit_len int32 [L][Hkv][B], the per-unit live lengths)."""

    def __init__(self, k, v, pos, seq_len, cur_pos, seq_start: Sequence[int],
                 cap_total: Optional[int] = None, unit_len=None):
        self.tensors = (k, v, pos, seq_len, cur_pos, unit_len)
        self._starts = (ctypes.c_int64 * len(seq_start))(*seq_start)
        cap = cap_total if cap_total is not None else (k.shape[2] if k is not None else 0)
        self.c = tria_cache(_ptr(k), _ptr(v), _ptr(pos), _ptr(seq_len), _ptr(cur_pos),
                            ctypes.cast(self._starts, ctypes.POINTER(ctypes.c_int64)), cap,
                            _ptr(unit_len))

    @classmethod
    def from_data(cls, data: dict) -> "Cache":
        return cls(data["k"], data["v"], data["pos"], data["seq_len"], data["cur_pos"],
                   data["seq_start"])


class Stats:
    """tria_stats over float32 device tensors centre [L][Hq][F][2], mean_norm, mrl [L][Hq][F]."""

    def __init__(self, centre, mean_norm, mrl):
        self.tensors = (centre, mean_norm, mrl)
        self.c = tria_stats(_ptr(centre), _ptr(mean_norm), _ptr(mrl))


def tria_workspace_size(cfg: Config, cache: Cache) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().tria_workspace_size(ctypes.byref(cfg.c), ctypes.byref(cache.c), ctypes.byref(n)),
           "tria_workspace_size")
    return int(n.value)


def workspace(cfg: Config, cache: Cache, device=None, stream=None) -> torch.Tensor:
    """Allocates (with torch) and initialises a workspace for this problem."""
    n = tria_workspace_size(cfg, cache)
    ws = torch.empty(n + 256, dtype=torch.uint8, device=device or "cuda")
    off = (-ws.data_ptr()) % 256
    ws = ws[off:off + n]
    tria_workspace_init(ws, stream)
    return ws


def tria_workspace_init(ws: torch.Tensor, stream=None):
    _check(lib().tria_workspace_init(_ptr(ws), ws.numel(), _stream(stream)), "tria_workspace_init")


def tria_calibrate(cfg: Config, q_pre: torch.Tensor, centre, mean_norm, mrl, stream=None):
    dtype = {torch.float32: DTYPE_F32, torch.bfloat16: DTYPE_BF16}[q_pre.dtype]
    _check(lib().tria_calibrate(ctypes.byref(cfg.c), _ptr(q_pre), dtype, q_pre.shape[1],
                                _ptr(centre), _ptr(mean_norm), _ptr(mrl), _stream(stream)),
           "tria_calibrate")


def calibrate(cfg: Config, q_pre: torch.Tensor, stream=None) -> Stats:
    L, N, Hq, D = q_pre.shape
    F = D // 2
    centre = torch.empty(L, Hq, F, 2, dtype=torch.float32, device=q_pre.device)
    mean_norm = torch.empty(L, Hq, F, dtype=torch.float32, device=q_pre.device)
    mrl = torch.empty(L, Hq, F, dtype=torch.float32, device=q_pre.device)
    tria_calibrate(cfg, q_pre, centre, mean_norm, mrl, stream)
    return Stats(centre, mean_norm, mrl)


def tria_score(cfg: Config, stats: Stats, cache: Cache, score: torch.Tensor,
               raw: Optional[torch.Tensor], ws: torch.Tensor, stream=None):
    _check(lib().tria_score(ctypes.byref(cfg.c), ctypes.byref(stats.c), ctypes.byref(cache.c),
                            _ptr(score), _ptr(raw), _ptr(ws), ws.numel(), _stream(stream)),
           "tria_score")


def tria_select(cfg: Config, cache: Cache, score: torch.Tensor, sel: torch.Tensor,
                ws: torch.Tensor, stream=None):
    _check(lib().tria_select(ctypes.byref(cfg.c), ctypes.byref(cache.c), _ptr(score), _ptr(sel),
                             _ptr(ws), ws.numel(), _stream(stream)), "tria_select")


def tria_compact(cfg: Config, cache: Cache, sel: torch.Tensor, ws: torch.Tensor, stream=None):
    _check(lib().tria_compact(ctypes.byref(cfg.c), ctypes.byref(cache.c), _ptr(sel), _ptr(ws),
                              ws.numel(), _stream(stream)), "tria_compact")


def tria_prune(cfg: Config, stats: Stats, cache: Cache, ws: torch.Tensor,
               sel_out: Optional[torch.Tensor] = None, stream=None):
    _check(lib().tria_prune(ctypes.byref(cfg.c), ctypes.byref(stats.c), ctypes.byref(cache.c),
                            _ptr(sel_out), _ptr(ws), ws.numel(), _stream(stream)), "tria_prune")


def tria_append(cfg: Config, cache: Cache, k_new: torch.Tensor, v_new: torch.Tensor,
                ws: torch.Tensor, stream=None):
    """k_new, v_new: bf16 [L][Hkv][B][D] device tensors, one new token per sequence."""
    _check(lib().tria_append(ctypes.byref(cfg.c), ctypes.byref(cache.c), _ptr(k_new),
                             _ptr(v_new), _ptr(ws), ws.numel(), _stream(stream)), "tria_append")


def tria_decode_attention(cfg: Config, cache: Cache, layer: int, q: torch.Tensor,
                          out: torch.Tensor, ws: torch.Tensor, scale: Optional[float] = None,
                          stream=None):
    """q: bf16 [B][Hq][D], out: float32 [B][Hq][D] device tensors; scale None (or
    <= 0) lets the library use 1/sqrt(D)."""
    if scale is None:
        scale = 0.0
    _check(lib().tria_decode_attention(ctypes.byref(cfg.c), ctypes.byref(cache.c), layer,
                                       _ptr(q), ctypes.c_float(scale), _ptr(out), _ptr(ws),
                                       ws.numel(), _stream(stream)), "tria_decode_attention")


def tria_prune_profiled(cfg: Config, stats: Stats, cache: Cache, ws: torch.Tensor, events,
                        sel_out: Optional[torch.Tensor] = None, stream=None):
    """events: PRUNE_MAX_STAGES + 1 torch.cuda.Event(enable_timing=True).
    Returns the kernel name of each stage (stage i runs between events i and i+1)."""
    for e in events:
        if not e.cuda_event:  # torch creates the CUDA event on its first record
            e.record(stream if stream is not None else torch.cuda.current_stream())
    arr = (ctypes.c_void_p * (PRUNE_MAX_STAGES + 1))(
        *[ctypes.c_void_p(e.cuda_event) for e in events])
    n = ctypes.c_int32(0)
    ids = (ctypes.c_int32 * PRUNE_MAX_STAGES)()
    _check(lib().tria_prune_profiled(ctypes.byref(cfg.c), ctypes.byref(stats.c),
                                     ctypes.byref(cache.c), _ptr(sel_out), _ptr(ws), ws.numel(),
                                     _stream(stream), arr, ctypes.byref(n), ids),
           "tria_prune_profiled")
    return [tria_prune_stage_name(ids[i]) for i in range(n.value)]


def tria_prune_noalloc(cfg: Config, stats: Stats, cache: Cache,
                       sel_out: Optional[torch.Tensor] = None,
                       device_error: Optional[torch.Tensor] = None, stream=None):
    """tria_prune without a workspace argument: the library's fixed device
    scratch array stands in for it (see include/tria.h).  device_error, if
    given, is an int32 device tensor of one element that receives the call's
    device error word."""
    _check(lib().tria_prune_noalloc(ctypes.byref(cfg.c), ctypes.byref(stats.c),
                                    ctypes.byref(cache.c), _ptr(sel_out), _ptr(device_error),
                                    _stream(stream)), "tria_prune_noalloc")


def tria_prune_stage_name(i: int) -> str:
    return lib().tria_prune_stage_name(i).decode()


def tria_get_device_error(ws: torch.Tensor, stream=None) -> int:
    code = ctypes.c_int32(0)
    st = lib().tria_get_device_error(_ptr(ws), ctypes.byref(code), _stream(stream))
    if st not in (OK, ERR_DEVICE_FLAG):
        raise TriaError(st, "tria_get_device_error")
    return int(code.value)


def tria_version() -> str:
    return lib().tria_version().decode()

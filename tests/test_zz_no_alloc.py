"""tria_prune_noalloc: the prune step with the library's fixed device scratch
array in place of a caller-allocated workspace.

It runs the same kernels as tria_prune on the same inputs, and those kernels
reduce in a fixed order, so the tolerance against tria_prune is zero: the
selection lists, the compacted K/V/pos rows and seq_len must be identical.
Consecutive calls share the scratch array, so each comparison follows a call
on a different problem, and the error word must not leak from one call into
the next.  The file is named to be collected last.
"""
import ctypes

import pytest
import torch

from kv_cache_eviction_trig_b200 import tria, workloads


def _small(name, **kw):
    d = dict(L=1, B=2, Hq=8, Hkv=2, D=128, theta=1e6, budget=100, offsets=range(1, 65),
             seq_lens=[1000, 333], seed=23, n_calib=128, slack=37)
    d.update(kw)
    return workloads.custom(name, **d)


class Pair:
    """One drawn problem, twice: a copy for tria_prune and one for tria_prune_noalloc."""

    def __init__(self, wl, seq_len=None):
        data = workloads.generate(wl, device="cuda")
        if seq_len is not None:
            data["seq_len"] = torch.tensor(seq_len, dtype=torch.int32, device="cuda")
        self.wl = wl
        self.cfg = tria.Config.from_workload(wl)
        self.stats = tria.calibrate(self.cfg, data["q_calib"])
        self.copies = []
        for _ in range(2):
            d = dict(data)
            for n in ("k", "v", "pos", "seq_len"):
                d[n] = data[n].clone()
            self.copies.append(d)
        self.caches = [tria.Cache.from_data(d) for d in self.copies]

    def sel(self):
        wl = self.wl
        return torch.full((wl.num_layers, wl.n_kv_heads, wl.batch, wl.budget), -7,
                          dtype=torch.int32, device="cuda")

    def run(self):
        """tria_prune on copy 0, tria_prune_noalloc on copy 1; returns both
        selections and both device error words."""
        ws = tria.workspace(self.cfg, self.caches[0])
        sel_ref, sel_na = self.sel(), self.sel()
        err_na = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        tria.tria_prune(self.cfg, self.stats, self.caches[0], ws, sel_out=sel_ref)
        tria.tria_prune_noalloc(self.cfg, self.stats, self.caches[1], sel_out=sel_na,
                                device_error=err_na)
        torch.cuda.synchronize()
        return sel_ref, sel_na, tria.tria_get_device_error(ws), int(err_na.item())

    def assert_same_cache(self):
        a, b = self.copies
        for n in ("k", "v", "pos"):
            assert torch.equal(a[n].view(torch.int16) if a[n].dtype == torch.bfloat16 else a[n],
                               b[n].view(torch.int16) if b[n].dtype == torch.bfloat16 else b[n]), n
        assert torch.equal(a["seq_len"], b["seq_len"])


@pytest.mark.gpu
def test_prune_noalloc_matches_prune_on_consecutive_calls():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from kv_cache_eviction_trig_b200 import build
    build.build()
    problems = [
        _small("noalloc-ragged"),
        workloads.workload(1),          # one 8B-shaped layer at 32K keys, about 4.4 MB of scratch
        _small("noalloc-two-layers", L=2, B=3, seq_lens=[129, 400, 90], budget=128,
               offsets=range(1, 33), seed=5),
    ]
    for wl in problems:
        pair = Pair(wl)
        sel_ref, sel_na, err_ref, err_na = pair.run()
        assert err_ref == 0 and err_na == 0, wl.name
        assert torch.equal(sel_ref, sel_na), wl.name
        pair.assert_same_cache()
        kept = [min(t, wl.budget) for t in wl.seq_lens]
        assert pair.copies[1]["seq_len"].cpu().tolist() == kept


@pytest.mark.gpu
def test_prune_noalloc_error_word_is_per_call():
    """A device error raised by one call is reported by that call only."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from kv_cache_eviction_trig_b200 import build
    build.build()
    bad = Pair(_small("noalloc-overflow", seq_lens=[300, 300], budget=50, slack=0),
               seq_len=[300, 301])            # sequence 1 claims more than its segment
    sel_ref, sel_na, err_ref, err_na = bad.run()
    assert err_ref & tria.DEVERR_SEQ_LEN and err_na == err_ref
    assert torch.equal(sel_ref, sel_na)
    bad.assert_same_cache()
    good = Pair(_small("noalloc-after-error"))
    sel_ref, sel_na, err_ref, err_na = good.run()
    assert err_ref == 0 and err_na == 0
    assert torch.equal(sel_ref, sel_na)
    good.assert_same_cache()


def test_prune_noalloc_rejects_problems_beyond_its_scratch():
    """Checked on the host before any CUDA call (fake, never dereferenced pointers)."""
    from kv_cache_eviction_trig_b200 import build
    build.build()
    L = tria.lib()
    fake = 0x7f0000000000

    keep = []

    def cache(seq_start, cap):
        starts = (ctypes.c_int64 * len(seq_start))(*seq_start)
        keep.append(starts)
        return tria.tria_cache(fake, fake + 0x10000000, fake + 0x20000000, fake + 0x30000000,
                               fake + 0x30000100,
                               ctypes.cast(starts, ctypes.POINTER(ctypes.c_int64)), cap)

    def call(cfg, seq_start, cap, device_error=None):
        stats = tria.tria_stats(fake + 0x40000000, fake + 0x50000000, fake + 0x60000000)
        return L.tria_prune_noalloc(ctypes.byref(cfg.c), ctypes.byref(stats),
                                    ctypes.byref(cache(seq_start, cap)), None, device_error, None)

    def need(cfg, seq_start, cap):
        n = ctypes.c_size_t(0)
        assert L.tria_workspace_size(ctypes.byref(cfg.c), ctypes.byref(cache(seq_start, cap)),
                                     ctypes.byref(n)) == tria.OK
        return n.value

    cfg = tria.Config(num_layers=2, batch=2, n_q_heads=8, n_kv_heads=2, head_dim=128,
                      rope_theta=1e6, budget=64, offsets=list(range(1, 9)))
    big = [0, 200000, 400000]            # raw scores alone: 2 * 8 * 400000 * 4 bytes = 25.6 MB
    assert need(cfg, big, 400000) > tria.NOALLOC_SCRATCH_BYTES
    assert call(cfg, big, 400000) == tria.ERR_UNSUPPORTED
    small = [0, 1000, 2000]
    assert need(cfg, small, 2000) <= tria.NOALLOC_SCRATCH_BYTES
    assert call(cfg, small, 2000, ctypes.c_void_p(fake + 2)) == tria.ERR_INVALID_ARG
    bad_cfg = tria.Config(num_layers=0, batch=2, n_q_heads=8, n_kv_heads=2, head_dim=128,
                          rope_theta=1e6, budget=64, offsets=[1])
    assert call(bad_cfg, small, 2000) == tria.ERR_INVALID_ARG


@pytest.mark.gpu
def test_prune_noalloc_second_call_reserves_no_device_memory():
    """The scratch array is loaded by the first call on a device; after that a call
    takes no device memory: free memory is the same before and after it."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from kv_cache_eviction_trig_b200 import build
    build.build()
    pair = Pair(_small("noalloc-memory"))
    sel = pair.sel()
    err = torch.zeros((1,), dtype=torch.int32, device="cuda")
    tria.tria_prune_noalloc(pair.cfg, pair.stats, pair.caches[1], sel_out=sel, device_error=err)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        tria.tria_prune_noalloc(pair.cfg, pair.stats, pair.caches[1], sel_out=sel,
                                device_error=err)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert int(err.item()) == 0
    assert free1 == free0

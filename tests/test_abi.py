"""The C ABI without a GPU: the library builds, loads, exports every entry
point include/tria.h declares, sizes workspaces, and rejects bad arguments
synchronously (before any CUDA call)."""
import ctypes
import os
import re

import pytest

from kv_cache_eviction_trig_b200 import build as tbuild
from kv_cache_eviction_trig_b200 import tria

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tria.h")


@pytest.fixture(scope="module")
def L():
    tbuild.build()
    return tria.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(tria_[a-z_0-9]+)\s*\(",
                                 text, flags=re.M)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert "tria_prune" in names and "tria_score" in names and len(names) >= 12
    for n in names:
        assert hasattr(L, n), f"{n} declared in tria.h but not exported"
    assert set(names) == set(tria.EXPORTS)


def test_header_constants_match_binding():
    text = open(HEADER).read()
    consts = dict(re.findall(r"#define (TRIA_[A-Z_0-9]+) \(?([0-9a-fx<\s]+?)u?\)?\s*(?:/\*|$)",
                             text, flags=re.M))
    assert eval(consts["TRIA_MAX_SEGMENT"]) == tria.MAX_SEGMENT
    assert int(consts["TRIA_MAX_BATCH"]) == tria.MAX_BATCH
    assert int(consts["TRIA_MAX_OFFSETS"]) == tria.MAX_OFFSETS
    assert int(consts["TRIA_NO_TRIG"]) == tria.NO_TRIG
    assert int(consts["TRIA_NO_CONC_WEIGHT"]) == tria.NO_CONC_WEIGHT
    assert int(consts["TRIA_PRUNE_MAX_STAGES"]) == tria.PRUNE_MAX_STAGES
    assert eval(consts["TRIA_NOALLOC_SCRATCH_BYTES"]) == tria.NOALLOC_SCRATCH_BYTES


def test_status_strings(L):
    for s, name in [(0, "TRIA_OK"), (1, "TRIA_ERR_INVALID_ARG"), (2, "TRIA_ERR_UNSUPPORTED"),
                    (3, "TRIA_ERR_WORKSPACE"), (4, "TRIA_ERR_CUDA"), (5, "TRIA_ERR_DEVICE_FLAG")]:
        assert tria.status_string(s) == name
    assert tria.tria_prune_stage_name(1) == "score_kernel"
    assert tria.tria_prune_stage_name(99) == ""


# ---------------------------------------------------------------- fake (never dereferenced) args

FAKE = 0x7f0000000000  # 256-aligned; validation fails before any pointer is used


def _cfg(**kw):
    d = dict(num_layers=1, batch=2, n_q_heads=8, n_kv_heads=2, head_dim=128, rope_theta=1e6,
             budget=64, offsets=list(range(1, 9)))
    d.update(kw)
    return tria.Config(**d)


def _cache(seq_start=(0, 100, 300), cap=300, k=FAKE, v=FAKE + 0x100000, pos=FAKE + 0x200000,
           seq_len=FAKE + 0x300000, cur=FAKE + 0x300100):
    c = tria.Cache.__new__(tria.Cache)
    c._starts = (ctypes.c_int64 * len(seq_start))(*seq_start)
    c.c = tria.tria_cache(k, v, pos, seq_len, cur,
                          ctypes.cast(c._starts, ctypes.POINTER(ctypes.c_int64)), cap)
    return c


def _stats(centre=FAKE + 0x400000, mean=FAKE + 0x500000, mrl=FAKE + 0x600000):
    s = tria.Stats.__new__(tria.Stats)
    s.c = tria.tria_stats(centre, mean, mrl)
    return s


def _prune(L, cfg, cache, stats=None, ws=FAKE + 0x1000000, ws_bytes=1 << 40):
    stats = stats or _stats()
    return L.tria_prune(ctypes.byref(cfg.c), ctypes.byref(stats.c), ctypes.byref(cache.c), None,
                        ctypes.c_void_p(ws), ws_bytes, None)


def test_workspace_size(L):
    cfg, cache = _cfg(), _cache()
    n = tria.tria_workspace_size(cfg, cache)
    F = 64
    need = 4 * 1 * 8 * 300 + 16 * 2 * F + 4 * 1 * 2 * 2 * 64   # raw + ea + sel at least
    assert n >= need and n % 256 == 0
    bigger = tria.tria_workspace_size(cfg, _cache(seq_start=(0, 100, 3000), cap=3000))
    assert bigger > n


@pytest.mark.parametrize("mutate,status", [
    (dict(num_layers=0), tria.ERR_INVALID_ARG),
    (dict(n_q_heads=7), tria.ERR_INVALID_ARG),           # not a multiple of Hkv
    (dict(head_dim=96), tria.ERR_UNSUPPORTED),
    (dict(n_q_heads=64), tria.ERR_UNSUPPORTED),          # G = 32
    (dict(budget=0), tria.ERR_INVALID_ARG),
    (dict(rope_theta=1.0), tria.ERR_INVALID_ARG),
    (dict(offsets=[1, 0, 3]), tria.ERR_INVALID_ARG),
    (dict(offsets=[]), tria.ERR_INVALID_ARG),
    (dict(offsets=list(range(1, 5000))), tria.ERR_UNSUPPORTED),
    (dict(rope_layout=2), tria.ERR_INVALID_ARG),
    (dict(flags=8), tria.ERR_INVALID_ARG),      # an unknown flag bit
    (dict(batch=300), tria.ERR_UNSUPPORTED),
    (dict(prune_window=-1), tria.ERR_INVALID_ARG),
])
def test_bad_config_rejected_before_launch(L, mutate, status):
    cfg = _cfg(**mutate)
    b = cfg.c.batch
    starts = tuple(range(0, 100 * (b + 1), 100))
    assert _prune(L, cfg, _cache(seq_start=starts, cap=100 * b)) == status


def test_bad_cache_and_workspace_rejected(L):
    cfg = _cfg()
    assert _prune(L, cfg, _cache(k=FAKE + 8)) == tria.ERR_INVALID_ARG          # misaligned K
    assert _prune(L, cfg, _cache(pos=0)) == tria.ERR_INVALID_ARG               # null pos
    assert _prune(L, cfg, _cache(seq_start=(0, 200, 100))) == tria.ERR_INVALID_ARG  # decreasing
    assert _prune(L, cfg, _cache(seq_start=(0, 100, 400))) == tria.ERR_INVALID_ARG  # > cap_total
    assert _prune(L, cfg, _cache(seq_start=(0, 1, 300000), cap=300000)) == tria.ERR_UNSUPPORTED
    assert _prune(L, cfg, _cache(), stats=_stats(centre=0)) == tria.ERR_INVALID_ARG
    assert _prune(L, cfg, _cache(), ws=FAKE + 16) == tria.ERR_WORKSPACE        # misaligned ws
    assert _prune(L, cfg, _cache(), ws_bytes=1000) == tria.ERR_WORKSPACE       # too small
    assert _prune(L, cfg, _cache(), ws=0) == tria.ERR_WORKSPACE


def test_select_and_compact_reject_bad_args(L):
    cfg, cache = _cfg(), _cache()
    ws = ctypes.c_void_p(FAKE + 0x1000000)
    assert L.tria_select(ctypes.byref(cfg.c), ctypes.byref(cache.c), None,
                         ctypes.c_void_p(FAKE), ws, 1 << 40, None) == tria.ERR_INVALID_ARG
    assert L.tria_compact(ctypes.byref(cfg.c), ctypes.byref(cache.c), None, ws, 1 << 40,
                          None) == tria.ERR_INVALID_ARG
    no_v = _cache(v=0)
    assert L.tria_compact(ctypes.byref(cfg.c), ctypes.byref(no_v.c), ctypes.c_void_p(FAKE), ws,
                          1 << 40, None) == tria.ERR_INVALID_ARG
    assert L.tria_calibrate(ctypes.byref(cfg.c), None, 0, 10, ctypes.c_void_p(FAKE),
                            ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), None) == tria.ERR_INVALID_ARG
    assert L.tria_calibrate(ctypes.byref(cfg.c), ctypes.c_void_p(FAKE), 7, 10,
                            ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE),
                            None) == tria.ERR_INVALID_ARG


def test_append_rejects_bad_args(L):
    cfg, cache = _cfg(), _cache()
    ws = ctypes.c_void_p(FAKE + 0x1000000)
    kn, vn = ctypes.c_void_p(FAKE + 0x700000), ctypes.c_void_p(FAKE + 0x800000)

    def app(cfg=cfg, cache=cache, kn=kn, vn=vn, ws=ws, ws_bytes=1 << 40):
        return L.tria_append(ctypes.byref(cfg.c), ctypes.byref(cache.c), kn, vn, ws, ws_bytes,
                             None)

    assert app(kn=None) == tria.ERR_INVALID_ARG
    assert app(vn=ctypes.c_void_p(FAKE + 0x800008)) == tria.ERR_INVALID_ARG  # misaligned
    assert app(cache=_cache(cur=0)) == tria.ERR_INVALID_ARG                  # no cur_pos
    assert app(cache=_cache(v=0)) == tria.ERR_INVALID_ARG
    assert app(cfg=_cfg(prune_window=-5)) == tria.ERR_INVALID_ARG
    assert app(cfg=_cfg(head_dim=100)) == tria.ERR_UNSUPPORTED               # not a multiple of 8
    assert app(ws_bytes=1000) == tria.ERR_WORKSPACE


def test_decode_attention_rejects_bad_args(L):
    cfg, cache = _cfg(), _cache()
    ws = ctypes.c_void_p(FAKE + 0x1000000)
    q, out = ctypes.c_void_p(FAKE + 0x700000), ctypes.c_void_p(FAKE + 0x800000)

    def att(cfg=cfg, cache=cache, layer=0, q=q, scale=0.1, out=out, ws_bytes=1 << 40):
        return L.tria_decode_attention(ctypes.byref(cfg.c), ctypes.byref(cache.c), layer, q,
                                       ctypes.c_float(scale), out, ws, ws_bytes, None)

    assert att(layer=1) == tria.ERR_INVALID_ARG                    # one layer only
    assert att(layer=-1) == tria.ERR_INVALID_ARG
    assert att(q=ctypes.c_void_p(FAKE + 0x700002)) == tria.ERR_INVALID_ARG  # misaligned
    assert att(out=None) == tria.ERR_INVALID_ARG
    assert att(scale=float("inf")) == tria.ERR_INVALID_ARG
    assert att(cache=_cache(v=0)) == tria.ERR_INVALID_ARG
    assert att(cfg=_cfg(head_dim=96)) == tria.ERR_UNSUPPORTED      # no kernel for D = 96
    assert att(ws_bytes=1000) == tria.ERR_WORKSPACE


def test_config_struct_matches_header():
    """The binding's tria_config has the header's fields in the header's order."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    body = re.search(r"typedef struct \{(.*?)\} tria_config;", text, flags=re.S).group(1)
    names = re.findall(r"([a-z_]+)\s*;", body)
    assert names == [f[0] for f in tria.tria_config._fields_]


def test_binding_refuses_host_tensors():
    import torch
    cfg = _cfg()
    with pytest.raises(ValueError):
        tria.Cache(torch.zeros(1, 2, 4, 128, dtype=torch.bfloat16), None, None, None, None,
                   [0, 4])


def test_product_path_has_no_oracle_or_fallback():
    """The package never imports the oracle and has no CPU scoring path."""
    pkg = os.path.join(ROOT, "kv_cache_eviction_trig_b200")
    for fn in os.listdir(pkg):
        if fn.endswith(".py"):
            src = open(os.path.join(pkg, fn)).read()
            assert "import oracle" not in src and "from oracle" not in src, fn


def test_every_declaration_cites_its_passage():
    """Each entry point in tria.h is preceded by a comment that cites the passage
    of the pages it follows (a review's page and section), or says that the
    paper has no counterpart."""
    text = open(HEADER).read()
    cite = re.compile(r"(romaanj|dimensionstp)\.github\.io[\s*]+review|no[\s*]+counterpart[\s*]+in[\s*]+the[\s*]+paper")
    for name in declared_functions():
        m = re.search(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*" + name + r"\s*\(", text, flags=re.M)
        assert m, name
        before = text[:m.start()]
        # the last comment block before the declaration (#define lines may sit between)
        end = before.rfind("*/")
        start = before.rfind("/*", 0, end)
        between = before[end + 2:]
        assert all(line.strip() == "" or line.strip().startswith("#define")
                   for line in between.splitlines()), name
        assert cite.search(before[start:end]), f"{name}: no passage cited"


def test_attention_scale_default_lives_in_the_library():
    """tria.py passes scale 0 when none is given; the C call picks 1/sqrt(D)."""
    import inspect
    src = inspect.getsource(tria.tria_decode_attention).split('"""')[-1]  # code, not docstring
    assert "sqrt" not in src and "** -0.5" not in src and "head_dim" not in src
    assert "TRIA_LIB" not in open(tria.__file__).read()

"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Tolerances (float32 accumulation over exact bf16 inputs):
  raw score   |s_gpu - s_ref| <= 1e-4 * max(|s_ref|, rms(s_ref over the sequence));
  z / score   |z_gpu - z_ref| <= 1e-4 * (2 + |z_ref|) * max_h rms_h / sigma_h, which is
              the 1e-4 relative raw tolerance carried through (s - mu) / sigma: an error
              of e*rms in s moves z by e*rms/sigma, and mu and sigma carry the same
              relative error (the 2 + |z| term).  Where rms_h/sigma_h is large (a head
              whose scores vary little around a large mean) this is wider than
              1e-4 * max(1, |z|); every check prints the factor and the largest
              |dz| / max(1, |z|) it saw, so the widening is on record;
  selection   same index set, except keys whose oracle score lies within that
              tolerance of the budget-th oracle score; ties go to the lower slot;
  compaction  bit-exact given the selection; selection on identical score
              values bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_eviction_trig_b200 import tria, workloads
from tests import common

pytestmark = pytest.mark.gpu

RAW_TOL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from kv_cache_eviction_trig_b200 import build
    build.build()
    tria.lib()


class Case:
    """One drawn workload on the GPU plus its oracle problem."""

    def __init__(self, wl, flags=0, seq_len=None, gen_device="cpu", calib_on_gpu=False,
                 fused=False):
        self.wl = wl
        data = workloads.generate(wl, device=gen_device)
        self.stats_np = common.stats_fp32(data["q_calib"], wl.rope_layout)
        self.host = {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in data.items()}
        if seq_len is not None:
            self.host["seq_len"] = torch.tensor(seq_len, dtype=torch.int32)
        self.dev = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in self.host.items()}
        self.pristine = {k: self.dev[k].clone() for k in ("k", "v", "pos", "seq_len")}
        self.cfg = tria.Config.from_workload(wl, flags=flags | (tria.FUSED_PRUNE if fused else 0))
        self.cache = tria.Cache.from_data(self.dev)
        self.stats = tria.Stats(*[torch.from_numpy(s).cuda() for s in self.stats_np])
        self.ws = tria.workspace(self.cfg, self.cache)
        self.prob = common.problem(wl, self.host, self.stats_np, flags=flags,
                                   seq_len=self.host["seq_len"].numpy())
        self.flags = flags

    @property
    def lens(self):
        return self.host["seq_len"].tolist()

    def segments(self):
        wl = self.wl
        for l in range(wl.num_layers):
            for g in range(wl.n_kv_heads):
                for b in range(wl.batch):
                    yield l, g, b, self.host["seq_start"][b], self.lens[b]

    def gpu_score(self):
        wl = self.wl
        score = torch.full((wl.num_layers, wl.n_kv_heads, wl.cap_total), float("nan"),
                           device="cuda")
        raw = torch.full((wl.num_layers, wl.n_q_heads, wl.cap_total), float("nan"),
                         device="cuda")
        tria.tria_score(self.cfg, self.stats, self.cache, score, raw, self.ws)
        torch.cuda.synchronize()
        assert tria.tria_get_device_error(self.ws) == 0
        return raw.double().cpu().numpy(), score.double().cpu().numpy()


def rms_over_sigma(ref_raw, case, l, g, b):
    """max over the group's query heads of rms(s_h) / sigma(s_h) (1 if every sigma is 0)."""
    s0, T = case.host["seq_start"][b], case.lens[b]
    G = case.wl.group
    worst = 0.0
    for h in range(g * G, (g + 1) * G):
        s = ref_raw[l, h, s0:s0 + T]
        sig = s.std()
        if sig > 0:
            worst = max(worst, np.sqrt(np.mean(s ** 2)) / sig)
    return max(worst, 1.0)


def z_tolerance(ref_raw, ref_z, case, l, g, b):
    return RAW_TOL * (2.0 + np.abs(ref_z)) * rms_over_sigma(ref_raw, case, l, g, b)


def report(what, case, **fields):
    """One line per check, so that the tolerance actually used is on record."""
    vals = " ".join(f"{k}={v:.3g}" if isinstance(v, float) else f"{k}={v}"
                    for k, v in fields.items())
    print(f"[{what}] {case.wl.name}: {vals}")


def check_raw(gpu_raw, ref_raw, case):
    wl = case.wl
    for l, g, b, s0, T in case.segments():
        for h in range(g * wl.group, (g + 1) * wl.group):
            ref = ref_raw[l, h, s0:s0 + T]
            got = gpu_raw[l, h, s0:s0 + T]
            if T == 0:
                continue
            scale = np.maximum(np.abs(ref), np.sqrt(np.mean(ref ** 2)))
            err = np.abs(got - ref)
            assert np.all(err <= RAW_TOL * scale + 1e-30), (l, h, b, float((err / scale).max()))


def check_score(gpu_score, ref_raw, ref_score, case):
    factor, rel = 1.0, 0.0
    for l, g, b, s0, T in case.segments():
        if T == 0:
            continue
        ref = ref_score[l, g, s0:s0 + T]
        got = gpu_score[l, g, s0:s0 + T]
        tol = z_tolerance(ref_raw, ref, case, l, g, b)
        assert np.all(np.abs(got - ref) <= tol), (l, g, b, float(np.abs(got - ref).max()))
        factor = max(factor, rms_over_sigma(ref_raw, case, l, g, b))
        rel = max(rel, float((np.abs(got - ref) / np.maximum(1.0, np.abs(ref))).max()))
    report("z", case, max_rms_over_sigma=factor, max_dz_rel=rel, bound_1e4=rel <= 1e-4)


def check_selection(gpu_sel, ref_sel, ref_raw, ref_score, case):
    budget = case.wl.budget
    excused = 0
    for l, g, b, s0, T in case.segments():
        got = gpu_sel[l, g, b]
        want = ref_sel[l, g, b]
        n = min(T, budget)
        assert np.all(got[n:] == -1) and np.all(np.diff(got[:n]) > 0)
        if T <= budget:
            assert got[:n].tolist() == list(range(T))
            continue
        sc = ref_score[l, g, s0:s0 + T]
        thr = np.sort(sc)[-budget]
        tol = z_tolerance(ref_raw, sc, case, l, g, b)
        diff = set(got[:n].tolist()) ^ set(want[:n].tolist())
        for t in diff:
            assert abs(sc[t] - thr) <= tol[t], (l, g, b, t, sc[t], thr)
        excused += len(diff) // 2
    report("select", case, keys_differing_within_tolerance=excused)


def check_compacted(case, sel, kept):
    """K, V, pos rows [0, kept) == pristine[sel]; rows [kept, capacity) untouched."""
    wl = case.wl
    k, v, pos = (case.dev[n].cpu() for n in ("k", "v", "pos"))
    pk, pv, pp = (case.pristine[n].cpu() for n in ("k", "v", "pos"))
    starts = case.host["seq_start"]
    for l, g, b, s0, T in case.segments():
        cap_b = starts[b + 1] - s0
        n = kept[b]
        idx = torch.from_numpy(sel[l, g, b, :n].astype(np.int64)) + s0
        assert torch.equal(k[l, g, s0:s0 + n].view(torch.int16), pk[l, g, idx].view(torch.int16))
        assert torch.equal(v[l, g, s0:s0 + n].view(torch.int16), pv[l, g, idx].view(torch.int16))
        assert torch.equal(pos[l, g, s0:s0 + n], pp[l, g, idx])
        assert torch.equal(k[l, g, s0 + n:s0 + cap_b].view(torch.int16),
                           pk[l, g, s0 + n:s0 + cap_b].view(torch.int16))
        assert torch.equal(pos[l, g, s0 + n:s0 + cap_b], pp[l, g, s0 + n:s0 + cap_b])


def small(name, **kw):
    d = dict(L=1, B=1, Hq=8, Hkv=2, D=128, theta=1e6, budget=100, offsets=range(1, 65),
             seq_lens=[1000], seed=11, n_calib=128)
    d.update(kw)
    return workloads.custom(name, **d)


CASES = {
    "tiny": lambda: workloads.workload(0),
    "ragged2seq": lambda: small("ragged2seq", B=2, seq_lens=[1000, 333], slack=37,
                                nu=lambda g: 0.3 if g == 0 else 1.5),
    "d64_interleaved": lambda: small("d64i", D=64, Hq=4, Hkv=2, seq_lens=[700], theta=1e4,
                                     rope_layout=workloads.INTERLEAVED),
    "g8": lambda: small("g8", Hq=8, Hkv=1, seq_lens=[515], budget=77),
    # G = 8 always takes the score kernel's tensor-core form: D = 64, interleaved RoPE,
    # two ragged sequences
    "d64_g8_interleaved": lambda: small("d64g8i", D=64, Hq=16, Hkv=2, B=2, seq_lens=[700, 333],
                                        theta=1e4, budget=60, rope_layout=workloads.INTERLEAVED),
    "d256": lambda: small("d256", D=256, Hq=4, Hkv=1, seq_lens=[300], budget=50),
    "g1": lambda: small("g1", Hq=4, Hkv=4, seq_lens=[260], budget=33),
    "g16_geometric": lambda: small("g16", D=64, Hq=16, Hkv=1, seq_lens=[200], budget=20,
                                   offsets=[2 ** i for i in range(17)]),
    "d128_g16": lambda: small("d128g16", Hq=16, Hkv=1, seq_lens=[130], budget=64),
    "two_layers": lambda: small("2l", L=2, B=3, seq_lens=[129, 400, 90], budget=128,
                                offsets=range(1, 33)),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_score_matches_oracle(name):
    case = Case(CASES[name]())
    ref_raw = oracle.raw_scores(case.prob)
    _, ref_score = oracle.zmax(case.prob, ref_raw)
    gpu_raw, gpu_score = case.gpu_score()
    check_raw(gpu_raw, ref_raw, case)
    check_score(gpu_score, ref_raw, ref_score, case)


@pytest.mark.parametrize("flags", [tria.NO_TRIG, tria.NO_CONC_WEIGHT])
def test_ablation_flags_match_oracle(flags):
    case = Case(CASES["ragged2seq"](), flags=flags)
    ref_raw = oracle.raw_scores(case.prob)
    _, ref_score = oracle.zmax(case.prob, ref_raw)
    gpu_raw, gpu_score = case.gpu_score()
    check_raw(gpu_raw, ref_raw, case)
    check_score(gpu_score, ref_raw, ref_score, case)


def test_calibrate_matches_oracle():
    wl = small("calib", L=2, Hq=8, D=128, n_calib=333)
    q = workloads.generate(wl)["q_calib"]
    for layout in (0, 1):
        cfg = tria.Config(num_layers=2, batch=1, n_q_heads=8, n_kv_heads=2, head_dim=128,
                          rope_theta=1e6, budget=1, offsets=[1], rope_layout=layout)
        for qd in (q, q.to(torch.bfloat16)):
            st = tria.calibrate(cfg, qd.cuda())
            torch.cuda.synchronize()
            c, m, r = oracle.calibrate(qd.double().numpy(), layout)
            np.testing.assert_allclose(st.tensors[0].cpu().numpy(), c, rtol=1e-6, atol=1e-7)
            np.testing.assert_allclose(st.tensors[1].cpu().numpy(), m, rtol=1e-6)
            np.testing.assert_allclose(st.tensors[2].cpu().numpy(), r, rtol=1e-6, atol=1e-7)


@pytest.mark.parametrize("name", ["tiny", "ragged2seq", "g8", "two_layers"])
def test_select_on_identical_scores_is_exact(name):
    """Given the same float32 scores, GPU and oracle selections are identical,
    including injected exact ties (ties to the lower slot)."""
    case = Case(CASES[name]())
    wl = case.wl
    rng = np.random.default_rng(5)
    score = rng.normal(size=(wl.num_layers, wl.n_kv_heads, wl.cap_total)).astype(np.float32)
    score[..., ::7] = score[..., 3:4]          # many exact ties
    score[..., 1::11] = 0.0
    score[..., 2::13] = -0.0                   # -0 and +0 tie
    sel = torch.full((wl.num_layers, wl.n_kv_heads, wl.batch, wl.budget), -7, dtype=torch.int32,
                     device="cuda")
    tria.tria_select(case.cfg, case.cache, torch.from_numpy(score).cuda(), sel, case.ws)
    ref = oracle.select(case.prob, score.astype(np.float64))
    np.testing.assert_array_equal(sel.cpu().numpy(), ref)


def _adversarial_sel(kind, T, budget, rng):
    if T <= budget:
        s = np.arange(T)
    elif kind == "first":
        s = np.arange(budget)
    elif kind == "last":
        s = np.arange(T - budget, T)
    elif kind == "alternating":
        s = np.arange(0, T, 2)[:budget]
        if len(s) < budget:
            s = np.sort(np.concatenate([s, np.arange(1, T, 2)[:budget - len(s)]]))
    else:
        s = np.sort(rng.choice(T, size=budget, replace=False))
    out = np.full(budget, -1, np.int32)
    out[:len(s)] = s
    return out


@pytest.mark.parametrize("kind", ["first", "last", "alternating", "random"])
def test_compact_in_place_is_bit_exact(kind):
    wl = small("compact", L=2, B=3, seq_lens=[1500, 90, 777], budget=400, slack=5, D=128)
    case = Case(wl)
    rng = np.random.default_rng(7)
    sel = np.stack([np.stack([np.stack([_adversarial_sel(kind, T, wl.budget, rng)
                                        for T in case.lens]) for _ in range(wl.n_kv_heads)])
                    for _ in range(wl.num_layers)])
    tria.tria_compact(case.cfg, case.cache, torch.from_numpy(sel).cuda(), case.ws)
    torch.cuda.synchronize()
    assert tria.tria_get_device_error(case.ws) == 0
    kept = [min(T, wl.budget) for T in case.lens]
    assert case.dev["seq_len"].cpu().tolist() == kept
    check_compacted(case, sel, kept)
    ok, ov, opos, osl = oracle.compact(case.prob, sel, common.bf16_bits(case.host["v"]))
    np.testing.assert_array_equal(common.bf16_bits(case.dev["k"]), ok)
    np.testing.assert_array_equal(common.bf16_bits(case.dev["v"]), ov)
    np.testing.assert_array_equal(case.dev["pos"].cpu().numpy(), opos)


@pytest.mark.parametrize("kind", ["last", "alternating", "random"])
@pytest.mark.parametrize("L,D,budget,T", [(2, 128, 3500, 4000), (2, 256, 2000, 2500),
                                          (1, 128, 3500, 4000)])
def test_compact_many_units_multi_batch(kind, L, D, budget, T):
    """Budgets larger than a unit's CTAs can stage at once are compacted in several
    batches: 16 units (one CTA each; about 330 rows of D=128 or 166 of D=256 per batch)
    and 8 units (one 8-CTA cluster each; about 2600 rows of D=128 per batch)."""
    wl = small("compact-multi", L=L, Hq=32, Hkv=8, B=1, D=D, seq_lens=[T], budget=budget)
    case = Case(wl)
    rng = np.random.default_rng(11)
    sel = np.stack([np.stack([np.stack([_adversarial_sel(kind, T, wl.budget, rng)
                                        for T in case.lens]) for _ in range(wl.n_kv_heads)])
                    for _ in range(wl.num_layers)])
    tria.tria_compact(case.cfg, case.cache, torch.from_numpy(sel).cuda(), case.ws)
    torch.cuda.synchronize()
    assert tria.tria_get_device_error(case.ws) == 0
    assert case.dev["seq_len"].cpu().tolist() == [budget]
    check_compacted(case, sel, [budget])


def test_four_cta_clusters_select_and_compact_exactly():
    """16 units whose segments (40000 and 36001 slots) do not fit one CTA: the unit kernel
    takes clusters of 4 CTAs (all resident at once). Selection on given scores with exact
    ties, then in-place compaction of a random selection, both against the oracle."""
    wl = small("cl4", Hq=16, Hkv=8, B=2, seq_lens=[40000, 36001], budget=3000,
               offsets=range(1, 5), n_calib=32)
    case = Case(wl)
    rng = np.random.default_rng(13)
    score = rng.normal(size=(wl.num_layers, wl.n_kv_heads, wl.cap_total)).astype(np.float32)
    score[..., ::7] = score[..., 3:4]          # many exact ties
    score[..., 1::11] = 0.0
    sel = torch.empty((wl.num_layers, wl.n_kv_heads, wl.batch, wl.budget), dtype=torch.int32,
                      device="cuda")
    tria.tria_select(case.cfg, case.cache, torch.from_numpy(score).cuda(), sel, case.ws)
    ref = oracle.select(case.prob, score.astype(np.float64))
    np.testing.assert_array_equal(sel.cpu().numpy(), ref)
    csel = np.stack([np.stack([np.stack([_adversarial_sel("random", T, wl.budget, rng)
                                         for T in case.lens]) for _ in range(wl.n_kv_heads)])
                     for _ in range(wl.num_layers)])
    tria.tria_compact(case.cfg, case.cache, torch.from_numpy(csel).cuda(), case.ws)
    torch.cuda.synchronize()
    assert tria.tria_get_device_error(case.ws) == 0
    assert case.dev["seq_len"].cpu().tolist() == [wl.budget] * wl.batch
    check_compacted(case, csel, [wl.budget] * wl.batch)


@pytest.mark.parametrize("fused", [False, True], ids=["kernels3", "fused"])
def test_prune_many_units_matches_oracle(fused):
    case = Case(small("prune-multi", L=2, Hq=32, Hkv=8, B=1, seq_lens=[4000], budget=3500,
                      offsets=range(1, 17)), fused=fused)
    wl = case.wl
    ref = oracle.prune(case.prob, common.bf16_bits(case.host["v"]))
    sel = torch.empty((wl.num_layers, wl.n_kv_heads, wl.batch, wl.budget), dtype=torch.int32,
                      device="cuda")
    tria.tria_prune(case.cfg, case.stats, case.cache, case.ws, sel_out=sel)
    torch.cuda.synchronize()
    assert tria.tria_get_device_error(case.ws) == 0
    gsel = sel.cpu().numpy()
    check_selection(gsel, ref["sel"], ref["raw"], ref["score"], case)
    check_compacted(case, gsel, [3500])


@pytest.mark.parametrize("fused", [False, True], ids=["kernels3", "fused"])
def test_prune_many_groups_matches_oracle(fused):
    """72 units: the single launch takes them in three groups of at most 32, so its
    per-group scratch slots are reused; lengths span short, pruned and long units."""
    case = Case(small("groups", L=3, Hq=16, Hkv=8, B=3, seq_lens=[700, 100, 1500], budget=128,
                      offsets=range(1, 17), slack=9), fused=fused)
    wl = case.wl
    ref = oracle.prune(case.prob, common.bf16_bits(case.host["v"]))
    sel = torch.full((wl.num_layers, wl.n_kv_heads, wl.batch, wl.budget), -7, dtype=torch.int32,
                     device="cuda")
    tria.tria_prune(case.cfg, case.stats, case.cache, case.ws, sel_out=sel)
    torch.cuda.synchronize()
    assert tria.tria_get_device_error(case.ws) == 0
    gsel = sel.cpu().numpy()
    check_selection(gsel, ref["sel"], ref["raw"], ref["score"], case)
    kept = [min(T, wl.budget) for T in case.lens]
    assert case.dev["seq_len"].cpu().tolist() == kept == ref["seq_len"].tolist()
    check_compacted(case, gsel, kept)


def test_compact_rejects_malformed_selection():
    wl = small("badsel", B=2, seq_lens=[300, 300], budget=50)
    case = Case(wl)
    sel = np.tile(np.arange(50, dtype=np.int32), (1, 2, 2, 1))
    sel[0, 1, 1, 10] = sel[0, 1, 1, 9]       # not strictly ascending
    sel[0, 0, 0, 49] = 400                   # beyond the segment
    tria.tria_compact(case.cfg, case.cache, torch.from_numpy(sel).cuda(), case.ws)
    torch.cuda.synchronize()
    assert tria.tria_get_device_error(case.ws) & tria.DEVERR_SELECTION
    # the malformed units are untouched
    assert torch.equal(case.dev["k"][0, 1, 300:600], case.pristine["k"][0, 1, 300:600])
    assert torch.equal(case.dev["k"][0, 0, 0:300], case.pristine["k"][0, 0, 0:300])


@pytest.mark.parametrize("name", ["tiny", "ragged2seq", "d64_interleaved", "g8", "two_layers",
                                  "g16_geometric", "d64_g8_interleaved"])
@pytest.mark.parametrize("fused", [False, True], ids=["kernels3", "fused"])
def test_prune_matches_oracle(name, fused):
    case = Case(CASES[name](), fused=fused)
    wl = case.wl
    ref = oracle.prune(case.prob, common.bf16_bits(case.host["v"]))
    sel = torch.full((wl.num_layers, wl.n_kv_heads, wl.batch, wl.budget), -7, dtype=torch.int32,
                     device="cuda")
    tria.tria_prune(case.cfg, case.stats, case.cache, case.ws, sel_out=sel)
    torch.cuda.synchronize()
    assert tria.tria_get_device_error(case.ws) == 0
    gsel = sel.cpu().numpy()
    check_selection(gsel, ref["sel"], ref["raw"], ref["score"], case)
    kept = [min(T, wl.budget) for T in case.lens]
    assert case.dev["seq_len"].cpu().tolist() == kept == ref["seq_len"].tolist()
    check_compacted(case, gsel, kept)


@pytest.mark.parametrize("fused", [False, True], ids=["kernels3", "fused"])
def test_prune_without_sel_out_equals_with(fused):
    a = Case(CASES["ragged2seq"](), fused=fused)
    b = Case(CASES["ragged2seq"](), fused=fused)
    wl = a.wl
    sel = torch.empty((wl.num_layers, wl.n_kv_heads, wl.batch, wl.budget), dtype=torch.int32,
                      device="cuda")
    tria.tria_prune(a.cfg, a.stats, a.cache, a.ws, sel_out=sel)
    tria.tria_prune(b.cfg, b.stats, b.cache, b.ws)
    torch.cuda.synchronize()
    for n in ("k", "v", "pos", "seq_len"):
        assert torch.equal(a.dev[n], b.dev[n])


@pytest.mark.parametrize("fused", [False, True], ids=["kernels3", "fused"])
def test_prune_edge_lengths(fused):
    """T = 0, T < budget, T = budget, T = budget + 1, and a long one, in one batch."""
    wl = small("edges", B=5, seq_lens=[0, 50, 100, 101, 900], budget=100, slack=3)
    case = Case(wl, fused=fused)
    ref = oracle.prune(case.prob, common.bf16_bits(case.host["v"]))
    sel = torch.empty((1, 2, 5, 100), dtype=torch.int32, device="cuda")
    tria.tria_prune(case.cfg, case.stats, case.cache, case.ws, sel_out=sel)
    torch.cuda.synchronize()
    assert tria.tria_get_device_error(case.ws) == 0
    assert case.dev["seq_len"].cpu().tolist() == [0, 50, 100, 100, 100]
    gsel = sel.cpu().numpy()
    check_selection(gsel, ref["sel"], ref["raw"], ref["score"], case)
    check_compacted(case, gsel, [0, 50, 100, 100, 100])


@pytest.mark.parametrize("fused", [False, True], ids=["kernels3", "fused"])
def test_prune_budget_one(fused):
    case = Case(small("b1", seq_lens=[333], budget=1), fused=fused)
    ref = oracle.prune(case.prob, common.bf16_bits(case.host["v"]))
    sel = torch.empty((1, 2, 1, 1), dtype=torch.int32, device="cuda")
    tria.tria_prune(case.cfg, case.stats, case.cache, case.ws, sel_out=sel)
    torch.cuda.synchronize()
    check_selection(sel.cpu().numpy(), ref["sel"], ref["raw"], ref["score"], case)
    check_compacted(case, sel.cpu().numpy(), [1])


@pytest.mark.parametrize("fused", [False, True], ids=["kernels3", "fused"])
def test_seq_len_beyond_capacity_sets_flag_and_skips_sequence(fused):
    wl = small("overflow", B=2, seq_lens=[300, 300], budget=50)
    case = Case(wl, seq_len=[300, 301], fused=fused)  # sequence 1 claims more than its segment
    case.cache = tria.Cache.from_data(case.dev)
    tria.tria_prune(case.cfg, case.stats, case.cache, case.ws)
    torch.cuda.synchronize()
    assert tria.tria_get_device_error(case.ws) & tria.DEVERR_SEQ_LEN
    assert case.dev["seq_len"].cpu().tolist() == [50, 301]
    assert torch.equal(case.dev["k"][:, :, 300:600], case.pristine["k"][:, :, 300:600])
    tria.tria_workspace_init(case.ws)
    assert tria.tria_get_device_error(case.ws) == 0


@pytest.mark.parametrize("fused", [False, True], ids=["kernels3", "fused"])
def test_repeated_prune_is_stable(fused):
    """A second prune of an already pruned cache (T = budget) changes nothing."""
    case = Case(CASES["ragged2seq"](), fused=fused)
    tria.tria_prune(case.cfg, case.stats, case.cache, case.ws)
    torch.cuda.synchronize()
    snap = {n: case.dev[n].clone() for n in ("k", "v", "pos", "seq_len")}
    tria.tria_prune(case.cfg, case.stats, case.cache, case.ws)
    torch.cuda.synchronize()
    for n, t in snap.items():
        assert torch.equal(case.dev[n], t)


# Problems with more than 15 units run one CTA per unit instead of one 8-CTA cluster.

@pytest.mark.parametrize("fused", [False, True], ids=["kernels3", "fused"])
def test_prune_edge_lengths_one_cta_per_unit(fused):
    """40 units (L2 x Hkv4 x B5): T = 0, < budget, = budget, budget + 1 and long."""
    wl = small("edges-1cta", L=2, B=5, Hq=8, Hkv=4, seq_lens=[0, 50, 100, 101, 900], budget=100,
               slack=3)
    case = Case(wl, fused=fused)
    ref = oracle.prune(case.prob, common.bf16_bits(case.host["v"]))
    sel = torch.full((2, 4, 5, 100), -7, dtype=torch.int32, device="cuda")
    tria.tria_prune(case.cfg, case.stats, case.cache, case.ws, sel_out=sel)
    torch.cuda.synchronize()
    assert tria.tria_get_device_error(case.ws) == 0
    assert case.dev["seq_len"].cpu().tolist() == [0, 50, 100, 100, 100]
    gsel = sel.cpu().numpy()
    check_selection(gsel, ref["sel"], ref["raw"], ref["score"], case)
    check_compacted(case, gsel, [0, 50, 100, 100, 100])


def test_score_one_cta_per_unit():
    case = Case(small("score-1cta", L=2, B=3, Hq=8, Hkv=4, seq_lens=[700, 129, 2000], budget=64,
                      offsets=[2 ** i for i in range(12)]))
    ref_raw = oracle.raw_scores(case.prob)
    _, ref_score = oracle.zmax(case.prob, ref_raw)
    gpu_raw, gpu_score = case.gpu_score()
    check_raw(gpu_raw, ref_raw, case)
    check_score(gpu_score, ref_raw, ref_score, case)


def test_select_on_identical_scores_one_cta_per_unit():
    case = Case(small("select-1cta", L=2, B=2, Hq=8, Hkv=4, seq_lens=[1500, 333], budget=200))
    wl = case.wl
    rng = np.random.default_rng(9)
    score = rng.normal(size=(wl.num_layers, wl.n_kv_heads, wl.cap_total)).astype(np.float32)
    score[..., ::5] = score[..., 2:3]          # many exact ties
    score[..., 1::7] = -0.0
    sel = torch.full((wl.num_layers, wl.n_kv_heads, wl.batch, wl.budget), -7, dtype=torch.int32,
                     device="cuda")
    tria.tria_select(case.cfg, case.cache, torch.from_numpy(score).cuda(), sel, case.ws)
    ref = oracle.select(case.prob, score.astype(np.float64))
    np.testing.assert_array_equal(sel.cpu().numpy(), ref)


# ------------------------------------------------------------------ large buckets and ties
# A bucket of more than 4096 keys at the threshold (massive ties, or scores packed into one
# histogram bin) takes the refinement rounds on the key bits and, when every key of the
# bucket is equal, the rule that ties go to the lowest slots (romaanj.github.io review,
# "Method": keep the top budget; ties to the lower position).  8 units run one 8-CTA
# cluster each; 16 units run one CTA each.

def _scores_only_case(L, Hkv, T, budget):
    """A problem with scores but no keys: tria_select reads only lengths and scores."""
    cfg = tria.Config(num_layers=L, batch=1, n_q_heads=Hkv, n_kv_heads=Hkv, head_dim=128,
                      rope_theta=1e6, budget=budget, offsets=[1])
    seq_len = torch.tensor([T], dtype=torch.int32, device="cuda")
    cache = tria.Cache(None, None, None, seq_len, None, [0, T], cap_total=T)
    ws = tria.workspace(cfg, cache)
    D = 8
    prob = oracle.Problem(k=np.zeros((L, Hkv, T, D), np.uint16), pos=np.zeros((L, Hkv, T), np.int32),
                          seq_start=[0, T], seq_len=[T], cur_pos=[T - 1],
                          centre=np.zeros((L, Hkv, D // 2, 2)), mean_norm=np.zeros((L, Hkv, D // 2)),
                          mrl=np.zeros((L, Hkv, D // 2)), theta=1e6, budget=budget, offsets=[1],
                          n_q_heads=Hkv)
    return cfg, cache, ws, prob


def _bucket_scores(pattern, L, Hkv, T, rng):
    if pattern == "one_bin":      # distinct values, all inside one 12-bit bin of the key
        return (1.0 + 1e-6 * np.stack([rng.permutation(T) for _ in range(L * Hkv)])).reshape(
            L, Hkv, T).astype(np.float32)
    if pattern == "all_equal":    # every key ties: the lowest slots are kept
        return np.full((L, Hkv, T), 0.5, np.float32)
    # three values 2^-20 apart, thousands of keys each: the threshold value ties
    vals = np.float32(1.0) + np.float32(2.0 ** -20) * np.arange(3, dtype=np.float32)
    return vals[rng.integers(0, 3, size=(L, Hkv, T))]


@pytest.mark.parametrize("pattern", ["one_bin", "all_equal", "three_values"])
@pytest.mark.parametrize("L", [1, 2])          # 8 units (clusters) or 16 units (one CTA each)
def test_select_large_bucket_is_exact(pattern, L):
    Hkv, T, budget = 8, 32768, 2048
    cfg, cache, ws, prob = _scores_only_case(L, Hkv, T, budget)
    score = _bucket_scores(pattern, L, Hkv, T, np.random.default_rng(L))
    sel = torch.full((L, Hkv, 1, budget), -7, dtype=torch.int32, device="cuda")
    tria.tria_select(cfg, cache, torch.from_numpy(score).cuda(), sel, ws)
    torch.cuda.synchronize()
    assert tria.tria_get_device_error(ws) == 0
    ref = oracle.select(prob, score.astype(np.float64))
    np.testing.assert_array_equal(sel.cpu().numpy(), ref)
    if pattern == "all_equal":
        assert np.all(ref == np.arange(budget))


@pytest.mark.parametrize("L", [1, 2])
@pytest.mark.parametrize("fused", [False, True], ids=["kernels3", "fused"])
def test_prune_degenerate_groups_keep_the_lowest_slots(L, fused):
    """KV groups whose query heads all have zero centre and zero mean norm score
    every key 0, so sigma = 0 and z = 0 (the z-score reading for sigma = 0): every
    key ties and the prune keeps slots 0..budget-1.  The other groups are ordinary."""
    wl = small("degenerate", L=L, Hq=32, Hkv=8, seq_lens=[8192], budget=2048, offsets=[1, 2, 3])
    case = Case(wl, fused=fused)
    c, m, r = (np.array(x) for x in case.stats_np)
    G = wl.group
    dead = [0, 5]
    for g in dead:
        c[:, g * G:(g + 1) * G] = 0.0
        m[:, g * G:(g + 1) * G] = 0.0
        r[:, g * G:(g + 1) * G] = 0.0
    case.stats_np = (c, m, r)
    case.stats = tria.Stats(*[torch.from_numpy(x).cuda() for x in case.stats_np])
    case.prob = common.problem(wl, case.host, case.stats_np, seq_len=case.host["seq_len"].numpy())
    ref = oracle.prune(case.prob, common.bf16_bits(case.host["v"]))
    sel = torch.full((L, 8, 1, wl.budget), -7, dtype=torch.int32, device="cuda")
    tria.tria_prune(case.cfg, case.stats, case.cache, case.ws, sel_out=sel)
    torch.cuda.synchronize()
    assert tria.tria_get_device_error(case.ws) == 0
    gsel = sel.cpu().numpy()
    for l in range(L):
        for g in dead:
            assert np.all(ref["sel"][l, g, 0] == np.arange(wl.budget))
            np.testing.assert_array_equal(gsel[l, g, 0], np.arange(wl.budget))
    check_selection(gsel, ref["sel"], ref["raw"], ref["score"], case)
    check_compacted(case, gsel, [wl.budget])

"""GPU parity of head-specific budgets (romaanj.github.io review, "Future work":
compression refined with a budget per head) against the oracle.

Every (layer, KV head) has its own budget and every (layer, KV head, sequence)
unit its own live length (tria_cache.unit_len), as after an earlier prune with
head budgets.  Checked through both prune paths (the fold, score and unit
kernels, and the single persistent launch), the separate select and compact calls
(one 8-CTA cluster per unit and one CTA per unit), a shape the single launch does
not take (head_dim 256 with 16 query heads per KV head), the decode-loop append
and the decode attention.  Tolerances as in test_gpu_parity: selections by the
threshold rule, compacted rows, lengths and selection lists of identical scores
bit-exact."""
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


class HeadCase:
    """A drawn cache with per-unit lengths and per-head budgets, on the GPU and in
    the oracle's form."""

    def __init__(self, wl, seed, budget_lo=1, len_lo=0.5, window=0, headroom=0, fused=False):
        rng = np.random.default_rng(seed)
        self.wl = wl
        data = workloads.generate(wl)
        self.stats_np = common.stats_fp32(data["q_calib"], wl.rope_layout)
        L, Hkv, B = wl.num_layers, wl.n_kv_heads, wl.batch
        caps = [wl.seq_start[b + 1] - wl.seq_start[b] for b in range(B)]
        self.unit_len = np.stack([np.stack([
            np.array([rng.integers(int(len_lo * c), c + 1 - headroom) if c else 0 for c in caps])
            for _ in range(Hkv)]) for _ in range(L)]).astype(np.int32)
        self.budgets = rng.integers(budget_lo, wl.budget + 1, size=(L, Hkv)).astype(np.int32)
        self.host = {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in data.items()}
        self.dev = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in self.host.items()}
        self.dev["unit_len"] = torch.from_numpy(self.unit_len.copy()).cuda()
        self.dev["budgets"] = torch.from_numpy(self.budgets.copy()).cuda()
        self.pristine = {k: self.dev[k].clone() for k in ("k", "v", "pos", "unit_len")}
        self.cfg = tria.Config.from_workload(wl, head_budgets=self.dev["budgets"],
                                             prune_window=window,
                                             flags=tria.FUSED_PRUNE if fused else 0)
        self.cache = tria.Cache(self.dev["k"], self.dev["v"], self.dev["pos"], None,
                                self.dev["cur_pos"], self.host["seq_start"],
                                unit_len=self.dev["unit_len"])
        self.stats = tria.Stats(*[torch.from_numpy(s).cuda() for s in self.stats_np])
        self.ws = tria.workspace(self.cfg, self.cache)
        c, m, r = self.stats_np
        self.prob = oracle.Problem(
            k=common.bf16_bits(self.host["k"]), pos=self.host["pos"].numpy(),
            seq_start=self.host["seq_start"], seq_len=self.host["seq_len"].numpy(),
            cur_pos=self.host["cur_pos"].numpy(), centre=c.astype(np.float64),
            mean_norm=m.astype(np.float64), mrl=r.astype(np.float64), theta=wl.rope_theta,
            budget=wl.budget, offsets=wl.offsets, n_q_heads=wl.n_q_heads,
            layout=wl.rope_layout, budgets=self.budgets, unit_len=self.unit_len)

    def units(self):
        wl = self.wl
        for l in range(wl.num_layers):
            for g in range(wl.n_kv_heads):
                for b in range(wl.batch):
                    yield l, g, b, self.host["seq_start"][b], int(self.unit_len[l, g, b]), \
                        int(self.budgets[l, g])


def z_tol(ref_raw, ref_z, case, l, g, s0, T):
    G = case.wl.group
    worst = 1.0
    for h in range(g * G, (g + 1) * G):
        s = ref_raw[l, h, s0:s0 + T]
        if s.std() > 0:
            worst = max(worst, np.sqrt(np.mean(s ** 2)) / s.std())
    return RAW_TOL * (2.0 + np.abs(ref_z)) * worst


def check_selection(case, gsel, ref):
    excused = 0
    for l, g, b, s0, T, bud in case.units():
        got = gsel[l, g, b]
        n = min(T, bud)
        assert np.all(got[n:] == -1), (l, g, b)
        assert np.all(np.diff(got[:n]) > 0) and (n == 0 or (got[0] >= 0 and got[n - 1] < T))
        if T <= bud:
            assert got[:n].tolist() == list(range(T))
            continue
        sc = ref["score"][l, g, s0:s0 + T]
        thr = np.sort(sc)[-bud]
        tol = z_tol(ref["raw"], sc, case, l, g, s0, T)
        diff = set(got[:n].tolist()) ^ set(ref["sel"][l, g, b, :n].tolist())
        for t in diff:
            assert abs(sc[t] - thr) <= tol[t], (l, g, b, t)
        excused += len(diff) // 2
    print(f"[head budgets] {case.wl.name}: keys differing within tolerance={excused}")


def check_compacted(case, gsel, lens_after):
    k, v, pos = (case.dev[n].cpu() for n in ("k", "v", "pos"))
    pk, pv, pp = (case.pristine[n].cpu() for n in ("k", "v", "pos"))
    for l, g, b, s0, T, bud in case.units():
        n = int(lens_after[l, g, b])
        idx = torch.from_numpy(gsel[l, g, b, :n].astype(np.int64)) + s0
        assert torch.equal(k[l, g, s0:s0 + n].view(torch.int16), pk[l, g, idx].view(torch.int16))
        assert torch.equal(v[l, g, s0:s0 + n].view(torch.int16), pv[l, g, idx].view(torch.int16))
        assert torch.equal(pos[l, g, s0:s0 + n], pp[l, g, idx])


def _small(name, **kw):
    d = dict(L=1, B=2, Hq=16, Hkv=4, D=128, theta=1e6, budget=300, offsets=range(1, 33),
             seq_lens=[1200, 700], seed=41, n_calib=128, slack=13)
    d.update(kw)
    return workloads.custom(name, **d)


SHAPES = {
    "g4": lambda: _small("hb-g4"),
    "g8_two_layers": lambda: _small("hb-g8", L=2, Hq=16, Hkv=2, seq_lens=[900, 2000, 50], B=3),
    "d64_interleaved": lambda: _small("hb-d64", D=64, theta=1e4, rope_layout=workloads.INTERLEAVED),
    "many_units": lambda: _small("hb-many", L=3, B=4, Hq=8, Hkv=4, seq_lens=[500, 64, 900, 333],
                                 budget=128),
}


@pytest.mark.parametrize("fused", [False, True], ids=["kernels3", "fused"])
@pytest.mark.parametrize("name", sorted(SHAPES))
def test_prune_with_head_budgets_matches_oracle(name, fused):
    case = HeadCase(SHAPES[name](), seed=len(name), fused=fused)
    wl = case.wl
    ref = oracle.prune(case.prob, common.bf16_bits(case.host["v"]))
    sel = torch.full((wl.num_layers, wl.n_kv_heads, wl.batch, wl.budget), -7, dtype=torch.int32,
                     device="cuda")
    tria.tria_prune(case.cfg, case.stats, case.cache, case.ws, sel_out=sel)
    torch.cuda.synchronize()
    assert tria.tria_get_device_error(case.ws) == 0
    got_len = case.dev["unit_len"].cpu().numpy()
    np.testing.assert_array_equal(got_len, ref["unit_len"])
    gsel = sel.cpu().numpy()
    check_selection(case, gsel, ref)
    check_compacted(case, gsel, got_len)


def test_three_kernel_prune_with_head_budgets_matches_oracle():
    """head_dim 256 with 16 query heads per KV head runs the fold, score and unit
    kernels even when the single-launch prune is asked for (that launch does not
    take this shape)."""
    case = HeadCase(_small("hb-d256g16", D=256, Hq=16, Hkv=1, seq_lens=[600, 300], budget=100),
                    seed=3, fused=True)
    wl = case.wl
    ref = oracle.prune(case.prob, common.bf16_bits(case.host["v"]))
    sel = torch.full((1, 1, 2, wl.budget), -7, dtype=torch.int32, device="cuda")
    names = tria.tria_prune_profiled(case.cfg, case.stats, case.cache, case.ws,
                                     [torch.cuda.Event(enable_timing=True)
                                      for _ in range(tria.PRUNE_MAX_STAGES + 1)], sel_out=sel)
    assert names == ["fold_kernel", "score_kernel", "unit_kernel"]
    torch.cuda.synchronize()
    assert tria.tria_get_device_error(case.ws) == 0
    got_len = case.dev["unit_len"].cpu().numpy()
    np.testing.assert_array_equal(got_len, ref["unit_len"])
    check_selection(case, sel.cpu().numpy(), ref)
    check_compacted(case, sel.cpu().numpy(), got_len)


@pytest.mark.parametrize("L", [1, 2])   # 8 units: 8-CTA clusters; 16 units: one CTA each
def test_select_and_compact_with_head_budgets_are_exact(L):
    """On the same float32 scores the selection equals the oracle's exactly (ties
    injected), and compaction moves exactly the selected rows."""
    wl = _small("hb-select", L=L, B=1, Hq=8, Hkv=8, seq_lens=[3000], budget=700)
    case = HeadCase(wl, seed=L)
    rng = np.random.default_rng(7)
    score = rng.normal(size=(L, 8, wl.cap_total)).astype(np.float32)
    score[..., ::9] = score[..., 4:5]
    sel = torch.full((L, 8, 1, wl.budget), -7, dtype=torch.int32, device="cuda")
    tria.tria_select(case.cfg, case.cache, torch.from_numpy(score).cuda(), sel, case.ws)
    torch.cuda.synchronize()
    assert tria.tria_get_device_error(case.ws) == 0
    ref_sel = oracle.select(case.prob, score.astype(np.float64))
    np.testing.assert_array_equal(sel.cpu().numpy(), ref_sel)
    tria.tria_compact(case.cfg, case.cache, sel, case.ws)
    torch.cuda.synchronize()
    assert tria.tria_get_device_error(case.ws) == 0
    want_len = np.minimum(case.unit_len, case.budgets[:, :, None])
    np.testing.assert_array_equal(case.dev["unit_len"].cpu().numpy(), want_len)
    ok, ov, opos, _, oul = oracle.compact_units(case.prob, ref_sel, common.bf16_bits(case.host["v"]))
    np.testing.assert_array_equal(oul, want_len)
    np.testing.assert_array_equal(common.bf16_bits(case.dev["k"]), ok)
    np.testing.assert_array_equal(common.bf16_bits(case.dev["v"]), ov)
    np.testing.assert_array_equal(case.dev["pos"].cpu().numpy(), opos)


def test_head_budget_out_of_range_sets_flag_and_skips_the_head():
    case = HeadCase(_small("hb-bad"), seed=9)
    bad = case.budgets.copy()
    bad[0, 1] = case.wl.budget + 1
    bad[0, 2] = 0
    case.dev["budgets"].copy_(torch.from_numpy(bad))
    tria.tria_prune(case.cfg, case.stats, case.cache, case.ws)
    torch.cuda.synchronize()
    assert tria.tria_get_device_error(case.ws) & tria.DEVERR_BUDGET
    got = case.dev["unit_len"].cpu().numpy()
    for g in (1, 2):  # untouched
        np.testing.assert_array_equal(got[0, g], case.unit_len[0, g])
        assert torch.equal(case.dev["k"][0, g], case.pristine["k"][0, g])
    for g in (0, 3):
        np.testing.assert_array_equal(got[0, g], np.minimum(case.unit_len[0, g], bad[0, g]))


@pytest.mark.parametrize("fused", [False, True], ids=["kernels3", "fused"])
def test_decode_loop_with_head_budgets_matches_oracle(fused):
    """Append a token to every sequence, then prune with a window, 12 times, with
    per-head budgets: lengths, cache and positions follow the oracle step by step
    (the selections are compared with the threshold rule, then the oracle continues
    from the GPU's state); attention over the result matches the oracle."""
    wl = _small("hb-loop", B=2, Hq=8, Hkv=2, seq_lens=[330, 310], budget=300, slack=40,
                offsets=range(1, 9))
    W = 4
    case = HeadCase(wl, seed=5, budget_lo=280, len_lo=0.9, window=W, headroom=1, fused=fused)
    gen = torch.Generator().manual_seed(0)
    L, Hkv, B, D = wl.num_layers, wl.n_kv_heads, wl.batch, wl.head_dim
    for step in range(12):
        kn = torch.randn(L, Hkv, B, D, generator=gen).to(torch.bfloat16)
        vn = torch.randn(L, Hkv, B, D, generator=gen).to(torch.bfloat16)
        before = {n: case.dev[n].cpu() for n in ("k", "v", "pos", "unit_len", "cur_pos")}
        tria.tria_append(case.cfg, case.cache, kn.cuda(), vn.cuda(), case.ws)
        torch.cuda.synchronize()
        k2, v2, p2, ul2, cp2, skipped = oracle.append(
            common.bf16_bits(before["k"]), common.bf16_bits(before["v"]),
            before["pos"].numpy(), case.host["seq_start"], None, before["cur_pos"].numpy(),
            common.bf16_bits(kn), common.bf16_bits(vn), unit_len=before["unit_len"].numpy())
        assert skipped == []
        np.testing.assert_array_equal(case.dev["unit_len"].cpu().numpy(), ul2)
        np.testing.assert_array_equal(case.dev["cur_pos"].cpu().numpy(), cp2)
        np.testing.assert_array_equal(common.bf16_bits(case.dev["k"]), k2)
        np.testing.assert_array_equal(case.dev["pos"].cpu().numpy(), p2)
        # the windowed prune, from the state after the append
        c, m, r = case.stats_np
        prob = oracle.Problem(k=k2, pos=p2, seq_start=case.host["seq_start"],
                              seq_len=case.host["seq_len"].numpy(), cur_pos=cp2,
                              centre=c.astype(np.float64), mean_norm=m.astype(np.float64),
                              mrl=r.astype(np.float64), theta=wl.rope_theta, budget=wl.budget,
                              offsets=wl.offsets, n_q_heads=wl.n_q_heads, budgets=case.budgets,
                              unit_len=ul2)
        ref = oracle.prune_window(prob, v2, W)
        pre = {n: case.dev[n].clone() for n in ("k", "v", "pos")}
        sel = torch.full((L, Hkv, B, wl.budget), -7, dtype=torch.int32, device="cuda")
        tria.tria_prune(case.cfg, case.stats, case.cache, case.ws, sel_out=sel)
        torch.cuda.synchronize()
        assert tria.tria_get_device_error(case.ws) == 0
        got_len = case.dev["unit_len"].cpu().numpy()
        np.testing.assert_array_equal(got_len, ref["unit_len"])
        gsel = sel.cpu().numpy()
        for l in range(L):
            for g in range(Hkv):
                for b in range(B):
                    T, bud = int(ul2[l, g, b]), int(case.budgets[l, g])
                    s0 = case.host["seq_start"][b]
                    if T < bud + W:
                        continue  # held back (or under budget): rows untouched, list not written
                    sc = ref["score"][l, g, s0:s0 + T]
                    thr = np.sort(sc)[-bud]
                    tol = z_tol(ref["raw"], sc, case, l, g, s0, T)
                    for t in set(gsel[l, g, b, :bud].tolist()) ^ set(ref["sel"][l, g, b, :bud].tolist()):
                        assert abs(sc[t] - thr) <= tol[t]
                    idx = torch.from_numpy(gsel[l, g, b, :bud].astype(np.int64)).cuda() + s0
                    assert torch.equal(case.dev["k"][l, g, s0:s0 + bud], pre["k"][l, g, idx])
                    assert torch.equal(case.dev["v"][l, g, s0:s0 + bud], pre["v"][l, g, idx])
    # attention over the final cache reads each unit's own live slots
    q = torch.randn(B, wl.n_q_heads, D, generator=gen).to(torch.bfloat16)
    out = torch.empty(B, wl.n_q_heads, D, device="cuda")
    tria.tria_decode_attention(case.cfg, case.cache, 0, q.cuda(), out, case.ws)
    torch.cuda.synchronize()
    want = oracle.decode_attention(common.bf16_bits(case.dev["k"]), common.bf16_bits(case.dev["v"]),
                                   case.host["seq_start"], None, 0, common.bf16_bits(q),
                                   D ** -0.5, unit_len=case.dev["unit_len"].cpu().numpy())
    from tests.test_gpu_decode import ATT_ATOL, ATT_RTOL
    assert np.allclose(out.cpu().numpy(), want, rtol=ATT_RTOL, atol=ATT_ATOL)

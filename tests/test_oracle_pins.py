"""Pins the CPU oracle to things other than itself: closed forms, special
cases, invariants and brute force (no GPU).

Each test names the property and the passage it follows.  Page references:
"Method" and "Key idea" are sections of the romaanj.github.io review;
"2-2", "3-2 (n)" are sections of the dimensionstp.github.io review.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from kv_cache_eviction_trig_b200 import workloads
from tests import common

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rope_real(vec, p, theta, layout):
    """Post-RoPE copy of a real D-vector (rotate-half / interleaved formulas)."""
    D = vec.shape[-1]
    F = D // 2
    out = np.empty_like(vec)
    for f in range(F):
        xi, yi = (f, f + F) if layout == 0 else (2 * f, 2 * f + 1)
        a = p * theta ** (-2.0 * f / D)
        out[xi] = vec[xi] * math.cos(a) - vec[yi] * math.sin(a)
        out[yi] = vec[xi] * math.sin(a) + vec[yi] * math.cos(a)
    return out


def _small(seed=0, D=16, G=2, Hkv=2, T=40, offsets=range(1, 9), layout=0, nu=0.5, B=1,
           budget=10, theta=1.0e4, L=1, position_mode="subset", seq_lens=None):
    wl = workloads.custom("pin", L=L, B=B, Hq=G * Hkv, Hkv=Hkv, D=D, theta=theta, budget=budget,
                          offsets=list(offsets), seq_lens=seq_lens or [T] * B, seed=seed,
                          nu=nu, rope_layout=layout, n_calib=64, position_mode=position_mode)
    data = workloads.generate(wl)
    stats = common.stats_fp32(data["q_calib"], layout)
    return wl, data, stats


def _key_float(data, l, g, slot):
    return common.bits_to_float(common.bf16_bits(data["k"][l, g, slot]))


# ---------------------------------------------------------------------------- golden

def test_worked_example_closed_form():
    """Hand-derived closed forms of the scoring rule (Method; 2-2)."""
    ex = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    keys = np.array(ex["keys"], dtype=np.float32)
    bits = keys.view(np.uint32) >> 16
    assert np.all((bits.astype(np.uint32) << 16).view(np.float32) == keys)  # bf16-exact
    T = len(keys)
    p = oracle.Problem(
        k=bits.astype(np.uint16).reshape(1, 1, T, ex["D"]),
        pos=np.array(ex["pos"], dtype=np.int32).reshape(1, 1, T),
        seq_start=[0, T], seq_len=[T], cur_pos=[ex["cur_pos"]],
        centre=np.array(ex["centre"]).reshape(1, 1, 2, 2),
        mean_norm=np.array(ex["mean_norm"]).reshape(1, 1, 2),
        mrl=np.array(ex["mrl"]).reshape(1, 1, 2), theta=ex["theta"], budget=1,
        offsets=ex["offsets"], n_q_heads=1)
    env = {"cos": math.cos, "sin": math.sin, "pi": math.pi}
    want = [eval(e, env) for e in ex["expected_raw"]]
    out = oracle.prune(p, np.zeros_like(p.k))
    np.testing.assert_allclose(out["raw"][0, 0], want, rtol=1e-13, atol=1e-13)
    hi = int(np.argmax(want))
    np.testing.assert_array_equal(out["z"][0, 0], [1.0 if i == hi else -1.0 for i in range(T)])
    assert out["sel"][0, 0, 0].tolist() == [hi]
    assert out["seq_len"].tolist() == [1]


# ---------------------------------------------------------------------------- calibration

def test_calibration_identical_queries_concentrate_fully():
    """N identical queries: centre = q_f, mean norm = |q_f|, R = 1 (Method)."""
    rng = np.random.default_rng(1)
    q1 = rng.normal(size=(2, 1, 3, 8))
    q = np.repeat(q1, 5, axis=1)
    for layout in (0, 1):
        c, m, r = oracle.calibrate(q, layout)
        for f in range(4):
            xi, yi = (f, f + 4) if layout == 0 else (2 * f, 2 * f + 1)
            np.testing.assert_allclose(c[:, :, f, 0], q1[:, 0, :, xi], rtol=1e-14)
            np.testing.assert_allclose(c[:, :, f, 1], q1[:, 0, :, yi], rtol=1e-14)
            np.testing.assert_allclose(m[:, :, f], np.hypot(q1[:, 0, :, xi], q1[:, 0, :, yi]),
                                       rtol=1e-14)
        np.testing.assert_allclose(r, 1.0, rtol=1e-14)


def test_calibration_antipodal_and_two_directions():
    """+q/-q pairs: centre 0, R = 0.  Two equal-norm queries 2a apart: R = cos a."""
    rng = np.random.default_rng(2)
    q1 = rng.normal(size=(1, 4, 2, 6))
    c, m, r = oracle.calibrate(np.concatenate([q1, -q1], axis=1))
    assert np.abs(c).max() < 1e-15 and np.abs(r).max() < 1e-15
    a = 0.3
    q = np.zeros((1, 2, 1, 2))
    q[0, 0, 0] = [2 * math.cos(1.0 + a), 2 * math.sin(1.0 + a)]
    q[0, 1, 0] = [2 * math.cos(1.0 - a), 2 * math.sin(1.0 - a)]
    c, m, r = oracle.calibrate(q)
    np.testing.assert_allclose(r[0, 0, 0], math.cos(a), rtol=1e-14)
    np.testing.assert_allclose(m[0, 0, 0], 2.0, rtol=1e-14)
    np.testing.assert_allclose(c[0, 0, 0], [2 * math.cos(a) * math.cos(1.0),
                                            2 * math.cos(a) * math.sin(1.0)], rtol=1e-13)


def test_calibration_full_circle_has_zero_centre():
    """Queries evenly spread on a circle in one band: E[q_f] = 0, R = 0."""
    n = 12
    ang = 2 * math.pi * np.arange(n) / n + 0.1
    q = np.zeros((1, n, 1, 2))
    q[0, :, 0, 0] = 3 * np.cos(ang)
    q[0, :, 0, 1] = 3 * np.sin(ang)
    c, m, r = oracle.calibrate(q)
    assert abs(c).max() < 1e-14 and abs(r).max() < 1e-14
    np.testing.assert_allclose(m, 3.0, rtol=1e-14)


# ---------------------------------------------------------------------------- score

@pytest.mark.parametrize("layout", [0, 1])
def test_offset_mean_matches_dirichlet_closed_form(layout):
    """Pin (1): for offsets {1..N} the mean of e^{i w delta} is the Dirichlet
    kernel e^{i w (N+1)/2} sin(N w/2) / (N sin(w/2)); the term-by-term trig
    sum must equal Re sum_f conj(ktilde_f) c_f e^{i w_f cur} D_N(w_f) plus the
    norm term (Method; 2-2)."""
    N = 37
    wl, data, stats = _small(seed=3, D=16, layout=layout, offsets=range(1, N + 1))
    p = common.problem(wl, data, stats)
    c, m, r = (s.astype(np.float64) for s in stats)
    D, F = wl.head_dim, wl.head_dim // 2
    cur = int(data["cur_pos"][0])
    for (g, t) in [(0, 0), (1, 17), (0, 39)]:
        kt = _key_float(data, 0, g, t)
        for h in range(g * wl.group, (g + 1) * wl.group):
            want = 0.0
            for f in range(F):
                xi, yi = (f, f + F) if layout == 0 else (2 * f, 2 * f + 1)
                w = wl.rope_theta ** (-2.0 * f / D)
                dn = np.exp(1j * w * (N + 1) / 2) * math.sin(N * w / 2) / (N * math.sin(w / 2))
                ktf = kt[xi] + 1j * kt[yi]
                cf = c[0, h, f, 0] + 1j * c[0, h, f, 1]
                want += (np.conj(ktf) * cf * np.exp(1j * w * cur) * dn).real
                want += (1.0 - r[0, h, f]) * m[0, h, f] * abs(ktf)
            got = oracle.key_score(p, 0, h, 0, t)
            assert abs(got - want) <= 1e-12 * max(1.0, abs(want)), (g, t, h, got, want)


@pytest.mark.parametrize("layout", [0, 1])
def test_zero_spread_equals_mean_post_rope_logit(layout):
    """Pin (2): queries with zero spread (calibrated from identical samples)
    give R = 1, no norm term, and S_trig = mean over offsets of the post-RoPE
    dot product <RoPE(c, cur + delta), ktilde> (Key idea; 2-2)."""
    wl, data, _ = _small(seed=4, D=12, layout=layout, offsets=[1, 2, 5, 11, 64])
    rng = np.random.default_rng(4)
    q1 = rng.normal(size=(1, 1, wl.n_q_heads, wl.head_dim))
    stats = oracle.calibrate(np.repeat(q1, 7, axis=1), layout)
    p = oracle.Problem(k=common.bf16_bits(data["k"]), pos=data["pos"].numpy(),
                       seq_start=data["seq_start"], seq_len=data["seq_len"].numpy(),
                       cur_pos=data["cur_pos"].numpy(), centre=stats[0], mean_norm=stats[1],
                       mrl=stats[2], theta=wl.rope_theta, budget=wl.budget, offsets=wl.offsets,
                       n_q_heads=wl.n_q_heads, layout=layout)
    cur = int(data["cur_pos"][0])
    for (g, t) in [(0, 3), (1, 25)]:
        kt = _key_float(data, 0, g, t)
        for h in range(g * wl.group, (g + 1) * wl.group):
            want = np.mean([np.dot(_rope_real(q1[0, 0, h], cur + d, wl.rope_theta, layout), kt)
                            for d in wl.offsets])
            got = oracle.key_score(p, 0, h, 0, t)
            assert abs(got - want) <= 1e-12 * max(1.0, abs(want))


def test_diffuse_queries_reduce_to_weighted_key_norm():
    """Pin (5): antipodal calibration (+q, -q) gives E[q_f] = 0 and R = 0, so the
    trig term vanishes and the score is sum_f E|q_f| |k_f| (Method; 3-2 (3)(4))."""
    wl, data, _ = _small(seed=5, D=16)
    rng = np.random.default_rng(5)
    q1 = rng.normal(size=(1, 9, wl.n_q_heads, wl.head_dim))
    c, m, r = oracle.calibrate(np.concatenate([q1, -q1], axis=1))
    p = oracle.Problem(k=common.bf16_bits(data["k"]), pos=data["pos"].numpy(),
                       seq_start=data["seq_start"], seq_len=data["seq_len"].numpy(),
                       cur_pos=data["cur_pos"].numpy(), centre=c, mean_norm=m, mrl=r,
                       theta=wl.rope_theta, budget=wl.budget, offsets=wl.offsets,
                       n_q_heads=wl.n_q_heads)
    F = wl.head_dim // 2
    for (g, t) in [(0, 1), (1, 30)]:
        kt = _key_float(data, 0, g, t)
        kn = np.hypot(kt[:F], kt[F:])
        for h in range(g * wl.group, (g + 1) * wl.group):
            want = float(np.dot(m[0, h], kn))
            assert abs(oracle.key_score(p, 0, h, 0, t) - want) <= 1e-12 * want


def test_key_position_cancels():
    """Pin (8): for a fixed stored (post-RoPE) key, the key's position drops out
    of the score: un-rotating by p and measuring distance from p cancel (2-1; 2-2)."""
    wl, data, stats = _small(seed=6, D=16, theta=1.0e6)
    p1 = common.problem(wl, data, stats)
    data2 = dict(data)
    data2["pos"] = data["pos"] * 0 + torch.randint(0, 100000, data["pos"].shape, dtype=torch.int32)
    p2 = common.problem(wl, data2, stats)
    r1, r2 = oracle.raw_scores(p1), oracle.raw_scores(p2)
    np.testing.assert_allclose(r1, r2, rtol=1e-9, atol=1e-9 * np.abs(r1).max())


def test_common_shift_of_queries_and_keys():
    """Pin (3): shifting every key position and the current position by the same
    amount leaves the scores unchanged.  The shifted cache is re-encoded from
    the same pre-RoPE keys, so only the bf16 rounding of the stored keys
    differs (relative 2^-8 per element)."""
    wl = workloads.custom("shift", L=1, B=1, Hq=4, Hkv=2, D=16, theta=1.0e4, budget=8,
                          offsets=range(1, 17), seq_lens=[30], seed=7, n_calib=64)
    base = workloads.generate(wl)
    stats = common.stats_fp32(base["q_calib"], 0)
    g = torch.Generator().manual_seed(99)
    L, Hkv, T, D = 1, 2, 30, 16
    kpre = torch.randn(L, Hkv, T, D, generator=g, dtype=torch.float64) + 1.0
    pos = torch.sort(torch.randperm(60, generator=g)[:T]).values.to(torch.int32).expand(L, Hkv, T)

    def scores(shift, cur):
        d = dict(base)
        d["k"] = workloads._rope_rotate(kpre, pos.to(torch.int64) + shift, wl.rope_theta,
                                        0).to(torch.bfloat16)
        d["pos"] = (pos + shift).contiguous()
        d["cur_pos"] = torch.tensor([cur + shift], dtype=torch.int32)
        return oracle.raw_scores(common.problem(wl, d, stats))

    a, b = scores(0, 59), scores(12345, 59)
    scale = np.sqrt(np.mean(a ** 2))
    assert np.abs(a - b).max() <= 2e-2 * scale
    # not vacuous: moving only the current position changes the scores far more
    wrong = scores(0, 66)
    assert np.abs(a - wrong).max() > 10 * np.abs(a - b).max()


def test_ablation_flags():
    """Ablations (Comparison section; 5-3): without the trig term the score is
    the (1-R)-weighted norm term; without concentration weighting the norm term
    uses E|q_f| alone."""
    wl, data, stats = _small(seed=8, D=16)
    c, m, r = (s.astype(np.float64) for s in stats)
    F = wl.head_dim // 2
    p0 = common.problem(wl, data, stats, flags=oracle.NO_TRIG)
    p1 = common.problem(wl, data, stats, flags=oracle.NO_CONC_WEIGHT)
    pf = common.problem(wl, data, stats)
    kt = _key_float(data, 0, 1, 11)
    kn = np.hypot(kt[:F], kt[F:])
    h = wl.group + 1
    want_norm = float(np.dot((1 - r[0, h]) * m[0, h], kn))
    assert abs(oracle.key_score(p0, 0, h, 0, 11) - want_norm) <= 1e-12 * abs(want_norm)
    full = oracle.key_score(pf, 0, h, 0, 11)
    trig = full - want_norm
    want1 = trig + float(np.dot(m[0, h], kn))
    assert abs(oracle.key_score(p1, 0, h, 0, 11) - want1) <= 1e-12 * max(1, abs(want1))


# ---------------------------------------------------------------------------- z-score + max

def test_zscore_invariants_and_max():
    """Per (layer, seq, query head) z has mean 0 and population std 1; the key
    score is the max of z over its GQA group (Method; 3-2 (6))."""
    wl, data, stats = _small(seed=9, D=16, G=3, Hkv=2, T=50, B=2, L=2,
                             seq_lens=[50, 33])
    p = common.problem(wl, data, stats)
    raw = oracle.raw_scores(p)
    z, score = oracle.zmax(p, raw)
    for l in range(2):
        for b, T in enumerate([50, 33]):
            s0 = data["seq_start"][b]
            for h in range(wl.n_q_heads):
                zz = z[l, h, s0:s0 + T]
                assert abs(zz.mean()) < 1e-13 and abs(zz.std() - 1) < 1e-13
            for g in range(wl.n_kv_heads):
                grp = z[l, g * 3:(g + 1) * 3, s0:s0 + T]
                np.testing.assert_array_equal(score[l, g, s0:s0 + T], grp.max(axis=0))


def test_zscore_degenerate_head_is_zero():
    """sigma = 0 gives z = 0: a head with zero statistics scores every key 0, so
    the group score is max(z_other, 0)."""
    wl, data, stats = _small(seed=10, D=16, G=2, Hkv=1, T=30)
    c, m, r = (s.copy() for s in stats)
    c[0, 1] = 0.0
    m[0, 1] = 0.0
    p = common.problem(wl, data, (c, m, r))
    raw = oracle.raw_scores(p)
    assert np.all(raw[0, 1, :30] == 0.0)
    z, score = oracle.zmax(p, raw)
    assert np.all(z[0, 1, :30] == 0.0)
    np.testing.assert_array_equal(score[0, 0, :30], np.maximum(z[0, 0, :30], 0.0))


def test_single_head_group_keeps_raw_ranking():
    """Pin (6): with G = 1 the z-score is a positive affine map of the raw score."""
    wl, data, stats = _small(seed=11, D=16, G=1, Hkv=3, T=64)
    p = common.problem(wl, data, stats)
    raw = oracle.raw_scores(p)
    _, score = oracle.zmax(p, raw)
    for g in range(3):
        assert np.array_equal(np.argsort(raw[0, g, :64], kind="stable"),
                              np.argsort(score[0, g, :64], kind="stable"))


def test_positive_scaling_of_head_statistics_leaves_z_unchanged():
    """Pin (7): scaling one head's centre and mean norm by alpha > 0 scales its
    raw scores by alpha, which the z-score removes."""
    wl, data, stats = _small(seed=12, D=16)
    c, m, r = (s.astype(np.float64) for s in stats)
    p1 = common.problem(wl, data, (c, m, r))
    c2, m2 = c.copy(), m.copy()
    c2[0, 1] *= 3.7
    m2[0, 1] *= 3.7
    p2 = common.problem(wl, data, (c2, m2, r))
    r1, r2 = oracle.raw_scores(p1), oracle.raw_scores(p2)
    np.testing.assert_allclose(r2[0, 1, :40], 3.7 * r1[0, 1, :40], rtol=1e-12)
    z1, _ = oracle.zmax(p1, r1)
    z2, _ = oracle.zmax(p2, r2)
    np.testing.assert_allclose(z1[:, :, :40], z2[:, :, :40], rtol=1e-11, atol=1e-11)


# ---------------------------------------------------------------------------- select / compact

def _brute_select(score, budget):
    T = len(score)
    if T <= budget:
        return list(range(T))
    keep = []
    for t in range(T):
        better = sum(1 for u in range(T) if score[u] > score[t] or (score[u] == score[t] and u < t))
        if better < budget:
            keep.append(t)
    return keep


@pytest.mark.parametrize("T,budget", [(64, 7), (64, 63), (5, 9), (33, 33), (1, 1), (40, 1)])
def test_select_equals_brute_force_with_ties(T, budget):
    """Pin (4): top-budget by (score desc, slot asc) equals a brute-force count of
    better keys, including injected exact ties (Method; 3-2 (5))."""
    rng = np.random.default_rng(T * 100 + budget)
    p = oracle.Problem(k=np.zeros((1, 1, T, 2), np.uint16), pos=np.arange(T, dtype=np.int32)[None, None],
                       seq_start=[0, T], seq_len=[T], cur_pos=[T], centre=np.zeros((1, 1, 1, 2)),
                       mean_norm=np.zeros((1, 1, 1)), mrl=np.zeros((1, 1, 1)), theta=1e4,
                       budget=budget, offsets=[1], n_q_heads=1)
    for trial in range(5):
        sc = rng.normal(size=T)
        if T > 3:
            sc[rng.integers(0, T, size=T // 3)] = sc[0]  # exact ties with slot 0
        sel = oracle.select(p, sc.reshape(1, 1, T))[0, 0, 0]
        want = _brute_select(sc, budget)
        assert sel[:len(want)].tolist() == want
        assert np.all(sel[len(want):] == -1)


def test_compaction_moves_selected_rows_in_order():
    """Pin (9): compaction writes old[sel] in ascending order to the front of each
    segment, sets seq_len to the number kept, and leaves sequences at or under
    the budget untouched (Method: prune back to budget)."""
    wl, data, stats = _small(seed=13, D=16, G=2, Hkv=2, T=40, B=3, budget=10,
                             seq_lens=[40, 10, 7])
    p = common.problem(wl, data, stats)
    out = oracle.prune(p, common.bf16_bits(data["v"]))
    k0, v0, pos0 = p.k, common.bf16_bits(data["v"]), p.pos
    assert out["seq_len"].tolist() == [10, 10, 7]
    for l in range(1):
        for g in range(2):
            for b, T in enumerate([40, 10, 7]):
                s0 = data["seq_start"][b]
                sel = out["sel"][l, g, b]
                n = min(T, 10)
                assert np.all(np.diff(sel[:n]) > 0) and np.all(sel[n:] == -1)
                np.testing.assert_array_equal(out["k"][l, g, s0:s0 + n], k0[l, g, s0 + sel[:n]])
                np.testing.assert_array_equal(out["v"][l, g, s0:s0 + n], v0[l, g, s0 + sel[:n]])
                np.testing.assert_array_equal(out["pos"][l, g, s0:s0 + n], pos0[l, g, s0 + sel[:n]])
                assert np.all(np.diff(out["pos"][l, g, s0:s0 + n]) > 0)
                if T <= 10:
                    np.testing.assert_array_equal(out["k"][l, g, s0:s0 + T], k0[l, g, s0:s0 + T])


def test_empty_segment_is_a_no_op():
    wl, data, stats = _small(seed=14, D=16, B=2, seq_lens=[20, 20], budget=5)
    p = common.problem(wl, data, stats, seq_len=np.array([20, 0], np.int32))
    out = oracle.prune(p, common.bf16_bits(data["v"]))
    assert out["seq_len"].tolist() == [5, 0]
    assert np.all(out["sel"][:, :, 1] == -1)
    s0 = data["seq_start"][1]
    np.testing.assert_array_equal(out["k"][:, :, s0:], p.k[:, :, s0:])


# ------------------------------------------------------- decode loop: append + windowed prune

def _decode_problem(seed, seq_lens, slack, budget, B=None):
    wl = workloads.custom("pin-decode", L=1, B=len(seq_lens), Hq=4, Hkv=2, D=16, theta=1.0e4,
                          budget=budget, offsets=list(range(1, 9)), seq_lens=seq_lens, seed=seed,
                          nu=0.5, n_calib=64, slack=slack)
    data = workloads.generate(wl)
    stats = common.stats_fp32(data["q_calib"], wl.rope_layout)
    return wl, data, stats


def test_prune_window_of_zero_or_one_is_the_plain_prune():
    """Window-based pruning (3-2 (5)) with a window of 0 or 1 prunes every
    sequence longer than the budget: it is the plain prune."""
    wl, data, stats = _decode_problem(21, [40, 11, 10], 0, 10)
    p = common.problem(wl, data, stats)
    v = common.bf16_bits(data["v"])
    a = oracle.prune(p, v)
    for w in (0, 1):
        b = oracle.prune_window(p, v, w)
        for key in ("k", "v", "pos", "seq_len", "sel"):
            np.testing.assert_array_equal(a[key], b[key])


def test_prune_window_threshold():
    """A sequence is pruned exactly when its length reaches budget + window: one
    key short it keeps everything, at the threshold it is pruned as by the plain
    prune, and a sequence within the budget is untouched either way (3-2 (5))."""
    budget, W = 10, 6
    lens = [budget + W - 1, budget + W, budget - 3]
    wl, data, stats = _decode_problem(22, lens, 0, budget)
    p = common.problem(wl, data, stats)
    v = common.bf16_bits(data["v"])
    full = oracle.prune(p, v)
    win = oracle.prune_window(p, v, W)
    assert win["seq_len"].tolist() == [budget + W - 1, budget, budget - 3]
    st = data["seq_start"]
    s0, e0 = st[0], st[1]
    np.testing.assert_array_equal(win["k"][:, :, s0:e0], p.k[:, :, s0:e0])
    np.testing.assert_array_equal(win["v"][:, :, s0:e0], v[:, :, s0:e0])
    np.testing.assert_array_equal(win["pos"][:, :, s0:e0], p.pos[:, :, s0:e0])
    assert np.all(win["sel"][:, :, 0] == -2)
    for b in (1, 2):
        s0, e0 = st[b], st[b + 1]
        for key in ("k", "v", "pos"):
            np.testing.assert_array_equal(win[key][:, :, s0:e0], full[key][:, :, s0:e0])
        np.testing.assert_array_equal(win["sel"][:, :, b], full["sel"][:, :, b])


def test_append_writes_the_next_slot_and_advances():
    """A decoded token joins the cache (Background): its rows land in slot
    seq_len[b] of every segment with position cur_pos[b] + 1, the length and the
    position advance by one, nothing else changes; a full segment is skipped."""
    rng = np.random.default_rng(5)
    L, Hkv, D = 2, 2, 8
    starts, lens, cur = [0, 5, 9, 12], [2, 3, 3], [100, 7, 50]  # segment 2 is full
    k = rng.integers(0, 1 << 16, size=(L, Hkv, 12, D), dtype=np.uint16)
    v = rng.integers(0, 1 << 16, size=(L, Hkv, 12, D), dtype=np.uint16)
    pos = rng.integers(0, 1000, size=(L, Hkv, 12), dtype=np.int32)
    kn = rng.integers(0, 1 << 16, size=(L, Hkv, 3, D), dtype=np.uint16)
    vn = rng.integers(0, 1 << 16, size=(L, Hkv, 3, D), dtype=np.uint16)
    k2, v2, pos2, sl, cp, skipped = oracle.append(k, v, pos, starts, lens, cur, kn, vn)
    assert skipped == [2]
    assert sl.tolist() == [3, 4, 3] and cp.tolist() == [101, 8, 50]
    changed = np.zeros(12, dtype=bool)
    for b in (0, 1):
        slot = starts[b] + lens[b]
        changed[slot] = True
        np.testing.assert_array_equal(k2[:, :, slot], kn[:, :, b])
        np.testing.assert_array_equal(v2[:, :, slot], vn[:, :, b])
        assert np.all(pos2[:, :, slot] == cur[b] + 1)
    np.testing.assert_array_equal(k2[:, :, ~changed], k[:, :, ~changed])
    np.testing.assert_array_equal(v2[:, :, ~changed], v[:, :, ~changed])
    np.testing.assert_array_equal(pos2[:, :, ~changed], pos[:, :, ~changed])


def test_decode_loop_lengths_follow_the_window_sawtooth():
    """One token appended per step and a windowed prune after each: a sequence
    grows by one per step until it reaches budget + W, and from then on returns
    to the budget every W steps (Method: one prune round per 128 decoded tokens,
    with W = 128).  Closed form of the length after step t for a
    start length s: s + t before the first prune, budget + (s + t - budget) mod W
    after it."""
    budget, W, steps = 8, 4, 17
    starts_len = [5, 11, 3]
    wl, data, stats = _decode_problem(23, starts_len, budget + W - min(starts_len), budget)
    rng = np.random.default_rng(9)
    k, v = common.bf16_bits(data["k"]), common.bf16_bits(data["v"])
    pos, cur = data["pos"].numpy(), data["cur_pos"].numpy()
    lens = np.array(starts_len, dtype=np.int32)
    st = data["seq_start"]
    for t in range(1, steps + 1):
        kn = common.bf16_bits(torch.randn(1, 2, 3, 16, dtype=torch.float32).to(torch.bfloat16))
        vn = rng.integers(0, 1 << 16, size=(1, 2, 3, 16), dtype=np.uint16)
        k, v, pos, lens, cur, skipped = oracle.append(k, v, pos, st, lens, cur, kn, vn)
        assert skipped == []
        c, m, r = stats
        p = oracle.Problem(k=k, pos=pos, seq_start=st, seq_len=lens, cur_pos=cur,
                           centre=c.astype(np.float64), mean_norm=m.astype(np.float64),
                           mrl=r.astype(np.float64), theta=wl.rope_theta, budget=budget,
                           offsets=wl.offsets, n_q_heads=wl.n_q_heads)
        out = oracle.prune_window(p, v, W)
        k, v, pos, lens = out["k"], out["v"], out["pos"], out["seq_len"]
        for b, s in enumerate(starts_len):
            want = s + t if s + t < budget + W else budget + (s + t - budget) % W
            assert lens[b] == want, (t, b, lens[b], want)
            seg = pos[0, 0, st[b]:st[b] + lens[b]]
            assert np.all(np.diff(seg) > 0)  # kept positions stay in order


# ------------------------------------------------- decode attention over the pruned cache

def _bits(x):
    """bf16-exact float values -> their bf16 bit patterns"""
    return (np.asarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _attn_arrays(rng, L, Hkv, G, D, lens, slack=2):
    starts = [0]
    for t in lens:
        starts.append(starts[-1] + t + slack)
    cap = starts[-1]
    k = _bits(rng.integers(-8, 9, size=(L, Hkv, cap, D)) / 4.0)  # exact in bf16
    v = _bits(rng.integers(-8, 9, size=(L, Hkv, cap, D)) / 4.0)
    q = _bits(rng.integers(-8, 9, size=(len(lens), Hkv * G, D)) / 8.0)
    return k, v, q, starts


def test_attention_single_key_returns_its_value():
    """With one live key the softmax weight is 1: the output is that key's value."""
    rng = np.random.default_rng(31)
    k, v, q, st = _attn_arrays(rng, 2, 2, 2, 8, [1, 1])
    out = oracle.decode_attention(k, v, st, [1, 1], 1, q, 0.3)
    for b in range(2):
        for h in range(4):
            np.testing.assert_array_equal(out[b, h], common.bits_to_float(v[1, h // 2, st[b]]))


def test_attention_two_keys_closed_form():
    """Two keys with logits a, b weigh their values by 1/(1+e^(b-a)) and 1/(1+e^(a-b))."""
    k = _bits(np.array([[[[2, 0, 0, 0], [-1, 0, 0, 0]]]], dtype=np.float32))
    v = _bits(np.array([[[[1, 0, 0, 0], [0, 1, 0, 0]]]], dtype=np.float32))
    q = _bits(np.array([[[1, 0, 0, 0]]], dtype=np.float32))
    out = oracle.decode_attention(k, v, [0, 2], [2], 0, q, 0.5)  # logits 1 and -0.5
    w0 = 1.0 / (1.0 + math.exp(-1.5))
    np.testing.assert_allclose(out[0, 0], [w0, 1.0 - w0, 0.0, 0.0], rtol=0, atol=1e-15)


def test_attention_equal_keys_average_the_values():
    """Equal keys get equal weights: the output is the mean of the values."""
    rng = np.random.default_rng(32)
    k, v, q, st = _attn_arrays(rng, 1, 1, 2, 8, [7])
    k[0, 0, :] = k[0, 0, 0]
    out = oracle.decode_attention(k, v, st, [7], 0, q, 0.7)
    want = common.bits_to_float(v[0, 0, 0:7]).mean(axis=0)
    for h in range(2):
        np.testing.assert_allclose(out[0, h], want, rtol=0, atol=1e-14)


def test_attention_query_heads_read_their_own_kv_head():
    """Query head h attends with KV head h // G: zero values in KV head 1 give zero
    outputs for its query heads and only for them (GQA grouping)."""
    rng = np.random.default_rng(33)
    k, v, q, st = _attn_arrays(rng, 1, 2, 2, 8, [9])
    v[0, 1] = 0
    v[0, 0] = _bits(rng.integers(1, 9, size=v[0, 0].shape) / 4.0)  # positive values
    out = oracle.decode_attention(k, v, st, [9], 0, q, 0.4)
    assert np.all(out[0, 2:4] == 0) and np.all(out[0, 0:2] > 0)


def test_attention_ignores_slot_order_and_empty_sequences():
    """Permuting the live (key, value) slots leaves the output unchanged; an empty
    sequence gives zeros."""
    rng = np.random.default_rng(34)
    k, v, q, st = _attn_arrays(rng, 1, 2, 2, 8, [11, 0])
    out = oracle.decode_attention(k, v, st, [11, 0], 0, q, 0.6)
    perm = rng.permutation(11)
    k2, v2 = k.copy(), v.copy()
    k2[:, :, 0:11] = k[:, :, perm]
    v2[:, :, 0:11] = v[:, :, perm]
    out2 = oracle.decode_attention(k2, v2, st, [11, 0], 0, q, 0.6)
    np.testing.assert_allclose(out2, out, rtol=0, atol=1e-13)
    assert np.all(out[1] == 0)


def test_attention_large_logits_pick_the_best_key():
    """With very large logits the softmax is the arg-max: the output is the value of
    the key most aligned with the query, and stays finite."""
    k = _bits(np.array([[[[1, 0], [3, 0], [-2, 0]]]], dtype=np.float32))
    v = _bits(np.array([[[[5, 6], [7, 8], [9, 10]]]], dtype=np.float32))
    q = _bits(np.array([[[4, 0]]], dtype=np.float32))
    out = oracle.decode_attention(k, v, [0, 3], [3], 0, q, 1.0e4)
    assert np.all(np.isfinite(out))
    np.testing.assert_array_equal(out[0, 0], [7.0, 8.0])


@pytest.mark.parametrize("layout,offsets,flags", [
    (0, range(1, 33), 0), (1, [2 ** i for i in range(17)], 0), (0, [3, 1, 200, 7], 0),
    (0, range(1, 9), oracle.NO_TRIG), (1, range(1, 9), oracle.NO_CONC_WEIGHT)])
def test_folded_scores_equal_term_by_term(layout, offsets, flags):
    """The folded CPU path (one weight per head and pair, no per-key trigonometry)
    equals the term-by-term scores: the key position cancels (2-1; 2-2), the offset
    mean factors out of the sum (Method).  Checked on ragged sequences with
    positions far from 0, both layouts, the pages' geometric offsets and both
    ablation flags."""
    wl, data, stats = _small(seed=21, D=16, B=2, seq_lens=[40, 23], offsets=offsets,
                             layout=layout, theta=1.0e6)
    data["pos"] = data["pos"] + 50000
    data["cur_pos"] = data["cur_pos"] + 50000
    p = common.problem(wl, data, stats, flags=flags)
    a, b = oracle.raw_scores(p), oracle.raw_scores_folded(p)
    live = ~np.isnan(a)
    assert np.array_equal(live, ~np.isnan(b))
    scale = np.abs(a[live]).max()
    np.testing.assert_allclose(b[live], a[live], rtol=0, atol=1e-10 * scale)


# ------------------------------------------------------- head-specific budgets
# romaanj.github.io review, "Future work": refined compression with budgets per head.
# The pages give no rule for choosing them, so they are an input per (layer, KV head);
# once heads keep different numbers of keys every unit has its own length.

def _budget_problem(seed, budgets, unit_len, seq_lens, budget_max, L=2, Hkv=3):
    wl = workloads.custom("pin-heads", L=L, B=len(seq_lens), Hq=2 * Hkv, Hkv=Hkv, D=16,
                          theta=1.0e4, budget=budget_max, offsets=list(range(1, 9)),
                          seq_lens=seq_lens, seed=seed, nu=0.5, n_calib=64)
    data = workloads.generate(wl)
    stats = common.stats_fp32(data["q_calib"], wl.rope_layout)
    c, m, r = stats
    p = oracle.Problem(k=common.bf16_bits(data["k"]), pos=data["pos"].numpy(),
                       seq_start=data["seq_start"], seq_len=data["seq_len"].numpy(),
                       cur_pos=data["cur_pos"].numpy(), centre=c.astype(np.float64),
                       mean_norm=m.astype(np.float64), mrl=r.astype(np.float64),
                       theta=wl.rope_theta, budget=budget_max, offsets=wl.offsets,
                       n_q_heads=wl.n_q_heads, budgets=budgets, unit_len=unit_len)
    return wl, data, stats, p


def test_uniform_head_budgets_are_the_plain_prune():
    """Every head at the same budget, every unit at its sequence's length: the
    per-head prune is the plain prune, byte for byte."""
    lens = [40, 12, 9]
    wl, data, stats, p = _budget_problem(31, np.full((2, 3), 10), np.broadcast_to(
        np.array(lens, np.int32), (2, 3, 3)), lens, 10)
    plain = oracle.prune(common.problem(wl, data, stats), common.bf16_bits(data["v"]))
    heads = oracle.prune(p, common.bf16_bits(data["v"]))
    for key in ("raw", "score", "sel", "k", "v", "pos", "unit_len"):
        np.testing.assert_array_equal(np.nan_to_num(plain[key], nan=-7.0),
                                      np.nan_to_num(heads[key], nan=-7.0), err_msg=key)


def test_head_budgets_keep_each_heads_top_b():
    """Ragged budgets and ragged unit lengths: each unit keeps exactly the top
    min(T_u, b_h) keys of its own scores (brute-force count of better keys, ties to
    the lower slot), in slot order; a head whose budget is at least the unit's
    length keeps the unit untouched; the z-score runs over the unit's own live
    keys (mean 0, population std 1 per query head)."""
    rng = np.random.default_rng(32)
    seq_lens = [30, 30]
    budgets = np.array([[4, 30, 11], [1, 7, 29]], np.int32)
    unit_len = rng.integers(5, 31, size=(2, 3, 2)).astype(np.int32)
    unit_len[0, 1, 0] = 30
    wl, data, stats, p = _budget_problem(33, budgets, unit_len, seq_lens, 30)
    v = common.bf16_bits(data["v"])
    out = oracle.prune(p, v)
    G = wl.group
    for l in range(2):
        for g in range(3):
            for b in range(2):
                T, bud = int(unit_len[l, g, b]), int(budgets[l, g])
                s0 = data["seq_start"][b]
                for h in range(g * G, (g + 1) * G):
                    z = out["z"][l, h, s0:s0 + T]
                    assert abs(z.mean()) < 1e-12 and abs(z.std() - 1.0) < 1e-12
                    assert np.all(np.isnan(out["z"][l, h, s0 + T:data["seq_start"][b + 1]]))
                sc = out["score"][l, g, s0:s0 + T]
                want = _brute_select(sc, bud)
                sel = out["sel"][l, g, b]
                assert sel[:len(want)].tolist() == want and np.all(sel[len(want):] == -1)
                n = min(T, bud)
                assert out["unit_len"][l, g, b] == n
                np.testing.assert_array_equal(out["k"][l, g, s0:s0 + n], p.k[l, g, s0 + sel[:n]])
                np.testing.assert_array_equal(out["v"][l, g, s0:s0 + n], v[l, g, s0 + sel[:n]])
                if T <= bud:  # untouched
                    np.testing.assert_array_equal(out["k"][l, g, s0:s0 + 30], p.k[l, g, s0:s0 + 30])


def test_head_budget_window_decides_per_unit():
    """With per-head budgets the prune window applies to each unit: a unit is pruned
    once its length reaches its own budget + window, else left as it is."""
    budgets = np.array([[5, 9]], np.int32)
    unit_len = np.array([[[9, 8]], [[12, 13]]], np.int32).reshape(1, 2, 2)
    wl, data, stats, p = _budget_problem(34, budgets, unit_len, [20, 20], 12, L=1, Hkv=2)
    v = common.bf16_bits(data["v"])
    full = oracle.prune(p, v)
    win = oracle.prune_window(p, v, 4)
    # head 0 (budget 5): 9 >= 5 + 4 is pruned, 8 is held back; head 1 (budget 9): 12 < 13
    # is held back, 13 is pruned
    assert win["unit_len"].tolist() == [[[5, 8], [12, 9]]]
    assert np.all(win["sel"][0, 0, 1] == -2) and np.all(win["sel"][0, 1, 0] == -2)
    np.testing.assert_array_equal(win["sel"][0, 0, 0], full["sel"][0, 0, 0])
    np.testing.assert_array_equal(win["sel"][0, 1, 1], full["sel"][0, 1, 1])
    s1 = data["seq_start"][1]
    np.testing.assert_array_equal(win["k"][0, 0, s1:], p.k[0, 0, s1:])


def test_append_and_attention_follow_each_units_length():
    """Per-unit lengths: a decoded token lands at each unit's own next slot, every
    unit grows by one; a sequence with a full unit is skipped whole; attention reads
    each unit's live slots only."""
    rng = np.random.default_rng(35)
    L, Hkv, D = 1, 2, 8
    starts, cur = [0, 6, 10], [40, 70]
    ul = np.array([[[3, 4], [5, 2]]], np.int32)            # [L][Hkv][B]; unit (0,1,1) has room
    k = rng.integers(0, 1 << 16, size=(L, Hkv, 10, D), dtype=np.uint16) & 0x3FFF
    v = rng.integers(0, 1 << 16, size=(L, Hkv, 10, D), dtype=np.uint16) & 0x3FFF
    pos = rng.integers(0, 100, size=(L, Hkv, 10), dtype=np.int32)
    kn = rng.integers(0, 1 << 16, size=(L, Hkv, 2, D), dtype=np.uint16) & 0x3FFF
    vn = rng.integers(0, 1 << 16, size=(L, Hkv, 2, D), dtype=np.uint16) & 0x3FFF
    k2, v2, pos2, ul2, cp, skipped = oracle.append(k, v, pos, starts, None, cur, kn, vn, unit_len=ul)
    assert skipped == [1] and cp.tolist() == [41, 70]     # segment 1 holds 4 slots; unit (0,0,1) full
    assert ul2.tolist() == [[[4, 4], [6, 2]]]
    for g in range(2):
        slot = ul[0, g, 0]
        np.testing.assert_array_equal(k2[0, g, slot], kn[0, g, 0])
        assert pos2[0, g, slot] == 41
    q = rng.integers(0, 1 << 16, size=(2, 4, D), dtype=np.uint16) & 0x3FFF
    out = oracle.decode_attention(k2, v2, starts, None, 0, q, 0.3, unit_len=ul2)
    for b in range(2):
        for h in range(4):
            g = h // 2
            T = ul2[0, g, b]
            one = oracle.decode_attention(k2[:, g:g + 1], v2[:, g:g + 1], starts, [T if bb == b else 0 for bb in range(2)],
                                          0, q[:, h:h + 1], 0.3)
            np.testing.assert_allclose(out[b, h], one[b, 0], rtol=1e-12, atol=0)

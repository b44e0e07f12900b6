"""GPU parity of the decode-loop steps against the oracle: tria_append, the
windowed tria_prune (dimensionstp.github.io review, section 3-2 (5): prune back
to the budget once per window of decoded tokens), and a decode loop of both,
run eagerly and replayed from a CUDA graph.

Tolerances as in test_gpu_parity: appended rows, lengths, positions and every
row a step does not select from are bit-exact; a pruned unit's selection equals
the oracle's except for keys within the score tolerance of the budget-th
oracle score; the compacted rows are bit-exact given the selection."""
import math

import numpy as np
import pytest
import torch

import oracle
from kv_cache_eviction_trig_b200 import tria, workloads
from tests import common
from tests.test_gpu_parity import Case, small, z_tolerance

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from kv_cache_eviction_trig_b200 import build
    build.build()
    tria.lib()


def _new_tokens(case, cur_next, gen):
    """One new token per sequence, drawn like the cache's keys (the KV head's
    centre plus noise, rotated to position cur_next[b]) and values ~ N(0, 1):
    bf16 [L][Hkv][B][D] on the host."""
    wl = case.wl
    L, Hkv, B, D = wl.num_layers, wl.n_kv_heads, wl.batch, wl.head_dim
    kc = case.host["k_centre"].double()
    nu = torch.tensor([wl.kv_noise(g) for g in range(Hkv)], dtype=torch.float64)
    scale = nu * kc.norm(dim=-1) / math.sqrt(D)
    noise = torch.randn(L, Hkv, B, D, generator=gen, dtype=torch.float64)
    pre = kc.unsqueeze(2) + scale[..., None, None] * noise
    p = torch.tensor(cur_next, dtype=torch.int64).view(1, 1, B).expand(L, Hkv, B)
    k = workloads._rope_rotate(pre, p, wl.rope_theta, wl.rope_layout).to(torch.bfloat16)
    v = torch.randn(L, Hkv, B, D, generator=gen, dtype=torch.float32).to(torch.bfloat16)
    return k.contiguous(), v.contiguous()


def _state(case):
    d = case.dev
    return {"k": common.bf16_bits(d["k"]), "v": common.bf16_bits(d["v"]),
            "pos": d["pos"].cpu().numpy(), "seq_len": d["seq_len"].cpu().numpy(),
            "cur_pos": d["cur_pos"].cpu().numpy()}


class _Lens:
    """What z_tolerance reads: the segments and their current lengths."""

    def __init__(self, wl, starts, lens):
        self.wl, self.host, self.lens = wl, {"seq_start": starts}, [int(t) for t in lens]


def _problem(case, k, pos, lens, cur):
    c, m, r = case.stats_np
    wl = case.wl
    return oracle.Problem(k=k, pos=pos, seq_start=case.host["seq_start"], seq_len=lens,
                          cur_pos=cur, centre=c.astype(np.float64),
                          mean_norm=m.astype(np.float64), mrl=r.astype(np.float64),
                          theta=wl.rope_theta, budget=wl.budget, offsets=wl.offsets,
                          n_q_heads=wl.n_q_heads, layout=wl.rope_layout)


def _check_windowed(case, window, before, after, gsel, ref):
    """`after` (GPU state) against the oracle's windowed prune `ref` of `before`."""
    wl = case.wl
    budget = wl.budget
    starts = case.host["seq_start"]
    lens = before["seq_len"]
    assert after["seq_len"].tolist() == ref["seq_len"].tolist()
    tol_case = _Lens(wl, starts, lens)
    for l in range(wl.num_layers):
        for g in range(wl.n_kv_heads):
            for b in range(wl.batch):
                s0, e0, T = starts[b], starts[b + 1], int(lens[b])
                row = gsel[l, g, b]
                if T < budget + max(window, 1):
                    for n in ("k", "v", "pos"):
                        assert np.array_equal(after[n][l, g, s0:e0], before[n][l, g, s0:e0]), (n, l, g, b)
                    if T <= budget:
                        assert row[:T].tolist() == list(range(T)) and np.all(row[T:] == -1)
                    else:
                        assert np.all(row == -7)  # held back: the row is not written
                    continue
                want = ref["sel"][l, g, b]
                assert np.all(np.diff(row) > 0) and row[0] >= 0 and row[-1] < T
                sc = ref["score"][l, g, s0:s0 + T]
                thr = np.sort(sc)[-budget]
                tol = z_tolerance(ref["raw"], sc, tol_case, l, g, b)
                for t in set(row.tolist()) ^ set(want.tolist()):
                    assert abs(sc[t] - thr) <= tol[t], (l, g, b, t, sc[t], thr)
                idx = s0 + row
                for n in ("k", "v", "pos"):
                    assert np.array_equal(after[n][l, g, s0:s0 + budget], before[n][l, g, idx]), n
                    assert np.array_equal(after[n][l, g, s0 + budget:e0],
                                          before[n][l, g, s0 + budget:e0]), n


def test_append_matches_oracle():
    wl = small("append", L=2, B=3, seq_lens=[300, 120, 301], budget=50, slack=2)
    case = Case(wl, seq_len=[300, 120, 303])  # the third segment is full
    case.cache = tria.Cache.from_data(case.dev)
    gen = torch.Generator().manual_seed(7)
    kn, vn = _new_tokens(case, (case.host["cur_pos"] + 1).tolist(), gen)
    before = _state(case)
    tria.tria_append(case.cfg, case.cache, kn.cuda(), vn.cuda(), case.ws)
    torch.cuda.synchronize()
    assert tria.tria_get_device_error(case.ws) == tria.DEVERR_SEGMENT_FULL
    k2, v2, pos2, sl, cp, skipped = oracle.append(
        before["k"], before["v"], before["pos"], case.host["seq_start"], before["seq_len"],
        before["cur_pos"], common.bf16_bits(kn), common.bf16_bits(vn))
    assert skipped == [2]
    after = _state(case)
    assert np.array_equal(after["k"], k2) and np.array_equal(after["v"], v2)
    assert np.array_equal(after["pos"], pos2)
    assert after["seq_len"].tolist() == sl.tolist() == [301, 121, 303]
    assert after["cur_pos"].tolist() == cp.tolist()


@pytest.mark.parametrize("fused", [False, True], ids=["kernels3", "fused"])
def test_prune_window_matches_oracle(fused):
    budget, W = 100, 40
    wl = small("window", B=4, seq_lens=[139, 140, 90, 500], budget=budget, slack=5)
    case = Case(wl)
    cfg = tria.Config.from_workload(wl, prune_window=W, flags=tria.FUSED_PRUNE if fused else 0)
    case.ws = tria.workspace(cfg, case.cache)
    before = _state(case)
    ref = oracle.prune_window(case.prob, before["v"], W)
    sel = torch.full((1, 2, 4, budget), -7, dtype=torch.int32, device="cuda")
    tria.tria_prune(cfg, case.stats, case.cache, case.ws, sel_out=sel)
    torch.cuda.synchronize()
    assert tria.tria_get_device_error(case.ws) == 0
    assert case.dev["seq_len"].cpu().tolist() == [139, 100, 90, 100]
    _check_windowed(case, W, before, _state(case), sel.cpu().numpy(), ref)


@pytest.mark.parametrize("fused", [False, True], ids=["kernels3", "fused"])
def test_decode_loop_matches_oracle_and_its_cuda_graph(fused):
    """40 decode steps (append, then the windowed prune) on three ragged
    sequences: every step against the oracle run from the GPU's state before it,
    and the same loop replayed from one captured CUDA graph ends bit-identical."""
    budget, W, steps = 48, 16, 40
    wl = small("decode", L=2, B=3, Hq=4, Hkv=2, D=64, theta=1e4, seq_lens=[40, 60, 63],
               budget=budget, slack=26, offsets=range(1, 33))
    a = Case(wl)
    cfg = tria.Config.from_workload(wl, prune_window=W, flags=tria.FUSED_PRUNE if fused else 0)
    a.ws = tria.workspace(cfg, a.cache)
    gen = torch.Generator().manual_seed(11)
    tokens, cur = [], a.host["cur_pos"].clone()
    for _ in range(steps):
        cur = cur + 1
        tokens.append(_new_tokens(a, cur.tolist(), gen))

    sel_a = torch.empty((2, 2, 3, budget), dtype=torch.int32, device="cuda")
    pruned_steps = 0
    for kn, vn in tokens:
        before = _state(a)
        sel_a.fill_(-7)
        tria.tria_append(cfg, a.cache, kn.cuda(), vn.cuda(), a.ws)
        tria.tria_prune(cfg, a.stats, a.cache, a.ws, sel_out=sel_a)
        torch.cuda.synchronize()
        assert tria.tria_get_device_error(a.ws) == 0
        k1, v1, pos1, sl1, cp1, skipped = oracle.append(
            before["k"], before["v"], before["pos"], a.host["seq_start"], before["seq_len"],
            before["cur_pos"], common.bf16_bits(kn), common.bf16_bits(vn))
        assert skipped == []
        ref = oracle.prune_window(_problem(a, k1, pos1, sl1, cp1), v1, W)
        appended = {"k": k1, "v": v1, "pos": pos1, "seq_len": sl1, "cur_pos": cp1}
        after = _state(a)
        assert after["cur_pos"].tolist() == cp1.tolist()
        _check_windowed(a, W, appended, after, sel_a.cpu().numpy(), ref)
        pruned_steps += int(np.any(sl1 >= budget + W))
    assert pruned_steps == 8  # sequences reach budget + W at steps 1, 4, 17, 20, 24, 33, 36, 40

    b = Case(wl)
    b.ws = tria.workspace(cfg, b.cache)
    kbuf = torch.empty_like(tokens[0][0], device="cuda")
    vbuf = torch.empty_like(tokens[0][1], device="cuda")
    sel_b = torch.empty_like(sel_a)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        tria.tria_append(cfg, b.cache, kbuf, vbuf, b.ws)
        tria.tria_prune(cfg, b.stats, b.cache, b.ws, sel_out=sel_b)
    for kn, vn in tokens:
        kbuf.copy_(kn)
        vbuf.copy_(vn)
        graph.replay()
    torch.cuda.synchronize()
    assert tria.tria_get_device_error(b.ws) == 0
    for n in ("k", "v", "pos", "seq_len", "cur_pos"):
        assert torch.equal(a.dev[n], b.dev[n]), n
    del graph


# --------------------------------------------------- decode attention over the pruned cache

ATT_RTOL = ATT_ATOL = 1e-4  # float32 dot products and weights against float64


def _queries(case, layer, gen):
    """One post-RoPE query per (sequence, query head), drawn like the calibration
    queries (the head's centre plus noise) and rotated to position cur_pos + 1:
    bf16 [B][Hq][D] on the device."""
    wl = case.wl
    B, Hq, D = wl.batch, wl.n_q_heads, wl.head_dim
    qc = case.host["q_centre"][layer].double()                       # [Hq, D]
    noise = torch.randn(B, Hq, D, generator=gen, dtype=torch.float64)
    pre = qc.unsqueeze(0) + 0.3 * qc.norm(dim=-1).view(1, Hq, 1) / math.sqrt(D) * noise
    p = (case.host["cur_pos"].to(torch.int64) + 1).view(B, 1).expand(B, Hq)
    q = workloads._rope_rotate(pre, p, wl.rope_theta, wl.rope_layout).to(torch.bfloat16)
    return q.contiguous().cuda()


def _check_attention(case, layer, q, out, scale):
    st = _state(case)
    ref = oracle.decode_attention(st["k"], st["v"], case.host["seq_start"], st["seq_len"], layer,
                                  common.bf16_bits(q), scale)
    got = out.double().cpu().numpy()
    assert np.allclose(got, ref, rtol=ATT_RTOL, atol=ATT_ATOL), float(np.abs(got - ref).max())
    return ref


ATT_CASES = {
    "d128_g4_ragged": lambda: small("att1", L=2, B=3, seq_lens=[2100, 1, 300]),
    "d64_g8": lambda: small("att2", D=64, Hq=8, Hkv=1, seq_lens=[515], theta=1e4),
    "d256_g1": lambda: small("att3", D=256, Hq=4, Hkv=4, seq_lens=[300]),
    "d128_g16_with_empty": lambda: small("att4", Hq=16, Hkv=1, B=2, seq_lens=[130, 0]),
    "d64_interleaved_g2": lambda: small("att5", D=64, Hq=4, Hkv=2, seq_lens=[700], theta=1e4,
                                        rope_layout=workloads.INTERLEAVED),
    # long segments over few (sequence, KV head) pairs: on the tensor-core path each pair's
    # keys spread over four 4-CTA clusters (stages reused), merged by the pair's last CTA;
    # a ragged last tile
    "d128_g4_long": lambda: small("att6", Hq=8, Hkv=2, seq_lens=[12001]),
    "d64_g2_long": lambda: small("att7", D=64, Hq=4, Hkv=2, seq_lens=[9000], theta=1e4),
    # G = 16 at D = 256 scores in two passes of 8 query heads
    "d256_g16_long": lambda: small("att8", D=256, Hq=16, Hkv=1, seq_lens=[3000]),
    # more pairs than SMs, ragged: one CTA per pair, no cluster
    "d128_g4_many_sequences": lambda: small("att9", B=80, Hq=8, Hkv=2,
                                            seq_lens=[700 - (b % 7) * 50 for b in range(80)]),
    # empty sequences around a long one: zero rows from split pairs with nothing to merge
    "d128_g4_empty_and_long": lambda: small("att10", Hq=8, Hkv=2, B=3, seq_lens=[0, 20000, 0]),
    # many pairs (1040): one CTA per pair, several waves
    "d64_g4_over_1024_pairs": lambda: small("att11", D=64, Hq=32, Hkv=8, B=130, theta=1e4,
                                            seq_lens=[1 + (b * 37) % 300 for b in range(130)]),
}


@pytest.mark.parametrize("name", sorted(ATT_CASES))
def test_decode_attention_matches_oracle(name):
    case = Case(ATT_CASES[name]())
    wl = case.wl
    layer = wl.num_layers - 1
    q = _queries(case, layer, torch.Generator().manual_seed(5))
    out = torch.full((wl.batch, wl.n_q_heads, wl.head_dim), float("nan"), device="cuda")
    tria.tria_decode_attention(case.cfg, case.cache, layer, q, out, case.ws)
    torch.cuda.synchronize()
    assert tria.tria_get_device_error(case.ws) == 0
    ref = _check_attention(case, layer, q, out, wl.head_dim ** -0.5)
    for b, T in enumerate(case.lens):
        if T == 0:
            assert torch.all(out[b] == 0)
        assert np.abs(ref[b]).max() > 0 or T == 0


def test_decode_attention_reads_the_pruned_cache():
    """Attention after a prune (the pruned cache is what decoding reads), with a
    scale other than 1/sqrt(D)."""
    case = Case(small("att-pruned", L=2, B=2, seq_lens=[1000, 333], budget=100, slack=5))
    tria.tria_prune(case.cfg, case.stats, case.cache, case.ws)
    q = _queries(case, 1, torch.Generator().manual_seed(6))
    out = torch.empty((2, case.wl.n_q_heads, case.wl.head_dim), device="cuda")
    tria.tria_decode_attention(case.cfg, case.cache, 1, q, out, case.ws, scale=0.05)
    torch.cuda.synchronize()
    assert tria.tria_get_device_error(case.ws) == 0
    assert case.dev["seq_len"].cpu().tolist() == [100, 100]
    _check_attention(case, 1, q, out, 0.05)


def test_decode_attention_flags_a_bad_length_and_skips_that_sequence():
    case = Case(small("att-bad", B=2, seq_lens=[300, 300], budget=50), seq_len=[300, 303])
    case.cache = tria.Cache.from_data(case.dev)
    q = _queries(case, 0, torch.Generator().manual_seed(7))
    out = torch.full((2, case.wl.n_q_heads, case.wl.head_dim), 7.0, device="cuda")
    tria.tria_decode_attention(case.cfg, case.cache, 0, q, out, case.ws)
    torch.cuda.synchronize()
    assert tria.tria_get_device_error(case.ws) & tria.DEVERR_SEQ_LEN
    assert torch.all(out[1] == 7.0)        # the bad sequence's rows are not written
    assert not torch.any(out[0] == 7.0)    # the good one's are

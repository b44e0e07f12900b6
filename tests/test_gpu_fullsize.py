"""Full-size workloads on the GPU, in the launch configuration the benchmark
times, checked on sampled outputs the oracle computes one by one and on
properties that hold at any size:

  * raw scores of sampled keys of sampled (layer, KV head, sequence) units
    against the oracle's term-by-term score (1e-4 relative to max(|s|, rms));
  * the group score equals max_h (s_h - mean) / std computed in float64 on
    the host from the GPU's raw scores of the whole unit;
  * the prune keeps exactly the top-`budget` of those scores (ties to the
    lower slot), in ascending order, and the compacted K/V/pos rows are
    bit-identical to the pristine rows at the kept slots.
"""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_eviction_trig_b200 import tria, workloads
from tests import common

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from kv_cache_eviction_trig_b200 import build
    build.build()
    tria.lib()


def _topk_slots(score, budget):
    order = np.lexsort((np.arange(len(score)), -score))  # score desc, slot asc
    return np.sort(order[:budget])


@pytest.mark.parametrize("index,n_units,n_keys", [(1, 8, 48), (4, 4, 12), (2, 6, 24), (3, 6, 16)])
def test_full_size_workload(index, n_units, n_keys):
    wl = workloads.workload(index)
    data = workloads.generate(wl, device="cuda")
    stats_np = common.stats_fp32(data["q_calib"], wl.rope_layout)
    del data["q_calib"]
    cfg = tria.Config.from_workload(wl)
    cache = tria.Cache.from_data(data)
    stats = tria.Stats(*[torch.from_numpy(s).cuda() for s in stats_np])
    ws = tria.workspace(cfg, cache)
    units = workloads.sample_units(wl, n_units, seed=index)
    starts = data["seq_start"]
    lens = data["seq_len"].cpu().tolist()

    # ---- scores of the whole cache
    score = torch.empty(wl.num_layers, wl.n_kv_heads, wl.cap_total, device="cuda")
    raw = torch.empty(wl.num_layers, wl.n_q_heads, wl.cap_total, device="cuda")
    tria.tria_score(cfg, stats, cache, score, raw, ws)
    torch.cuda.synchronize()
    assert tria.tria_get_device_error(ws) == 0

    # the oracle sees only the sampled units' rows (same bytes as the device)
    host_k = {}
    pristine = {}
    for (l, g, b) in units:
        s0, T = starts[b], lens[b]
        pristine[(l, g, b)] = tuple(data[n][l, g, s0:s0 + T].clone() for n in ("k", "v", "pos"))
    rng = np.random.default_rng(index)
    G = wl.group
    for (l, g, b) in units:
        s0, T = starts[b], lens[b]
        gr = raw[l, g * G:(g + 1) * G, s0:s0 + T].double().cpu().numpy()
        gs = score[l, g, s0:s0 + T].double().cpu().numpy()
        # sampled raw parity against the oracle (one-unit problem)
        kk = np.unique(np.concatenate([[0, T - 1], rng.integers(0, T, n_keys)]))
        sub = {"k": pristine[(l, g, b)][0][None, None], "pos": pristine[(l, g, b)][2][None, None],
               "seq_start": [0, T], "seq_len": torch.tensor([T], dtype=torch.int32),
               "cur_pos": data["cur_pos"][b:b + 1].cpu()}
        c, m, r = stats_np
        sl = slice(g * G, (g + 1) * G)
        prob = oracle.Problem(k=common.bf16_bits(sub["k"]), pos=sub["pos"].cpu().numpy(),
                              seq_start=[0, T], seq_len=[T], cur_pos=sub["cur_pos"].numpy(),
                              centre=c[l:l + 1, sl].astype(np.float64),
                              mean_norm=m[l:l + 1, sl].astype(np.float64),
                              mrl=r[l:l + 1, sl].astype(np.float64), theta=wl.rope_theta,
                              budget=wl.budget, offsets=wl.offsets, n_q_heads=G,
                              layout=wl.rope_layout)
        for j in range(G):
            rms = np.sqrt(np.mean(gr[j] ** 2))
            for t in kk:
                ref = oracle.key_score(prob, 0, j, 0, int(t))
                assert abs(gr[j, t] - ref) <= 1e-4 * max(abs(ref), rms), (l, g, b, j, t)
        # group max of standardised raw scores (float64 on the host)
        z = (gr - gr.mean(axis=1, keepdims=True)) / gr.std(axis=1, keepdims=True)
        want = z.max(axis=0)
        assert np.all(np.abs(gs - want) <= 1e-6 * (1 + np.abs(want)))
        host_k[(l, g, b)] = gs

    # ---- the prune, as the benchmark launches it
    sel = torch.empty(wl.num_layers, wl.n_kv_heads, wl.batch, wl.budget, dtype=torch.int32,
                      device="cuda")
    tria.tria_prune(cfg, stats, cache, ws, sel_out=sel)
    torch.cuda.synchronize()
    assert tria.tria_get_device_error(ws) == 0
    assert data["seq_len"].cpu().tolist() == [min(T, wl.budget) for T in lens]
    for (l, g, b), gs in host_k.items():
        s0, T = starts[b], lens[b]
        got = sel[l, g, b].cpu().numpy()
        assert np.array_equal(got, _topk_slots(gs, wl.budget))
        idx = torch.from_numpy(got.astype(np.int64)).cuda()
        pk, pv, pp = pristine[(l, g, b)]
        n = wl.budget
        assert torch.equal(data["k"][l, g, s0:s0 + n].view(torch.int16), pk[idx].view(torch.int16))
        assert torch.equal(data["v"][l, g, s0:s0 + n].view(torch.int16), pv[idx].view(torch.int16))
        assert torch.equal(data["pos"][l, g, s0:s0 + n], pp[idx])

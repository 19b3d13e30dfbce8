"""Oracle parity at full size for the two workloads whose reduced forms are
checked elsewhere: the 128K tiered-storage workload (history K/V and group
summaries in pinned host memory, a group-summary cache in HBM for a quarter
of the groups, the final 4096 queries) and the 32K budget sweep (top chunks 4,
8, 16, 64 and all, top groups twice that).  The GPU runs each whole workload;
the oracle recomputes sampled (query block, KV head) units: the first and last
block of every KV head plus random ones.

Sources: "Long-Context Fine-Tuning with Limited VRAM", section 2.1
(exact-token attention over the routed groups plus sink and local windows),
section 2.2 (tiered storage: history in host RAM, summaries cached in VRAM)
and section 4.5 (the top-k chunk sweep).  With every chunk and group kept,
routed attention must equal dense causal attention (the router disabled)."""
import functools

import numpy as np
import pytest
import torch

import hga_inputs as gi
from oracle import hga_oracle as ho
import parity

pytestmark = pytest.mark.gpu


def _units(w, n_random, seed=0):
    """First and last block of every KV head plus n_random (block, head)."""
    nb = -(-w.Tq // w.qblock)
    units = set()
    for h in range(w.n_kv_heads):
        units.update({(0, h), (nb - 1, h)})
    rng = np.random.default_rng(seed)
    while len(units) < 2 * w.n_kv_heads + n_random:
        units.add((int(rng.integers(nb)), int(rng.integers(w.n_kv_heads))))
    return sorted(units)


def test_tiered_128k_full_size_matches_all_hbm_and_oracle():
    from test_gpu_tier import _setup, _tiered_run
    w = gi.TIERED_128K
    hga, p, inp, q, k_all, v_all, full, tier = _setup(w)
    hga.forward(p, q, w.q0, k_all, v_all, full)           # all-HBM step
    assert hga.check() == 0
    b1 = _tiered_run(hga, p, w, q, k_all, v_all, full, tier)
    assert torch.equal(b1.chunk_idx, full.chunk_idx)
    assert torch.equal(b1.group_idx, full.group_idx)
    assert torch.equal(b1.o, full.o) and torch.equal(b1.lse, full.lse)
    hits, misses = tier.stats.tolist()
    assert hits == 0 and misses > 0                        # the first step is cold
    g = parity.GpuResult(np.zeros(1), np.zeros(1),
                         b1.chunk_idx.cpu().numpy(), b1.chunk_cnt.cpu().numpy(),
                         b1.group_idx.cpu().numpy(), b1.group_cnt.cpu().numpy(),
                         b1.o.double().cpu().numpy(), b1.lse.double().cpu().numpy())
    del k_all, v_all, full, b1, tier
    torch.cuda.empty_cache()
    units = _units(w, 8)
    rep = parity.compare(w, inp, g, units=units, check_summaries=False)
    print(w.name, rep)
    assert rep.ok(), rep
    assert rep.compared_units == len(units) == 24


@functools.lru_cache(maxsize=1)
def _sweep_inputs():
    """The sweep budgets share one set of inputs (the budget is not part of
    the input recipe), with the oracle's float64 copies and summaries."""
    w = gi.SWEEP_32K
    inp = gi.make_inputs(w)
    f64 = (gi.to_f64(inp.q), gi.to_f64(inp.k), gi.to_f64(inp.v))
    summ = ho.build_summaries(f64[1], parity.oracle_params(w), 0, w.T)
    return inp, f64, summ


@pytest.mark.parametrize("kc", gi.SWEEP_BUDGETS)
def test_sweep_32k_full_size_every_budget(kc):
    w = gi.SWEEP_32K.with_(top_chunks=kc, top_groups=2 * kc)
    inp, f64, summ = _sweep_inputs()
    g = parity.run_gpu(w, inp, v_f16=True)                # the bench's launch configuration
    units = _units(w, 6, seed=kc)
    rep = parity.compare(w, inp, g, units=units, summaries=summ, f64=f64)
    print(w.name, kc, rep)
    assert rep.ok(), rep
    assert rep.compared_units == len(units)
    if kc == 0:
        # every chunk and group kept: dense causal attention of the same rows
        q, k, v = f64
        atol, rtol = parity.TOL["bf16"]
        assert abs(rep.density - 1.0) < 1e-12
        for (b, h) in units[::3]:
            b0 = w.q0 + b * w.qblock
            b1 = min(b0 + w.qblock, w.T)
            hs = slice(h * w.G, (h + 1) * w.G)
            o_d, l_d = ho.dense_causal_attention(q[b0 - w.q0:b1 - w.q0, hs], k[h:h + 1, :b1],
                                                 v[h:h + 1, :b1], b0, w.G)
            o_g = g.o[b0 - w.q0:b1 - w.q0, hs]
            assert (np.abs(o_g - o_d) <= atol + rtol * np.abs(o_d)).all(), (b, h)
            l_g = g.lse[b0 - w.q0:b1 - w.q0, hs]
            assert (np.abs(l_g - l_d) <= atol + rtol * np.abs(l_d)).all(), (b, h)

"""Host-memory tier on a B200: history K/V and group summaries in pinned host
memory, group-summary cache in HBM, routed groups gathered on a side stream.
The tiered step must reproduce the all-HBM step exactly (indices and O), and
the oracle on sampled units; the cache must start cold and then hit."""
import numpy as np
import pytest
import torch

import hga_inputs as gi
import parity

pytestmark = pytest.mark.gpu


def _setup(w):
    from long_context_hga_b200 import hga
    p = hga.Params.from_workload(w)
    inp = gi.make_inputs(w)
    dev = torch.device("cuda:0")
    T, q0 = w.T, w.q0
    k_all = inp.k.to(dev)
    v_all = inp.v.to(dev)
    q = inp.q.to(dev)
    # commit of the history: chunk summaries stay in HBM, group summaries and
    # K/V go to pinned host memory
    full = hga.allocate(p, T, w.Tq, device=dev)
    hga.build_summaries(p, k_all, 0, q0, full.chunk_sum, full.group_sum)
    tier = hga.make_host_tier(p, inp.k.pin_memory(), inp.v.pin_memory(),
                              full.group_sum.cpu().pin_memory(), t_hist=q0)
    return hga, p, inp, q, k_all, v_all, full, tier


def _tiered_run(hga, p, w, q, k_all, v_all, full, tier):
    dev = q.device
    bufs = hga.allocate(p, w.T, w.Tq, device=dev)
    bufs.chunk_sum.copy_(full.chunk_sum)            # resident chunk summaries
    nan = torch.tensor(float("nan"), dtype=k_all.dtype, device=dev)
    bufs.group_sum.fill_(nan)                       # history rows must come from the tier
    bufs.group_sum[:, w.q0 // w.group:] = 0
    k_dev = torch.full_like(k_all, float("nan"))
    v_dev = torch.full_like(v_all, float("nan"))
    k_dev[:, w.q0:] = k_all[:, w.q0:]               # the segment's own K/V is in HBM
    v_dev[:, w.q0:] = v_all[:, w.q0:]
    hga.tiered_step(p, q, w.q0, tier, k_dev, v_dev, bufs)
    assert hga.check() == 0
    return bufs


def test_tiered_equals_all_hbm_and_oracle():
    w = gi.TIERED_128K.with_(T=12288, q0=10240, n_needles=16)
    hga, p, inp, q, k_all, v_all, full, tier = _setup(w)
    # all-HBM reference run
    hga.forward(p, q, w.q0, k_all, v_all, full)
    assert hga.check() == 0
    b1 = _tiered_run(hga, p, w, q, k_all, v_all, full, tier)
    assert torch.equal(b1.chunk_idx, full.chunk_idx)
    assert torch.equal(b1.group_idx, full.group_idx)
    assert torch.equal(b1.o, full.o)
    hits1, misses1 = tier.stats.tolist()
    assert hits1 == 0 and misses1 > 0               # cold cache
    gathered = int(tier.bytes.item())
    assert 0 < gathered <= w.n_kv_heads * (w.q0 // w.group) * 2 * w.group * w.head_dim * 2
    # second step on the same segment: installed entries now hit
    b2 = _tiered_run(hga, p, w, q, k_all, v_all, full, tier)
    assert torch.equal(b2.group_idx, full.group_idx) and torch.equal(b2.o, full.o)
    hits2, misses2 = (tier.stats - torch.tensor([hits1, misses1], device=tier.stats.device)).tolist()
    assert hits2 > 0 and hits2 + misses2 == hits1 + misses1
    print(f"cache: cold {misses1} misses; warm hit rate {hits2 / (hits2 + misses2):.3f}; "
          f"gathered {gathered} B")
    # oracle on sampled units of the tiered outputs
    g = parity.GpuResult(np.zeros(1), np.zeros(1),
                         b1.chunk_idx.cpu().numpy(), b1.chunk_cnt.cpu().numpy(),
                         b1.group_idx.cpu().numpy(), b1.group_cnt.cpu().numpy(),
                         b1.o.double().cpu().numpy(), b1.lse.double().cpu().numpy())
    rep = parity.compare(w, inp, g, units=parity.sample_units(w, 10), check_summaries=False)
    assert rep.ok(), rep

"""File-backed K/V store on a B200: the history's exact K/V in a file, read
through a bounded page cache in pinned host memory and gathered into the
device mirrors ("Long-Context Fine-Tuning with Limited VRAM", section 2.2,
the filesystem store with RAM as a page cache).  A step through the store
must reproduce the all-HBM step exactly (indices and O) and the oracle on
sampled units, also when the cache is too small for two steps and evicts."""
import numpy as np
import pytest
import torch

import hga_inputs as gi
import parity

pytestmark = pytest.mark.gpu

W = gi.TIERED_128K.with_(T=12288, q0=10240, n_needles=16)


def _setup(w):
    from long_context_hga_b200 import hga
    p = hga.Params.from_workload(w)
    inp = gi.make_inputs(w)
    dev = torch.device("cuda:0")
    k_all, v_all, q = inp.k.to(dev), inp.v.to(dev), inp.q.to(dev)
    full = hga.allocate(p, w.T, w.Tq, device=dev)
    hga.build_summaries(p, k_all, 0, w.q0, full.chunk_sum, full.group_sum)
    hga.forward(p, q, w.q0, k_all, v_all, full)             # the all-HBM reference
    assert hga.check() == 0
    tier = hga.make_host_tier(p, None, None, full.group_sum.cpu().pin_memory(), t_hist=w.q0)
    return hga, p, inp, q, k_all, v_all, full, tier


def _store_run(hga, p, w, q, k_all, v_all, full, tier, store):
    dev = q.device
    bufs = hga.allocate(p, w.T, w.Tq, device=dev)
    bufs.chunk_sum.copy_(full.chunk_sum)
    nan = torch.tensor(float("nan"), dtype=k_all.dtype, device=dev)
    bufs.group_sum.fill_(nan)                           # history rows come from the tier
    bufs.group_sum[:, w.q0 // w.group:] = 0
    k_dev = torch.full_like(k_all, float("nan"))         # history K/V only via the store
    v_dev = torch.full_like(v_all, float("nan"))
    k_dev[:, w.q0:] = k_all[:, w.q0:]
    v_dev[:, w.q0:] = v_all[:, w.q0:]
    stats = hga.store_step(p, q, w.q0, tier, store, k_dev, v_dev, bufs)
    assert hga.check() == 0
    return bufs, stats


@pytest.mark.parametrize("direct", [False, True])
def test_store_step_equals_all_hbm_and_oracle(tmp_path, direct):
    hga, p, inp, q, k_all, v_all, full, tier = _setup(W)
    try:
        store = hga.KVStore(p, str(tmp_path / "kv.bin"), W.T, 64, cache_pages=2048,
                            direct=direct)
    except hga.HgaError as e:
        if direct and e.code == hga.HGA_ERR_IO:
            pytest.skip("O_DIRECT refused by this filesystem")
        raise
    store.append(inp.k[:, :W.q0], inp.v[:, :W.q0])
    b1, st1 = _store_run(hga, p, W, q, k_all, v_all, full, tier, store)
    assert torch.equal(b1.chunk_idx, full.chunk_idx)
    assert torch.equal(b1.group_idx, full.group_idx)
    assert torch.equal(b1.o, full.o)
    assert st1["hits"] == 0 and st1["misses"] == st1["pages_needed"] > 0
    assert st1["bytes_read"] == st1["misses"] * store.page_bytes
    b2, st2 = _store_run(hga, p, W, q, k_all, v_all, full, tier, store)   # warm cache
    assert torch.equal(b2.o, full.o)
    assert st2["hits"] == st1["pages_needed"] and st2["misses"] == 0
    print(f"store: {st1['pages_needed']} pages of {store.page_bytes} B per step; "
          f"direct={direct}")
    g = parity.GpuResult(np.zeros(1), np.zeros(1),
                         b1.chunk_idx.cpu().numpy(), b1.chunk_cnt.cpu().numpy(),
                         b1.group_idx.cpu().numpy(), b1.group_cnt.cpu().numpy(),
                         b1.o.double().cpu().numpy(), b1.lse.double().cpu().numpy())
    rep = parity.compare(W, inp, g, units=parity.sample_units(W, 10), check_summaries=False)
    assert rep.ok(), rep
    store.close()


def test_store_with_evictions_between_steps(tmp_path):
    """Two query sets over one history, alternating, with one-group pages and
    a cache sized for the larger single step: steps evict and each still
    matches its own all-HBM result."""
    w = W.with_(q0=W.T - 256)
    hga, p, inp, q_a, k_all, v_all, full_a, tier = _setup(w)
    g = torch.Generator().manual_seed(7)                 # a second query set, same history
    q_b = (torch.randn(q_a.shape, generator=g) * q_a.float().std().item()).to(
        q_a.dtype).to(q_a.device)
    full_b = hga.allocate(p, w.T, w.Tq, device=q_a.device)
    full_b.chunk_sum.copy_(full_a.chunk_sum)
    full_b.group_sum.copy_(full_a.group_sum)
    hga.forward(p, q_b, w.q0, k_all, v_all, full_b)
    assert hga.check() == 0
    assert not torch.equal(full_b.group_idx, full_a.group_idx)
    probe = hga.KVStore(p, str(tmp_path / "probe.bin"), w.T, 8, cache_pages=4096)
    probe.append(inp.k[:, :w.q0], inp.v[:, :w.q0])
    _, sa = _store_run(hga, p, w, q_a, k_all, v_all, full_a, tier, probe)
    _, sb = _store_run(hga, p, w, q_b, k_all, v_all, full_b, tier, probe)
    probe.close()
    cap = max(sa["pages_needed"], sb["pages_needed"])
    store = hga.KVStore(p, str(tmp_path / "kv.bin"), w.T, 8, cache_pages=cap)
    store.append(inp.k[:, :w.q0], inp.v[:, :w.q0])
    evicted = 0
    for q, full in ((q_a, full_a), (q_b, full_b), (q_a, full_a), (q_b, full_b)):
        b, st = _store_run(hga, p, w, q, k_all, v_all, full, tier, store)
        assert torch.equal(b.group_idx, full.group_idx)
        assert torch.equal(b.o, full.o)
        evicted += st["evictions"]
    assert evicted > 0
    store.close()


def test_gather_without_prepare_reports_absent_pages(tmp_path):
    """The kernel's own check: a group whose page is not resident is skipped
    and reported (HGA_ERR_DEVICE_CHECK), never read."""
    hga, p, inp, q, k_all, v_all, full, tier = _setup(W)
    store = hga.KVStore(p, str(tmp_path / "kv.bin"), W.T, 64, cache_pages=16)
    store.append(inp.k[:, :W.q0], inp.v[:, :W.q0])
    k_dev = torch.zeros_like(k_all)
    v_dev = torch.zeros_like(v_all)
    hga.gather_store(p, store, W.q0, W.Tq, W.q0, full.group_idx, full.group_cnt, k_dev, v_dev,
                     tier.gen, 1, tier.bytes)
    assert hga.check() == hga.HGA_ERR_DEVICE_CHECK
    assert not k_dev.any() and not v_dev.any()
    assert hga.check() == 0
    store.close()

"""hga_gather_history_noalloc: the history gather with its generation stamps in
the library's fixed device array instead of a caller buffer.  It must copy
exactly what hga_gather_history copies, on every call (the stamps are cleared
per call), and refuse capacities beyond its fixed array before any launch.
Named to be collected last: the fixed array is shared by every call in the
process, so the test must also pass after all the others ran."""
import ctypes

import pytest
import torch

import hga_inputs as gi


def _lib():
    from long_context_hga_b200 import hga
    return hga


def test_noalloc_rejects_capacity_beyond_fixed_array():
    hga = _lib()
    w = gi.TIERED_128K                       # 8 KV heads, 8-token groups
    p = hga.Params.from_workload(w)
    t_cap = (1 << 18) + 64                   # 8 * t_cap / 8 stamps > 2^18
    q_start = 1 << 18
    fake = ctypes.c_void_p(256)              # never dereferenced: refused first
    rc = hga.LIB.hga_gather_history_noalloc(
        ctypes.byref(p.c()), q_start, 64, t_cap, q_start, fake, fake, fake, fake, fake,
        fake, None, None)
    assert rc == hga.HGA_ERR_UNSUPPORTED
    # argument errors still come first, as in hga_gather_history
    rc = hga.LIB.hga_gather_history_noalloc(
        ctypes.byref(p.c()), 64 * 3, 64, 1024, 8 * 5 + 1, fake, fake, fake, fake, fake,
        fake, None, None)
    assert rc == hga.HGA_ERR_INVALID_ARG


def _bits(t):
    return t.view(torch.int16) if t.element_size() == 2 else t.view(torch.int32)


@pytest.mark.gpu
def test_noalloc_gather_matches_caller_stamped_gather_twice():
    hga = _lib()
    w = gi.TIERED_128K.with_(T=12288, q0=10240, n_needles=16)
    p = hga.Params.from_workload(w)
    inp = gi.make_inputs(w)
    dev = torch.device("cuda:0")
    q, k_all, v_all = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    full = hga.allocate(p, w.T, w.Tq, device=dev)
    hga.forward(p, q, w.q0, k_all, v_all, full)
    assert hga.check() == 0
    tier = hga.make_host_tier(p, inp.k.pin_memory(), inp.v.pin_memory(),
                              full.group_sum.cpu().pin_memory(), t_hist=w.q0)

    def mirrors():
        return (torch.full_like(k_all, float("nan")), torch.full_like(v_all, float("nan")))

    for call in range(2):                    # two calls in a row through each entry point
        k1, v1 = mirrors()
        before = int(tier.bytes.item())
        hga.gather_history(p, w.q0, w.Tq, w.T, tier, full.group_idx, full.group_cnt, k1, v1)
        assert hga.check() == 0
        bytes1 = int(tier.bytes.item()) - before

        k2, v2 = mirrors()
        before = int(tier.bytes.item())
        hga.gather_history_noalloc(p, w.q0, w.Tq, w.T, tier, full.group_idx, full.group_cnt,
                                   k2, v2)
        assert hga.check() == 0
        bytes2 = int(tier.bytes.item()) - before

        assert bytes1 > 0 and bytes2 == bytes1, (call, bytes1, bytes2)
        assert torch.equal(_bits(k2), _bits(k1)) and torch.equal(_bits(v2), _bits(v1)), call
        copied = ~torch.isnan(k2[..., 0])
        assert int(copied.sum()) * 2 * w.head_dim * 2 == bytes2
        assert torch.equal(k2[copied], k_all[copied]) and torch.equal(v2[copied], v_all[copied])
        assert not bool(copied[:, w.q0:].any())   # only history below t_hist is gathered

"""Failure detection on a B200 without a GPU fault: every wait of the
tensor-core kernels is bounded.  A wait that nothing completes must give up
after the (settable) limit, report HGA_ERR_TIMEOUT through the status word and
leave the device usable; the attention kernel with a K/V copy that never
arrives must drain, free its TMEM and return, and the next call must be
exact again."""
import numpy as np
import pytest
import torch

import hga_inputs as gi

pytestmark = pytest.mark.gpu

LIMIT_NS = 50_000_000          # 50 ms


@pytest.fixture
def hga():
    from long_context_hga_b200 import hga as mod
    assert mod.check() == 0
    mod.set_wait_limit_ns(LIMIT_NS)
    yield mod
    mod.debug_stall_next_attend(-1)
    mod.set_wait_limit_ns(2_000_000_000)
    mod.check()


def test_wait_without_arrival_times_out(hga):
    for _ in range(2):
        elapsed = hga.selftest_wait()
        assert hga.check() == hga.HGA_ERR_TIMEOUT
        assert hga.check() == 0                      # read and cleared
        ns = int(elapsed.item())
        assert LIMIT_NS <= ns < 20 * LIMIT_NS, ns


def _case():
    w = gi.QWEN3_30B_64K.with_(T=8168, q0=6144, n_needles=16)
    return w, gi.make_inputs(w)


@pytest.mark.parametrize("stall", [0, 1, 5, 12])
def test_attention_with_a_lost_copy_returns_and_recovers(hga, stall):
    """stall = ring load index (K loads even, V loads odd) that every CTA
    never issues; its consumers wait, time out and abort the CTA."""
    import dataclasses
    w, inp = _case()
    p = hga.Params.from_workload(w)
    pf = dataclasses.replace(p, v_f16=True)
    dev = torch.device("cuda:0")
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    v16 = torch.empty(v.shape, dtype=torch.float16, device=dev)
    hga.convert_v(p, v, 0, w.T, v16)
    bufs = hga.allocate(p, w.T, w.Tq, device=dev)
    hga.build_summaries(p, k, 0, w.T, bufs.chunk_sum, bufs.group_sum)
    hga.route_chunks(p, q, w.q0, bufs.chunk_sum, w.T, bufs.chunk_idx, bufs.chunk_cnt)
    hga.route_groups(p, q, w.q0, bufs.group_sum, w.T, bufs.chunk_idx, bufs.chunk_cnt,
                     bufs.group_idx, bufs.group_cnt)
    o_ref = torch.empty_like(bufs.o)
    hga.attend(pf, q, w.q0, k, v16, bufs.group_idx, bufs.group_cnt, o_ref)
    assert hga.check() == 0

    o_bad = torch.full_like(bufs.o, float("nan"))
    hga.debug_stall_next_attend(stall)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    hga.attend(pf, q, w.q0, k, v16, bufs.group_idx, bufs.group_cnt, o_bad)
    t1.record()
    assert hga.check() == hga.HGA_ERR_TIMEOUT
    ms = t0.elapsed_time(t1)
    assert LIMIT_NS / 1e6 <= ms < 60 * LIMIT_NS / 1e6, ms
    assert bool(torch.isnan(o_bad.float()).any())    # the aborted items wrote nothing

    o_again = torch.empty_like(bufs.o)               # the hook was one-shot
    hga.attend(pf, q, w.q0, k, v16, bufs.group_idx, bufs.group_cnt, o_again)
    assert hga.check() == 0
    assert torch.equal(o_again, o_ref)

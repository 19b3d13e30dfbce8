"""Strictly causal routing variant on a B200 (hga_forward_causal).

"Long-Context Fine-Tuning with Limited VRAM", section 6.1 names a strictly
causal routing variant and leaves its design open; the library routes block b
on the queries of the block before it.  Checked here: parity with the
oracle's variant (every unit on reduced shapes with ragged tails, sampled
units at the 64K size), equality with the routing and attention calls made
separately on the shifted queries, and strict causality of the device
outputs (inputs after position t do not change any output at or before t)."""
import numpy as np
import pytest
import torch

import hga_inputs as gi
from oracle import hga_oracle as ho
import parity

pytestmark = pytest.mark.gpu


def _check(w, units=None):
    inp = gi.make_inputs(w)
    qb = gi.make_q_before(w)
    g = parity.run_gpu_causal(w, inp, qb)
    q_route = ho.causal_route_queries(gi.to_f64(qb), gi.to_f64(inp.q))
    rep = parity.compare(w, inp, g, units=units, q_route=q_route)
    print(w.name, rep)
    assert rep.ok(), rep
    return g, inp, qb


def test_causal_tiny_fp32_from_position_zero():
    _check(gi.TINY_FP32)


def test_causal_tiny_fp32_ragged_segment():
    _check(gi.TINY_FP32.with_(T=1000, q0=256))


def test_causal_qwen3_30b_shape_reduced_ragged():
    _check(gi.QWEN3_30B_64K.with_(T=8168, q0=6144, n_needles=16))


def test_causal_qwen3_8b_shape_reduced():
    _check(gi.QWEN3_8B_16K.with_(T=4136, q0=2048, n_needles=8))


def test_causal_full_size_sampled():
    w = gi.QWEN3_30B_64K
    _check(w, units=parity.sample_units(w, 8))


def _device_inputs(w):
    from long_context_hga_b200 import hga
    p = hga.Params.from_workload(w)
    inp = gi.make_inputs(w)
    dev = torch.device("cuda:0")
    q_ext = torch.cat([gi.make_q_before(w), inp.q]).to(dev)
    return hga, p, q_ext, inp.k.to(dev), inp.v.to(dev)


def _forward_causal(hga, p, w, q_ext, k, v):
    bufs = hga.allocate(p, w.T, w.Tq, device=q_ext.device)
    hga.build_summaries(p, k, 0, w.q0, bufs.chunk_sum, bufs.group_sum)
    hga.forward_causal(p, q_ext, w.q0, k, v, bufs)
    assert hga.check() == 0
    return bufs


def test_causal_equals_shifted_routing_then_attention():
    w = gi.QWEN3_30B_64K.with_(T=8168, q0=6144, n_needles=16)
    hga, p, q_ext, k, v = _device_inputs(w)
    a = _forward_causal(hga, p, w, q_ext, k, v)
    b = hga.allocate(p, w.T, w.Tq, device=q_ext.device)
    hga.build_summaries(p, k, 0, w.T, b.chunk_sum, b.group_sum)
    q_route, q = q_ext[:w.Tq], q_ext[w.qblock:]
    hga.route_chunks(p, q_route, w.q0, b.chunk_sum, w.T, b.chunk_idx, b.chunk_cnt)
    hga.route_groups(p, q_route, w.q0, b.group_sum, w.T, b.chunk_idx, b.chunk_cnt,
                     b.group_idx, b.group_cnt)
    hga.attend(p, q, w.q0, k, v, b.group_idx, b.group_cnt, b.o, b.lse)
    assert hga.check() == 0
    for name in ("chunk_idx", "chunk_cnt", "group_idx", "group_cnt", "o", "lse"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name


@pytest.mark.parametrize("t_rel", [63, 64, 1000, 1500])
def test_causal_outputs_ignore_later_inputs(t_rel):
    """Random q, k, v after position t = q0 + t_rel: outputs and LSE at
    positions <= t are bit-identical."""
    w = gi.QWEN3_30B_64K.with_(T=8168, q0=6144, n_needles=16)
    hga, p, q_ext, k, v = _device_inputs(w)
    a = _forward_causal(hga, p, w, q_ext, k, v)
    t = w.q0 + t_rel
    g = torch.Generator(device="cpu").manual_seed(t_rel)
    q2, k2, v2 = q_ext.clone(), k.clone(), v.clone()
    rows = q2[w.qblock + t_rel + 1:]
    q2[w.qblock + t_rel + 1:] = (torch.randn(rows.shape, generator=g) * 3).to(q2.dtype).to(
        q2.device)
    k2[:, t + 1:] = (torch.randn(k2[:, t + 1:].shape, generator=g) * 3).to(k2.dtype).to(k2.device)
    v2[:, t + 1:] = (torch.randn(v2[:, t + 1:].shape, generator=g) * 3).to(v2.dtype).to(v2.device)
    b = _forward_causal(hga, p, w, q2, k2, v2)
    n = t_rel + 1
    assert torch.equal(a.o[:n], b.o[:n])
    assert torch.equal(a.lse[:n], b.lse[:n])
    assert not torch.equal(a.o[n:], b.o[n:])

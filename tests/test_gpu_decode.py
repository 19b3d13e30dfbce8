"""Decode steps (hga_decode_step) vs the oracle and vs prefill (needs a B200).

A generation step at position pos routes the token's query block on the
queries present (positions b0 .. pos), so its output row must equal the
oracle's forward of the context [0, pos + 1) with the segment [b0, pos + 1),
within the bf16 output bound, and bit-for-bit the prefill call on that
segment.  Steps at the first, a middle and the last position of a block, with
the history committed first and the step committing its own token.
"""
import dataclasses

import numpy as np
import pytest
import torch

import hga_inputs as gi
from oracle import hga_oracle as ho

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("v16", [True, False])
def test_decode_steps_match_oracle_and_prefill(v16):
    from long_context_hga_b200 import hga
    w = gi.QWEN3_30B_64K.with_(T=4160, q0=4096, n_needles=4)
    inp = gi.make_inputs(w)
    p = hga.Params.from_workload(w)
    dev = torch.device("cuda:0")
    q_all, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)   # q_all: positions 4096 .. 4159
    b0 = w.q0
    bufs = hga.allocate(p, w.T, p.qblock, device=dev)
    v_f16 = torch.zeros(v.shape, dtype=torch.float16, device=dev) if v16 else None
    hga.commit(p, k, v, 0, b0, bufs.chunk_sum, bufs.group_sum, v_f16)   # the history
    op = ho.Params(w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk, w.group, w.qblock,
                   w.sink, w.local, w.top_chunks, w.top_groups, w.dtype)
    f = lambda t: t.detach().to(torch.float64).cpu().numpy()
    for pos in (b0, b0 + 17, b0 + 63):
        n = pos - b0 + 1
        row = hga.decode_step(p, q_all, pos, k, v, bufs, v_f16=v_f16)
        assert hga.check() == 0
        got = f(row)
        # prefill of the same segment: the same kernels on the same inputs
        pre = hga.allocate(p, w.T, n, device=dev)
        pre.chunk_sum.copy_(bufs.chunk_sum)
        pre.group_sum.copy_(bufs.group_sum)
        p_att = dataclasses.replace(p, v_f16=True) if v16 else p
        hga.route_chunks(p, q_all[:n], b0, pre.chunk_sum, w.T, pre.chunk_idx, pre.chunk_cnt)
        hga.route_groups(p, q_all[:n], b0, pre.group_sum, w.T, pre.chunk_idx, pre.chunk_cnt,
                         pre.group_idx, pre.group_cnt)
        hga.attend(p_att, q_all[:n], b0, k, v_f16 if v16 else v, pre.group_idx, pre.group_cnt,
                   pre.o, pre.lse)
        assert hga.check() == 0
        assert torch.equal(row, pre.o[n - 1])
        assert torch.equal(bufs.lse[n - 1], pre.lse[n - 1])
        # the oracle on the context [0, pos + 1), segment [b0, pos + 1)
        qd, kd, vd = f(q_all[:n]), f(k[:, :pos + 1]), f(v[:, :pos + 1])
        res = ho.hga_forward(qd, kd, vd, b0, op)
        O, _ = ho.assemble_output(res, b0, pos + 1, op, w.head_dim)
        ref = O[n - 1]
        err = np.abs(got - ref)
        assert np.all(err <= 2e-3 + 1e-2 * np.abs(ref)), (pos, float(err.max()))
        # the routed groups agree wherever the oracle's margin is clear
        gi_np, gc_np = bufs.group_idx.cpu().numpy(), bufs.group_cnt.cpu().numpy()
        for h in range(w.n_kv_heads):
            if res.group_margin[(0, h)] > 1e-4 and res.chunk_margin[(0, h)] > 1e-4:
                assert list(gi_np[h, 0, :gc_np[h, 0]]) == res.group_idx[(0, h)], (pos, h)


def test_lockstep_requests_as_heads_equal_separate_steps():
    """Requests decoding at the same position can share one call: request r's
    KV heads become heads r*Hkv .. of one cache and its query heads r*Hq ..;
    every (block, KV head) unit is independent, so the outputs equal the
    per-request steps bit for bit."""
    from long_context_hga_b200 import hga
    dev = torch.device("cuda:0")
    ws = [gi.QWEN3_30B_64K.with_(T=2112, q0=2048, seed=s, n_needles=2) for s in (0, 1)]
    p = hga.Params.from_workload(ws[0])
    pos = 2048 + 40
    outs, qs, ks, vs = [], [], [], []
    for w in ws:
        inp = gi.make_inputs(w)
        q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
        bufs = hga.allocate(p, w.T, p.qblock, device=dev)
        hga.commit(p, k, v, 0, w.q0, bufs.chunk_sum, bufs.group_sum)
        outs.append(hga.decode_step(p, q, pos, k, v, bufs).clone())
        qs.append(q)
        ks.append(k)
        vs.append(v)
    pb = dataclasses.replace(p, n_q_heads=2 * p.n_q_heads, n_kv_heads=2 * p.n_kv_heads)
    kb, vb = torch.cat(ks, 0), torch.cat(vs, 0)
    qb = torch.cat(qs, 1).contiguous()
    bb = hga.allocate(pb, ws[0].T, p.qblock, device=dev)
    hga.commit(pb, kb, vb, 0, ws[0].q0, bb.chunk_sum, bb.group_sum)
    row = hga.decode_step(pb, qb, pos, kb, vb, bb)
    assert hga.check() == 0
    assert torch.equal(row[:p.n_q_heads], outs[0])
    assert torch.equal(row[p.n_q_heads:], outs[1])

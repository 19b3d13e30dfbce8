"""Backward of the gathered attention (routing held fixed) vs the oracle's
backward, through the C ABI (needs a B200).

Both sides take the same inputs: q, k, v as stored, the group lists of the
GPU forward pass, its O and LSE, and a seeded dO.  The kernel computes in
fp32 (bf16 inputs are exact in fp32); the bound below allows the rounding of
fp32 dot products over d terms and sums over up to a few thousand attended
tokens or query rows: |err| <= 2e-4 * (1 + max|ref|) per tensor.
"""
import numpy as np
import pytest
import torch

import hga_inputs as gi
from oracle import hga_oracle as ho

pytestmark = pytest.mark.gpu

CASES = {
    "tiny_fp32": gi.TINY_FP32,
    "30b_ragged": gi.QWEN3_30B_64K.with_(T=2600, q0=2048, n_needles=4),
    "d64_g1": gi.Workload("d64_g1", 4, 4, 64, 1536, 512, 1e6, 64, 128, 3, 10, n_needles=4),
    "budget_all": gi.SWEEP_32K.with_(T=704, q0=320, top_chunks=0, top_groups=0, n_needles=2),
}


def _run(w):
    from long_context_hga_b200 import hga
    p = hga.Params.from_workload(w)
    inp = gi.make_inputs(w)
    dev = torch.device("cuda:0")
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    bufs = hga.allocate(p, w.T, w.Tq, device=dev)
    if w.q0 > 0:
        hga.build_summaries(p, k, 0, w.q0, bufs.chunk_sum, bufs.group_sum)
    hga.forward(p, q, w.q0, k, v, bufs)
    g = torch.Generator().manual_seed(17)
    d_o = torch.randn(q.shape, generator=g).to(q.dtype).to(dev)
    d_q = torch.full(q.shape, float("nan"), dtype=torch.float32, device=dev)
    d_k = torch.full(k.shape, float("nan"), dtype=torch.float32, device=dev)
    d_v = torch.full(v.shape, float("nan"), dtype=torch.float32, device=dev)
    hga.attend_backward(p, q, w.q0, k, v, bufs.group_idx, bufs.group_cnt, bufs.o, bufs.lse,
                        d_o, d_q, d_k, d_v)
    assert hga.check() == 0
    f = lambda t: t.detach().to(torch.float64).cpu().numpy()
    gi_np, gc_np = bufs.group_idx.cpu().numpy(), bufs.group_cnt.cpu().numpy()
    groups = {(b, h): [int(x) for x in gi_np[h, b, :gc_np[h, b]]]
              for h in range(w.n_kv_heads) for b in range(gc_np.shape[1])}
    op = ho.Params(w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk, w.group, w.qblock,
                   w.sink, w.local, w.top_chunks, w.top_groups, w.dtype)
    ref = ho.hga_backward(f(q), f(k), f(v), w.q0, op, groups, f(bufs.o), f(bufs.lse), f(d_o))
    return (f(d_q), f(d_k), f(d_v)), ref


@pytest.mark.parametrize("case", sorted(CASES))
def test_backward_matches_oracle(case):
    w = CASES[case]
    got, ref = _run(w)
    for name, x, r in zip(("dq", "dk", "dv"), got, ref):
        if name != "dq":   # tokens past the context are not touched
            x, r = x[:, :w.T], r[:, :w.T]
        assert np.all(np.isfinite(x)), name
        err = float(np.max(np.abs(x - r)))
        scale = 1.0 + float(np.max(np.abs(r)))
        print(case, name, "max|err|", err, "max|ref|", scale - 1)
        assert err <= 2e-4 * scale, (case, name, err, scale)

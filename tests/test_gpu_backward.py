"""Backward of the gathered attention (routing held fixed) vs the oracle's
backward, through the C ABI (needs a B200).

Both sides take the same inputs: q, k, v as stored, the group lists of the
GPU forward pass, its O and LSE, and a seeded dO.

Tolerance, elementwise, from the kernels' arithmetic.  Every output element
is a sum of terms (dv_t = sum_r p_rt dO_r, dk_t = sum_r ds_rt q_r / sqrt(d),
dq_r = sum_t ds_rt k_t / sqrt(d)).  The bound is c * M + d * 2^-24 * E:
  * M is the sum of the terms' absolute values.  The multiplier c covers the
    rounding of the terms: bf16 inputs run on the tensor cores, which take p
    and ds rounded to bf16 (relative 2^-9 each) while everything else
    accumulates in fp32, so c = 2^-8; fp32 inputs (and bf16 shapes the
    tensor-core kernels do not take) run in fp32 on the CUDA cores, c = 2^-16.
  * E covers the fp32 dot products inside ds = p (dp - D) (dp = dO.v, D =
    dO.o and s = q.k, each with a relative error of at most d * 2^-24 of the
    sum of its products' absolute values).  ds can be much smaller than
    p |dp| when dp and D nearly cancel, which M alone does not see:
    E = sum of p (|dO|.|v| + |dO|.|o|) (1 + |q|.|k| / sqrt(d)) times |k| or
    |q| / sqrt(d), like M.
Both are computed below in float64 from the definition.
"""
import math

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
    "g16": gi.Workload("g16", 16, 1, 128, 1600, 1024, 1e6, 128, 128, 5, 12, n_needles=4),
    # context not a multiple of the group size: the CUDA-core kernel
    "context_ragged": gi.QWEN3_30B_64K.with_(T=2604, q0=2048, n_needles=4),
}


def _run(w, variant=0):
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
    hga.set_kernel_variant(variant)
    try:
        hga.attend_backward(p, q, w.q0, k, v, bufs.group_idx, bufs.group_cnt, bufs.o, bufs.lse,
                            d_o, d_q, d_k, d_v)
    finally:
        hga.set_kernel_variant(0)
    assert hga.check() == 0
    f = lambda t: t.detach().to(torch.float64).cpu().numpy()
    gi_np, gc_np = bufs.group_idx.cpu().numpy(), bufs.group_cnt.cpu().numpy()
    groups = {(b, h): [int(x) for x in gi_np[h, b, :gc_np[h, b]]]
              for h in range(w.n_kv_heads) for b in range(gc_np.shape[1])}
    op = ho.Params(w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk, w.group, w.qblock,
                   w.sink, w.local, w.top_chunks, w.top_groups, w.dtype)
    args = (f(q), f(k), f(v), w.q0, op, groups, f(bufs.o), f(bufs.lse), f(d_o))
    ref = ho.hga_backward(*args)
    return (f(d_q), f(d_k), f(d_v)), ref, _magnitudes(*args)


def _magnitudes(q, k, v, q0, p, groups, O, L, dO):
    """Per output element: M, the sum of the absolute values of its terms, and
    E, the scale of the fp32 dot-product errors inside ds (see above); float64
    from the definition."""
    T = k.shape[1]
    d = q.shape[-1]
    sc = 1.0 / math.sqrt(d)
    Mq, Mk, Mv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    Eq, Ek = np.zeros_like(q), np.zeros_like(k)
    for (b, h), gr in groups.items():
        b0 = q0 + b * p.qblock
        hs = slice(h * p.G, (h + 1) * p.G)
        for pos in range(b0, min(b0 + p.qblock, T)):
            R = ho.attention_set(b0, pos, gr, p)
            qr, gr_ = q[pos - q0, hs], dO[pos - q0, hs]                     # [G][d]
            kr, vr = k[h, R], v[h, R]
            pr = np.exp(qr @ kr.T * sc - L[pos - q0, hs][:, None])         # [G][|R|]
            D = np.sum(gr_ * O[pos - q0, hs], axis=1)
            ds = pr * (gr_ @ vr.T - D[:, None])
            e = pr * (np.abs(gr_) @ np.abs(vr).T +
                      np.sum(np.abs(gr_ * O[pos - q0, hs]), axis=1)[:, None]) * \
                (1.0 + np.abs(qr) @ np.abs(kr).T * sc)
            Mq[pos - q0, hs] = np.abs(ds) @ np.abs(kr) * sc
            Eq[pos - q0, hs] = e @ np.abs(kr) * sc
            Mk[h, R] += np.abs(ds).T @ np.abs(qr) * sc
            Ek[h, R] += e.T @ np.abs(qr) * sc
            Mv[h, R] += np.abs(pr).T @ np.abs(gr_)
    return (Mq, Mk, Mv), (Eq, Ek, np.zeros_like(v))


def _check(case, w, got, ref, mag, c):
    (M, E), d = mag, w.head_dim
    for name, x, r, m, e in zip(("dq", "dk", "dv"), got, ref, M, E):
        if name != "dq":   # tokens past the context are not touched
            x, r, m, e = x[:, :w.T], r[:, :w.T], m[:, :w.T], e[:, :w.T]
        assert np.all(np.isfinite(x)), name
        err = np.abs(x - r)
        bound = c * m + d * 2.0 ** -24 * e + 1e-7
        worst = float(np.max(err / bound))
        print(case, name, "max|err|", float(err.max()), "max|ref|", float(np.abs(r).max()),
              "worst err/bound", worst)
        assert worst <= 1.0, (case, name, worst)


@pytest.mark.parametrize("case", sorted(CASES))
def test_backward_matches_oracle(case):
    w = CASES[case]
    got, ref, mag = _run(w)
    tensor_cores = w.dtype == "bf16" and w.T % w.group == 0
    _check(case, w, got, ref, mag, 2.0 ** -8 if tensor_cores else 2.0 ** -16)


def test_tensor_core_and_cuda_core_backward_agree():
    """The tensor-core kernels and the fp32 CUDA-core kernel (variant 1) on
    the same bf16 inputs: each within its own bound of the oracle."""
    w = CASES["30b_ragged"]
    got_tc, ref, mag = _run(w, variant=0)
    got_cc, _, _ = _run(w, variant=1)
    _check("tc", w, got_tc, ref, mag, 2.0 ** -8)
    _check("cuda_core", w, got_cc, ref, mag, 2.0 ** -16)
    assert not np.array_equal(got_tc[0], got_cc[0])     # two different kernels ran


def test_backward_full_size_64k_sampled_dq():
    """The 64K workload as the bench times it (tensor cores, fp16-free bf16
    inputs): dq of sampled (block, KV head) units against the oracle's
    backward of those units (a unit's dq depends on that unit alone)."""
    from long_context_hga_b200 import hga
    w = gi.QWEN3_30B_64K
    p = hga.Params.from_workload(w)
    inp = gi.make_inputs(w)
    dev = torch.device("cuda:0")
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    bufs = hga.allocate(p, w.T, w.Tq, device=dev)
    hga.build_summaries(p, k, 0, w.q0, bufs.chunk_sum, bufs.group_sum)
    hga.forward(p, q, w.q0, k, v, bufs)
    g = torch.Generator().manual_seed(17)
    d_o = torch.randn(q.shape, generator=g).to(q.dtype).to(dev)
    d_q = torch.full(q.shape, float("nan"), dtype=torch.float32, device=dev)
    d_k = torch.empty(k.shape, dtype=torch.float32, device=dev)
    d_v = torch.empty(v.shape, dtype=torch.float32, device=dev)
    hga.attend_backward(p, q, w.q0, k, v, bufs.group_idx, bufs.group_cnt, bufs.o, bufs.lse,
                        d_o, d_q, d_k, d_v)
    assert hga.check() == 0
    f = lambda t: t.detach().to(torch.float64).cpu().numpy()
    gi_np, gc_np = bufs.group_idx.cpu().numpy(), bufs.group_cnt.cpu().numpy()
    op = ho.Params(w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk, w.group, w.qblock,
                   w.sink, w.local, w.top_chunks, w.top_groups, w.dtype)
    qd, kd, vd, O, L, dO = f(q), f(k), f(v), f(bufs.o), f(bufs.lse), f(d_o)
    got = f(d_q)
    nb = w.Tq // w.qblock
    units = [(0, 0), (nb - 1, w.n_kv_heads - 1), (nb // 2, 1), (7, 2), (nb - 5, 3)]
    groups = {(b, h): [int(x) for x in gi_np[h, b, :gc_np[h, b]]] for (b, h) in units}
    (Mq, _, _), (Eq, _, _) = _magnitudes(qd, kd, vd, w.q0, op, groups, O, L, dO)
    for (b, h) in units:
        r0, r1 = b * w.qblock, (b + 1) * w.qblock
        hs = slice(h * w.G, (h + 1) * w.G)
        dq, _, _ = ho.attend_unit_backward(qd, kd, vd, w.q0, w.T, groups[(b, h)], op, b, h,
                                           O[r0:r1, hs], L[r0:r1, hs], dO[r0:r1, hs])
        err = np.abs(got[r0:r1, hs] - dq)
        bound = 2.0 ** -8 * Mq[r0:r1, hs] + w.head_dim * 2.0 ** -24 * Eq[r0:r1, hs] + 1e-7
        worst = float(np.max(err / bound))
        print("64k unit", (b, h), "max|err|", float(err.max()), "worst err/bound", worst)
        assert worst <= 1.0, ((b, h), worst)

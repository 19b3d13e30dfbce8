"""CUDA path vs CPU oracle through the C ABI (needs a B200).

Small sizes compare every (query block, KV head) unit; the full-size
workloads run in the same launch configuration as bench.py and compare
sampled units.  Ragged tails (a last query block shorter than 64) and the
first blocks (sink, local and diagonal overlapping) are covered.
"""
import numpy as np
import pytest
import torch

import hga_inputs as gi
from oracle import hga_oracle as ho
import parity

pytestmark = pytest.mark.gpu


def _check(w, units=None, split_history=True, t_cap=None, v_f16=False):
    inp = gi.make_inputs(w)
    g = parity.run_gpu(w, inp, t_cap=t_cap, split_history=split_history, v_f16=v_f16)
    rep = parity.compare(w, inp, g, units=units)
    print(w.name, rep)
    assert rep.ok(), rep
    return rep, g, inp


def test_tiny_fp32_all_units():
    _check(gi.TINY_FP32)


def test_tiny_fp32_ragged_and_capacity():
    # context not a multiple of 64, t_cap larger than the context
    _check(gi.TINY_FP32.with_(T=1000), t_cap=1088)


def test_qwen3_8b_shape_reduced_ragged():
    _check(gi.QWEN3_8B_16K.with_(T=2088, n_needles=8), split_history=False)


def test_qwen3_30b_shape_reduced_ragged():
    _check(gi.QWEN3_30B_64K.with_(T=8168, q0=6144, n_needles=16))


def test_head_dim_64_bf16_no_gqa():
    w = gi.Workload("d64_g1", 4, 4, 64, 1536, 512, 1e6, 64, 128, 3, 10,
                    n_needles=4)
    _check(w)


def test_gqa16_rows_span_slices():
    # 16 query heads per KV head: 1024 rows per block, several row slices
    w = gi.Workload("g16", 16, 1, 128, 1600, 1024, 1e6, 128, 128, 5, 12,
                    n_needles=4)
    _check(w)


def test_budget_covers_everything_is_dense():
    """Full budget must reproduce dense causal attention."""
    w = gi.SWEEP_32K.with_(T=1280, top_chunks=0, top_groups=0, n_needles=4)
    rep, g, inp = _check(w)
    q, k, v = gi.to_f64(inp.q), gi.to_f64(inp.k), gi.to_f64(inp.v)
    Od, Ld = ho.dense_causal_attention(q, k, v, w.q0, w.n_q_heads)
    atol, rtol = parity.TOL["bf16"]
    assert (np.abs(g.o - Od) <= atol + rtol * np.abs(Od)).all()
    assert abs(rep.density - 1.0) < 1e-12


@pytest.mark.parametrize("kc", [4, 8, 16, 64, 0])
def test_budget_sweep_reduced(kc):
    w = gi.SWEEP_32K.with_(T=4096, top_chunks=kc,
                           top_groups=2 * kc if kc > 0 else 0, n_needles=8)
    units = parity.sample_units(w, 40)
    _check(w, units=units)


def test_exact_ties_go_to_lower_index():
    """Identical chunk summaries give exactly equal scores on both sides;
    the lower chunk / group index must win."""
    w = gi.Workload("ties", 8, 2, 128, 2048, 1536, 1e6, 64, 128, 5, 7)
    inp = gi.make_inputs(w)
    k = inp.k.clone()
    base = k[:, 64:128].clone()
    for c in range(1, 2048 // 64):      # every candidate chunk identical
        k[:, 64 * c:64 * (c + 1)] = base
    inp = gi.Inputs(w, inp.q, k, inp.v, [])
    g = parity.run_gpu(w, inp)
    for h in range(2):
        for b in range(8):
            ch = list(g.chunk_idx[h, b, :g.chunk_cnt[h, b]])
            assert ch == [1, 2, 3, 4, 5], ch
    rep = parity.compare(w, inp, g)
    assert rep.chunk_mismatch == 0 and rep.invalid_choice == 0


def test_empty_and_tiny_segments():
    from long_context_hga_b200 import hga
    w = gi.TINY_FP32.with_(dtype="bf16", T=64)
    p = hga.Params.from_workload(w)
    dev = "cuda:0"
    bufs = hga.allocate(p, 64, 0, device=dev)
    k = torch.zeros(1, 64, 64, dtype=torch.bfloat16, device=dev)
    q = torch.zeros(0, 2, 64, dtype=torch.bfloat16, device=dev)
    n0 = hga.launch_count()
    hga.forward(p, q, 0, k, k, bufs)            # n_q = 0: nothing launched
    assert hga.launch_count() == n0
    for T in (1, 7, 8, 63, 65):
        _check(gi.TINY_FP32.with_(T=T, dtype="bf16"), t_cap=128)


def test_bad_group_index_sets_device_status():
    """Out-of-range routed groups are skipped and reported, never read."""
    from long_context_hga_b200 import hga
    w = gi.TINY_FP32.with_(dtype="bf16")
    inp = gi.make_inputs(w)
    p = hga.Params.from_workload(w)
    dev = "cuda:0"
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    bufs = hga.allocate(p, w.T, w.Tq, device=dev)
    hga.forward(p, q, 0, k, v, bufs)
    assert hga.check() == 0
    gi_bad = bufs.group_idx.clone()
    gi_bad[0, -1, 0] = 10 ** 6          # far outside the context
    gi_bad[0, -2, 0] = gi_bad[0, -2, 1]  # duplicate -> not ascending
    o2 = torch.empty_like(bufs.o)
    hga.attend(p, q, 0, k, v, gi_bad, bufs.group_cnt, o2)
    assert hga.check() == hga.HGA_ERR_DEVICE_CHECK
    assert hga.check() == 0             # cleared
    assert torch.isfinite(o2.float()).all()
    ci_bad = bufs.chunk_idx.clone()
    ci_bad[0, -1, 0] = -5
    hga.route_groups(p, q, 0, bufs.group_sum, w.T, ci_bad, bufs.chunk_cnt,
                     bufs.group_idx, bufs.group_cnt)
    assert hga.check() == hga.HGA_ERR_DEVICE_CHECK


@pytest.mark.parametrize("v_f16", [True, False])
@pytest.mark.parametrize("name", ["qwen3_30b_a3b_64k_last2k",
                                  "qwen3_8b_prefill_16k"])
def test_full_size_sampled(name, v_f16):
    """Full-size workloads; with fp16 V storage this is the benchmark's launch
    configuration.  The oracle recomputes a sample of units."""
    w = gi.WORKLOADS[name]
    units = parity.sample_units(w, 12)
    rep, _, _ = _check(w, units=units, v_f16=v_f16)
    assert rep.compared_units >= 10


@pytest.mark.parametrize("variant", [1, 0])
def test_attend_variants_agree_with_oracle(variant):
    """Both bf16 attention kernels (portable mma.sync and tcgen05) pass the
    same parity check, with a ragged tail and GQA 8."""
    from long_context_hga_b200 import hga
    hga.set_kernel_variant(variant)
    try:
        _check(gi.QWEN3_30B_64K.with_(T=4136, q0=2048, n_needles=8))
    finally:
        hga.set_kernel_variant(0)


def test_software_exp2_matches_cuda_exp2f():
    """The FMA-pipe 2^x used for part of each softmax row stays within 8e-5
    relative of CUDA's exp2f over the range the kernel feeds it, and gives
    ~0 for -inf (masked scores)."""
    from long_context_hga_b200 import hga
    x = torch.linspace(-125.0, 8.0, 1 << 20, device="cuda", dtype=torch.float32)
    x = torch.cat([x, torch.rand(1 << 18, device="cuda") * 16 - 8,
                   torch.tensor([0.0, -0.5, 0.5, 7.99, -124.9], device="cuda")])
    y = hga.selftest_exp2(x)
    ref = torch.exp2(x.double())
    rel = ((y.double() - ref).abs() / ref).max().item()
    assert rel < 8e-5, rel
    z = hga.selftest_exp2(torch.tensor([-float("inf"), -1e30, -200.0], device="cuda"))
    assert (z >= 0).all() and (z < 3e-38).all()


@pytest.mark.parametrize("case", ["30b_64k", "8b_ragged", "g16", "d64_g1", "budget_all", "tiny_fp32"])
def test_fused_route_equals_two_calls(case):
    """hga_route (chunk and group routing in one CTA per unit) writes exactly
    what hga_route_chunks followed by hga_route_groups write."""
    from long_context_hga_b200 import hga
    w = {"30b_64k": gi.QWEN3_30B_64K,
         "8b_ragged": gi.QWEN3_8B_16K.with_(T=4136, q0=2048, n_needles=8),
         "g16": gi.Workload("g16", 16, 1, 128, 1600, 1024, 1e6, 128, 128, 5, 12, n_needles=4),
         "d64_g1": gi.Workload("d64_g1", 4, 4, 64, 1536, 512, 1e6, 64, 128, 3, 10, n_needles=4),
         "budget_all": gi.SWEEP_32K.with_(T=4096, q0=2048, top_chunks=0, top_groups=0),
         "tiny_fp32": gi.TINY_FP32}[case]
    p = hga.Params.from_workload(w)
    inp = gi.make_inputs(w)
    dev = torch.device("cuda:0")
    q, k = inp.q.to(dev), inp.k.to(dev)
    a = hga.allocate(p, w.T, w.Tq, device=dev)
    b = hga.allocate(p, w.T, w.Tq, device=dev)
    hga.build_summaries(p, k, 0, w.T, a.chunk_sum, a.group_sum)
    hga.route_chunks(p, q, w.q0, a.chunk_sum, w.T, a.chunk_idx, a.chunk_cnt)
    hga.route_groups(p, q, w.q0, a.group_sum, w.T, a.chunk_idx, a.chunk_cnt, a.group_idx,
                     a.group_cnt)
    b.group_idx.fill_(12345)
    b.chunk_idx.fill_(12345)
    hga.route(p, q, w.q0, a.chunk_sum, a.group_sum, w.T, b.chunk_idx, b.chunk_cnt, b.group_idx,
              b.group_cnt)
    assert hga.check() == 0
    assert torch.equal(a.chunk_cnt, b.chunk_cnt) and torch.equal(a.chunk_idx, b.chunk_idx)
    assert torch.equal(a.group_cnt, b.group_cnt) and torch.equal(a.group_idx, b.group_idx)


@pytest.mark.parametrize("case", ["30b_ragged", "budget_all", "g16", "d64_g1"])
def test_q_ready_calls_equal_the_default(case):
    """With q_ready the routing and attention kernels request q before waiting
    for the previous kernel (each call here follows one of the library's own
    kernels, as the promise requires).  Their outputs equal the default
    path's bit for bit; the full budget takes the routing exits that score
    nothing (and must wait for that early copy before leaving)."""
    import dataclasses
    from long_context_hga_b200 import hga
    w = {"30b_ragged": gi.QWEN3_30B_64K.with_(T=4136, q0=2048, n_needles=8),
         "budget_all": gi.SWEEP_32K.with_(T=4096, q0=2048, top_chunks=0, top_groups=0),
         "g16": gi.Workload("g16", 16, 1, 128, 1600, 1024, 1e6, 128, 128, 5, 12, n_needles=4),
         "d64_g1": gi.Workload("d64_g1", 4, 4, 64, 1536, 512, 1e6, 64, 128, 3, 10,
                               n_needles=4)}[case]
    p = hga.Params.from_workload(w)
    pr = dataclasses.replace(p, q_ready=True)
    inp = gi.make_inputs(w)
    dev = torch.device("cuda:0")
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    out = []
    for pp in (p, pr):
        bb = hga.allocate(p, w.T, w.Tq, device=dev)
        bb.o.fill_(float("nan"))
        hga.commit(p, k, v, 0, w.T, bb.chunk_sum, bb.group_sum)
        for _ in range(2):          # the second pass starts right after the first's attention
            hga.route_chunks(pp, q, w.q0, bb.chunk_sum, w.T, bb.chunk_idx, bb.chunk_cnt)
            hga.route_groups(pp, q, w.q0, bb.group_sum, w.T, bb.chunk_idx, bb.chunk_cnt,
                             bb.group_idx, bb.group_cnt)
            hga.attend(pp, q, w.q0, k, v, bb.group_idx, bb.group_cnt, bb.o, bb.lse)
        assert hga.check() == 0
        out.append(bb)
    a, b = out
    for name in ("chunk_cnt", "chunk_idx", "group_cnt", "group_idx", "o", "lse"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    assert torch.isfinite(b.o.float()).all()

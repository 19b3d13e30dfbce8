"""V stored as fp16 (params.v_f16 = 1, filled by hga_convert_v).

The attention kernels keep P in fp16 and always multiply it by fp16 V. With
bf16 V they convert each gathered tile on chip; with fp16 V they read it as
is. Both routes must give bit-identical O and LSE. hga_convert_v must round
exactly as IEEE round-to-nearest-even (checked against torch's conversion),
touch only the requested tokens, and report overflow through the device
status word."""
import dataclasses

import numpy as np
import pytest
import torch

import hga_inputs as gi
import parity

pytestmark = pytest.mark.gpu


def _hga():
    from long_context_hga_b200 import hga
    return hga


def _params(hga, w, v_f16):
    return dataclasses.replace(hga.Params.from_workload(w), v_f16=v_f16)


def test_convert_v_rounds_like_ieee_and_keeps_other_tokens():
    hga = _hga()
    w = gi.QWEN3_30B_64K.with_(T=1024, q0=0)
    p = hga.Params.from_workload(w)
    g = torch.Generator().manual_seed(3)
    mag = torch.exp2(torch.randint(-30, 14, (4, 1024, 128), generator=g).float())
    v = (torch.randn(4, 1024, 128, generator=g).clamp(-3.9, 3.9) * mag).to(torch.bfloat16)
    v = v.cuda()
    out = torch.full(v.shape, 7.0, dtype=torch.float16, device="cuda")
    hga.convert_v(p, v, 64, 960, out)
    assert hga.check() == 0
    ref = v.float().half()
    assert torch.equal(out[:, 64:960].view(torch.int16), ref[:, 64:960].view(torch.int16))
    assert bool((out[:, :64] == 7.0).all()) and bool((out[:, 960:] == 7.0).all())
    # in place: the fp16 bits replace the bf16 bits of the same tokens
    inplace = v.clone()
    hga.convert_v(p, inplace, 0, 1024, inplace)
    assert hga.check() == 0
    assert torch.equal(inplace.view(torch.int16), ref.view(torch.int16))


def test_convert_v_overflow_sets_device_status():
    hga = _hga()
    w = gi.QWEN3_30B_64K.with_(T=256, q0=0)
    p = hga.Params.from_workload(w)
    v = torch.zeros(4, 256, 128, dtype=torch.bfloat16, device="cuda")
    v[1, 5, 3] = 70000.0
    out = torch.zeros(v.shape, dtype=torch.float16, device="cuda")
    hga.convert_v(p, v, 0, 256, out)
    assert hga.check() == hga.HGA_ERR_DEVICE_CHECK
    assert torch.isinf(out[1, 5, 3]) and int(torch.isinf(out).sum()) == 1
    assert hga.check() == 0                       # the status word was cleared


@pytest.mark.parametrize("d", [128, 64])
def test_commit_equals_summaries_and_convert(d):
    """One launch gives the summaries of build_summaries and the fp16 V of
    convert_v, bit for bit, over a range that ends in a partial chunk; tokens
    outside the range keep their bytes; in place works too."""
    hga = _hga()
    w = gi.QWEN3_30B_64K.with_(T=1024, q0=0, head_dim=d)
    p = hga.Params.from_workload(w)
    g = torch.Generator().manual_seed(11)
    k = torch.randn(4, 1024, d, generator=g).to(torch.bfloat16).cuda()
    mag = torch.exp2(torch.randint(-20, 12, (4, 1024, d), generator=g).float())
    v = (torch.randn(4, 1024, d, generator=g).clamp(-3.9, 3.9) * mag).to(torch.bfloat16).cuda()
    t0, t1 = 128, 1000                                   # 1000 = 15 chunks + 40 tokens
    ref_b = hga.allocate(p, 1024, 64, device="cuda")
    got_b = hga.allocate(p, 1024, 64, device="cuda")
    for b in (ref_b, got_b):
        b.chunk_sum.fill_(3.0)
        b.group_sum.fill_(3.0)
    ref_v = torch.full(v.shape, 7.0, dtype=torch.float16, device="cuda")
    got_v = ref_v.clone()
    hga.build_summaries(p, k, t0, t1, ref_b.chunk_sum, ref_b.group_sum)
    hga.convert_v(p, v, t0, t1, ref_v)
    hga.commit(p, k, v, t0, t1, got_b.chunk_sum, got_b.group_sum, got_v)
    assert hga.check() == 0
    assert torch.equal(got_b.chunk_sum.view(torch.int16), ref_b.chunk_sum.view(torch.int16))
    assert torch.equal(got_b.group_sum.view(torch.int16), ref_b.group_sum.view(torch.int16))
    assert torch.equal(got_v.view(torch.int16), ref_v.view(torch.int16))
    assert bool((got_v[:, :t0] == 7.0).all()) and bool((got_v[:, t1:] == 7.0).all())
    inplace = v.clone()
    hga.commit(p, k, inplace, t0, t1, got_b.chunk_sum, got_b.group_sum, inplace)
    assert hga.check() == 0
    assert torch.equal(inplace[:, t0:t1].view(torch.int16), ref_v[:, t0:t1].view(torch.int16))
    assert torch.equal(inplace[:, :t0], v[:, :t0]) and torch.equal(inplace[:, t1:], v[:, t1:])


def test_commit_overflow_sets_device_status():
    hga = _hga()
    w = gi.QWEN3_30B_64K.with_(T=256, q0=0)
    p = hga.Params.from_workload(w)
    k = torch.zeros(4, 256, 128, dtype=torch.bfloat16, device="cuda")
    v = torch.zeros(4, 256, 128, dtype=torch.bfloat16, device="cuda")
    v[2, 200, 7] = -1.0e5
    b = hga.allocate(p, 256, 64, device="cuda")
    out = torch.zeros(v.shape, dtype=torch.float16, device="cuda")
    hga.commit(p, k, v, 0, 256, b.chunk_sum, b.group_sum, out)
    assert hga.check() == hga.HGA_ERR_DEVICE_CHECK
    assert torch.isinf(out[2, 200, 7]) and int(torch.isinf(out).sum()) == 1
    assert hga.check() == 0


CASES = {
    "30b_ragged": gi.QWEN3_30B_64K.with_(T=8168, q0=6144, n_needles=16),
    "8b_ragged": gi.QWEN3_8B_16K.with_(T=4136, q0=2048, n_needles=8),
    "d64_g1": gi.Workload("d64_g1", 4, 4, 64, 1536, 512, 1e6, 64, 128, 3, 10, n_needles=4),
}


@pytest.mark.parametrize("variant", [2, 1])
@pytest.mark.parametrize("case", sorted(CASES))
def test_fp16_v_gives_identical_attention(case, variant):
    # variants 2 (same as the default tensor-core kernel) and 1 (mma.sync):
    # the fp16-V and bf16-V forms run the same arithmetic
    hga = _hga()
    w = CASES[case]
    inp = gi.make_inputs(w)
    dev = torch.device("cuda:0")
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    p = _params(hga, w, False)
    p16 = _params(hga, w, True)
    v16 = torch.empty(v.shape, dtype=torch.float16, device=dev)
    hga.convert_v(p, v, 0, w.T, v16)
    hga.set_kernel_variant(variant)
    try:
        b1 = hga.allocate(p, w.T, w.Tq, device=dev)
        hga.build_summaries(p, k, 0, w.q0, b1.chunk_sum, b1.group_sum)
        hga.forward(p, q, w.q0, k, v, b1)
        b2 = hga.allocate(p, w.T, w.Tq, device=dev)
        hga.build_summaries(p16, k, 0, w.q0, b2.chunk_sum, b2.group_sum)
        hga.forward(p16, q, w.q0, k, v16, b2)
        assert hga.check() == 0
    finally:
        hga.set_kernel_variant(0)
    assert torch.equal(b1.group_idx, b2.group_idx)
    assert torch.equal(b1.o.view(torch.int16), b2.o.view(torch.int16))
    assert torch.equal(b1.lse, b2.lse)
    # and the fp16-V result passes the oracle on sampled units
    f = lambda t: t.detach().to(torch.float64).cpu().numpy()
    g = parity.GpuResult(f(b2.chunk_sum), f(b2.group_sum), b2.chunk_idx.cpu().numpy(),
                         b2.chunk_cnt.cpu().numpy(), b2.group_idx.cpu().numpy(),
                         b2.group_cnt.cpu().numpy(), f(b2.o),
                         b2.lse.cpu().numpy().astype(np.float64))
    rep = parity.compare(w, inp, g, units=parity.sample_units(w, 6))
    assert rep.ok(), rep


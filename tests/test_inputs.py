"""The seeded generator: shapes, determinism, RoPE norm preservation, needle
placement (each needle group is a routing candidate of its target block)."""
import numpy as np
import torch

import hga_inputs as gi


def test_shapes_and_determinism():
    w = gi.QWEN3_8B_16K.with_(T=2048, n_needles=4)
    a = gi.make_inputs(w)
    b = gi.make_inputs(w)
    assert a.q.shape == (2048, 32, 128) and a.q.dtype == torch.bfloat16
    assert a.k.shape == (8, 2048, 128) and a.v.shape == (8, 2048, 128)
    assert torch.equal(a.q, b.q) and torch.equal(a.k, b.k)
    assert a.needles == b.needles and len(a.needles) == 8 * 4
    c = gi.make_inputs(w, seed=1)
    assert not torch.equal(a.q, c.q)


def test_rope_preserves_pair_norms():
    w = gi.TINY_FP32.with_(T=256)
    x = gi.make_inputs(w)
    rng = np.random.Generator(np.random.PCG64(0))
    q = rng.standard_normal((256, 2, 64), dtype=np.float32).astype(np.float64)
    got = x.q.double().numpy()
    n_raw = q[..., :32] ** 2 + q[..., 32:] ** 2
    n_rot = got[..., :32] ** 2 + got[..., 32:] ** 2
    np.testing.assert_allclose(n_rot, n_raw, rtol=1e-5, atol=1e-5)
    # position 0 is not rotated
    np.testing.assert_allclose(got[0], q[0], rtol=1e-6, atol=1e-6)


def test_needles_are_candidates():
    w = gi.QWEN3_30B_64K.with_(T=8192, q0=6144, n_needles=16)
    x = gi.make_inputs(w)
    assert len(x.needles) == 4 * 16
    for h, j, b in x.needles:
        b0 = w.q0 + b * w.qblock
        c = j * w.group // w.chunk
        assert c * w.chunk >= w.sink and (c + 1) * w.chunk <= b0 - w.local
        assert 0 <= b < w.Tq // w.qblock


def test_q_before_shape_determinism_and_rotation():
    """The queries before a segment: [qblock][Hq][d] in the storage dtype,
    the same draw every call, zero when no earlier position exists, and
    rotated at their own positions (RoPE keeps each pair's norm)."""
    w = gi.QWEN3_30B_64K.with_(T=8168, q0=6144)
    a, b = gi.make_q_before(w), gi.make_q_before(w)
    assert a.shape == (w.qblock, w.n_q_heads, w.head_dim) and a.dtype == torch.bfloat16
    assert torch.equal(a, b)
    assert not gi.make_q_before(gi.TINY_FP32).any()
    rng = np.random.Generator(np.random.PCG64(w.seed + 2))
    raw = rng.standard_normal((w.qblock, w.n_q_heads, w.head_dim), dtype=np.float32)
    half = w.head_dim // 2
    norm = lambda x: np.sqrt(x[..., :half] ** 2 + x[..., half:] ** 2)
    got = a.float().numpy().astype(np.float64)
    assert np.allclose(norm(got), norm(raw.astype(np.float64)), rtol=2e-2, atol=2e-2)
    assert not np.allclose(got, raw, atol=1e-2)          # rotated, not the raw draw

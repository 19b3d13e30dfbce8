"""Pins of the oracle's strictly causal routing variant.

"Long-Context Fine-Tuning with Limited VRAM", section 6.1: one routing set is
shared by every position of a block and depends on the scores of all its
query positions, so an earlier token can learn about later ones through it
(a causal side channel); a strictly causal routing variant is named there and
its design left open.  The reading implemented in the oracle: block b is
routed on the queries of the block before it (as many rows as b has), so the
output at a position depends on no later input.

The pins check, without retyping the oracle:
  * strict causality: changing q, k, v at positions after t leaves every
    output at positions <= t unchanged, while the block-shared routing fails
    the same check on a constructed case (the side channel is real and the
    check sees it);
  * which rows route: a needle query placed at the first or last row of the
    previous block steers block b, one placed in block b steers block b + 1
    instead, and for a ragged last block of n rows only the previous block's
    first n rows count;
  * at full budget the variant is dense causal attention (torch SDPA).
Planted mistakes in the variant's row choice each fail one of them."""
import numpy as np
import pytest
import torch

from oracle import hga_oracle as ho

D = 16


def _p(**kw):
    base = dict(n_q_heads=2, n_kv_heads=1, head_dim=D, sink=64, local=64, top_chunks=2,
                top_groups=4)
    base.update(kw)
    return ho.Params(**base)


def _inputs(T, q0, p, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T - q0, p.n_q_heads, D))
    k = rng.standard_normal((p.n_kv_heads, T, D))
    v = rng.standard_normal((p.n_kv_heads, T, D))
    qb = rng.standard_normal((p.qblock, p.n_q_heads, D))
    return q, k, v, qb


def _causal_out(q, k, v, qb, q0, p):
    res = ho.hga_forward(q, k, v, q0, p, q_route=ho.causal_route_queries(qb, q))
    return ho.assemble_output(res, q0, k.shape[1], p, D)[0], res


def _std_out(q, k, v, q0, p):
    res = ho.hga_forward(q, k, v, q0, p)
    return ho.assemble_output(res, q0, k.shape[1], p, D)[0], res


def pin_strict_causality(seed=0):
    """Outputs at positions <= t do not move when anything after t does."""
    p = _p()
    T, q0 = 448, 64
    q, k, v, qb = _inputs(T, q0, p, seed)
    O, _ = _causal_out(q, k, v, qb, q0, p)
    rng = np.random.default_rng(seed + 100)
    for t in (191, 192, 255, 300, 383):
        q2, k2, v2 = q.copy(), k.copy(), v.copy()
        q2[t + 1 - q0:] = rng.standard_normal(q2[t + 1 - q0:].shape) * 5
        k2[:, t + 1:] = rng.standard_normal(k2[:, t + 1:].shape) * 5
        v2[:, t + 1:] = rng.standard_normal(v2[:, t + 1:].shape) * 5
        O2, _ = _causal_out(q2, k2, v2, qb, q0, p)
        if not np.array_equal(O2[:t + 1 - q0], O[:t + 1 - q0]):
            return False
    return True


def _needle_case(p, T, q0, c_star, needle_pos, seed=1):
    """Keys of chunk c_star point along e0, every other key and every query is
    zero except the needle query (along e0) at position needle_pos (which may
    lie before q0, i.e. in q_before)."""
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((p.n_kv_heads, T, D)) * 0.01
    k[:, :, 0] = 0.0
    k[:, c_star * p.chunk:(c_star + 1) * p.chunk, 0] = 1.0
    v = rng.standard_normal((p.n_kv_heads, T, D))
    q = np.zeros((T - q0, p.n_q_heads, D))
    qb = np.zeros((p.qblock, p.n_q_heads, D))
    if needle_pos >= q0:
        q[needle_pos - q0, :, 0] = 50.0
    else:
        qb[needle_pos - (q0 - p.qblock), :, 0] = 50.0
    return q, k, v, qb


def pin_previous_block_rows(T=640, q0=128):
    """Block b (b0 = 448) is steered by a needle at b0 - 64 or b0 - 1; a needle
    at b0 steers block b + 1 instead; a needle before q0 (in q_before) steers
    the segment's first block."""
    p = _p(top_chunks=1, top_groups=8, local=64, sink=64)
    c_star = 4                                   # a candidate of blocks at b0 >= 384
    b0 = 448
    b = (b0 - q0) // p.qblock
    for pos, steered in ((b0 - 64, b), (b0 - 1, b), (b0, b + 1), (b0 + 63, b + 1)):
        q, k, v, qb = _needle_case(p, T, q0, c_star, pos)
        res = ho.hga_forward(q, k, v, q0, p, q_route=ho.causal_route_queries(qb, q),
                             with_attention=False)
        for bb in range(ho.n_blocks(q0, T, p)):
            picked = res.chunk_idx[(bb, 0)] == [c_star]
            if picked != (bb == steered):
                return False
    # the first block of a segment at q0 = 384 is routed by q_before
    q0b = 384
    q, k, v, qb = _needle_case(p, T, q0b, c_star - 1, q0b - 10)
    res = ho.hga_forward(q, k, v, q0b, p, q_route=ho.causal_route_queries(qb, q),
                         with_attention=False)
    return res.chunk_idx[(0, 0)] == [c_star - 1] and res.chunk_idx[(1, 0)] != [c_star - 1]


def pin_ragged_last_block():
    """The last block of n = 20 rows (positions 576..595) is routed on
    positions 512..531: a needle at 531 steers it, one at 532 does not."""
    p = _p(top_chunks=1, top_groups=8, local=64, sink=64)
    T, q0, c_star = 596, 128, 5
    last = ho.n_blocks(q0, T, p) - 1
    out = []
    for pos in (531, 532):
        q, k, v, qb = _needle_case(p, T, q0, c_star, pos)
        res = ho.hga_forward(q, k, v, q0, p, q_route=ho.causal_route_queries(qb, q),
                             with_attention=False)
        out.append(res.chunk_idx[(last, 0)] == [c_star])
    return out == [True, False]


def pin_full_budget_is_dense(seed=3):
    """With every candidate kept the variant is dense causal attention."""
    p = _p(top_chunks=0, top_groups=0, n_q_heads=4, n_kv_heads=2)
    T, q0 = 300, 70 - 70 % 64
    q, k, v, qb = _inputs(T, q0, p, seed)
    O, _ = _causal_out(q, k, v, qb, q0, p)
    from torch.nn.attention.bias import causal_lower_right
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(
        qt, torch.from_numpy(k)[None], torch.from_numpy(v)[None],
        attn_mask=causal_lower_right(T - q0, T), enable_gqa=True)[0].permute(1, 0, 2).numpy()
    return np.allclose(O, ref, atol=1e-12, rtol=1e-10)


PINS = (pin_strict_causality, pin_previous_block_rows, pin_ragged_last_block,
        pin_full_budget_is_dense)


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    assert pin()


def test_block_shared_routing_fails_the_causality_check():
    """The side channel of section 6.1 exists in the block-shared routing: a
    needle query late in a block changes the output at the block's first
    position.  The same change leaves the causal variant's output alone."""
    p = _p(top_chunks=1, top_groups=8, local=64, sink=64)
    T, q0, c_star, b0 = 640, 128, 4, 448
    q, k, v, qb = _needle_case(p, T, q0, c_star, b0 + 40)
    q_quiet = q.copy()
    q_quiet[b0 + 40 - q0] = 0.0
    q[b0 - q0, :, 1:] = q_quiet[b0 - q0, :, 1:] = 0.3    # the position we watch
    O_std, r_std = _std_out(q, k, v, q0, p)
    O_std_quiet, r_quiet = _std_out(q_quiet, k, v, q0, p)
    b = (b0 - q0) // p.qblock
    assert r_std.chunk_idx[(b, 0)] == [c_star] != r_quiet.chunk_idx[(b, 0)]
    assert not np.array_equal(O_std[b0 - q0], O_std_quiet[b0 - q0])
    O_c, _ = _causal_out(q, k, v, qb, q0, p)
    O_c_quiet, _ = _causal_out(q_quiet, k, v, qb, q0, p)
    assert np.array_equal(O_c[:b0 + 40 - q0], O_c_quiet[:b0 + 40 - q0])


def _rows_own_block(q, q0, T, p, b, h, q_route=None):      # ignores q_route
    return ho.block_rows(q, q0, T, p, b, h)


def _rows_shift_one(q, q0, T, p, b, h, q_route=None):      # one position late
    rows, b0, b1 = ho.block_rows(q, q0, T, p, b, h)
    if q_route is None:
        return rows, b0, b1
    full = np.concatenate([q_route, q[-1:]], axis=0)
    i0 = b * p.qblock + 1
    r = full[i0:i0 + (b1 - b0), h * p.G:(h + 1) * p.G, :]
    return r.reshape(-1, q.shape[-1]), b0, b1


def _rows_full_prev_block(q, q0, T, p, b, h, q_route=None):  # always qblock rows
    rows, b0, b1 = ho.block_rows(q, q0, T, p, b, h)
    if q_route is None:
        return rows, b0, b1
    # row j = the query at position q0 + j - qblock, for j < Tq + qblock
    full = np.concatenate([q_route, q[q.shape[0] - p.qblock:]], axis=0)
    i0 = b * p.qblock
    r = full[i0:i0 + p.qblock, h * p.G:(h + 1) * p.G, :]
    return r.reshape(-1, q.shape[-1]), b0, b1


@pytest.mark.parametrize("mistake", [_rows_own_block, _rows_shift_one, _rows_full_prev_block],
                         ids=lambda f: f.__name__)
def test_planted_row_mistakes_fail_a_pin(mistake, monkeypatch):
    monkeypatch.setattr(ho, "routing_rows", mistake)
    assert not all(pin() for pin in PINS), mistake.__name__

"""Pins of the oracle's backward pass (gradients of the routed attention with
the routing held fixed) against what the mathematics fixes:

* central finite differences of L = sum(dO * O) through the oracle's own
  forward attention, at sampled entries of q, k and v, on a case whose
  routing keeps only some groups (sink, routed groups, local window and the
  causal diagonal all carry gradient);
* the full-budget case, where routed attention is dense causal attention:
  the gradients equal torch autograd of the textbook dense attention in
  float64.

A dropped term (the D = dO . O correction), a wrong scale, or a transposed
operand fails one of them.
"""
import math

import numpy as np
import torch

from oracle import hga_oracle as ho


def _fixed_routing_loss(q, k, v, q0, p, groups, d_o):
    """sum(dO * O) with O from the oracle's attention over fixed groups."""
    T = k.shape[1]
    total = 0.0
    for h in range(p.n_kv_heads):
        for b in range(ho.n_blocks(q0, T, p)):
            o, _, _ = ho.attend_unit(q, k, v, q0, T, groups[(b, h)], p, b, h)
            r0 = b * p.qblock
            total += float(np.sum(d_o[r0:r0 + o.shape[0], h * p.G:(h + 1) * p.G] * o))
    return total


def _case(seed=0, T=256, q0=128, d=8, Hq=2, Hkv=1, top_chunks=1, top_groups=2):
    p = ho.Params(n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, sink=64, local=64,
                  top_chunks=top_chunks, top_groups=top_groups, dtype="fp32")
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T - q0, Hq, d))
    k = rng.standard_normal((Hkv, T, d))
    v = rng.standard_normal((Hkv, T, d))
    d_o = rng.standard_normal((T - q0, Hq, d))
    return p, q, k, v, d_o


def test_backward_matches_finite_differences():
    p, q, k, v, d_o = _case()
    T, q0 = k.shape[1], 128
    res = ho.hga_forward(q, k, v, q0, p)
    # the second block routes a proper subset of the candidate groups
    assert any(0 < len(g) < 8 for g in res.group_idx.values())
    O, L = ho.assemble_output(res, q0, T, p, q.shape[-1])
    dQ, dK, dV = ho.hga_backward(q, k, v, q0, p, res.group_idx, O, L, d_o)
    rng = np.random.default_rng(5)
    eps = 1e-6
    checked = 0
    for name, x, g in (("q", q, dQ), ("k", k, dK), ("v", v, dV)):
        flat = x.reshape(-1)
        idx = rng.choice(flat.size, size=24, replace=False)
        if name != "q":   # also tokens of the routed groups and of the windows
            extra = [(0, t, 0) for t in (3, 70, 120, 190, 250)]
            idx = np.concatenate([idx, [np.ravel_multi_index(e, x.shape) for e in extra]])
        for i in idx:
            old = flat[i]
            flat[i] = old + eps
            lp = _fixed_routing_loss(q, k, v, q0, p, res.group_idx, d_o)
            flat[i] = old - eps
            lm = _fixed_routing_loss(q, k, v, q0, p, res.group_idx, d_o)
            flat[i] = old
            fd = (lp - lm) / (2 * eps)
            an = g.reshape(-1)[i]
            assert abs(fd - an) <= 1e-6 + 1e-6 * abs(an), (name, int(i), fd, an)
            checked += 1
    assert checked >= 3 * 24


def test_backward_full_budget_equals_dense_autograd():
    p, q, k, v, d_o = _case(seed=1, T=320, q0=64, d=16, Hq=4, Hkv=2, top_chunks=0, top_groups=0)
    T, q0 = k.shape[1], 64
    res = ho.hga_forward(q, k, v, q0, p)
    O, L = ho.assemble_output(res, q0, T, p, q.shape[-1])
    dQ, dK, dV = ho.hga_backward(q, k, v, q0, p, res.group_idx, O, L, d_o)
    qt = torch.tensor(q, requires_grad=True)
    kt = torch.tensor(k, requires_grad=True)
    vt = torch.tensor(v, requires_grad=True)
    G = p.G
    outs = []
    for hq in range(p.n_q_heads):
        h = hq // G
        s = qt[:, hq, :] @ kt[h].T / math.sqrt(q.shape[-1])
        pos = torch.arange(q0, T)[:, None]
        s = s.masked_fill(torch.arange(T)[None, :] > pos, float("-inf"))
        outs.append(torch.softmax(s, dim=1) @ vt[h])
    Ot = torch.stack(outs, dim=1)
    (Ot * torch.tensor(d_o)).sum().backward()
    assert np.allclose(O, Ot.detach().numpy(), atol=1e-12, rtol=1e-12)
    assert np.allclose(dQ, qt.grad.numpy(), atol=1e-10, rtol=1e-10)
    assert np.allclose(dK, kt.grad.numpy(), atol=1e-10, rtol=1e-10)
    assert np.allclose(dV, vt.grad.numpy(), atol=1e-10, rtol=1e-10)


# ---------------------------------------------------------------- mutations

def _backward_no_d(q, k, v, q0, T, groups, p, b, h, o, lse, d_o):
    """Plants the classic mistake: ds = p * dp (the D = dO . o term dropped)."""
    zero_o = np.zeros_like(o)
    return _ORIG(q, k, v, q0, T, groups, p, b, h, zero_o, lse, d_o)


def _backward_dk_unscaled(q, k, v, q0, T, groups, p, b, h, o, lse, d_o):
    """Plants a missing 1/sqrt(d) on dk (dq kept right)."""
    dq, dk, dv = _ORIG(q, k, v, q0, T, groups, p, b, h, o, lse, d_o)
    return dq, dk * math.sqrt(q.shape[-1]), dv


def _backward_dv_transposed_heads(q, k, v, q0, T, groups, p, b, h, o, lse, d_o):
    """Plants dv accumulated with the wrong query head's dO."""
    return _ORIG(q, k, v, q0, T, groups, p, b, h, o, lse, d_o[:, ::-1])


_ORIG = ho.attend_unit_backward


def test_planted_backward_mistakes_fail_a_pin(monkeypatch):
    import pytest
    for bad in (_backward_no_d, _backward_dk_unscaled, _backward_dv_transposed_heads):
        monkeypatch.setattr(ho, "attend_unit_backward", bad)
        failed = False
        for pin in (test_backward_matches_finite_differences,
                    test_backward_full_budget_equals_dense_autograd):
            try:
                pin()
            except AssertionError:
                failed = True
                break
        monkeypatch.setattr(ho, "attend_unit_backward", _ORIG)
        assert failed, bad.__name__

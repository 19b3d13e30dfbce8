"""Pins of the CPU oracle against what the pages and the mathematics fix.

The pages print no worked numbers for the routed path, so the oracle is pinned
by: hand-derived golden cases (tests/golden), exact rational arithmetic for the
summaries and their rounding, brute-force subset search for the selection,
equality with torch's CPU scaled_dot_product_attention when the routing budget
covers everything (the router disabled = dense attention, page "Long-Context
Fine-Tuning with Limited VRAM", section 4.2), and set invariants.  Each pin is
a plain function so that test_oracle_mutations.py can plant mistakes in the
oracle and check that some pin fails.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import hga_oracle as ho

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- helpers

def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _geometry_inputs(keys_x, T, q0, qvec, d=2):
    k = np.zeros((1, T, d))
    k[0, :, 0] = np.asarray(keys_x[:T], dtype=np.float64)
    q = np.zeros((T - q0, 1, d))
    q[:, 0, :] = qvec
    return q, k


def _close(a, b, tol=1e-12):
    if b is None:
        return a == math.inf
    return abs(a - b) <= tol


def rne_fraction_bf16(m: Fraction) -> Fraction:
    """Independent exact round-to-nearest-even of a rational to bfloat16."""
    if m == 0:
        return Fraction(0)
    sign = -1 if m < 0 else 1
    a = abs(m)
    e = 0
    while a >= 2:
        a /= 2
        e += 1
    while a < 1:
        a *= 2
        e -= 1
    # |m| in [2**e, 2**(e+1)); 8 significant bits; subnormal floor 2**-133
    qe = max(e - 7, -133)
    q = Fraction(2) ** qe
    n = abs(m) / q
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * fl * q


# ---------------------------------------------------------------- pins

def pin_golden_routing():
    g = _load("hand_routing.json")
    pr = g["params"]
    for case in g["cases"]:
        p = ho.Params(1, 1, 2, chunk=pr["chunk"], group=pr["group"],
                      qblock=pr["qblock"], sink=pr["sink"], local=pr["local"],
                      top_chunks=case["top_chunks"],
                      top_groups=case["top_groups"], dtype="fp32")
        q, k = _geometry_inputs(g["keys_x"], case["T"], case["q0"], g["query"])
        res = ho.hga_forward(q, k, k, case["q0"], p, with_attention=False)
        assert list(res.chunk_idx[(0, 0)]) == case["chunks"], case
        assert list(res.group_idx[(0, 0)]) == case["groups"], case
        assert _close(res.chunk_margin[(0, 0)], case["chunk_margin"]), case
        assert _close(res.group_margin[(0, 0)], case["group_margin"]), case


def pin_golden_attention():
    g = _load("hand_attention.json")
    pr = g["params"]
    p = ho.Params(1, 1, 2, chunk=pr["chunk"], group=pr["group"],
                  qblock=pr["qblock"], sink=pr["sink"], local=pr["local"],
                  top_chunks=pr["top_chunks"], top_groups=pr["top_groups"],
                  dtype="fp32")
    T, q0 = pr["T"], pr["q0"]
    q, k = _geometry_inputs(g["keys_x"], T, q0, [g["a"], 0.0])
    v = np.zeros((1, T, 2))
    v[0, :, 1] = 1.0
    for t in g["v_first_tokens"]:
        v[0, t] = [1.0, 0.0]
    res = ho.hga_forward(q, k, v, q0, p)
    assert list(res.chunk_idx[(0, 0)]) == g["chunks"]
    assert list(res.group_idx[(0, 0)]) == g["groups"]
    o = res.o[(0, 0)][:, 0, :]
    np.testing.assert_allclose(o, np.array(g["o"]), rtol=0, atol=1e-13)
    np.testing.assert_allclose(res.lse[(0, 0)][:, 0], g["lse"], rtol=0,
                               atol=1e-13)
    assert abs(res.density - g["density"]) < 1e-15


def pin_bf16_rounding():
    rng = np.random.default_rng(5)
    # fp32-representable values: torch's float32 -> bfloat16 cast is one RNE.
    x = (rng.standard_normal(20000) *
         10.0 ** rng.integers(-40, 38, 20000)).astype(np.float32)
    x = np.concatenate([x, np.array([0.0, -0.0, 1e-45, 3.3e38, -2.5e-40],
                                    dtype=np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    got = ho.round_bf16(x.astype(np.float64))
    assert np.array_equal(ref, got)
    # float64 values that a detour through float32 would round twice.
    cases = [1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, 1 + 2.0 ** -8 + 2.0 ** -40,
             -(1 + 2.0 ** -8 + 2.0 ** -40), 2.0 ** -134, 3 * 2.0 ** -134,
             2.0 ** -134 + 2.0 ** -160, 255.5, 256.5 + 2.0 ** -30]
    for c in cases:
        want = rne_fraction_bf16(Fraction(c))
        assert Fraction(float(ho.round_bf16(np.array([c]))[0])) == want, c


def pin_summaries_exact():
    """Summaries equal the exact rational mean, rounded once (RNE)."""
    rng = np.random.default_rng(11)
    Hkv, T, d = 2, 192, 8
    k = ho.round_bf16(rng.standard_normal((Hkv, T, d)) * 3)
    p = ho.Params(2, 2, d, chunk=64, group=8, dtype="bf16")
    csum, gsum = ho.build_summaries(k, p, 64, 192)
    assert sorted(csum[0]) == [1, 2] and sorted(gsum[1]) == list(range(8, 24))
    for h in range(Hkv):
        for c, vec in csum[h].items():
            for i in range(d):
                m = sum(Fraction(float(k[h, t, i]))
                        for t in range(64 * c, 64 * c + 64)) / 64
                assert Fraction(float(vec[i])) == rne_fraction_bf16(m)
        for j, vec in gsum[h].items():
            for i in range(d):
                m = sum(Fraction(float(k[h, t, i]))
                        for t in range(8 * j, 8 * j + 8)) / 8
                assert Fraction(float(vec[i])) == rne_fraction_bf16(m)
    # constant keys: the summary is the key itself
    kc = np.ones((1, 128, 4)) * 0.3125
    cs, gs = ho.build_summaries(kc, ho.Params(1, 1, 4, dtype="fp32"), 0, 128)
    assert all((v == 0.3125).all() for v in cs[0].values())
    assert all((v == 0.3125).all() for v in gs[0].values())
    # a partial trailing chunk/group gets no summary
    cs, gs = ho.build_summaries(kc, ho.Params(1, 1, 4, dtype="fp32"), 0, 100)
    assert sorted(cs[0]) == [0] and sorted(gs[0]) == list(range(12))


def _brute_score(q, summ, q0, T, p, b, h):
    """Block score by explicit loops: max over rows of sum_i q_i s_i / sqrt(d)."""
    d = q.shape[-1]
    b0 = q0 + b * p.qblock
    best = -math.inf
    for pos in range(b0, min(b0 + p.qblock, T)):
        for hq in range(h * p.G, (h + 1) * p.G):
            acc = 0.0
            for i in range(d):
                acc += q[pos - q0, hq, i] * summ[i]
            best = max(best, acc / math.sqrt(d))
    return best


def _brute_select(cands, scores, k):
    """The unique subset whose every member beats every non-member in
    (higher score, then lower index); found by enumeration."""
    k_eff = len(cands) if k <= 0 else min(k, len(cands))
    found = []
    for sub in itertools.combinations(range(len(cands)), k_eff):
        inside = set(sub)
        ok = all((scores[i] > scores[u]) or
                 (scores[i] == scores[u] and cands[i] < cands[u])
                 for i in inside for u in range(len(cands)) if u not in inside)
        if ok:
            found.append(sorted(cands[i] for i in sub))
    assert len(found) == 1
    return found[0]


def pin_bruteforce_routing(seed=3, integer_valued=True):
    rng = np.random.default_rng(seed)
    Hq, Hkv, d, T, q0 = 4, 2, 4, 72, 24
    p = ho.Params(Hq, Hkv, d, chunk=8, group=2, qblock=8, sink=8, local=8,
                  top_chunks=2, top_groups=3, dtype="fp32")
    if integer_valued:   # many exact ties
        q = rng.integers(-1, 2, (T - q0, Hq, d)).astype(np.float64)
        k = rng.integers(-1, 2, (Hkv, T, d)).astype(np.float64)
    else:
        q = rng.standard_normal((T - q0, Hq, d))
        k = rng.standard_normal((Hkv, T, d))
    csum, gsum = ho.build_summaries(k, p, 0, T)
    res = ho.hga_forward(q, k, k, q0, p, csum=csum, gsum=gsum,
                         with_attention=False)
    n_checked = 0
    for (b, h), chunks in res.chunk_idx.items():
        b0 = q0 + b * p.qblock
        cands = [c for c in range(T // p.chunk)
                 if c * p.chunk >= p.sink and (c + 1) * p.chunk <= b0 - p.local]
        sc = [_brute_score(q, csum[h][c], q0, T, p, b, h) for c in cands]
        assert chunks == _brute_select(cands, sc, p.top_chunks)
        per = p.chunk // p.group
        gc = [c * per + i for c in chunks for i in range(per)]
        gsc = [_brute_score(q, gsum[h][j], q0, T, p, b, h) for j in gc]
        assert res.group_idx[(b, h)] == _brute_select(gc, gsc, p.top_groups)
        n_checked += len(cands) > 0
    assert n_checked >= 4


def _sdpa_dense(q, k, v, q0):
    """torch's CPU scaled_dot_product_attention (float64), causal aligned to
    the bottom-right corner (query i sits at position q0 + i)."""
    from torch.nn.attention.bias import causal_lower_right
    Tq, Hq, d = q.shape
    T = k.shape[1]
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    kt = torch.from_numpy(k)[None]
    vt = torch.from_numpy(v)[None]
    mask = causal_lower_right(Tq, T)
    o = torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=mask, enable_gqa=True)
    return o[0].permute(1, 0, 2).numpy()


def pin_dense_equivalence(q0=0, T=200, seed=7):
    rng = np.random.default_rng(seed)
    Hq, Hkv, d = 4, 2, 16
    q = rng.standard_normal((T - q0, Hq, d))
    k = rng.standard_normal((Hkv, T, d))
    v = rng.standard_normal((Hkv, T, d))
    p = ho.Params(Hq, Hkv, d, chunk=16, group=4, qblock=16, sink=16, local=32,
                  top_chunks=0, top_groups=0, dtype="fp32")
    res = ho.hga_forward(q, k, v, q0, p)
    O, L = ho.assemble_output(res, q0, T, p, d)
    Od, Ld = ho.dense_causal_attention(q, k, v, q0, Hq)
    np.testing.assert_allclose(O, Od, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Ld, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Od, _sdpa_dense(q, k, v, q0), rtol=0, atol=1e-12)
    assert abs(res.density - 1.0) < 1e-15


def pin_invariants(seed=9):
    rng = np.random.default_rng(seed)
    Hq, Hkv, d, T, q0 = 4, 2, 16, 1000, 320
    q = rng.standard_normal((T - q0, Hq, d))
    k = rng.standard_normal((Hkv, T, d))
    v = rng.standard_normal((Hkv, T, d))
    p = ho.Params(Hq, Hkv, d, chunk=64, group=8, qblock=64, sink=64, local=128,
                  top_chunks=3, top_groups=5, dtype="fp32")
    res = ho.hga_forward(q, k, v, q0, p)
    for (b, h), ch in res.chunk_idx.items():
        b0 = q0 + b * p.qblock
        n_cand = len(ho.chunk_candidates(b0, p))
        assert len(ch) == min(3, n_cand) and ch == sorted(set(ch))
        for c in ch:     # closed, outside sink and local, strictly in the past
            assert c * 64 >= p.sink and (c + 1) * 64 <= b0 - p.local
        gr = res.group_idx[(b, h)]
        assert len(gr) == min(5, 8 * len(ch)) and gr == sorted(set(gr))
        assert all(j // 8 in ch for j in gr)
        for pos in range(b0, min(b0 + 64, T)):
            R = ho.attention_set(b0, pos, gr, p)
            assert R.max() == pos                            # no future token
            assert set(range(min(64, pos + 1))) <= set(R)    # sink
            assert set(range(max(0, b0 - 128), pos + 1)) <= set(R)  # local+diag
            assert len(R) == len(set(R.tolist()))
    O, _ = ho.assemble_output(res, q0, T, p, d)
    assert np.isfinite(O).all()
    # every output row is a convex combination of true V rows: inside the
    # per-dimension hull of V
    assert (O <= v.max(axis=(0, 1)) + 1e-12).all()
    assert (O >= v.min(axis=(0, 1)) - 1e-12).all()


# ---------------------------------------------------------------- tests

def test_golden_routing():
    pin_golden_routing()


def test_golden_attention():
    pin_golden_attention()


def test_bf16_rounding():
    pin_bf16_rounding()


def test_summaries_exact():
    pin_summaries_exact()


@pytest.mark.parametrize("seed,integer_valued",
                         [(3, True), (4, True), (5, False)])
def test_bruteforce_routing(seed, integer_valued):
    pin_bruteforce_routing(seed, integer_valued)


@pytest.mark.parametrize("q0,T", [(0, 200), (48, 200), (64, 256), (0, 17)])
def test_dense_equivalence(q0, T):
    pin_dense_equivalence(q0, T)


def test_invariants():
    pin_invariants()


def test_dense_reference_is_sdpa_gqa():
    """The textbook dense reference itself agrees with torch's SDPA."""
    rng = np.random.default_rng(1)
    q = rng.standard_normal((30, 6, 8))
    k = rng.standard_normal((2, 50, 8))
    v = rng.standard_normal((2, 50, 8))
    O, _ = ho.dense_causal_attention(q, k, v, 20, 6)
    np.testing.assert_allclose(O, _sdpa_dense(q, k, v, 20), atol=1e-12)

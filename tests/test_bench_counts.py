"""The benchmark's algorithmic counts (the numerators of its roofline
fractions and its density) against what the oracle actually attends and
scores, on small workloads (no GPU).

The bench counts from the routed group counts alone: per query row, the sink,
the routed groups' tokens, the local window and the causal diagonal, and per
(block, KV head) the candidate chunks and the kept chunks' groups.  The
oracle builds every attention set explicitly; the two must agree exactly."""
import os
import sys

import numpy as np
import pytest

import hga_inputs as gi
from oracle import hga_oracle as ho

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    sys.path.insert(0, ROOT)
    import bench as mod
    return mod


CASES = [
    gi.TINY_FP32,
    gi.TINY_FP32.with_(T=1000, q0=256),
    gi.Workload("small_gqa", 8, 2, 32, 1536, 640, 1e6, 64, 256, 3, 5, n_needles=2),
    gi.Workload("small_all", 4, 1, 32, 900, 320, 1e6, 0, 0, 0, 0),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_counts_match_the_oracle(bench, w):
    p = ho.Params(w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk, w.group, w.qblock,
                  w.sink, w.local, w.top_chunks, w.top_groups, w.dtype)
    inp = gi.make_inputs(w)
    q, k, v = gi.to_f64(inp.q), gi.to_f64(inp.k), gi.to_f64(inp.v)
    res = ho.hga_forward(q, k, v, w.q0, p)
    nb = ho.n_blocks(w.q0, w.T, p)
    gcnt = np.zeros((w.n_kv_heads, nb), dtype=np.int64)
    route_chunk_pairs = route_group_pairs = 0
    for (b, h), groups in res.group_idx.items():
        gcnt[h, b] = len(groups)
        b0 = w.q0 + b * w.qblock
        rows = min(b0 + w.qblock, w.T) - b0
        route_chunk_pairs += rows * w.G * len(ho.chunk_candidates(b0, p))
        route_group_pairs += rows * w.G * len(res.chunk_idx[(b, h)]) * (w.chunk // w.group)
    c = bench.algorithmic_counts(w, gcnt)
    # attention: 4 d flops per (query row, attended token); the oracle counts
    # |R| per (position, query head)
    assert c["attn_flops"] == 4 * w.head_dim * res.attended
    assert c["density"] == pytest.approx(res.density, rel=1e-12)
    assert c["route_chunk_flops"] == 2 * w.head_dim * route_chunk_pairs
    assert c["route_group_flops"] == 2 * w.head_dim * route_group_pairs

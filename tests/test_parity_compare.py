"""The parity checker itself (CPU): compare() must accept a result that follows
the method, reject one whose output, padding or routing is off, and, where
the GPU may legitimately pick differently (an exact tie), check the output
against the oracle's attention over the groups the GPU picked."""
import copy

import numpy as np

import hga_inputs as gi
from oracle import hga_oracle as ho
import parity

W = gi.TINY_FP32.with_(T=1024)


def _oracle_as_gpu(w, inp, csum, gsum):
    """A GpuResult holding the oracle's own routing and outputs."""
    p = parity.oracle_params(w)
    q, k, v = gi.to_f64(inp.q), gi.to_f64(inp.k), gi.to_f64(inp.v)
    res = ho.hga_forward(q, k, v, w.q0, p, csum=csum, gsum=gsum)
    nb = ho.n_blocks(w.q0, w.T, p)
    cap_c, cap_g = w.top_chunks, w.top_groups
    ci = np.full((p.n_kv_heads, nb, cap_c), -1, np.int32)
    gi_ = np.full((p.n_kv_heads, nb, cap_g), -1, np.int32)
    cc = np.zeros((p.n_kv_heads, nb), np.int32)
    gc = np.zeros((p.n_kv_heads, nb), np.int32)
    for (b, h), ch in res.chunk_idx.items():
        ci[h, b, :len(ch)] = ch
        cc[h, b] = len(ch)
        gr = res.group_idx[(b, h)]
        gi_[h, b, :len(gr)] = gr
        gc[h, b] = len(gr)
    O, L = ho.assemble_output(res, w.q0, w.T, p, w.head_dim)
    return parity.GpuResult(np.zeros(1), np.zeros(1), ci, cc, gi_, gc, O, L), res


def _setup():
    inp = gi.make_inputs(W)
    csum, gsum = parity.oracle_summaries(W, inp)
    return inp, csum, gsum


def test_oracle_result_passes_and_every_unit_is_compared():
    inp, csum, gsum = _setup()
    g, _ = _oracle_as_gpu(W, inp, csum, gsum)
    rep = parity.compare(W, inp, g, check_summaries=False, summaries=(csum, gsum))
    assert rep.ok(), rep
    assert rep.compared_units == rep.units == 16 and rep.worst_excess < 0


def test_wrong_output_padding_or_routing_fails():
    inp, csum, gsum = _setup()
    g, _ = _oracle_as_gpu(W, inp, csum, gsum)
    bad_o = copy.deepcopy(g)
    bad_o.o[64 * 9 + 3, 1, 7] += 1e-3                 # one element of block 9
    rep = parity.compare(W, inp, bad_o, check_summaries=False, summaries=(csum, gsum))
    assert not rep.ok() and rep.worst_excess > 0
    bad_pad = copy.deepcopy(g)
    b = 15
    bad_pad.group_cnt[0, b] -= 1                      # count too small: slot left non -1
    rep = parity.compare(W, inp, bad_pad, check_summaries=False, summaries=(csum, gsum),
                         units=[(b, 0)])
    assert not rep.ok() and rep.pad_mismatch == 1
    bad_route = copy.deepcopy(g)
    bad_route.chunk_idx[0, b, 0], bad_route.chunk_idx[0, b, 1] = (
        bad_route.chunk_idx[0, b, 1], bad_route.chunk_idx[0, b, 0])   # not ascending
    rep = parity.compare(W, inp, bad_route, check_summaries=False, summaries=(csum, gsum),
                         units=[(b, 0)])
    assert not rep.ok()


def test_tie_choice_is_checked_on_the_gpu_groups():
    """Make the weakest kept group of the last block tie exactly with the best
    dropped one.  A GPU that keeps the other one of the pair (valid at a tie)
    passes only if its O is attention over the groups it kept."""
    inp, csum, gsum = _setup()
    p = parity.oracle_params(W)
    q = gi.to_f64(inp.q)
    b, h = 15, 0
    ch, _ = ho.route_chunks_unit(q, W.q0, W.T, csum[h], p, b, h)
    gr, _ = ho.route_groups_unit(q, W.q0, W.T, gsum[h], ch, p, b, h)
    rows, _, _ = ho.routing_rows(q, W.q0, W.T, p, b, h)
    cands = [c * 8 + i for c in ch for i in range(8)]
    sc = ho.block_scores(rows, np.stack([gsum[h][j] for j in cands]))
    score = dict(zip(cands, sc))
    j_min = min(gr, key=lambda j: (score[j], -j))
    j_out = max((j for j in cands if j not in gr), key=lambda j: (score[j], -j))
    gsum = copy.deepcopy(gsum)
    gsum[h][j_out] = gsum[h][j_min].copy()           # identical summaries: exact tie
    g, res = _oracle_as_gpu(W, inp, csum, gsum)
    gr_o = res.group_idx[(b, h)]
    assert min(j_min, j_out) in gr_o and max(j_min, j_out) not in gr_o
    swapped = sorted([j for j in gr_o if j != min(j_min, j_out)] + [max(j_min, j_out)])
    k, v = gi.to_f64(inp.k), gi.to_f64(inp.v)
    o_sw, l_sw, _ = ho.attend_unit(q, k, v, W.q0, W.T, swapped, p, b, h)
    tie = copy.deepcopy(g)
    tie.group_idx[h, b, :len(swapped)] = swapped
    rep = parity.compare(W, inp, tie, check_summaries=False, summaries=(csum, gsum))
    assert not rep.ok() and rep.worst_excess > 0      # O still over the oracle's groups
    b0 = b * 64
    tie.o[b0:b0 + 64, h * 2:(h + 1) * 2] = o_sw
    tie.lse[b0:b0 + 64, h * 2:(h + 1) * 2] = l_sw
    rep = parity.compare(W, inp, tie, check_summaries=False, summaries=(csum, gsum))
    assert rep.ok(), rep
    assert rep.tie_units_compared == 1 and rep.group_near_ties >= 1

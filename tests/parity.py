"""Parity helpers: run the CUDA path through the C ABI and compare it with the
CPU oracle on the same seeded inputs.

Rules (the routed path's stated tolerance):
  * summaries: bit-exact (both sides round the exact mean once);
  * routed chunk / group index sets: identical wherever the oracle's top-k
    margin exceeds NEAR_TIE (1e-4, scaled score units); near-ties are counted
    and the GPU's choice must still be a valid top-k within that band; where
    the chunk decision is a near-tie the group decision is excluded too;
  * outputs and LSE: |gpu - ref| <= atol + rtol*|ref| elementwise on every
    compared unit, against the oracle's attention over the groups the GPU
    attended (the oracle's own groups outside near-ties); bf16: atol 2e-3,
    rtol 1e-2; fp32: 1e-5 and 1e-5;
  * index slots past each count are -1 on every unit.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

import hga_inputs as gi
from oracle import hga_oracle as ho

NEAR_TIE = 1e-4
TOL = {"bf16": (2e-3, 1e-2), "fp32": (1e-5, 1e-5)}


def oracle_params(w: gi.Workload) -> ho.Params:
    return ho.Params(w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk, w.group,
                     w.qblock, w.sink, w.local, w.top_chunks, w.top_groups,
                     w.dtype)


@dataclasses.dataclass
class GpuResult:
    chunk_sum: np.ndarray
    group_sum: np.ndarray
    chunk_idx: np.ndarray
    chunk_cnt: np.ndarray
    group_idx: np.ndarray
    group_cnt: np.ndarray
    o: np.ndarray
    lse: np.ndarray


def run_gpu_causal(w: gi.Workload, inp: gi.Inputs, q_before) -> GpuResult:
    """Strictly causal routing variant: history summaries [0, q0) first, then
    hga_forward_causal on q_before followed by the segment's queries."""
    from long_context_hga_b200 import hga
    p = hga.Params.from_workload(w)
    dev = torch.device("cuda:0")
    q_ext = torch.cat([q_before, inp.q]).to(dev)
    k, v = inp.k.to(dev), inp.v.to(dev)
    bufs = hga.allocate(p, w.T, w.Tq, device=dev)
    if w.q0 > 0:
        hga.build_summaries(p, k, 0, w.q0, bufs.chunk_sum, bufs.group_sum)
    hga.forward_causal(p, q_ext, w.q0, k, v, bufs)
    st = hga.check()
    assert st == 0, f"device status {hga.status_string(st)}"
    f = lambda t: t.detach().to(torch.float64).cpu().numpy()
    return GpuResult(f(bufs.chunk_sum), f(bufs.group_sum),
                     bufs.chunk_idx.cpu().numpy(), bufs.chunk_cnt.cpu().numpy(),
                     bufs.group_idx.cpu().numpy(), bufs.group_cnt.cpu().numpy(),
                     f(bufs.o), bufs.lse.cpu().numpy().astype(np.float64))


def run_gpu(w: gi.Workload, inp: gi.Inputs, t_cap: Optional[int] = None,
            split_history: bool = True, v_f16: bool = False) -> GpuResult:
    """History summaries [0, q0) are built first (the committed history), then
    hga_forward runs summaries of the segment + routing + attention.  With
    v_f16 the attention reads V stored as fp16 (converted by the library), as
    the benchmark does."""
    from long_context_hga_b200 import hga
    p = hga.Params.from_workload(w)
    p_att = dataclasses.replace(p, v_f16=True) if v_f16 else p
    t_cap = t_cap or w.T
    dev = torch.device("cuda:0")
    q = inp.q.to(dev)
    k = torch.zeros(w.n_kv_heads, t_cap, w.head_dim, dtype=inp.k.dtype, device=dev)
    v = torch.zeros_like(k)
    k[:, :w.T] = inp.k.to(dev)
    v[:, :w.T] = inp.v.to(dev)
    bufs = hga.allocate(p, t_cap, w.Tq, device=dev)
    v_att = v
    if v_f16:
        v_att = torch.empty(v.shape, dtype=torch.float16, device=dev)
        hga.convert_v(p, v, 0, t_cap, v_att)
    if split_history and w.q0 > 0:
        hga.build_summaries(p, k, 0, w.q0, bufs.chunk_sum, bufs.group_sum)
        hga.forward(p_att, q, w.q0, k, v_att, bufs)
    else:
        hga.build_summaries(p, k, 0, w.T, bufs.chunk_sum, bufs.group_sum)
        hga.route_chunks(p, q, w.q0, bufs.chunk_sum, t_cap, bufs.chunk_idx,
                         bufs.chunk_cnt)
        hga.route_groups(p, q, w.q0, bufs.group_sum, t_cap, bufs.chunk_idx,
                         bufs.chunk_cnt, bufs.group_idx, bufs.group_cnt)
        hga.attend(p_att, q, w.q0, k, v_att, bufs.group_idx, bufs.group_cnt, bufs.o,
                   bufs.lse)
    st = hga.check()
    assert st == 0, f"device status {hga.status_string(st)}"
    f = lambda t: t.detach().to(torch.float64).cpu().numpy()
    return GpuResult(f(bufs.chunk_sum), f(bufs.group_sum),
                     bufs.chunk_idx.cpu().numpy(), bufs.chunk_cnt.cpu().numpy(),
                     bufs.group_idx.cpu().numpy(), bufs.group_cnt.cpu().numpy(),
                     f(bufs.o), bufs.lse.cpu().numpy().astype(np.float64))


@dataclasses.dataclass
class Report:
    units: int = 0
    chunk_near_ties: int = 0
    group_near_ties: int = 0
    chunk_mismatch: int = 0        # outside the near-tie band (must be 0)
    group_mismatch: int = 0
    pad_mismatch: int = 0          # index slots past the count that are not -1
    invalid_choice: int = 0        # near-tie choice that is not a valid top-k
    compared_units: int = 0
    tie_units_compared: int = 0    # compared on the GPU's own near-tie choice
    max_abs: float = 0.0
    max_rel: float = 0.0
    worst_excess: float = -math.inf   # max(|err| - (atol + rtol|ref|))
    lse_worst_excess: float = -math.inf
    density: float = 0.0

    def ok(self) -> bool:
        return (self.chunk_mismatch == 0 and self.group_mismatch == 0 and
                self.pad_mismatch == 0 and self.invalid_choice == 0 and
                self.worst_excess <= 0 and self.lse_worst_excess <= 0 and
                self.compared_units == self.units and self.units > 0)


def _valid_choice(chosen, cands, scores, k, band=NEAR_TIE) -> bool:
    """GPU choice is a top-k up to the near-tie band: right size, candidates
    only, and nobody outside beats anybody inside by more than the band."""
    k_eff = len(cands) if k <= 0 else min(k, len(cands))
    if len(chosen) != k_eff or len(set(chosen)) != k_eff:
        return False
    pos = {c: i for i, c in enumerate(cands)}
    if any(c not in pos for c in chosen):
        return False
    if sorted(chosen) != list(chosen):
        return False
    inside = set(chosen)
    if k_eff in (0, len(cands)):
        return True
    worst_in = min(scores[pos[c]] for c in inside)
    best_out = max(scores[i] for i, c in enumerate(cands) if c not in inside)
    return best_out <= worst_in + band


def oracle_summaries(w: gi.Workload, inp: gi.Inputs):
    """The oracle's chunk and group summaries of the whole context (reusable
    across compare() calls on the same inputs)."""
    return ho.build_summaries(gi.to_f64(inp.k), oracle_params(w), 0, w.T)


def compare(w: gi.Workload, inp: gi.Inputs, gpu: GpuResult, units=None,
            check_summaries: bool = True, q_route=None, summaries=None,
            f64=None) -> Report:
    """q_route (float64, from oracle causal_route_queries) compares against
    the strictly causal routing variant instead of the block-shared one.

    Every compared unit gets its outputs checked.  Where the GPU's chunk or
    group choice differs from the oracle's inside the near-tie band (and is a
    valid top-k there), the oracle routes the next level on the GPU's chunks
    and attends over the GPU's groups, so O and LSE are still compared
    against the oracle elementwise."""
    p = oracle_params(w)
    if f64 is None:
        f64 = (gi.to_f64(inp.q), gi.to_f64(inp.k), gi.to_f64(inp.v))
    q, k, v = f64
    T, q0 = w.T, w.q0
    csum, gsum = summaries if summaries is not None else ho.build_summaries(k, p, 0, T)
    if check_summaries:
        C, G = ho.summaries_as_arrays(csum, gsum, T // p.chunk, T // p.group,
                                      w.head_dim)
        n_c, n_g = T // p.chunk, T // p.group
        assert np.array_equal(gpu.chunk_sum[:, :n_c], C), "chunk summaries differ"
        assert np.array_equal(gpu.group_sum[:, :n_g], G), "group summaries differ"
    nb = ho.n_blocks(q0, T, p)
    if units is None:
        units = [(b, h) for h in range(p.n_kv_heads) for b in range(nb)]
    atol, rtol = TOL[w.dtype]
    rep = Report()
    att_total = 0
    causal_total = 0
    per = p.chunk // p.group
    for (b, h) in units:
        rep.units += 1
        rows, b0, b1 = ho.routing_rows(q, q0, T, p, b, h, q_route)
        ch_ref, ch_margin = ho.route_chunks_unit(q, q0, T, csum[h], p, b, h, q_route)
        ch_gpu = [int(x) for x in gpu.chunk_idx[h, b, :gpu.chunk_cnt[h, b]]]
        gr_gpu = [int(x) for x in gpu.group_idx[h, b, :gpu.group_cnt[h, b]]]
        pad_ok = ((gpu.chunk_idx[h, b, gpu.chunk_cnt[h, b]:] == -1).all() and
                  (gpu.group_idx[h, b, gpu.group_cnt[h, b]:] == -1).all())
        if not pad_ok:
            rep.pad_mismatch += 1
        cands = ho.chunk_candidates(b0, p)
        chunk_same = ch_gpu == ch_ref
        tie_path = False
        if ch_margin <= NEAR_TIE:
            rep.chunk_near_ties += 1
            if not chunk_same:
                sc = ho.block_scores(rows, np.stack([csum[h][c] for c in cands]))
                if not _valid_choice(ch_gpu, cands, sc, p.top_chunks):
                    rep.invalid_choice += 1
                    continue
                tie_path = True
        elif not chunk_same:
            rep.chunk_mismatch += 1
            continue
        # group routing on the chunks the GPU kept (the oracle's own, except
        # after a valid near-tie difference)
        gr_ref, gr_margin = ho.route_groups_unit(q, q0, T, gsum[h], ch_gpu, p, b, h,
                                                 q_route)
        group_same = gr_gpu == gr_ref
        if gr_margin <= NEAR_TIE or ch_margin <= NEAR_TIE:
            rep.group_near_ties += 1
            if not group_same:
                gc = [c * per + i for c in ch_gpu for i in range(per)]
                sc = ho.block_scores(rows, np.stack([gsum[h][j] for j in gc]))
                if not _valid_choice(gr_gpu, gc, sc, p.top_groups):
                    rep.invalid_choice += 1
                    continue
                tie_path = True
        elif not group_same:
            rep.group_mismatch += 1
            continue
        # attention over the groups the GPU attended
        o_ref, lse_ref, att = ho.attend_unit(q, k, v, q0, T, gr_gpu, p, b, h)
        att_total += att
        causal_total += p.G * sum(pos + 1 for pos in range(b0, b1))
        o_gpu = gpu.o[b0 - q0:b1 - q0, h * p.G:(h + 1) * p.G]
        l_gpu = gpu.lse[b0 - q0:b1 - q0, h * p.G:(h + 1) * p.G]
        err = np.abs(o_gpu - o_ref)
        rep.max_abs = max(rep.max_abs, float(err.max()))
        rep.max_rel = max(rep.max_rel,
                          float((err / np.maximum(np.abs(o_ref), 1e-6)).max()))
        rep.worst_excess = max(rep.worst_excess,
                               float((err - (atol + rtol * np.abs(o_ref))).max()))
        lerr = np.abs(l_gpu - lse_ref)
        rep.lse_worst_excess = max(rep.lse_worst_excess,
                                   float((lerr - (atol + rtol * np.abs(lse_ref))).max()))
        rep.compared_units += 1
        rep.tie_units_compared += int(tie_path)
    rep.density = att_total / max(1, causal_total)
    return rep


def sample_units(w: gi.Workload, n: int, seed: int = 0):
    """First and last block of every KV head plus n random (block, head)."""
    nb = -(-w.Tq // w.qblock)
    rng = np.random.default_rng(seed)
    units = {(0, 0), (nb - 1, w.n_kv_heads - 1), (nb // 2, 0)}
    while len(units) < n + 3:
        units.add((int(rng.integers(nb)), int(rng.integers(w.n_kv_heads))))
    return sorted(units)

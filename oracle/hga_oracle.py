"""CPU oracle for HGA exact-token two-level routed causal attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only the tests, the smoke check and the benchmark's CPU-baseline leg call it.
It shares no code with the CUDA library and is deliberately plain and slow:
NumPy float64, one (query block, KV head) unit at a time, library matmuls as
the only primitive.

What it follows ("Long-Context Fine-Tuning with Limited VRAM", section 2.1
"Exact-token hierarchical routing"):
  * the context is cut into 64-token chunks and 8-token groups and a summary
    is kept for each closed chunk and each group  -> build_summaries
  * the current query block scores the chunk summaries and keeps the most
    relevant chunks, besides fixed sink and local windows  -> route_chunks
  * the chosen chunks are opened at group level and the best groups inside
    them are kept  -> route_groups
  * exact token K/V of the chosen groups (plus the windows) feed ordinary
    softmax attention; summaries are never values  -> attend
The page's section 6.1 ("Long-horizon causal leakage") says one routing
decision is shared by all positions of a block; hence one routed set per
(query block, KV head).

Readings where the pages are silent (each is also listed in the design notes):
  * summary = mean of the post-RoPE keys of the chunk / group, computed in
    float64 and rounded once (round-to-nearest-even) to the storage dtype;
  * block score of a summary s = max over the block's query positions and the
    query heads sharing the KV head of (q . s) / sqrt(d);
  * candidate chunks of a block starting at b0: sink/C <= c < (b0 - local)/C
    (closed, outside the sink and the local window);
  * local window = the `local` tokens before the block, plus the block's own
    causal diagonal; sink = tokens [0, sink);
  * selection = first min(k, n) candidates in the order (score desc, index
    asc); k <= 0 means all; the group budget is global over the groups of the
    chosen chunks;
  * margin = k-th selected score minus best unselected score (+inf when all
    candidates are taken), in scaled units;
  * strictly causal routing variant (section 6.1 names it and leaves its
    design to future work): block b is routed on the queries of the block
    before it (positions b0 - qblock .. b0 - qblock + n - 1 for a block of n
    rows), so no position's output depends on a later input.

Parity pins (none of the pages' worked numbers exist; see tests/): dense
equivalence at full budget against torch's CPU scaled_dot_product_attention,
brute-force subset search for the selection on tiny inputs, closed-form
summaries, a hand-derived golden example, and set invariants.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np


# ---------------------------------------------------------------- rounding

def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even), returned as
    float64.  bfloat16: 8 significant bits, exponent range of float32
    (normal down to 2**-126, subnormal quantum 2**-133)."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = (x != 0) & np.isfinite(x)
    m, e = np.frexp(x[nz])                 # x = m * 2**e, 0.5 <= |m| < 1
    # 8 significant bits -> quantum 2**(e-8); never finer than the subnormal
    # quantum 2**-133.
    q_exp = np.maximum(e - 8, -133)
    scaled = np.ldexp(x[nz], -q_exp)       # exact (power-of-two scaling)
    r = np.rint(scaled)                    # round half to even
    out[nz] = np.ldexp(r, q_exp)
    big = np.abs(out) > 3.3895313892515355e38   # largest finite bfloat16
    out[big] = np.sign(out[big]) * np.inf
    out[~np.isfinite(x)] = x[~np.isfinite(x)]
    return out


def round_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return round_bf16(x)
    if dtype == "fp32":
        return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)
    raise ValueError(dtype)


# ---------------------------------------------------------------- params

@dataclass(frozen=True)
class Params:
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    chunk: int = 64
    group: int = 8
    qblock: int = 64
    sink: int = 64
    local: int = 128
    top_chunks: int = 4     # <= 0: all
    top_groups: int = 8     # <= 0: all
    dtype: str = "bf16"

    @property
    def G(self) -> int:
        return self.n_q_heads // self.n_kv_heads


# ---------------------------------------------------------------- step 1

def build_summaries(k: np.ndarray, p: Params, t_begin: int, t_end: int):
    """Chunk and group summaries of the keys in [t_begin, t_end).

    k: [Hkv][T][d] float64 (post-RoPE keys).  Returns (csum, gsum) with
    csum[h][c] for every chunk c fully inside [t_begin, t_end) and gsum[h][j]
    for every such group, as dicts {index: vector} per head, rounded to the
    storage dtype.  Only closed (complete) chunks/groups get a summary.
    """
    Hkv = k.shape[0]
    csum = [dict() for _ in range(Hkv)]
    gsum = [dict() for _ in range(Hkv)]
    for h in range(Hkv):
        for c in range(-(-t_begin // p.chunk), t_end // p.chunk):
            toks = k[h, c * p.chunk:(c + 1) * p.chunk, :]
            csum[h][c] = round_storage(toks.mean(axis=0), p.dtype)
        for j in range(-(-t_begin // p.group), t_end // p.group):
            toks = k[h, j * p.group:(j + 1) * p.group, :]
            gsum[h][j] = round_storage(toks.mean(axis=0), p.dtype)
    return csum, gsum


def summaries_as_arrays(csum, gsum, n_chunks: int, n_groups: int, d: int):
    """Dense [Hkv][n][d] arrays (NaN where no summary was built)."""
    Hkv = len(csum)
    C = np.full((Hkv, n_chunks, d), np.nan)
    Gs = np.full((Hkv, n_groups, d), np.nan)
    for h in range(Hkv):
        for c, vec in csum[h].items():
            C[h, c] = vec
        for j, vec in gsum[h].items():
            Gs[h, j] = vec
    return C, Gs


# ---------------------------------------------------------------- step 2/3

def block_rows(q: np.ndarray, q0: int, T: int, p: Params, b: int, h: int):
    """Query vectors of block b (positions b0..min(b0+B,T)-1) for the query
    heads h*G .. h*G+G-1, as an [n_pos * G][d] matrix, plus b0 and positions."""
    b0 = q0 + b * p.qblock
    b1 = min(b0 + p.qblock, T)
    rows = q[b0 - q0:b1 - q0, h * p.G:(h + 1) * p.G, :]
    return rows.reshape(-1, q.shape[-1]), b0, b1


def chunk_candidates(b0: int, p: Params) -> list:
    """Closed chunks outside the sink and the local window of a block at b0."""
    lo = p.sink // p.chunk
    hi = (b0 - p.local) // p.chunk if b0 - p.local > 0 else 0
    return list(range(lo, hi)) if hi > lo else []


def block_scores(rows: np.ndarray, summaries: np.ndarray) -> np.ndarray:
    """Max over the block's rows of (q . s) / sqrt(d), one per summary."""
    d = rows.shape[1]
    if summaries.shape[0] == 0:
        return np.zeros(0)
    s = rows @ summaries.T / math.sqrt(d)        # [rows][cands]
    return s.max(axis=0)


def select_top(cands: list, scores: np.ndarray, k: int):
    """First min(k, n) candidates in the order (score desc, index asc).
    Returns (chosen ascending, margin)."""
    n = len(cands)
    k_eff = n if k <= 0 else min(k, n)
    order = sorted(range(n), key=lambda i: (-scores[i], cands[i]))
    chosen = sorted(cands[i] for i in order[:k_eff])
    if k_eff == n or k_eff == 0:
        margin = math.inf
    else:
        margin = float(scores[order[k_eff - 1]] - scores[order[k_eff]])
    return chosen, margin


def causal_route_queries(q_before: np.ndarray, q: np.ndarray) -> np.ndarray:
    """Routing queries of the strictly causal variant, indexed like q: row i
    is the query at position q0 + i - qblock.  q_before [qblock][Hq][d] holds
    the queries of the qblock positions before q0 (any values when q0 = 0:
    the first block of a sequence has no candidates)."""
    return np.concatenate([q_before, q], axis=0)[:q.shape[0]]


def routing_rows(q, q0, T, p: Params, b: int, h: int, q_route=None):
    """Rows that score the summaries for block b, as an [n * G][d] matrix,
    plus b0 and b1.  Standard HGA (section 2.1; section 6.1 notes that one
    routing decision serves every position of the block): the block's own
    queries.  Strictly causal variant (section 6.1 leaves its design open;
    reading: the block is routed on the queries of the block before it, as
    many rows as the block has): rows b*qblock .. b*qblock + n - 1 of
    q_route (see causal_route_queries), i.e. positions b0 - qblock ..
    b1 - qblock - 1, all before the block's first token."""
    rows, b0, b1 = block_rows(q, q0, T, p, b, h)
    if q_route is None:
        return rows, b0, b1
    i0 = b * p.qblock
    r = q_route[i0:i0 + (b1 - b0), h * p.G:(h + 1) * p.G, :]
    return r.reshape(-1, q.shape[-1]), b0, b1


def route_chunks_unit(q, q0, T, csum_h, p: Params, b: int, h: int, q_route=None):
    rows, b0, _ = routing_rows(q, q0, T, p, b, h, q_route)
    cands = chunk_candidates(b0, p)
    if not cands:
        return [], math.inf
    S = np.stack([csum_h[c] for c in cands])
    return select_top(cands, block_scores(rows, S), p.top_chunks)


def route_groups_unit(q, q0, T, gsum_h, chunks: list, p: Params, b: int,
                      h: int, q_route=None):
    rows, _, _ = routing_rows(q, q0, T, p, b, h, q_route)
    per = p.chunk // p.group
    cands = [c * per + i for c in chunks for i in range(per)]
    if not cands:
        return [], math.inf
    S = np.stack([gsum_h[j] for j in cands])
    return select_top(cands, block_scores(rows, S), p.top_groups)


# ---------------------------------------------------------------- step 4

def attention_set(b0: int, pos: int, groups: list, p: Params) -> np.ndarray:
    """Token indices attended by the query at position pos of the block at b0:
    sink U routed groups' tokens U local window U causal diagonal, as a set."""
    toks = set(range(0, min(p.sink, pos + 1)))
    for j in groups:
        toks.update(range(j * p.group, (j + 1) * p.group))
    toks.update(range(max(0, b0 - p.local), b0))
    toks.update(range(b0, pos + 1))
    return np.array(sorted(toks), dtype=np.int64)


def attend_unit(q, k, v, q0, T, groups: list, p: Params, b: int, h: int):
    """Exact-token softmax attention of block b, KV head h over its routed set.
    Returns (o [n_pos][G][d], lse [n_pos][G] natural log of the scaled
    scores' sum of exponentials, attended token count summed over rows)."""
    d = q.shape[-1]
    b0 = q0 + b * p.qblock
    b1 = min(b0 + p.qblock, T)
    o = np.zeros((b1 - b0, p.G, d))
    lse = np.zeros((b1 - b0, p.G))
    attended = 0
    for pos in range(b0, b1):
        R = attention_set(b0, pos, groups, p)
        Kr = k[h, R, :]
        Vr = v[h, R, :]
        for gi in range(p.G):
            qv = q[pos - q0, h * p.G + gi, :]
            s = Kr @ qv / math.sqrt(d)
            m = s.max()
            e = np.exp(s - m)
            z = e.sum()
            o[pos - b0, gi] = (e @ Vr) / z
            lse[pos - b0, gi] = m + math.log(z)
        attended += len(R) * p.G
    return o, lse, attended


# ---------------------------------------------------------------- whole pass

@dataclass
class Result:
    chunk_idx: dict = field(default_factory=dict)     # (b, h) -> list
    chunk_margin: dict = field(default_factory=dict)  # (b, h) -> float
    group_idx: dict = field(default_factory=dict)
    group_margin: dict = field(default_factory=dict)
    o: dict = field(default_factory=dict)             # (b, h) -> [n_pos][G][d]
    lse: dict = field(default_factory=dict)
    attended: int = 0
    causal_total: int = 0

    @property
    def density(self) -> float:
        return self.attended / max(1, self.causal_total)


def n_blocks(q0: int, T: int, p: Params) -> int:
    return -(-(T - q0) // p.qblock)


def hga_forward(q, k, v, q0: int, p: Params, units=None, csum=None,
                gsum=None, with_attention: bool = True, q_route=None) -> Result:
    """Run the four steps for the query segment [q0, T).

    q [Tq][Hq][d], k and v [Hkv][T][d], float64 holding the exact storage
    values.  `units` restricts the work to a list of (block, kv_head) pairs
    (default: all).  Summaries cover [0, T) unless given.  q_route (from
    causal_route_queries) selects the strictly causal routing variant;
    attention always uses q."""
    T = k.shape[1]
    if csum is None or gsum is None:
        csum, gsum = build_summaries(k, p, 0, T)
    if units is None:
        units = [(b, h) for h in range(p.n_kv_heads)
                 for b in range(n_blocks(q0, T, p))]
    res = Result()
    for (b, h) in units:
        ch, cm = route_chunks_unit(q, q0, T, csum[h], p, b, h, q_route)
        gr, gm = route_groups_unit(q, q0, T, gsum[h], ch, p, b, h, q_route)
        res.chunk_idx[(b, h)] = ch
        res.chunk_margin[(b, h)] = cm
        res.group_idx[(b, h)] = gr
        res.group_margin[(b, h)] = gm
        if with_attention:
            o, lse, att = attend_unit(q, k, v, q0, T, gr, p, b, h)
            res.o[(b, h)] = o
            res.lse[(b, h)] = lse
            res.attended += att
            b0 = q0 + b * p.qblock
            b1 = min(b0 + p.qblock, T)
            res.causal_total += p.G * sum(pos + 1 for pos in range(b0, b1))
    return res


def assemble_output(res: Result, q0: int, T: int, p: Params, d: int):
    """Gather per-unit outputs into O [Tq][Hq][d] and LSE [Tq][Hq]."""
    Tq = T - q0
    O = np.full((Tq, p.n_q_heads, d), np.nan)
    L = np.full((Tq, p.n_q_heads), np.nan)
    for (b, h), o in res.o.items():
        b0 = b * p.qblock
        O[b0:b0 + o.shape[0], h * p.G:(h + 1) * p.G] = o
        L[b0:b0 + o.shape[0], h * p.G:(h + 1) * p.G] = res.lse[(b, h)]
    return O, L


# ---------------------------------------------------------------- dense

def dense_causal_attention(q, k, v, q0: int, n_q_heads: int):
    """Textbook causal softmax attention with grouped KV heads: query at
    position p (query head hq) attends to keys 0..p of KV head hq // G."""
    Tq, Hq, d = q.shape
    Hkv = k.shape[0]
    G = Hq // Hkv
    O = np.zeros_like(q)
    L = np.zeros((Tq, Hq))
    for hq in range(Hq):
        h = hq // G
        s = q[:, hq, :] @ k[h].T / math.sqrt(d)            # [Tq][T]
        pos = np.arange(q0, q0 + Tq)[:, None]
        s = np.where(np.arange(k.shape[1])[None, :] <= pos, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        z = e.sum(axis=1, keepdims=True)
        O[:, hq, :] = (e @ v[h]) / z
        L[:, hq] = (m + np.log(z))[:, 0]
    return O, L


# ---------------------------------------------------------------- backward

def attend_unit_backward(q, k, v, q0, T, groups: list, p: Params, b: int, h: int,
                         o, lse, d_o):
    """Gradients of the exact-token attention of block b, KV head h, with the
    routed groups held fixed (the selection is piecewise constant, so no
    gradient flows into the summaries): for a row with attended set R,
        s_j = q . k_j / sqrt(d),  p_j = exp(s_j - lse),  o = sum_j p_j v_j,
        dp_j = dO . v_j,  D = dO . o,  ds_j = p_j (dp_j - D),
        dq = sum_j ds_j k_j / sqrt(d),  dk_j += ds_j q / sqrt(d),  dv_j += p_j dO.
    o [n_pos][G][d] and lse [n_pos][G] are the forward's outputs as given (the
    caller's O and LSE, so D and p use the same values a kernel would).
    Returns (dq [n_pos][G][d], dk [T][d], dv [T][d]) for this unit."""
    d = q.shape[-1]
    b0 = q0 + b * p.qblock
    b1 = min(b0 + p.qblock, T)
    dq = np.zeros((b1 - b0, p.G, d))
    dk = np.zeros((T, d))
    dv = np.zeros((T, d))
    for pos in range(b0, b1):
        R = attention_set(b0, pos, groups, p)
        Kr = k[h, R, :]
        Vr = v[h, R, :]
        for gi in range(p.G):
            qv = q[pos - q0, h * p.G + gi, :]
            g = d_o[pos - b0, gi]
            s = Kr @ qv / math.sqrt(d)
            pj = np.exp(s - lse[pos - b0, gi])
            dp = Vr @ g
            D = float(g @ o[pos - b0, gi])
            ds = pj * (dp - D)
            dq[pos - b0, gi] = ds @ Kr / math.sqrt(d)
            dk[R] += np.outer(ds, qv) / math.sqrt(d)
            dv[R] += np.outer(pj, g)
    return dq, dk, dv


def hga_backward(q, k, v, q0: int, p: Params, group_idx: dict, O, L, dO):
    """Gradients of the routed attention for the segment [q0, T) with the
    routing (group lists per (block, KV head)) of a forward pass held fixed.
    q [Tq][Hq][d], k, v [Hkv][T][d], O and dO [Tq][Hq][d], L [Tq][Hq] (natural
    log), all float64.  Returns dQ [Tq][Hq][d], dK and dV [Hkv][T][d]."""
    T = k.shape[1]
    Tq, Hq, d = q.shape
    dQ = np.zeros((Tq, Hq, d))
    dK = np.zeros_like(k)
    dV = np.zeros_like(v)
    for h in range(p.n_kv_heads):
        for b in range(n_blocks(q0, T, p)):
            r0 = b * p.qblock
            r1 = min(r0 + p.qblock, Tq)
            hs = slice(h * p.G, (h + 1) * p.G)
            dq, dk, dv = attend_unit_backward(q, k, v, q0, T, group_idx[(b, h)], p, b, h,
                                              O[r0:r1, hs], L[r0:r1, hs], dO[r0:r1, hs])
            dQ[r0:r1, hs] = dq
            dK[h] += dk
            dV[h] += dv
    return dQ, dK, dV

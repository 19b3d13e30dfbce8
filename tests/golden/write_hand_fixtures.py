"""Writes the hand-derived golden fixtures in this folder.

Every value here is a closed form worked out by hand from the routing rules of
"Long-Context Fine-Tuning with Limited VRAM", section 2.1; the derivation text
is stored beside the numbers.  Nothing is computed by the oracle or the GPU.
Run from the repository root: python tests/golden/write_hand_fixtures.py
"""
import json
import math
import os

HERE = os.path.dirname(os.path.abspath(__file__))


def main():
    a = math.sqrt(2) * math.log(4.5) / 3
    routing = {
        "citation": "Long-Context Fine-Tuning with Limited VRAM, section 2.1 (Exact-token hierarchical routing): closed-chunk summaries scored by the query block, chosen besides fixed sink and local windows; chosen chunks opened at group level, best groups kept.",
        "derivation": "d=2, one KV head, one query head, chunk 4, group 2, query block 4, sink 4, local 4. Key x-components per token: chunk0 (tokens 0-3) = 10, chunk1 = 0, chunk2 = 1,1,3,3, chunk3 = 1, chunk4 (16-19) = 10, tokens 20-23 = 10; y = 0. Queries (1, 0). Summary = mean key, so chunk x-means are 10,0,2,1,10 and group x-means 10,10,0,0,1,3,1,1,10,10,... A block at b0 may route only chunks c with sink/chunk <= c < (b0-local)/chunk: for b0=20 that is chunks 1..3 (chunk0 is the sink, chunk4 is the local window, so the two 10-valued chunks must never be routed). Scores are x-mean/sqrt(2); ties go to the lower index; margins are the k-th kept score minus the best dropped one.",
        "keys_x": [10, 10, 10, 10, 0, 0, 0, 0, 1, 1, 3, 3, 1, 1, 1, 1,
                   10, 10, 10, 10, 10, 10, 10, 10],
        "query": [1.0, 0.0],
        "params": {"chunk": 4, "group": 2, "qblock": 4, "sink": 4, "local": 4},
        "cases": [
            {"T": 24, "q0": 20, "top_chunks": 1, "top_groups": 1,
             "chunks": [2], "groups": [5],
             "chunk_margin": 1 / math.sqrt(2), "group_margin": 2 / math.sqrt(2)},
            {"T": 24, "q0": 20, "top_chunks": 2, "top_groups": 2,
             "chunks": [2, 3], "groups": [4, 5],
             "chunk_margin": 1 / math.sqrt(2), "group_margin": 0.0},
            {"T": 24, "q0": 20, "top_chunks": 0, "top_groups": 3,
             "chunks": [1, 2, 3], "groups": [4, 5, 6],
             "chunk_margin": None, "group_margin": 0.0},
            {"T": 24, "q0": 20, "top_chunks": 0, "top_groups": 0,
             "chunks": [1, 2, 3], "groups": [2, 3, 4, 5, 6, 7],
             "chunk_margin": None, "group_margin": None},
            {"T": 12, "q0": 8, "top_chunks": 1, "top_groups": 1,
             "chunks": [], "groups": [],
             "chunk_margin": None, "group_margin": None},
            {"T": 16, "q0": 12, "top_chunks": 1, "top_groups": 1,
             "chunks": [1], "groups": [2],
             "chunk_margin": None, "group_margin": 0.0},
        ],
        "note": "margin null means +infinity (every candidate kept or none exists).",
    }
    attn = {
        "citation": "Long-Context Fine-Tuning with Limited VRAM, section 2.1: only the exact token K/V of the selected groups (with the sink and local windows) enter softmax attention; summaries are never values.",
        "derivation": "Same geometry as hand_routing.json with x-components chunk0 = 0, chunk1 = 0, chunk2 = 1,1,3,3, chunk3 = 1, chunk4 = 0, tokens 20-23 = 0, y = 0, one chunk and one group routed. Queries (a, 0) with a = sqrt(2)*ln(4.5)/3, so chunk 2 (x-mean 2) beats chunk 3 (1) and chunk 1 (0), and group 5 (tokens 10, 11; x = 3) beats group 4. A query at position p attends tokens 0-3 (sink), 10-11 (routed), 16-19 (local) and 20..p (diagonal). Tokens 10 and 11 score a*3/sqrt(2) = ln 4.5, all others 0, so the softmax weights are 4.5 and 1. V is (1,0) at tokens 10, 11 and (0,1) elsewhere, giving o = (9, n0)/(9 + n0) with n0 = 9 + (p - 20) zero-score tokens, and lse = ln(9 + n0).",
        "a": a,
        "keys_x": [0, 0, 0, 0, 0, 0, 0, 0, 1, 1, 3, 3, 1, 1, 1, 1,
                   0, 0, 0, 0, 0, 0, 0, 0],
        "v_first_tokens": [10, 11],
        "params": {"chunk": 4, "group": 2, "qblock": 4, "sink": 4, "local": 4,
                   "top_chunks": 1, "top_groups": 1, "T": 24, "q0": 20},
        "chunks": [2], "groups": [5],
        "o": [[9 / 18, 9 / 18], [9 / 19, 10 / 19], [9 / 20, 11 / 20],
              [9 / 21, 12 / 21]],
        "lse": [math.log(18), math.log(19), math.log(20), math.log(21)],
        "density": 50 / 90,
    }
    with open(os.path.join(HERE, "hand_routing.json"), "w") as f:
        json.dump(routing, f, indent=1)
    with open(os.path.join(HERE, "hand_attention.json"), "w") as f:
        json.dump(attn, f, indent=1)


if __name__ == "__main__":
    main()

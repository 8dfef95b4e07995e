"""Pure-Python brute force of MLA decode attention -- TEST INFRASTRUCTURE ONLY.

Scalar loops over Python lists, for tiny shapes (a few heads, a handful of
tokens).  It is written independently of ``mla_oracle`` (no NumPy, no shared
helpers) so that agreement between the two pins both.  Same definition:
order 1 of the MLA matrix-absorption notes (§2.1 Steps 2-3 for the logits,
§3.1 Steps 1-2 for the output) plus the RoPE-MQA score of the izhida.com
answer, standard softmax with the query of index i among s new tokens
attending keys t <= T - s + i.
"""
from __future__ import annotations

import math


def brute_decode(q_nope, q_rope, caches, W_UK, W_UV, s_q, scale, visible=None):
    """Nested lists in, nested lists out.

    q_nope[n][h][d], q_rope[n][h][r], caches[b][t][k + r] (latent then rope),
    W_UK[k][h][d], W_UV[k][h][v].  Returns (out[n][h][v], lse[n][h]).
    ``visible`` (optional): visible[b][i] is the list of key positions query
    i of sequence b attends, in place of 0 .. T - s + i.
    """
    n_rows = len(q_nope)
    H = len(q_nope[0])
    d = len(q_nope[0][0])
    R = len(q_rope[0][0])
    dc = len(W_UK)
    v = len(W_UV[0][0])
    out = [[[0.0] * v for _ in range(H)] for _ in range(n_rows)]
    lse = [[0.0] * H for _ in range(n_rows)]
    for b, cache in enumerate(caches):
        T = len(cache)
        for i in range(s_q):
            n = b * s_q + i
            keys = list(range(T - s_q + i + 1)) if visible is None else list(visible[b][i])
            for h in range(H):
                logits = []
                for t in keys:
                    acc = 0.0
                    for j in range(d):
                        kj = 0.0
                        for c in range(dc):
                            kj += cache[t][c] * W_UK[c][h][j]
                        acc += q_nope[n][h][j] * kj
                    for r in range(R):
                        acc += q_rope[n][h][r] * cache[t][dc + r]
                    logits.append(acc * scale)
                m = max(logits)
                w = [math.exp(x - m) for x in logits]
                z = sum(w)
                lse[n][h] = m + math.log(z)
                for j in range(v):
                    acc = 0.0
                    for a, t in enumerate(keys):
                        vj = 0.0
                        for c in range(dc):
                            vj += cache[t][c] * W_UV[c][h][j]
                        acc += (w[a] / z) * vj
                    out[n][h][j] = acc
    return out, lse

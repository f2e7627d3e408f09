"""Pure-Python brute force of the same block attention, for tiny inputs.

TEST INFRASTRUCTURE ONLY (see oracle/oracle.py for who may use it).

Written independently of oracle.py: no numpy arithmetic, one explicit loop
per query row over every visible key, Python floats (IEEE double) and
``math.exp`` / ``math.log``.  It follows the same statement of the method
(paperfeed.app review of arXiv 2606.26493, section "The idea: freeze the
reader, train the writer": layer-i queries of the noisy block attend to the
context tower's layer-i cache followed by the block's own KV, one softmax;
section "Training and sampling" for the c_{<b} conditioning of block b).

Visibility is decided per (query position, key position) by an explicit
predicate rather than by slicing, so a slicing mistake in the oracle and a
predicate mistake here cannot cancel.
"""
from __future__ import annotations

import math


def _row(qv, keys, vals, scale):
    scores = []
    for kv in keys:
        acc = 0.0
        for a, b in zip(qv, kv):
            acc += a * b
        scores.append(scale * acc)
    m = max(scores)
    w = [math.exp(s - m) for s in scores]
    z = 0.0
    for x in w:
        z += x
    D = len(vals[0])
    out = [0.0] * D
    for wi, vv in zip(w, vals):
        for d in range(D):
            out[d] += wi * vv[d]
    return [o / z for o in out], m + math.log(z)


def brute_block_attn(q, k_ctx, v_ctx, k_blk, v_blk, ctx_lens, scale=None):
    """Same contract as oracle.block_attn; nested lists or arrays accepted.

    Returns (out, lse) as nested Python lists [B][S][Hq][D] and [B][Hq][S].
    """
    B, S, Hq, D = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    Hkv, Lcap = len(k_ctx[0]), len(k_ctx[0][0])
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out = [[[None] * Hq for _ in range(S)] for _ in range(B)]
    lse = [[[None] * S for _ in range(Hq)] for _ in range(B)]
    for n in range(B):
        for j in range(Hq):
            # query head j reads KV head floor(j * Hkv / Hq)
            h = (j * Hkv) // Hq
            keys, vals = [], []
            for l in range(Lcap):
                if l < int(ctx_lens[n]):
                    keys.append([float(x) for x in k_ctx[n][h][l]])
                    vals.append([float(x) for x in v_ctx[n][h][l]])
            for u in range(S):
                keys.append([float(x) for x in k_blk[n][u][h]])
                vals.append([float(x) for x in v_blk[n][u][h]])
            for t in range(S):
                o, l = _row([float(x) for x in q[n][t][j]], keys, vals, scale)
                out[n][t][j] = o
                lse[n][j][t] = l
    return out, lse


def brute_block_causal(q, k_ctx, v_ctx, k_blk, v_blk, block_size, scale=None):
    """Whole-sequence form by an explicit visibility predicate.

    Query position p (block b = p // S) sees context position c iff
    c < S*b (clean context of earlier blocks only) and block position u iff
    u // S == b (its own block, bidirectionally).  Keys are visited context
    first, then block, matching the concatenation order of the method.
    """
    B, N, Hq, D = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    Hkv = len(k_ctx[0])
    S = int(block_size)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out = [[[None] * Hq for _ in range(N)] for _ in range(B)]
    lse = [[[None] * N for _ in range(Hq)] for _ in range(B)]
    for n in range(B):
        for j in range(Hq):
            h = (j * Hkv) // Hq
            for p in range(N):
                b = p // S
                keys, vals = [], []
                for c in range(N):
                    if c < S * b:
                        keys.append([float(x) for x in k_ctx[n][h][c]])
                        vals.append([float(x) for x in v_ctx[n][h][c]])
                for u in range(N):
                    if u // S == b:
                        keys.append([float(x) for x in k_blk[n][u][h]])
                        vals.append([float(x) for x in v_blk[n][u][h]])
                o, l = _row([float(x) for x in q[n][p][j]], keys, vals, scale)
                out[n][p][j] = o
                lse[n][j][p] = l
    return out, lse

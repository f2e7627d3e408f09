"""Float64 CPU oracle for TwoTower layer-aligned block attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It
shares no code, constant or helper with the CUDA library; the only thing both
sides see is the seeded input generator, which holds none of the method's
arithmetic.

What it computes (sources: the paperfeed.app review of arXiv 2606.26493,
"Nemotron-Labs-TwoTower: Diffusion Language Modeling with Pretrained
Autoregressive Context", section "The idea: freeze the reader, train the
writer", the paragraphs on the context tower and on the denoiser's layer-i
attention; and section "Training and sampling" for the block-causal form):

* the denoiser's queries come from the S noisy tokens of the current block;
* the keys and values are the concatenation of the frozen context tower's
  layer-i KV cache over the committed tokens with the denoiser's own KV for
  the block (same section: the page describes the denoiser's layer-i keys and
  values as the context cache of the earlier blocks joined to the block's own);
* the cache is fully visible to every block query (only the context tower
  itself is causal), and attention inside the block is bidirectional, still-masked
  positions included (same section, on the block's own attention);
* one softmax runs over the concatenation.  The equation itself did not
  survive the page extraction; the joint softmax is the plain reading of the
  surrounding prose.

Readings the pages leave open (each also listed in the design notes):
  scale = 1/sqrt(head_dim) unless given; query head j uses KV head j // g
  (g = Hq / Hkv, contiguous groups); context rows at or beyond ctx_lens[n]
  are never read; lse is in natural log; no dropout, softcap, sink or bias.

Every routine below is the definition written out: explicit max, exp, sum
and divide over the concatenated keys, with numpy matmul as the only library
primitive.  Pinned by tests/test_oracle.py (closed forms, invariants,
brute force, and independent library routines).
"""
from __future__ import annotations

import numpy as np

__all__ = ["block_attn", "block_causal", "attend_rows"]


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def attend_rows(qrows, keys, vals, scale):
    """Softmax attention of query rows over one key set.

    qrows [R, D], keys [K, D], vals [K, D] (float64).  Returns (out [R, D],
    lse [R]).  This is the single joint softmax of the denoiser's layer-i
    attention: s = scale * q.k for every key, out = sum_k e^{s_k - m} v_k /
    sum_k e^{s_k - m} with m the row maximum, lse = m + ln(sum_k e^{s_k - m}).
    """
    s = scale * (qrows @ keys.T)                 # [R, K] scores
    m = s.max(axis=1, keepdims=True)             # row maximum
    e = np.exp(s - m)                            # unnormalised weights
    z = e.sum(axis=1, keepdims=True)             # partition function
    out = (e @ vals) / z
    lse = m[:, 0] + np.log(z[:, 0])
    return out, lse


def block_attn(q, k_ctx, v_ctx, k_blk, v_blk, ctx_lens, scale=None):
    """Decode-time block attention for one denoising step of one layer.

    q      [B, S, Hq, D]   queries of the S noisy block tokens
    k_ctx  [B, Hkv, Lcap, D], v_ctx likewise: context-tower layer-i cache
    k_blk  [B, S, Hkv, D], v_blk likewise: the denoiser's own block KV
    ctx_lens [B]: committed context length L_n of each sequence (0..Lcap)
    Returns out [B, S, Hq, D] and lse [B, Hq, S], float64.

    For sequence n and query head j (KV head h = j // g) the key set is
    {k_ctx[n, h, l] : l < L_n} followed by {k_blk[n, u, h] : u < S}; every
    block row t attends to all of it (context fully visible, block
    bidirectional), with one softmax over the union.
    """
    q = _f64(q)
    B, S, Hq, D = q.shape
    Hkv = k_ctx.shape[1]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    g = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    out = np.empty((B, S, Hq, D), dtype=np.float64)
    lse = np.empty((B, Hq, S), dtype=np.float64)
    for n in range(B):
        L = int(ctx_lens[n])
        if L < 0 or L > k_ctx.shape[2]:
            raise ValueError("ctx_lens out of range")
        for h in range(Hkv):
            keys = np.concatenate([_f64(k_ctx[n, h, :L]), _f64(k_blk[n, :, h])], axis=0)
            vals = np.concatenate([_f64(v_ctx[n, h, :L]), _f64(v_blk[n, :, h])], axis=0)
            for j in range(h * g, (h + 1) * g):
                o, l = attend_rows(q[n, :, j, :], keys, vals, scale)
                out[n, :, j, :] = o
                lse[n, j, :] = l
    return out, lse


def block_causal(q, k_ctx, v_ctx, k_blk, v_blk, block_size, scale=None, blocks=None):
    """Whole-sequence (training / prefill) form of the same attention.

    q [B, N, Hq, D]; k_ctx, v_ctx [B, Hkv, N, D] (the context tower's cache
    over the clean sequence); k_blk, v_blk [B, N, Hkv, D] (the denoiser's own
    KV over the noisy sequence).  N is a multiple of the block size S.

    Block b (tokens S*b .. S*b+S-1) conditions on the clean context of the
    earlier blocks only, c_{<b} (section "Training and sampling": the loss is
    conditioned on the noisy block, the timestep and the frozen caches
    c_{<b}), plus its own block bidirectionally.  So block b is exactly one
    decode call with L = S*b on the matching slices.  Returns out
    [B, N, Hq, D] and lse [B, Hq, N].  ``blocks`` optionally restricts the
    computation to a subset of block indices (other rows are left NaN).
    """
    q = _f64(q)
    B, N, Hq, D = q.shape
    S = int(block_size)
    if S <= 0 or N % S:
        raise ValueError("sequence length must be a multiple of the block size")
    nb = N // S
    out = np.full((B, N, Hq, D), np.nan)
    lse = np.full((B, Hq, N), np.nan)
    for b in (range(nb) if blocks is None else blocks):
        lo, hi = S * b, S * b + S
        o, l = block_attn(q[:, lo:hi], k_ctx, v_ctx, k_blk[:, lo:hi], v_blk[:, lo:hi],
                          np.full(B, lo, dtype=np.int64), scale=scale)
        out[:, lo:hi] = o
        lse[:, :, lo:hi] = l
    return out, lse

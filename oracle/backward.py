"""Float64 CPU oracle of the block-causal backward pass (gradients of the training loss).

TEST INFRASTRUCTURE ONLY (same rule as ``oracle.oracle``): only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may use it.

What it computes (paperfeed.app review of arXiv 2606.26493, section "Training and
sampling"): the denoiser is trained with the loss conditioned on the noisy block and
on the frozen caches c_{<b}; the context tower runs once per sequence without
gradients.  So the gradients of the block attention flow to the denoiser's queries
and to its own block keys and values only:

    given dO = dL/dout for every query row r of block b,
    s_k  = scale <q_r, k_k>            over the keys k of the block's key set
    p_k  = exp(s_k - lse_r)            (the forward softmax weights)
    dp_k = <dO_r, v_k>
    ds_k = p_k (dp_k - sum_j p_j dp_j)   (softmax derivative; sum_j p_j dp_j = <dO_r, out_r>)
    dq_r        = scale * sum_k ds_k k_k          (all keys: context and block)
    dk_blk[u]  += scale * ds_u q_r                 (block keys only)
    dv_blk[u]  += p_u dO_r                         (block keys only)

summed over the g query heads that share a KV head and over the S rows of the block.
Nothing flows into the context cache (frozen).  This is the chain rule through the
definition in ``oracle.attend_rows``, written out per block.
"""
from __future__ import annotations

import numpy as np

__all__ = ["block_causal_backward"]


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def block_causal_backward(q, k_ctx, v_ctx, k_blk, v_blk, dout, block_size, scale=None, blocks=None):
    """Gradients of sum(dout * out) for the block-causal attention.

    Shapes as ``oracle.block_causal``; dout [B, N, Hq, D].  Returns dq [B, N, Hq, D],
    dk_blk [B, N, Hkv, D], dv_blk [B, N, Hkv, D] (float64).  ``blocks`` restricts the
    work to some block indices (other rows of dq / dk_blk / dv_blk stay NaN).
    """
    q = _f64(q)
    dout = _f64(dout)
    B, N, Hq, D = q.shape
    Hkv = k_ctx.shape[1]
    g = Hq // Hkv
    S = int(block_size)
    if S <= 0 or N % S:
        raise ValueError("sequence length must be a multiple of the block size")
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    dq = np.full((B, N, Hq, D), np.nan)
    dk = np.full((B, N, Hkv, D), np.nan)
    dv = np.full((B, N, Hkv, D), np.nan)
    for b in (range(N // S) if blocks is None else blocks):
        lo, hi = S * b, S * b + S
        for n in range(B):
            for h in range(Hkv):
                keys = np.concatenate([_f64(k_ctx[n, h, :lo]), _f64(k_blk[n, lo:hi, h])], axis=0)
                vals = np.concatenate([_f64(v_ctx[n, h, :lo]), _f64(v_blk[n, lo:hi, h])], axis=0)
                dkb = np.zeros((S, D))
                dvb = np.zeros((S, D))
                for j in range(h * g, (h + 1) * g):
                    qr = q[n, lo:hi, j, :]                       # [S, D] rows of this head
                    do = dout[n, lo:hi, j, :]
                    s = scale * (qr @ keys.T)                    # [S, K]
                    m = s.max(axis=1, keepdims=True)
                    e = np.exp(s - m)
                    p = e / e.sum(axis=1, keepdims=True)         # forward weights
                    dp = do @ vals.T                             # [S, K]
                    ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
                    dq[n, lo:hi, j, :] = scale * (ds @ keys)
                    dkb += scale * (ds[:, lo:].T @ qr)           # block keys are the last S columns
                    dvb += p[:, lo:].T @ do
                dk[n, lo:hi, h, :] = dkb
                dv[n, lo:hi, h, :] = dvb
    return dq, dk, dv

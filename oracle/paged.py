"""CPU oracle of decode block attention over a paged context cache.

TEST INFRASTRUCTURE ONLY (same rule as ``oracle.oracle``).

Serving keeps each sequence's context-tower cache in fixed-size pages drawn from a
shared pool.  Only the context tower holds sequence-length-dependent state (paperfeed
review of arXiv 2606.26493, "What this changes, and what to be skeptical of"), and
committed blocks are ingested one after another ("Training and sampling").  Logical
position l of sequence n lives in
page page_table[n, l // P] at offset l % P; the pool is [num_pages, Hkv, P, D].  The
attention itself is unchanged: gathering the pages back into a contiguous cache and
calling ``oracle.block_attn`` is the definition.
"""
from __future__ import annotations

import numpy as np

from .oracle import block_attn

__all__ = ["gather_pages", "block_attn_paged"]


def gather_pages(pages, page_table, ctx_lens, capacity):
    """Contiguous [B, Hkv, capacity, D] copy of the first ctx_lens[n] positions of every
    sequence (rows beyond stay zero)."""
    pages = np.asarray(pages)
    B = len(ctx_lens)
    _, Hkv, P, D = pages.shape
    out = np.zeros((B, Hkv, capacity, D), dtype=pages.dtype)
    for n in range(B):
        for pos in range(int(ctx_lens[n])):
            out[n, :, pos] = pages[page_table[n][pos // P], :, pos % P]
    return out


def block_attn_paged(q, k_pages, v_pages, page_table, k_blk, v_blk, ctx_lens, capacity, scale=None):
    k_ctx = gather_pages(k_pages, page_table, ctx_lens, capacity)
    v_ctx = gather_pages(v_pages, page_table, ctx_lens, capacity)
    return block_attn(q, k_ctx, v_ctx, k_blk, v_blk, ctx_lens, scale=scale)

"""Float64/bit-level CPU oracle of the committed-block cache update.

TEST INFRASTRUCTURE ONLY (same rule as ``oracle.oracle``): only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may use it.

What it computes (paperfeed.app review of arXiv 2606.26493, section "The idea:
freeze the reader, train the writer", last paragraphs): once every token of a
block is resolved the block is committed and the frozen context tower ingests
it causally, which extends its per-layer caches.  The context tower's layer-i keys and
values of the S committed positions (computed by the caller) are written into
the cache right after the L_n tokens already committed, and the committed
length grows by S.  Plain reading of a step the page states only in words:
positions [L_n, L_n + S) of sequence n receive the new rows in token order;
every other cache row is left as it was; a sequence without room for S more
rows (L_n + S > capacity) or with L_n < 0 is an error and nothing of it is
written.
"""
from __future__ import annotations

import numpy as np

__all__ = ["kv_append"]


def kv_append(k_new, v_new, k_ctx, v_ctx, ctx_lens, advance=True):
    """Return (k_ctx', v_ctx', lens', bad) without modifying the inputs.

    k_new, v_new [B, S, Hkv, D]; k_ctx, v_ctx [B, Hkv, Lcap, D] (any dtype, copied
    exactly); ctx_lens [B] int.  bad[n] is True for a sequence that had no room;
    its rows and length are unchanged.
    """
    k_out = np.array(k_ctx, copy=True)
    v_out = np.array(v_ctx, copy=True)
    lens = np.array(ctx_lens, dtype=np.int64, copy=True)
    B, S, Hkv, _ = np.shape(k_new)
    cap = np.shape(k_ctx)[2]
    bad = np.zeros(B, dtype=bool)
    for n in range(B):
        L = int(ctx_lens[n])
        if L < 0 or L + S > cap:
            bad[n] = True
            continue
        for t in range(S):
            for h in range(Hkv):
                k_out[n, h, L + t] = k_new[n, t, h]
                v_out[n, h, L + t] = v_new[n, t, h]
        if advance:
            lens[n] = L + S
    return k_out, v_out, lens, bad

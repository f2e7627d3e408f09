"""Float64 CPU oracle of the confidence-unmasking step of block sampling.

TEST INFRASTRUCTURE ONLY (same rule as ``oracle.oracle``).

What it computes (paperfeed.app review of arXiv 2606.26493, section "Training and
sampling"; the kongchang explainer, section "Sudoku"): at each denoising step all
masked positions of the block are predicted in parallel; every prediction whose
confidence is above the threshold gamma = 0.8 is committed, the rest stay masked for
the next step.  Readings of what the pages leave open:

* confidence = the softmax probability of the predicted token, and the prediction is
  the most probable token (argmax of the logits; among equal maxima the lowest
  vocabulary index);
* "above" is strict: p > gamma;
* with ``min_one``, a step in which no masked position of a sequence passes the
  threshold commits the single most confident masked position (the lowest position
  among equals), so that a block of S tokens finishes within S steps, as the pages'
  "up to T steps" per block requires of a sampler; without it nothing is committed;
* committed positions are never revisited.
"""
from __future__ import annotations

import numpy as np

__all__ = ["confidence_unmask"]


def confidence_unmask(logits, tokens, masked, gamma=0.8, min_one=True):
    """logits [B, S, V] (float); tokens [B, S] int; masked [B, S] bool.

    Returns (tokens', masked', p [B, S] float64, arg [B, S] int64, n_committed [B]).
    p and arg are reported for the positions masked on entry (p = 0 and arg = -1
    elsewhere); only those positions can commit.
    """
    x = np.asarray(logits, dtype=np.float64)
    B, S, V = x.shape
    m = x.max(axis=2)
    arg = np.argmax(x, axis=2)                       # numpy returns the first maximum
    p = 1.0 / np.exp(x - m[:, :, None]).sum(axis=2)  # probability of the argmax token
    tok = np.array(tokens, dtype=np.int64, copy=True)
    msk = np.array(masked, dtype=bool, copy=True)
    p = np.where(msk, p, 0.0)
    arg = np.where(msk, arg, -1)
    n_commit = np.zeros(B, dtype=np.int64)
    for n in range(B):
        commit = msk[n] & (p[n] > gamma)
        if min_one and not commit.any() and msk[n].any():
            cand = np.where(msk[n], p[n], -np.inf)
            commit = np.zeros(S, dtype=bool)
            commit[int(np.argmax(cand))] = True        # first position among equal confidences
        tok[n, commit] = arg[n, commit]
        msk[n, commit] = False
        n_commit[n] = int(commit.sum())
    return tok, msk, p, arg, n_commit

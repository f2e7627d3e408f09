"""Checks that pin the float64 oracle to facts outside itself.

Each ``pin_*`` takes a decode implementation with the oracle's signature
``attn(q, k_ctx, v_ctx, k_blk, v_blk, ctx_lens, scale=None) -> (out, lse)``
and raises AssertionError when the implementation disagrees with what the
method and the mathematics fix.  ``tests/test_oracle.py`` runs them on the
oracle; ``tests/test_oracle_mutations.py`` runs them on deliberately broken
copies of it and requires every copy to be caught.

Sources for the facts: the method's statement (paperfeed.app review of arXiv
2606.26493, section "The idea: freeze the reader, train the writer": the
block queries attend to the context tower's layer-i cache concatenated with
the block's own KV; inside the block attention is bidirectional; "Training
and sampling": block b conditions on c_{<b}), and textbook properties of a
softmax-weighted average.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from oracle.brute import brute_block_attn

TOL = 1e-10


def rand_case(seed, B=2, S=3, Hq=4, Hkv=2, D=5, Lcap=7, lens=None, std=1.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, S, Hq, D)) * std
    k_ctx = rng.standard_normal((B, Hkv, Lcap, D)) * std
    v_ctx = rng.standard_normal((B, Hkv, Lcap, D)) * std
    k_blk = rng.standard_normal((B, S, Hkv, D)) * std
    v_blk = rng.standard_normal((B, S, Hkv, D)) * std
    if lens is None:
        lens = rng.integers(0, Lcap, size=B, endpoint=True)
    return q, k_ctx, v_ctx, k_blk, v_blk, np.asarray(lens)


def _close(a, b, tol=TOL, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} != {b.shape}"
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.1e}"


def sdpa_reference(q, k_ctx, v_ctx, k_blk, v_blk, lens, scale=None):
    """torch float64 scaled_dot_product_attention on the explicitly concatenated
    [context ; block] keys, KV heads repeated in contiguous groups, plus
    torch.logsumexp of the scores.  An independent library route."""
    B, S, Hq, D = q.shape
    Hkv = k_ctx.shape[1]
    g = Hq // Hkv
    sc = (1.0 / math.sqrt(D)) if scale is None else scale
    out = np.empty((B, S, Hq, D))
    lse = np.empty((B, Hq, S))
    for n in range(B):
        L = int(lens[n])
        K = torch.cat([torch.from_numpy(np.ascontiguousarray(k_ctx[n, :, :L])),
                       torch.from_numpy(np.ascontiguousarray(k_blk[n].transpose(1, 0, 2)))], dim=1)
        V = torch.cat([torch.from_numpy(np.ascontiguousarray(v_ctx[n, :, :L])),
                       torch.from_numpy(np.ascontiguousarray(v_blk[n].transpose(1, 0, 2)))], dim=1)
        K = K.double().repeat_interleave(g, dim=0)
        V = V.double().repeat_interleave(g, dim=0)
        Q = torch.from_numpy(np.ascontiguousarray(q[n].transpose(1, 0, 2))).double()  # [Hq, S, D]
        o = torch.nn.functional.scaled_dot_product_attention(Q, K, V, scale=sc)
        out[n] = o.permute(1, 0, 2).numpy()
        lse[n] = torch.logsumexp(sc * (Q @ K.transpose(1, 2)), dim=-1).numpy()
    return out, lse


# ---------------------------------------------------------------- pins ----

def pin_brute_force(attn):
    """Tiny random problems (GQA, ragged, empty context) against the pure-Python
    per-row loop with an explicit visibility predicate."""
    for seed, kw in [(1, {}), (2, dict(B=3, S=1, Hq=2, Hkv=1, D=3, Lcap=4, lens=[0, 4, 2])),
                     (3, dict(B=1, S=4, Hq=6, Hkv=3, D=2, Lcap=5, lens=[5]))]:
        case = rand_case(seed, **kw)
        o, l = attn(*case)
        bo, bl = brute_block_attn(*case)
        _close(o, bo, 1e-12, "brute out")
        _close(l, bl, 1e-12, "brute lse")


def pin_sdpa(attn):
    """Against torch's float64 SDPA on the concatenated keys (library routine)."""
    for seed, kw in [(11, dict(B=3, S=4, Hq=8, Hkv=2, D=16, Lcap=33)),
                     (12, dict(B=2, S=16, Hq=4, Hkv=1, D=8, Lcap=40, lens=[40, 17])),
                     (13, dict(B=2, S=5, Hq=6, Hkv=3, D=4, Lcap=9, lens=[0, 9], std=3.0))]:
        case = rand_case(seed, **kw)
        o, l = attn(*case)
        ro, rl = sdpa_reference(*case)
        _close(o, ro, 1e-12, "sdpa out")
        _close(l, rl, 1e-12, "sdpa lse")
    case = rand_case(14, B=1, S=3, Hq=2, Hkv=1, D=6, Lcap=5)
    o, l = attn(*case, scale=0.37)
    ro, rl = sdpa_reference(*case, scale=0.37)
    _close(o, ro, 1e-12, "sdpa out (explicit scale)")
    _close(l, rl, 1e-12, "sdpa lse (explicit scale)")


def pin_empty_context(attn):
    """With L_n = 0 the result is plain bidirectional self-attention of the block:
    every block row sees every block key and nothing else."""
    q, k_ctx, v_ctx, k_blk, v_blk, _ = rand_case(21, B=2, S=6, Hq=4, Hkv=2, D=8, Lcap=5)
    # poison the cache: none of it may be read when L_n = 0
    k_ctx[:] = np.nan
    v_ctx[:] = np.nan
    o, l = attn(q, k_ctx, v_ctx, k_blk, v_blk, np.zeros(2, dtype=np.int64))
    for n in range(2):
        for j in range(4):
            h = j // 2
            Q = torch.from_numpy(q[n, :, j]).double()[None]
            K = torch.from_numpy(np.ascontiguousarray(k_blk[n, :, h])).double()[None]
            V = torch.from_numpy(np.ascontiguousarray(v_blk[n, :, h])).double()[None]
            ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V)[0].numpy()
            _close(o[n, :, j], ref, 1e-12, "empty-context self-attention")


def pin_closed_form_weights(attn):
    """Scores ln 1, ln 2, ln 3 (scale 1, one-hot query) give softmax weights
    1/6, 2/6, 3/6 exactly, and lse = ln 6."""
    D = 3
    q = np.zeros((1, 1, 1, D)); q[0, 0, 0, 0] = 1.0
    k_ctx = np.zeros((1, 1, 4, D)); v_ctx = np.zeros((1, 1, 4, D))
    k_ctx[0, 0, 0, 0] = math.log(1.0); v_ctx[0, 0, 0] = [1.0, 0.0, 5.0]
    k_ctx[0, 0, 1, 0] = math.log(2.0); v_ctx[0, 0, 1] = [0.0, 1.0, -1.0]
    k_ctx[0, 0, 2:, :] = 100.0                      # beyond L_n = 2: must be ignored
    k_blk = np.zeros((1, 1, 1, D)); v_blk = np.zeros((1, 1, 1, D))
    k_blk[0, 0, 0, 0] = math.log(3.0); v_blk[0, 0, 0] = [2.0, 2.0, 0.0]
    o, l = attn(q, k_ctx, v_ctx, k_blk, v_blk, np.array([2]), scale=1.0)
    expect = (1.0 * np.array([1.0, 0.0, 5.0]) + 2.0 * np.array([0.0, 1.0, -1.0])
              + 3.0 * np.array([2.0, 2.0, 0.0])) / 6.0
    _close(o[0, 0, 0], expect, 1e-14, "closed-form weights")
    _close(l[0, 0, 0], math.log(6.0), 1e-14, "closed-form lse")


def pin_equal_keys(attn):
    """All visible keys equal: the output is the mean of the visible values and
    lse = scale*<q,k> + ln(L_n + S)."""
    B, S, Hq, Hkv, D, Lcap = 2, 4, 4, 2, 6, 9
    rng = np.random.default_rng(31)
    q = rng.standard_normal((B, S, Hq, D))
    kvec = rng.standard_normal(D)
    k_ctx = np.broadcast_to(kvec, (B, Hkv, Lcap, D)).copy()
    k_blk = np.broadcast_to(kvec, (B, S, Hkv, D)).copy()
    v_ctx = rng.standard_normal((B, Hkv, Lcap, D))
    v_blk = rng.standard_normal((B, S, Hkv, D))
    lens = np.array([9, 3])
    o, l = attn(q, k_ctx, v_ctx, k_blk, v_blk, lens)
    sc = 1.0 / math.sqrt(D)
    for n in range(B):
        for j in range(Hq):
            h = j // 2
            mean = np.concatenate([v_ctx[n, h, :lens[n]], v_blk[n, :, h]]).mean(axis=0)
            for t in range(S):
                _close(o[n, t, j], mean, 1e-12, "equal keys -> mean of V")
                _close(l[n, j, t], sc * q[n, t, j] @ kvec + math.log(lens[n] + S), 1e-12,
                       "equal keys lse")


def pin_dominant_key(attn):
    """One key far ahead of all others takes all the weight: output = its value."""
    q, k_ctx, v_ctx, k_blk, v_blk, _ = rand_case(41, B=1, S=2, Hq=2, Hkv=1, D=4, Lcap=6)
    lens = np.array([6])
    q[0, :, :, :] = np.array([1.0, 0.0, 0.0, 0.0])
    k_ctx[0, 0, 3] = np.array([2000.0, 0.0, 0.0, 0.0])
    o, _ = attn(q, k_ctx, v_ctx, k_blk, v_blk, lens)
    for t in range(2):
        for j in range(2):
            _close(o[0, t, j], v_ctx[0, 0, 3], 1e-12, "dominant context key")
    k_blk[0, 1, 0] = np.array([4000.0, 0.0, 0.0, 0.0])
    o, _ = attn(q, k_ctx, v_ctx, k_blk, v_blk, lens)
    _close(o[0, 0, 0], v_blk[0, 1, 0], 1e-12, "dominant block key")


def pin_affine_values(attn):
    """out(alpha*V + beta) = alpha*out(V) + beta (weights sum to one); lse unchanged."""
    case = rand_case(51, B=2, S=3, Hq=4, Hkv=1, D=5, Lcap=6)
    q, k_ctx, v_ctx, k_blk, v_blk, lens = case
    o, l = attn(*case)
    beta = np.linspace(-1, 1, 5)
    o2, l2 = attn(q, k_ctx, -2.5 * v_ctx + beta, k_blk, -2.5 * v_blk + beta, lens)
    _close(o2, -2.5 * o + beta, 1e-12, "affine V")
    _close(l2, l, 1e-12, "affine V lse")


def pin_key_shift(attn):
    """Adding one vector c to every key shifts each row's scores by scale*<q,c>:
    out unchanged, lse shifted by exactly that amount."""
    case = rand_case(61, B=2, S=3, Hq=4, Hkv=2, D=5, Lcap=6)
    q, k_ctx, v_ctx, k_blk, v_blk, lens = case
    c = np.array([0.3, -1.2, 0.5, 2.0, -0.7])
    o, l = attn(*case)
    o2, l2 = attn(q, k_ctx + c, v_ctx, k_blk + c, v_blk, lens)
    _close(o2, o, 1e-12, "key shift out")
    shift = np.einsum("bthd,d->bht", q, c) / math.sqrt(5)
    _close(l2, l + shift, 1e-12, "key shift lse")


def pin_context_permutation(attn):
    """Permuting the visible context positions together with their V changes nothing."""
    case = rand_case(71, B=2, S=3, Hq=2, Hkv=1, D=4, Lcap=8, lens=[8, 5])
    q, k_ctx, v_ctx, k_blk, v_blk, lens = case
    o, l = attn(*case)
    k2, v2 = k_ctx.copy(), v_ctx.copy()
    rng = np.random.default_rng(72)
    for n in range(2):
        p = rng.permutation(int(lens[n]))
        for h in range(k_ctx.shape[1]):
            k2[n, h, :lens[n]] = k_ctx[n, h][p]
            v2[n, h, :lens[n]] = v_ctx[n, h][p]
    o2, l2 = attn(q, k2, v2, k_blk, v_blk, lens)
    _close(o2, o, 1e-12, "context permutation out")
    _close(l2, l, 1e-12, "context permutation lse")


def pin_block_permutation(attn):
    """Bidirectional block: permuting block positions (queries and block KV together)
    permutes the output rows the same way."""
    case = rand_case(81, B=1, S=5, Hq=4, Hkv=2, D=4, Lcap=3)
    q, k_ctx, v_ctx, k_blk, v_blk, lens = case
    o, l = attn(*case)
    p = np.array([3, 0, 4, 1, 2])
    o2, l2 = attn(q[:, p], k_ctx, v_ctx, k_blk[:, p], v_blk[:, p], lens)
    _close(o2, o[:, p], 1e-12, "block permutation out")
    _close(l2, l[:, :, p], 1e-12, "block permutation lse")


def pin_ignores_beyond_len(attn):
    """Context rows at or beyond L_n are never read, whatever they hold."""
    case = rand_case(91, B=2, S=2, Hq=2, Hkv=1, D=3, Lcap=6, lens=[2, 6])
    q, k_ctx, v_ctx, k_blk, v_blk, lens = case
    o, l = attn(*case)
    k2, v2 = k_ctx.copy(), v_ctx.copy()
    k2[0, :, 2:] = np.nan
    v2[0, :, 2:] = np.inf
    o2, l2 = attn(q, k2, v2, k_blk, v_blk, lens)
    _close(o2, o, 0.0, "poisoned padding out")
    _close(l2, l, 0.0, "poisoned padding lse")


def pin_softmax_stability(attn):
    """Huge common score offsets (scores ~ 1e4) must not overflow: out is the same
    as for the shifted-down problem, lse shifted by the offset."""
    case = rand_case(95, B=1, S=2, Hq=2, Hkv=1, D=3, Lcap=4, lens=[4])
    q, k_ctx, v_ctx, k_blk, v_blk, lens = case
    q = q.copy(); q[..., 0] = 1.0; q[..., 1:] = 0.0
    o, l = attn(q, k_ctx, v_ctx, k_blk, v_blk, lens)
    off = 2e4
    o2, l2 = attn(q, k_ctx + np.array([off, 0, 0]), v_ctx, k_blk + np.array([off, 0, 0]), v_blk, lens)
    assert np.all(np.isfinite(o2)), "overflow in softmax"
    _close(o2, o, 1e-9, "large offset out")
    _close(l2, l + off / math.sqrt(3), 1e-9, "large offset lse")


ALL_PINS = [pin_brute_force, pin_sdpa, pin_empty_context, pin_closed_form_weights, pin_equal_keys,
            pin_dominant_key, pin_affine_values, pin_key_shift, pin_context_permutation,
            pin_block_permutation, pin_ignores_beyond_len, pin_softmax_stability]

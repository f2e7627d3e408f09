"""Seeded synthetic workloads for TwoTower block attention.

This module only draws inputs; it holds none of the attention arithmetic, so
the CUDA path, the float64 oracle, the tests and the benchmark can all share
it.  Everything is numpy on the host; tensors come back as bf16 bit patterns
(uint16) plus int32 context lengths.

Recipe (the pages run no attention benchmark, so these shapes stand in for
their decoding regime: 16-token blocks over a growing committed context):

* ``numpy.random.default_rng(seed)``; the named workloads use seed 1234 + id.
* Draw order is fixed: q, k_ctx, v_ctx, k_blk, v_blk, then the peaky-key
  selection (decode L=4096 workload), then the ragged context lengths.
* Every tensor is float32 standard normal times ``std``, rounded to bf16 with
  round-to-nearest-even.  The peaky workload multiplies 1% of key rows
  (every context and block key row is picked independently) by 8 after the
  rounding, which is exact in bf16.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "Workload", "DecodeInputs", "CausalInputs", "WORKLOADS", "bf16_bits", "bf16_to_f32",
    "bf16_to_f64", "make_decode", "make_causal", "make_workload",
]


def bf16_bits(x) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); return the bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(bits) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_to_f64(bits) -> np.ndarray:
    return bf16_to_f32(bits).astype(np.float64)


@dataclass
class Workload:
    """One named workload; ``kind`` is "decode" or "causal"."""
    wid: int
    name: str
    kind: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    ctx: int = 0                 # decode: context length (or capacity when ragged)
    ragged: tuple | None = None  # decode: (lo, hi) inclusive range of L_n
    seq_len: int = 0             # causal: N
    std: float = 1.0
    peaky_frac: float = 0.0
    peaky_mult: float = 8.0

    @property
    def seed(self) -> int:
        return 1234 + self.wid

    def describe(self) -> dict:
        d = {"workload": self.name, "batch": self.batch, "q_heads": self.num_q_heads,
             "kv_heads": self.num_kv_heads, "head_dim": self.head_dim, "block": self.block_size}
        if self.kind == "decode":
            d["ctx"] = (f"U[{self.ragged[0]},{self.ragged[1]}]" if self.ragged else self.ctx)
        else:
            d["seq_len"] = self.seq_len
        return d


WORKLOADS = {
    1: Workload(1, "tiny-decode-B1-Hq4-Hkv1-D64-L256", "decode", 1, 4, 1, 64, 16, ctx=256),
    2: Workload(2, "decode-B8-Hq32-Hkv2-D128-L4096-peaky", "decode", 8, 32, 2, 128, 16, ctx=4096,
                peaky_frac=0.01),
    3: Workload(3, "ragged-decode-B64-Hq32-Hkv2-D128-L512..16384", "decode", 64, 32, 2, 128, 16,
                ctx=16384, ragged=(512, 16384)),
    4: Workload(4, "long-decode-B4-Hq32-Hkv2-D128-L131072", "decode", 4, 32, 2, 128, 16, ctx=131072,
                std=0.5),
    5: Workload(5, "block-causal-B8-N8192-S16-Hq32-Hkv2-D128", "causal", 8, 32, 2, 128, 16,
                seq_len=8192),
}


@dataclass
class DecodeInputs:
    q: np.ndarray        # [B, S, Hq, D] bf16 bits
    k_ctx: np.ndarray    # [B, Hkv, Lcap, D]
    v_ctx: np.ndarray
    k_blk: np.ndarray    # [B, S, Hkv, D]
    v_blk: np.ndarray
    ctx_lens: np.ndarray  # [B] int32
    meta: dict = field(default_factory=dict)

    @property
    def shape(self):
        B, S, Hq, D = self.q.shape
        return B, S, Hq, self.k_ctx.shape[1], D, self.k_ctx.shape[2]


@dataclass
class CausalInputs:
    q: np.ndarray        # [B, N, Hq, D]
    k_ctx: np.ndarray    # [B, Hkv, N, D]
    v_ctx: np.ndarray
    k_blk: np.ndarray    # [B, N, Hkv, D]
    v_blk: np.ndarray
    block_size: int
    meta: dict = field(default_factory=dict)


def _draw(rng, shape, std):
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return bf16_bits(x)


def _scale_rows(bits, rows_mask, mult):
    """Multiply whole D-vectors (last axis) selected by rows_mask by a power of two."""
    if not rows_mask.any():
        return bits
    vals = bf16_to_f32(bits)
    vals[rows_mask] *= np.float32(mult)
    return bf16_bits(vals)


def make_decode(batch, block, q_heads, kv_heads, head_dim, ctx_cap, seed, ctx_lens=None,
                ragged=None, std=1.0, peaky_frac=0.0, peaky_mult=8.0) -> DecodeInputs:
    """Draw one decode problem.  ``ctx_lens`` defaults to the capacity for every sequence,
    or to ``rng.integers(lo, hi, endpoint=True)`` when ``ragged=(lo, hi)`` is given."""
    rng = np.random.default_rng(seed)
    B, S, Hq, Hkv, D, L = batch, block, q_heads, kv_heads, head_dim, ctx_cap
    q = _draw(rng, (B, S, Hq, D), std)
    k_ctx = _draw(rng, (B, Hkv, L, D), std)
    v_ctx = _draw(rng, (B, Hkv, L, D), std)
    k_blk = _draw(rng, (B, S, Hkv, D), std)
    v_blk = _draw(rng, (B, S, Hkv, D), std)
    if peaky_frac > 0.0:
        k_ctx = _scale_rows(k_ctx, rng.random((B, Hkv, L)) < peaky_frac, peaky_mult)
        k_blk = _scale_rows(k_blk, rng.random((B, S, Hkv)) < peaky_frac, peaky_mult)
    if ragged is not None:
        lens = rng.integers(ragged[0], ragged[1], size=B, endpoint=True)
    elif ctx_lens is not None:
        lens = np.asarray(ctx_lens)
    else:
        lens = np.full(B, L)
    return DecodeInputs(q, k_ctx, v_ctx, k_blk, v_blk, np.ascontiguousarray(lens, dtype=np.int32),
                        meta={"seed": seed, "std": std, "peaky_frac": peaky_frac})


def make_causal(batch, seq_len, block, q_heads, kv_heads, head_dim, seed, std=1.0) -> CausalInputs:
    rng = np.random.default_rng(seed)
    B, N, S, Hq, Hkv, D = batch, seq_len, block, q_heads, kv_heads, head_dim
    q = _draw(rng, (B, N, Hq, D), std)
    k_ctx = _draw(rng, (B, Hkv, N, D), std)
    v_ctx = _draw(rng, (B, Hkv, N, D), std)
    k_blk = _draw(rng, (B, N, Hkv, D), std)
    v_blk = _draw(rng, (B, N, Hkv, D), std)
    return CausalInputs(q, k_ctx, v_ctx, k_blk, v_blk, S, meta={"seed": seed, "std": std})


def make_workload(wid: int, batch: int | None = None):
    """Inputs of a named workload (optionally with a smaller batch, same per-sequence recipe)."""
    w = WORKLOADS[wid]
    B = w.batch if batch is None else batch
    if w.kind == "decode":
        return make_decode(B, w.block_size, w.num_q_heads, w.num_kv_heads, w.head_dim, w.ctx,
                           w.seed, ragged=w.ragged, std=w.std, peaky_frac=w.peaky_frac,
                           peaky_mult=w.peaky_mult)
    return make_causal(B, w.seq_len, w.block_size, w.num_q_heads, w.num_kv_heads, w.head_dim,
                       w.seed, std=w.std)


def decode_cost(B, S, Hq, Hkv, D, lens, out_bytes=4):
    """Algorithmic bytes and flops of one decode call.

    Bytes: the K and V rows actually visible (context rows below L_n and the
    block rows, bf16), Q (bf16) and the output at its dtype.  Flops: two
    contractions (QK^T and PV) of 2*D flops per (query row, key).
    """
    lens = np.asarray(lens, dtype=np.int64)
    kv = int(Hkv * D * 2 * 2 * (lens.sum() + B * S))
    qb = B * S * Hq * D * 2
    ob = B * S * Hq * D * out_bytes
    flops = int(4 * Hq * S * D * (lens + S).sum())
    return {"bytes": kv + qb + ob, "kv_bytes": kv, "flops": flops}


def causal_cost(B, N, S, Hq, Hkv, D, out_bytes=4):
    nb = N // S
    keys_per_row = sum(S * b + S for b in range(nb))      # per query position of a block
    flops = 4 * B * Hq * D * S * keys_per_row
    kv = 2 * 2 * B * Hkv * D * N * 2                       # ctx + block, K and V, bf16
    qb = B * N * Hq * D * 2
    ob = B * N * Hq * D * out_bytes
    return {"bytes": kv + qb + ob, "kv_bytes": kv, "flops": flops}


@dataclass
class PagedCache:
    """A decode cache laid out as a shared page pool (bf16 bit patterns)."""
    k_pages: np.ndarray      # [num_pages, Hkv, P, D] uint16
    v_pages: np.ndarray
    page_table: np.ndarray   # [B, pages_per_seq] int32; entries past ceil(L_n / P) are -1
    page_size: int


def make_paged(inp: DecodeInputs, page_size: int, seed: int, spare_pages: int = 3,
               fill_bits: int = 0x7FC0) -> PagedCache:
    """Scatter the first L_n rows of every sequence of ``inp`` into pages of ``page_size``
    rows drawn in a shuffled order from one pool.  Rows past L_n inside a sequence's last
    page and ``spare_pages`` pages that no sequence owns hold ``fill_bits`` (bf16 NaN by
    default), so any read of them shows; unused table entries are -1."""
    rng = np.random.default_rng(seed)
    B, Hkv, Lcap, D = inp.k_ctx.shape
    P = page_size
    per = -(-Lcap // P) if Lcap else 0
    need = [-(-int(L) // P) for L in inp.ctx_lens]
    num_pages = sum(need) + spare_pages
    order = rng.permutation(num_pages)
    k_pages = np.full((num_pages, Hkv, P, D), fill_bits, dtype=np.uint16)
    v_pages = np.full_like(k_pages, fill_bits)
    table = np.full((B, per), -1, dtype=np.int32)
    nxt = 0
    for n in range(B):
        L = int(inp.ctx_lens[n])
        for i in range(need[n]):
            pg = int(order[nxt])
            nxt += 1
            table[n, i] = pg
            rows = min(P, L - i * P)
            k_pages[pg, :, :rows] = inp.k_ctx[n, :, i * P:i * P + rows]
            v_pages[pg, :, :rows] = inp.v_ctx[n, :, i * P:i * P + rows]
    return PagedCache(k_pages, v_pages, table, P)

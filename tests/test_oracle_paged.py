"""Pins of the paged-cache gather (CPU only): brute-force placement, and attention over
a shuffled page pool equals attention over the contiguous cache."""
import numpy as np

from oracle import block_attn, block_attn_paged, gather_pages


def _pool_from_contiguous(k_ctx, P, rng):
    """Scatter a contiguous cache into a shuffled pool; return (pool, page_table)."""
    B, Hkv, L, D = k_ctx.shape
    per = (L + P - 1) // P
    perm = rng.permutation(B * per + 3)              # spare pages stay unused
    pool = rng.standard_normal((B * per + 3, Hkv, P, D))
    table = perm[:B * per].reshape(B, per)
    for n in range(B):
        for i in range(per):
            seg = k_ctx[n, :, i * P:(i + 1) * P]
            pool[table[n, i], :, :seg.shape[1]] = seg
    return pool, table


def test_gather_places_every_position():
    rng = np.random.default_rng(1)
    pool = rng.standard_normal((7, 2, 4, 3))
    table = np.array([[5, 0, 3], [6, 1, 2]])
    lens = np.array([10, 3])
    g = gather_pages(pool, table, lens, 12)
    for n in range(2):
        for pos in range(12):
            want = pool[table[n, pos // 4], :, pos % 4] if pos < lens[n] else 0.0
            assert np.array_equal(g[n, :, pos], np.broadcast_to(want, g[n, :, pos].shape))


def test_paged_attention_equals_contiguous():
    rng = np.random.default_rng(2)
    B, S, Hq, Hkv, D, L, P = 2, 3, 4, 2, 5, 13, 4
    q = rng.standard_normal((B, S, Hq, D))
    k_ctx = rng.standard_normal((B, Hkv, L, D))
    v_ctx = rng.standard_normal((B, Hkv, L, D))
    k_blk = rng.standard_normal((B, S, Hkv, D))
    v_blk = rng.standard_normal((B, S, Hkv, D))
    lens = np.array([13, 6])
    kp, table = _pool_from_contiguous(k_ctx, P, np.random.default_rng(3))
    vp, table2 = _pool_from_contiguous(v_ctx, P, np.random.default_rng(3))
    assert np.array_equal(table, table2)
    o1, l1 = block_attn(q, k_ctx, v_ctx, k_blk, v_blk, lens)
    o2, l2 = block_attn_paged(q, kp, vp, table, k_blk, v_blk, lens, L)
    assert np.allclose(o1, o2, atol=1e-14) and np.allclose(l1, l2, atol=1e-14)


def test_make_paged_places_rows_and_fills_the_rest():
    """The pool builder the GPU tests use: row l of sequence n sits at row l % P of page
    table[n][l // P]; unused entries are -1; spare pages and rows past L_n hold the fill."""
    from two_tower_block_b200.workloads import make_decode, make_paged
    inp = make_decode(3, 4, 4, 2, 64, 100, seed=9, ctx_lens=[100, 0, 33])
    P = 16
    pc = make_paged(inp, P, seed=4, spare_pages=2, fill_bits=0x7FC0)
    need = [-(-int(L) // P) for L in inp.ctx_lens]
    assert pc.k_pages.shape == (sum(need) + 2, 2, P, 64) and pc.page_table.shape == (3, 7)
    owned = set()
    for n, L in enumerate(inp.ctx_lens):
        assert (pc.page_table[n, need[n]:] == -1).all()
        for l in range(int(L)):
            pg = pc.page_table[n, l // P]
            assert np.array_equal(pc.k_pages[pg, :, l % P], inp.k_ctx[n, :, l])
            assert np.array_equal(pc.v_pages[pg, :, l % P], inp.v_ctx[n, :, l])
        for i in range(need[n]):
            owned.add(int(pc.page_table[n, i]))
        last = pc.page_table[n, need[n] - 1] if need[n] else None
        if last is not None:
            assert (pc.k_pages[last, :, int(L) - (need[n] - 1) * P:] == 0x7FC0).all()
    assert len(owned) == sum(need)                      # no page is shared
    spare = sorted(set(range(pc.k_pages.shape[0])) - owned)
    assert len(spare) == 2 and (pc.k_pages[spare] == 0x7FC0).all() and (pc.v_pages[spare] == 0x7FC0).all()

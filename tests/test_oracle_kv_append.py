"""Pins of the committed-block cache update oracle (CPU only)."""
import numpy as np

from oracle import attend_rows, kv_append


def _case(seed, B=3, S=4, Hkv=2, D=6, cap=11, lens=(0, 5, 7)):
    rng = np.random.default_rng(seed)
    k_new = rng.standard_normal((B, S, Hkv, D))
    v_new = rng.standard_normal((B, S, Hkv, D))
    k_ctx = rng.standard_normal((B, Hkv, cap, D))
    v_ctx = rng.standard_normal((B, Hkv, cap, D))
    return k_new, v_new, k_ctx, v_ctx, np.array(lens, dtype=np.int32)


def test_rows_land_after_the_committed_length_and_nothing_else_moves():
    k_new, v_new, k_ctx, v_ctx, lens = _case(1)
    k2, v2, l2, bad = kv_append(k_new, v_new, k_ctx, v_ctx, lens)
    S = k_new.shape[1]
    assert not bad.any()
    assert (l2 == lens + S).all()
    for n in range(len(lens)):
        L = lens[n]
        # the new rows, transposed from [S, Hkv, D] to [Hkv, S, D]
        assert np.array_equal(k2[n, :, L:L + S], np.transpose(k_new[n], (1, 0, 2)))
        assert np.array_equal(v2[n, :, L:L + S], np.transpose(v_new[n], (1, 0, 2)))
        # every other row is untouched
        keep = np.ones(k_ctx.shape[2], dtype=bool)
        keep[L:L + S] = False
        assert np.array_equal(k2[n][:, keep], k_ctx[n][:, keep])
        assert np.array_equal(v2[n][:, keep], v_ctx[n][:, keep])


def test_no_advance_keeps_lengths():
    k_new, v_new, k_ctx, v_ctx, lens = _case(2)
    _, _, l2, _ = kv_append(k_new, v_new, k_ctx, v_ctx, lens, advance=False)
    assert (l2 == lens).all()


def test_full_cache_is_an_error_and_writes_nothing():
    k_new, v_new, k_ctx, v_ctx, lens = _case(3, lens=(8, -1, 7))   # cap 11, S 4: 8+4 > 11
    k2, v2, l2, bad = kv_append(k_new, v_new, k_ctx, v_ctx, lens)
    assert list(bad) == [True, True, False]
    for n in (0, 1):
        assert np.array_equal(k2[n], k_ctx[n]) and np.array_equal(v2[n], v_ctx[n]) and l2[n] == lens[n]


def test_attention_over_the_grown_cache_equals_attention_over_the_concatenation():
    """After the update, attending to the first L+S cache rows is attending to the old
    L rows followed by the committed block's rows: the cache the next block sees."""
    k_new, v_new, k_ctx, v_ctx, lens = _case(4, B=2, lens=(3, 6))
    k2, v2, l2, _ = kv_append(k_new, v_new, k_ctx, v_ctx, lens)
    rng = np.random.default_rng(5)
    for n in range(2):
        for h in range(k_new.shape[2]):
            q = rng.standard_normal((3, k_new.shape[3]))
            L = lens[n]
            keys = np.concatenate([k_ctx[n, h, :L], k_new[n, :, h]], axis=0)
            vals = np.concatenate([v_ctx[n, h, :L], v_new[n, :, h]], axis=0)
            o1, s1 = attend_rows(q, keys, vals, 0.4)
            o2, s2 = attend_rows(q, k2[n, h, :l2[n]], v2[n, h, :l2[n]], 0.4)
            assert np.allclose(o1, o2, atol=1e-14) and np.allclose(s1, s2, atol=1e-14)


def test_bf16_bit_patterns_are_copied_exactly():
    rng = np.random.default_rng(6)
    k_new = rng.integers(0, 65535, size=(2, 3, 1, 8), dtype=np.uint16)
    v_new = rng.integers(0, 65535, size=(2, 3, 1, 8), dtype=np.uint16)
    k_ctx = np.zeros((2, 1, 9, 8), dtype=np.uint16)
    v_ctx = np.zeros((2, 1, 9, 8), dtype=np.uint16)
    k2, v2, _, _ = kv_append(k_new, v_new, k_ctx, v_ctx, np.array([0, 6]))
    assert k2.dtype == np.uint16 and np.array_equal(k2[1, 0, 6:9], k_new[1, :, 0])

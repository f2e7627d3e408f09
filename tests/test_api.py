"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every symbol the header declares, rejects malformed descriptors before
touching a device, and its work split covers every tile exactly once."""
import os
import re

import numpy as np
import pytest

from two_tower_block_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_symbols():
    src = open(os.path.join(ROOT, "include", "tt_block_attn.h")).read()
    return sorted(set(re.findall(r"TT_API\s+[\w\s\*]*?\b(tt_\w+)\s*\(", src)))


def test_header_symbols_are_exported():
    L = ops.lib()
    syms = header_symbols()
    assert len(syms) >= 13
    for s in syms:
        assert hasattr(L, s), f"{s} declared in the header but not exported"
    assert sorted(ops.EXPORTED_SYMBOLS) == syms


def test_exported_symbols_via_nm():
    import shutil
    import subprocess
    nm = shutil.which("nm")
    if nm is None:
        pytest.skip("nm not available")
    out = subprocess.run([nm, "-D", "--defined-only", ops.library_path], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (tt_\w+)", out))
    assert set(header_symbols()) <= exported


def test_status_strings():
    L = ops.lib()
    for s in range(6):
        assert L.tt_status_string(s)
    assert b"timed out" in L.tt_status_string(ops.TT_ERR_TIMEOUT)


@pytest.mark.parametrize("bad,code", [
    (dict(head_dim=96), ops.TT_ERR_UNSUPPORTED),
    (dict(num_q_heads=6, num_kv_heads=4), ops.TT_ERR_INVALID_ARG),
    (dict(block_size=0), ops.TT_ERR_INVALID_ARG),
    (dict(block_size=32, num_q_heads=32, num_kv_heads=2), ops.TT_ERR_UNSUPPORTED),  # S*g = 512
    (dict(seq_len=100, block_size=16), ops.TT_ERR_INVALID_ARG),
    (dict(batch=-1), ops.TT_ERR_INVALID_ARG),
    (dict(scale=-1.0), ops.TT_ERR_INVALID_ARG),
    (dict(kernel=9), ops.TT_ERR_INVALID_ARG),
    (dict(flags=4), ops.TT_ERR_INVALID_ARG),
])
def test_descriptor_validation_before_device(bad, code):
    import ctypes
    d = dict(batch=2, num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16, ctx_capacity=64,
             seq_len=0, scale=0.0, kernel=0, num_ctas=0, flags=0, wait_timeout_us=0)
    d.update(bad)
    desc = ops.Desc(**d)
    h = ctypes.c_void_p()
    st = ops.lib().tt_block_attn_plan(ctypes.byref(desc), 0, ctypes.byref(h))
    assert st == code, ops.lib().tt_last_error_detail()
    assert not h.value


def test_null_arguments():
    L = ops.lib()
    assert L.tt_block_attn_plan(None, 0, None) == ops.TT_ERR_INVALID_ARG
    assert L.tt_block_attn(None, *([None] * 9)) == ops.TT_ERR_INVALID_ARG
    assert L.tt_block_attn_check(None, None) == ops.TT_ERR_INVALID_ARG
    assert L.tt_kv_append(None, *([None] * 5), 1, None) == ops.TT_ERR_INVALID_ARG
    assert L.tt_block_attn_block_causal_backward(None, *([None] * 12)) == ops.TT_ERR_INVALID_ARG
    assert L.tt_block_attn_paged(None, None, None, None, None, 0, 64, 0, None, None, None, None, None,
                                 None) == ops.TT_ERR_INVALID_ARG
    L.tt_block_attn_plan_destroy(None)  # no-op


@pytest.mark.parametrize("B,S,V", [(-1, 16, 10), (1, 0, 10), (1, 1025, 10), (1, 16, 0)])
def test_confidence_unmask_rejects_bad_shapes_before_the_device(B, S, V):
    import ctypes
    L = ops.lib()
    L.tt_confidence_unmask.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                                       ctypes.c_int] + [ctypes.c_void_p] * 6
    assert L.tt_confidence_unmask(None, B, S, V, 0.8, 1, None, None, None, None, None, None) == ops.TT_ERR_INVALID_ARG


def test_confidence_unmask_rejects_null_tensors_and_empty_batch_is_a_noop():
    import ctypes
    L = ops.lib()
    L.tt_confidence_unmask.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                                       ctypes.c_int] + [ctypes.c_void_p] * 6
    assert L.tt_confidence_unmask(None, 2, 16, 100, 0.8, 1, None, None, None, None, None, None) == ops.TT_ERR_INVALID_ARG
    assert L.tt_confidence_unmask(None, 0, 16, 100, 0.8, 1, None, None, None, None, None, None) == ops.TT_OK


@pytest.mark.parametrize("tiles,C", [
    ([3, 5, 1, 7], 4), ([1] * 17, 5), ([40], 148), ([2, 2], 7), ([33] * 16, 148), ([5], 592),
    (list(np.random.default_rng(0).integers(1, 130, 128)), 148), ([1], 1),
])
def test_work_split_partition(tiles, C):
    """Ranges partition [0, T) into near-equal pieces; every unit is touched by the
    contiguous ranges [first, last]; at most one cut unit begins in any range, which
    bounds the partial slots at two per range."""
    starts, first, last = ops.work_split([int(t) for t in tiles], C)
    T = int(sum(tiles))
    Ce = min(C, T)
    assert starts[0] == 0 and starts[-1] == T
    sizes = np.diff(starts)
    # the first min(C, T) ranges are non-empty and near-equal; the rest are empty
    assert sizes[:Ce].min() >= max(1, T // Ce) and sizes[:Ce].max() <= -(-T // Ce)
    assert not sizes[Ce:].any()
    Tu = np.concatenate([[0], np.cumsum(tiles)])
    for u in range(len(tiles)):
        # brute force: ranges whose [start, end) meets [Tu, Tu + tiles)
        touching = [c for c in range(C) if starts[c] < Tu[u + 1] and starts[c + 1] > Tu[u]]
        assert touching == list(range(first[u], last[u] + 1))
    cut_starts = [first[u] for u in range(len(tiles)) if last[u] > first[u]]
    assert len(cut_starts) == len(set(cut_starts))


def _causal_tiles(B, Hkv, N, S, kt):
    """Key tiles of each block-causal unit in the kernel's order ((n, h) major, block b minor):
    the block's own S keys, then its S*b context keys, key_tile at a time."""
    one = [-(-S // kt) + -(-S * b // kt) for b in range(N // S)]
    return one * (B * Hkv)


def _modelled_range_times(tiles, starts, unit_cost):
    """Per range: its tiles plus unit_cost for every unit it touches (a cut unit counts in each
    range that holds a piece of it: each piece loads Q and writes an epilogue)."""
    Tu = np.concatenate([[0], np.cumsum(tiles)])
    out = []
    for c in range(len(starts) - 1):
        s, e = starts[c], starts[c + 1]
        if e <= s:
            continue
        u0 = np.searchsorted(Tu, s, side="right") - 1
        u1 = np.searchsorted(Tu, e, side="left")
        out.append((e - s) + unit_cost * (u1 - u0))
    return np.array(out, dtype=np.float64)


@pytest.mark.parametrize("B,Hkv,N,S,kt,C", [
    (8, 2, 8192, 16, 64, 148), (1, 2, 8192, 16, 64, 148), (2, 4, 4096, 32, 64, 148), (1, 1, 2048, 16, 128, 37),
    (3, 2, 1024, 16, 64, 148), (1, 1, 64, 16, 64, 148), (1, 1, 16, 16, 64, 148), (1, 1, 256, 16, 64, 1),
])
def test_causal_split_weighs_units(B, Hkv, N, S, kt, C):
    """The block-causal boundaries partition [0, T) into min(C, T) non-empty ranges; with no
    unit cost they are the even split; with the default cost the modelled range times (tiles +
    8 per touched unit) are balanced far better than the even split's, which puts the many
    short early blocks of each (n, h) into a few ranges."""
    tiles = _causal_tiles(B, Hkv, N, S, kt)
    T = sum(tiles)
    Ce = min(C, T)
    even = ops.causal_split(B, Hkv, N, S, kt, C, 0)
    assert even == ops.work_split(tiles, C)[0]
    starts = ops.causal_split(B, Hkv, N, S, kt, C)
    assert starts[0] == 0 and starts[Ce] == T and all(x == T for x in starts[Ce:])
    assert all(starts[c] < starts[c + 1] for c in range(Ce))
    # the partial-slot bound of the split holds for the table too: at most one cut unit begins in
    # any range (brute force over the units)
    Tu = np.concatenate([[0], np.cumsum(tiles)])
    cut_first = []
    for u in range(len(tiles)):
        touching = [c for c in range(Ce) if starts[c] < Tu[u + 1] and starts[c + 1] > Tu[u]]
        assert touching == list(range(touching[0], touching[-1] + 1))
        if len(touching) > 1:
            cut_first.append(touching[0])
    assert len(cut_first) == len(set(cut_first))
    if T <= C:
        assert starts == even   # one tile per range: nothing to weigh
        return
    w = _modelled_range_times(tiles, starts, 8)
    e = _modelled_range_times(tiles, even, 8)
    # a boundary moves by at most one unit's fixed cost to stay off it: within one unit cost
    # of the mean (the even split is off by 1.6 to 2.1 x the mean on these shapes)
    assert w.max() - w.mean() <= 8 + 1
    assert w.max() <= e.max()
    if (B, N) == (1, 8192):
        assert e.max() / e.mean() > 1.6 and w.max() / w.mean() < 1.02


def test_causal_split_rejects_bad_geometry():
    for args in [(0, 1, 64, 16, 64, 4), (1, 1, 60, 16, 64, 4), (1, 1, 64, 16, 0, 4), (1, 1, 64, 16, 64, 0),
                 (1, 0, 64, 16, 64, 4), (1, 1, 8, 16, 64, 4)]:
        with pytest.raises(RuntimeError):
            ops.causal_split(*args)


def test_no_device_plan_creation_reports_cuda_error():
    """Without a visible GPU a valid descriptor yields TT_ERR_CUDA (never a CPU path)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("GPU present")
    import ctypes
    desc = ops.Desc(1, 4, 1, 64, 16, 256, 0, 0.0, 0, 0, 0, 0)
    h = ctypes.c_void_p()
    st = ops.lib().tt_block_attn_plan(ctypes.byref(desc), 0, ctypes.byref(h))
    assert st in (ops.TT_ERR_CUDA, ops.TT_ERR_INVALID_ARG)
    assert not h.value


@pytest.mark.parametrize("page_size,num_pages,pages_per_seq", [
    (0, 1, 1), (8, 1, 1), (48, 1, 1), (1 << 17, 1, 1), (-64, 1, 1), (64, -1, 1), (64, 1, -1)])
def test_paged_rejects_bad_page_geometry_before_the_device(page_size, num_pages, pages_per_seq):
    """Page size must be a power of two in [16, 65536] and the counts non-negative; the
    check precedes every use of the plan or the device."""
    L = ops.lib()
    st = L.tt_block_attn_paged(None, None, None, None, None, num_pages, page_size, pages_per_seq, None, None, None,
                               None, None, None)
    assert st == ops.TT_ERR_INVALID_ARG
    assert b"page" in L.tt_last_error_detail()


def _shape_only_plan(**kw):
    """A Plan object with a shape but no library handle: the binding's argument checks
    run before any library call, so they can be exercised without a GPU."""
    p = object.__new__(ops.Plan)
    d = dict(batch=2, q_heads=8, kv_heads=2, head_dim=64, block=4, ctx_capacity=32, seq_len=0)
    d.update(kw)
    p.shape = ops.Shape(**d)
    p.device = 0
    p._h = None
    return p


def test_binding_rejects_wrong_dtype_and_size_before_the_library():
    import torch
    plan = _shape_only_plan()
    B, S, Hq, Hkv, D, L = 2, 4, 8, 2, 64, 32
    q = torch.zeros(B, S, Hq, D, dtype=torch.bfloat16)
    kc = torch.zeros(B, Hkv, L, D, dtype=torch.bfloat16)
    kb = torch.zeros(B, S, Hkv, D, dtype=torch.bfloat16)
    lens = torch.zeros(B, dtype=torch.int32)
    out = torch.zeros(B, S, Hq, D)
    with pytest.raises(TypeError, match="q: dtype"):              # fp16 is not bf16
        plan.block_attn(q.half(), kc, kc, kb, kb, lens, out=out)
    with pytest.raises(ValueError, match="k_blk: .* elements"):   # one KV head short
        plan.block_attn(q, kc, kc, kb[:, :, :1], kb, lens, out=out)
    with pytest.raises(ValueError, match="k_ctx: .* elements"):   # capacity 16, plan has 32
        plan.block_attn(q, kc[:, :, :16], kc, kb, kb, lens, out=out)
    with pytest.raises(TypeError, match="ctx_lens"):              # int64 lengths
        plan.block_attn(q, kc, kc, kb, kb, lens.long(), out=out)
    with pytest.raises(TypeError, match="out"):                   # bf16 output
        plan.block_attn(q, kc, kc, kb, kb, lens, out=out.bfloat16())
    with pytest.raises(ValueError, match="cuda:0"):               # right sizes, host memory
        plan.block_attn(q, kc, kc, kb, kb, lens, out=out)


def test_binding_checks_paged_pool_and_table_shapes():
    import torch
    plan = _shape_only_plan(ctx_capacity=0)
    B, S, Hq, Hkv, D = 2, 4, 8, 2, 64
    q = torch.zeros(B, S, Hq, D, dtype=torch.bfloat16)
    kb = torch.zeros(B, S, Hkv, D, dtype=torch.bfloat16)
    lens = torch.zeros(B, dtype=torch.int32)
    out = torch.zeros(B, S, Hq, D)
    pool = torch.zeros(5, Hkv, 16, D, dtype=torch.bfloat16)
    table = torch.zeros(B, 3, dtype=torch.int32)
    with pytest.raises(ValueError, match="k_pages: shape"):       # KV heads and head_dim swapped
        plan.block_attn_paged(q, pool.view(5, D, 16, Hkv), pool, table, kb, kb, lens, out=out)
    with pytest.raises(ValueError, match="v_pages: .* elements"):
        plan.block_attn_paged(q, pool, pool[:4], table, kb, kb, lens, out=out)
    with pytest.raises(ValueError, match="page_table: shape"):    # one row per sequence
        plan.block_attn_paged(q, pool, pool, table[:1], kb, kb, lens, out=out)
    with pytest.raises(TypeError, match="page_table"):
        plan.block_attn_paged(q, pool, pool, table.long(), kb, kb, lens, out=out)


def test_binding_accepts_bf16_bit_patterns_as_two_byte_integers():
    import torch
    ops._arg(torch.zeros(6, dtype=torch.int16), "x", 6, "bf16", None)
    ops._arg(torch.zeros(6, dtype=torch.bfloat16), "x", 6, "bf16", None)
    with pytest.raises(TypeError):
        ops._arg(torch.zeros(6, dtype=torch.float16), "x", 6, "bf16", None)
    ops._arg(torch.zeros(1, dtype=torch.int32), "status", 1, "w32", None)
    with pytest.raises(TypeError):
        ops._arg(torch.zeros(1, dtype=torch.float32), "status", 1, "w32", None)
    ops._arg(torch.zeros(3), "out", 3, "f32", "host")


def test_binding_paged_without_context_needs_no_pool():
    """No pools and no table: the binding passes NULLs through (valid only without
    context; the library rejects pages_per_seq > 0 without a pool)."""
    import torch
    plan = _shape_only_plan(ctx_capacity=0)
    B, S, Hq, Hkv, D = 2, 4, 8, 2, 64
    q = torch.zeros(B, S, Hq, D, dtype=torch.bfloat16)
    kb = torch.zeros(B, S, Hkv, D, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="q: expected on cuda:0"):    # sizes pass; host memory is refused
        plan.block_attn_paged(q, None, None, None, kb, kb, torch.zeros(B, dtype=torch.int32),
                              out=torch.zeros(B, S, Hq, D))


def test_binding_marshals_page_geometry_from_tensor_shapes(monkeypatch):
    """The paged call hands the library num_pages = pool.shape[0], page_size =
    pool.shape[2] and pages_per_seq = table.shape[1], in the header's argument order
    (recorded by a stand-in library; device checks are off for host tensors here)."""
    import torch
    seen = {}

    class Rec:
        def tt_block_attn_paged(self, *a):
            seen["args"] = a
            return ops.TT_OK

    monkeypatch.setattr(ops, "lib", lambda: Rec())
    real_arg = ops._arg
    monkeypatch.setattr(ops, "_arg", lambda t, n, k, kind, dev: real_arg(t, n, k, kind, None))
    plan = _shape_only_plan(ctx_capacity=0)
    B, S, Hq, Hkv, D = 2, 4, 8, 2, 64
    pool = torch.zeros(7, Hkv, 32, D, dtype=torch.bfloat16)
    table = torch.zeros(B, 5, dtype=torch.int32)
    q = torch.zeros(B, S, Hq, D, dtype=torch.bfloat16)
    kb = torch.zeros(B, S, Hkv, D, dtype=torch.bfloat16)
    lens = torch.zeros(B, dtype=torch.int32)
    out = torch.zeros(B, S, Hq, D)
    monkeypatch.setattr(ops, "_stream", lambda s: None)
    plan.block_attn_paged(q, pool, pool, table, kb, kb, lens, out=out)
    a = seen["args"]
    assert a[5:8] == (7, 32, 5)                                   # num_pages, page_size, pages_per_seq
    assert a[1].value == q.data_ptr() and a[4].value == table.data_ptr() and a[10].value == lens.data_ptr()
    assert a[11].value == out.data_ptr() and a[12] is None        # no lse requested


def test_binding_bf16_output_plan_wants_bf16_out():
    """A plan made with out_bf16=True takes a bf16 `out` (2-byte elements) and rejects fp32."""
    import torch
    plan = _shape_only_plan()
    plan.out_dtype = torch.bfloat16
    B, S, Hq, Hkv, D, L = 2, 4, 8, 2, 64, 32
    q = torch.zeros(B, S, Hq, D, dtype=torch.bfloat16)
    kc = torch.zeros(B, Hkv, L, D, dtype=torch.bfloat16)
    kb = torch.zeros(B, S, Hkv, D, dtype=torch.bfloat16)
    lens = torch.zeros(B, dtype=torch.int32)
    with pytest.raises(TypeError, match="out"):
        plan.block_attn(q, kc, kc, kb, kb, lens, out=torch.zeros(B, S, Hq, D))
    with pytest.raises(ValueError, match="cuda:0"):               # right dtype and size, host memory
        plan.block_attn(q, kc, kc, kb, kb, lens, out=torch.zeros(B, S, Hq, D, dtype=torch.bfloat16))


def test_plan_flag_values_match_the_header():
    import re
    hdr = open(os.path.join(os.path.dirname(__file__), "..", "include", "tt_block_attn.h")).read()
    flags = {m.group(1): int(m.group(2)) for m in re.finditer(r"#define (TT_PLAN_\w+) (\d+)", hdr)}
    assert flags == {"TT_PLAN_HOST_IO": ops.PLAN_HOST_IO, "TT_PLAN_OUT_BF16": ops.PLAN_OUT_BF16}

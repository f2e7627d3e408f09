"""GPU parity: the CUDA kernels through the C ABI against the float64 oracle.

Tolerance (bf16 inputs, fp32 accumulation): max-abs <= 1e-2 and relative
L2 <= 5e-3, on `out` and on `lse`.  Context rows beyond L_n are NaN on the
device in every decode case, so any read of them would show.
"""
import os

import numpy as np
import pytest
import torch

from oracle import block_attn as oracle_attn
from oracle import block_causal as oracle_causal
from tests.gpu_util import assert_parity, dev, errors, f64, poison_beyond
from two_tower_block_b200 import ops
from two_tower_block_b200.workloads import WORKLOADS, bf16_bits, make_causal, make_decode, make_workload

pytestmark = pytest.mark.gpu

# (kernel, plan-time tuning knobs): the tcgen05 kernel with two 64-key S buffers per
# M-tile (default), with one 128-key buffer (TT_TCGEN05_KEY_TILE=128), and the
# transposed-PV kernel for head_dim 128 (TT_TCGEN05_VARIANT=2), the 2-SM kernel
# (TT_TCGEN05_VARIANT=3; head_dim 128 with 128 % g == 0, else the default), the default kernel with
# the split combine fused into its tail (TT_FUSED_COMBINE=1); the mma.sync baseline
KERNELS = [pytest.param((ops.KERNEL_TCGEN05, {}), id="tcgen05"),
           pytest.param((ops.KERNEL_TCGEN05, {"TT_TCGEN05_KEY_TILE": "128"}), id="tcgen05_k128"),
           pytest.param((ops.KERNEL_TCGEN05, {"TT_TCGEN05_VARIANT": "2"}), id="tcgen05_pt"),
           pytest.param((ops.KERNEL_TCGEN05, {"TT_TCGEN05_VARIANT": "3"}), id="tcgen05_2sm"),
           pytest.param((ops.KERNEL_TCGEN05, {"TT_FUSED_COMBINE": "1"}), id="tcgen05_fused"),
           pytest.param((ops.KERNEL_MMA_SYNC, {}), id="mma_sync")]
KNOBS = ("TT_TCGEN05_KEY_TILE", "TT_TCGEN05_VARIANT", "TT_FUSED_COMBINE")


def make_plan(kernel, *args, **kw):
    """ops.Plan for a (kernel, knobs) parameter; the knobs are read at plan creation."""
    kind, knobs = kernel
    old = {k: os.environ.pop(k, None) for k in KNOBS}
    try:
        os.environ.update(knobs)
        plan = ops.Plan(*args, kernel=kind, **kw)
    finally:
        for k in KNOBS:
            os.environ.pop(k, None)
            if old[k] is not None:
                os.environ[k] = old[k]
    if "TT_TCGEN05_KEY_TILE" in knobs:
        assert plan.info().key_tile == int(knobs["TT_TCGEN05_KEY_TILE"])
    return plan


def run_decode(inp, kernel, num_ctas=0, poison=True):
    B, S, Hq, Hkv, D, Lcap = inp.shape
    plan = make_plan(kernel, B, Hq, Hkv, D, S, ctx_capacity=Lcap, num_ctas=num_ctas)
    kc = poison_beyond(inp.k_ctx, inp.ctx_lens) if poison else inp.k_ctx
    vc = poison_beyond(inp.v_ctx, inp.ctx_lens) if poison else inp.v_ctx
    out, lse = plan.block_attn(dev(inp.q), dev(kc), dev(vc), dev(inp.k_blk), dev(inp.v_blk),
                               torch.from_numpy(inp.ctx_lens).cuda(), want_lse=True)
    plan.check()
    return out, lse


def oracle_decode(inp, idx=None):
    sl = slice(None) if idx is None else idx
    return oracle_attn(f64(inp.q[sl]), f64(inp.k_ctx[sl]), f64(inp.v_ctx[sl]), f64(inp.k_blk[sl]),
                       f64(inp.v_blk[sl]), inp.ctx_lens[sl])


SMALL = {
    "tiny-workload": lambda: make_workload(1),
    "gqa16-ragged": lambda: make_decode(3, 16, 32, 2, 128, 777, seed=7, ctx_lens=[0, 300, 777]),
    "d64-g4": lambda: make_decode(2, 16, 8, 2, 64, 200, seed=8, ctx_lens=[129, 64]),
    "odd-block-S5-g3": lambda: make_decode(2, 5, 6, 2, 128, 150, seed=9, ctx_lens=[150, 1]),
    "S256-g1": lambda: make_decode(1, 256, 2, 2, 64, 300, seed=10, ctx_lens=[300]),
    "S1-g16": lambda: make_decode(4, 1, 16, 1, 128, 513, seed=11, ctx_lens=[513, 0, 1, 255]),
    "no-context": lambda: make_decode(2, 16, 4, 1, 64, 0, seed=12),
    "peaky-std3": lambda: make_decode(2, 16, 16, 1, 128, 400, seed=13, std=3.0, peaky_frac=0.05,
                                      ctx_lens=[400, 385]),
}


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("case", list(SMALL))
def test_decode_small(case, kernel):
    inp = SMALL[case]()
    out, lse = run_decode(inp, kernel)
    ro, rl = oracle_decode(inp)
    assert_parity(out, ro, f"{case} out")
    assert_parity(lse, rl, f"{case} lse")


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("num_ctas", [1, 3, 37, 148, 300])
def test_split_count_invariance(kernel, num_ctas):
    """Any cut of the key list into segments recombines to the same softmax."""
    inp = make_decode(3, 16, 32, 2, 128, 1000, seed=21, ctx_lens=[1000, 517, 3])
    out, lse = run_decode(inp, kernel, num_ctas=num_ctas)
    ro, rl = oracle_decode(inp)
    assert_parity(out, ro, f"C={num_ctas} out")
    assert_parity(lse, rl, f"C={num_ctas} lse")


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("num_ctas", [40, 65])
def test_combine_many_segments(kernel, num_ctas):
    """One long unit cut into more than 32 segments: the combine folds its sweeps of 32
    segments online (running maximum and rescaled sums)."""
    inp = make_decode(1, 16, 16, 1, 128, 8192, seed=23, ctx_lens=[8192])
    out, lse = run_decode(inp, kernel, num_ctas=num_ctas)
    ro, rl = oracle_decode(inp)
    assert_parity(out, ro, f"C={num_ctas} out")
    assert_parity(lse, rl, f"C={num_ctas} lse")


@pytest.fixture(scope="module")
def wl2():
    return make_workload(2)


@pytest.mark.parametrize("kernel", KERNELS)
def test_decode_L4096_peaky_full(wl2, kernel):
    """Full decode workload (B=8, Hq=32, Hkv=2, D=128, L=4096, 1% keys x8): every output."""
    out, lse = run_decode(wl2, kernel)
    ro, rl = oracle_decode(wl2)
    assert_parity(out, ro, "L4096 out")
    assert_parity(lse, rl, "L4096 lse")


@pytest.mark.parametrize("kernel", KERNELS)
def test_decode_ragged_B64_sampled(kernel):
    """Full ragged workload on the GPU; oracle on sampled sequences (shortest,
    longest, first, one more)."""
    inp = make_workload(3)
    out, lse = run_decode(inp, kernel, poison=True)
    lens = inp.ctx_lens
    for n in sorted({int(np.argmin(lens)), int(np.argmax(lens)), 0, 33}):
        ro, rl = oracle_decode(inp, slice(n, n + 1))
        assert_parity(out[n:n + 1], ro, f"ragged n={n} L={lens[n]} out")
        assert_parity(lse[n:n + 1], rl, f"ragged n={n} lse")


@pytest.mark.parametrize("kernel", KERNELS)
def test_decode_long_L131072_sampled(kernel):
    """Full long-context workload (B=4, L=131072, std 0.5) on the GPU; oracle on
    sequence 2 (both KV heads), which spans many segments."""
    inp = make_workload(4)
    out, lse = run_decode(inp, kernel, poison=False)
    assert torch.isfinite(out).all()
    ro, rl = oracle_decode(inp, slice(2, 3))
    assert_parity(out[2:3], ro, "long out")
    assert_parity(lse[2:3], rl, "long lse")


def run_causal(inp, kernel, num_ctas=0):
    B, N, Hq, D = inp.q.shape
    Hkv = inp.k_ctx.shape[1]
    plan = make_plan(kernel, B, Hq, Hkv, D, inp.block_size, seq_len=N, num_ctas=num_ctas)
    out, lse = plan.block_attn_block_causal(dev(inp.q), dev(inp.k_ctx), dev(inp.v_ctx), dev(inp.k_blk),
                                            dev(inp.v_blk), want_lse=True)
    plan.check()
    return out, lse


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("shape", [(2, 64, 16, 8, 2, 128), (1, 40, 4, 8, 1, 64), (2, 300, 20, 4, 2, 128)],
                         ids=["S16-g4", "S4-g8-d64", "S20-g2"])
def test_block_causal_small(kernel, shape):
    B, N, S, Hq, Hkv, D = shape
    inp = make_causal(B, N, S, Hq, Hkv, D, seed=31)
    out, lse = run_causal(inp, kernel)
    ro, rl = oracle_causal(f64(inp.q), f64(inp.k_ctx), f64(inp.v_ctx), f64(inp.k_blk), f64(inp.v_blk), S)
    assert_parity(out, ro, "causal out")
    assert_parity(lse, rl, "causal lse")


@pytest.mark.parametrize("kernel", KERNELS)
def test_block_causal_full_sampled(kernel):
    """Full training/prefill workload (B=8, N=8192, 512 blocks of 16) on the GPU;
    oracle on sampled blocks of two sequences."""
    w = WORKLOADS[5]
    inp = make_workload(5)
    out, lse = run_causal(inp, kernel)
    S = w.block_size
    for n, blocks in [(0, [0, 1, 8, 100, 511]), (7, [255, 511])]:
        sl = slice(n, n + 1)
        ro, rl = oracle_causal(f64(inp.q[sl]), f64(inp.k_ctx[sl]), f64(inp.v_ctx[sl]), f64(inp.k_blk[sl]),
                               f64(inp.v_blk[sl]), S, blocks=blocks)
        for b in blocks:
            p = slice(S * b, S * b + S)
            assert_parity(out[n:n + 1, p], ro[:, p], f"causal n={n} b={b} out")
            assert_parity(lse[n:n + 1, :, p], rl[:, :, p], f"causal n={n} b={b} lse")


@pytest.mark.parametrize("kernel", KERNELS)
def test_block_causal_equals_decode(kernel):
    """Block b of the block-causal entry is the decode entry with L = S*b on the
    same sequence (GPU against GPU, same kernel)."""
    B, N, S, Hq, Hkv, D = 2, 96, 16, 8, 2, 128
    inp = make_causal(B, N, S, Hq, Hkv, D, seed=41)
    out_c, lse_c = run_causal(inp, kernel)
    for b in [0, 1, 5]:
        p = slice(S * b, S * b + S)
        plan = make_plan(kernel, B, Hq, Hkv, D, S, ctx_capacity=N)
        lens = torch.full((B,), S * b, dtype=torch.int32, device="cuda")
        out_d, lse_d = plan.block_attn(dev(np.ascontiguousarray(inp.q[:, p])), dev(inp.k_ctx), dev(inp.v_ctx),
                                       dev(np.ascontiguousarray(inp.k_blk[:, p])),
                                       dev(np.ascontiguousarray(inp.v_blk[:, p])), lens, want_lse=True)
        plan.check()
        torch.testing.assert_close(out_d, out_c[:, p], atol=2e-5, rtol=1e-4)
        torch.testing.assert_close(lse_d, lse_c[:, :, p], atol=2e-5, rtol=1e-4)


@pytest.mark.parametrize("kernel", KERNELS)
def test_host_io_entry_matches_device_entry(kernel):
    inp = make_decode(2, 16, 32, 2, 128, 600, seed=51, ctx_lens=[600, 257])
    B, S, Hq, Hkv, D, Lcap = inp.shape
    out_dev, lse_dev = run_decode(inp, kernel, poison=False)
    plan = make_plan(kernel, B, Hq, Hkv, D, S, ctx_capacity=Lcap, host_io=True)

    def pinned(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    out = torch.empty((B, S, Hq, D), dtype=torch.float32).pin_memory()
    lse = torch.empty((B, Hq, S), dtype=torch.float32).pin_memory()
    plan.block_attn_host(pinned(inp.q), pinned(inp.k_ctx), pinned(inp.v_ctx), pinned(inp.k_blk),
                         pinned(inp.v_blk), torch.from_numpy(inp.ctx_lens).pin_memory(), out, lse)
    plan.check()
    torch.testing.assert_close(out, out_dev.cpu(), atol=0, rtol=0)
    torch.testing.assert_close(lse, lse_dev.cpu(), atol=0, rtol=0)


@pytest.mark.parametrize("kernel", KERNELS)
def test_ctx_len_out_of_range_is_reported(kernel):
    inp = make_decode(2, 16, 8, 2, 64, 100, seed=61, ctx_lens=[100, 50])
    B, S, Hq, Hkv, D, Lcap = inp.shape
    plan = make_plan(kernel, B, Hq, Hkv, D, S, ctx_capacity=Lcap)
    args = [dev(inp.q), dev(inp.k_ctx), dev(inp.v_ctx), dev(inp.k_blk), dev(inp.v_blk)]
    bad = torch.tensor([101, 50], dtype=torch.int32, device="cuda")
    plan.block_attn(*args, bad)
    assert plan.check_status() == ops.TT_ERR_DEVICE_ARG
    bad = torch.tensor([-3, 50], dtype=torch.int32, device="cuda")
    plan.block_attn(*args, bad)
    assert plan.check_status() == ops.TT_ERR_DEVICE_ARG
    # the error word was cleared and the context still works
    out = plan.block_attn(*args, torch.from_numpy(inp.ctx_lens).cuda())
    plan.check()
    ro, _ = oracle_decode(inp)
    assert_parity(out, ro, "after device error")


def test_wait_timeout_selftest():
    """A wait on a barrier nothing arrives at gives up after its limit and reports
    TT_ERR_TIMEOUT; the device stays usable."""
    assert ops.selftest_wait_timeout(0, 20000) == ops.TT_ERR_TIMEOUT
    x = torch.ones(1024, device="cuda")
    assert float(x.sum()) == 1024.0


@pytest.mark.parametrize("kernel", KERNELS)
def test_empty_batch_is_noop(kernel):
    plan = make_plan(kernel, 0, 8, 2, 128, 16, ctx_capacity=64)
    e = torch.empty(0, dtype=torch.bfloat16, device="cuda")
    lens = torch.empty(0, dtype=torch.int32, device="cuda")
    out = torch.empty(0, dtype=torch.float32, device="cuda")
    plan.block_attn(e, e, e, e, e, lens, out=out)
    plan.check()


@pytest.mark.parametrize("kernel", KERNELS)
def test_profile_hook_counts_launches(kernel):
    inp = make_decode(2, 16, 32, 2, 128, 2048, seed=71)
    B, S, Hq, Hkv, D, Lcap = inp.shape
    plan = make_plan(kernel, B, Hq, Hkv, D, S, ctx_capacity=Lcap)
    args = [dev(inp.q), dev(inp.k_ctx), dev(inp.v_ctx), dev(inp.k_blk), dev(inp.v_blk),
            torch.from_numpy(inp.ctx_lens).cuda()]
    plan.profile(True)
    for _ in range(5):
        plan.block_attn(*args)
    n, ms = plan.profile_read(0)
    plan.profile(False)
    assert n == 5 and ms > 0


# --- committed-block cache update -------------------------------------------------
def _bits(shape, rng):
    """Random 16-bit patterns (every bf16 value, NaN and Inf patterns included)."""
    return rng.integers(0, 1 << 16, size=shape, dtype=np.uint16)


def _dev_bits(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("advance", [True, False])
def test_kv_append_bit_exact(D, advance):
    from oracle import kv_append as oracle_append
    rng = np.random.default_rng(31 + D)
    B, S, Hkv, Lcap = 4, 16, 2, 100
    lens = np.array([0, 50, 84, 85], dtype=np.int32)          # the last has no room
    k_new, v_new = _bits((B, S, Hkv, D), rng), _bits((B, S, Hkv, D), rng)
    k_ctx, v_ctx = _bits((B, Hkv, Lcap, D), rng), _bits((B, Hkv, Lcap, D), rng)
    plan = ops.Plan(B, 4, Hkv, D, S, ctx_capacity=Lcap)
    dk, dv, dl = _dev_bits(k_ctx), _dev_bits(v_ctx), torch.from_numpy(lens).cuda()
    plan.kv_append(_dev_bits(k_new), _dev_bits(v_new), dk, dv, dl, advance=advance)
    assert plan.check_status() == ops.TT_ERR_DEVICE_ARG         # sequence 3 was reported
    rk, rv, rl, bad = oracle_append(k_new, v_new, k_ctx, v_ctx, lens, advance=advance)
    assert list(bad) == [False, False, False, True]
    assert np.array_equal(dk.cpu().numpy().view(np.uint16), rk)
    assert np.array_equal(dv.cpu().numpy().view(np.uint16), rv)
    assert np.array_equal(dl.cpu().numpy(), rl.astype(np.int32))


def test_kv_append_then_decode_equals_decode_with_block_in_context():
    """Commit block b (its context-tower K/V) and decode the next block: the same as
    decoding that block with the committed rows already in the cache."""
    from oracle import kv_append as oracle_append
    inp = make_decode(2, 16, 32, 2, 128, 600, seed=33, ctx_lens=[300, 584])
    k_new = make_decode(2, 16, 32, 2, 128, 1, seed=35).k_blk      # bf16 bits [B, S, Hkv, D]
    v_new = make_decode(2, 16, 32, 2, 128, 1, seed=36).v_blk
    plan = ops.Plan(2, 32, 2, 128, 16, ctx_capacity=600)
    dk, dv, dl = dev(inp.k_ctx).clone(), dev(inp.v_ctx).clone(), torch.from_numpy(inp.ctx_lens).cuda()
    plan.kv_append(dev(k_new), dev(v_new), dk, dv, dl)
    out, lse = plan.block_attn(dev(inp.q), dk, dv, dev(inp.k_blk), dev(inp.v_blk), dl, want_lse=True)
    plan.check()
    rk, rv, rl, _ = oracle_append(k_new, v_new, inp.k_ctx, inp.v_ctx, inp.ctx_lens)
    ro, rlse = oracle_attn(f64(inp.q), f64(rk), f64(rv), f64(inp.k_blk), f64(inp.v_blk), rl)
    assert_parity(out, ro, "out after append")
    assert_parity(lse, rlse, "lse after append")


# --- block-causal backward ------------------------------------------------------------
def run_backward(inp, dout_bits, kernel=(ops.KERNEL_TCGEN05, {}), bwd="tcgen05"):
    """Forward and backward through the C ABI.  bwd: "tcgen05" (the tensor-memory kernel,
    where the shape allows it) or "mma_sync" (the warp-level kernel, TT_BWD_KERNEL)."""
    B, N, Hq, D = inp.q.shape
    Hkv = inp.k_ctx.shape[1]
    plan = make_plan(kernel, B, Hq, Hkv, D, inp.block_size, seq_len=N)
    q, kc, vc, kb, vb = dev(inp.q), dev(inp.k_ctx), dev(inp.v_ctx), dev(inp.k_blk), dev(inp.v_blk)
    out, lse = plan.block_attn_block_causal(q, kc, vc, kb, vb, want_lse=True)
    old = os.environ.pop("TT_BWD_KERNEL", None)
    try:
        if bwd == "mma_sync":
            os.environ["TT_BWD_KERNEL"] = "mma_sync"
        dq, dk, dv = plan.block_causal_backward(q, kc, vc, kb, vb, out, lse, dev(dout_bits))
        plan.check()
    finally:
        os.environ.pop("TT_BWD_KERNEL", None)
        if old is not None:
            os.environ["TT_BWD_KERNEL"] = old
    return dq, dk, dv


@pytest.mark.parametrize("bwd", ["tcgen05", "mma_sync"])
@pytest.mark.parametrize("shape", [(2, 64, 16, 8, 2, 128), (1, 40, 4, 8, 1, 64), (2, 300, 20, 4, 2, 128),
                                   (1, 256, 128, 2, 1, 64), (1, 128, 16, 16, 1, 128), (2, 96, 16, 32, 2, 64),
                                   (1, 200, 8, 24, 1, 128)],
                         ids=["S16-g4-D128", "S4-g8-D64", "S20-g2-D128-ragged", "S128-g2-D64",
                              "S16-g16-D128-two-Mtiles", "S16-g16-D64-two-Mtiles", "S8-g24-D128-partial-Mtile"])
def test_block_causal_backward_small(shape, bwd):
    """Small shapes spanning several key tiles, ragged tails (S = 20: blocks and context tiles
    that are not multiples of 16), both head dims, one and two 128-row M-tiles (S*g = 256) and
    a partial second M-tile (S*g = 192, g = 24 does not divide 128: the warp-level kernel)."""
    from oracle import block_causal_backward
    B, N, S, Hq, Hkv, D = shape
    inp = make_causal(B, N, S, Hq, Hkv, D, seed=41)
    dout = bf16_bits(np.random.default_rng(42).standard_normal((B, N, Hq, D)).astype(np.float32))
    dq, dk, dv = run_backward(inp, dout, bwd=bwd)
    rq, rk, rv = block_causal_backward(f64(inp.q), f64(inp.k_ctx), f64(inp.v_ctx), f64(inp.k_blk),
                                       f64(inp.v_blk), f64(dout), S)
    errs = {w: errors(a, r) for w, a, r in (("dq", dq, rq), ("dk_blk", dk, rk), ("dv_blk", dv, rv))}
    print({w: (f"{e[0]:.2e}", f"{e[1]:.2e}") for w, e in errs.items()})
    assert_parity(dq, rq, "dq")
    assert_parity(dk, rk, "dk_blk")
    assert_parity(dv, rv, "dv_blk")


def test_block_causal_backward_full_sampled():
    """The full N=8192 training workload on the GPU; oracle on a few blocks spread over
    the sequence (early, middle, last) of sequence 0."""
    from oracle import block_causal_backward
    inp = make_workload(5)
    B, N, Hq, D = inp.q.shape
    S = inp.block_size
    dout = bf16_bits(np.random.default_rng(43).standard_normal((B, N, Hq, D)).astype(np.float32))
    dq, dk, dv = run_backward(inp, dout)
    assert torch.isfinite(dq).all() and torch.isfinite(dk).all() and torch.isfinite(dv).all()
    blocks = [0, 1, 255, 511]
    rq, rk, rv = block_causal_backward(f64(inp.q[:1]), f64(inp.k_ctx[:1]), f64(inp.v_ctx[:1]),
                                       f64(inp.k_blk[:1]), f64(inp.v_blk[:1]), f64(dout[:1]), S,
                                       blocks=blocks)
    for b in blocks:
        sl = slice(S * b, S * b + S)
        assert_parity(dq[:1, sl], rq[:, sl], f"dq block {b}")
        assert_parity(dk[:1, sl], rk[:, sl], f"dk_blk block {b}")
        assert_parity(dv[:1, sl], rv[:, sl], f"dv_blk block {b}")


# --- confidence-unmasking step --------------------------------------------------------
@pytest.mark.parametrize("V", [131072, 1001], ids=["V131072", "V1001-unaligned"])
@pytest.mark.parametrize("min_one", [True, False])
def test_confidence_unmask(V, min_one):
    from oracle import confidence_unmask as oracle_unmask
    rng = np.random.default_rng(51 + V % 7)
    B, S = 4, 16
    x = rng.standard_normal((B, S, V)).astype(np.float32)
    # a few confident positions (p near 0.95 or 0.5, far from the 0.8 threshold)
    for (n, s_, boost) in [(0, 3, 30.0), (0, 9, 30.0), (1, 0, 30.0), (2, 5, np.log(V) + 0.2), (3, 15, 30.0)]:
        x[n, s_, (n * 1000 + s_ * 7) % V] = boost
    bits = bf16_bits(x)
    tokens = np.full((B, S), -1, dtype=np.int32)
    masked = np.ones((B, S), dtype=np.uint8)
    masked[0, 9] = 0           # already committed: untouched even though confident
    masked[3, :8] = 0
    tokens[masked == 0] = 7
    rt, rm, rp, ra, rn = oracle_unmask(f64(bits), tokens, masked.astype(bool), gamma=0.8, min_one=min_one)
    # the test inputs keep every decision unambiguous: no masked confidence near 0.8 and, where
    # the fallback may decide, a unique most confident position
    assert np.all(np.abs(rp[masked == 1] - 0.8) > 1e-3)
    dt, dm = torch.from_numpy(tokens).cuda(), torch.from_numpy(masked).cuda()
    p_max, arg, n_c = ops.confidence_unmask(dev(bits), dt, dm, gamma=0.8, min_one=min_one)
    torch.cuda.synchronize()
    assert np.array_equal(arg.cpu().numpy(), ra)
    gp = p_max.cpu().numpy()
    assert np.allclose(gp, rp, rtol=1e-4, atol=1e-9)
    assert np.array_equal(dt.cpu().numpy(), rt)
    assert np.array_equal(dm.cpu().numpy().astype(bool), rm)
    assert np.array_equal(n_c.cpu().numpy(), rn)

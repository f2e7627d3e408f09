"""The allocation-free decode entry point (tt_block_attn_noalloc) through the C ABI.

It serves callers that may not call cudaMalloc (engines that own all device
memory, serving loops that must not stall on an allocation).  It must give the
same answer as the plan-based entry point, call after call, although every call
reuses one fixed scratch array.  Collected last on purpose (file name), so a
failure here comes after every other test has run.
"""
import numpy as np
import pytest
import torch

from tests.gpu_util import assert_parity, dev, poison_beyond
from two_tower_block_b200 import ops
from two_tower_block_b200.workloads import make_decode

pytestmark = pytest.mark.gpu


def _inputs(inp):
    return [dev(inp.q), dev(poison_beyond(inp.k_ctx, inp.ctx_lens)), dev(poison_beyond(inp.v_ctx, inp.ctx_lens)),
            dev(inp.k_blk), dev(inp.v_blk), torch.from_numpy(inp.ctx_lens).cuda()]


def _plan_entry(inp, args):
    B, S, Hq, Hkv, D, Lcap = inp.shape
    plan = ops.Plan(B, Hq, Hkv, D, S, ctx_capacity=Lcap)
    out, lse = plan.block_attn(*args, want_lse=True)
    plan.check()
    return out, lse


def test_noalloc_matches_plan_entry_two_calls_in_a_row():
    # two different problems back to back: the second call must not see the first's scratch
    cases = [make_decode(3, 16, 32, 2, 128, 1000, seed=91, ctx_lens=[1000, 517, 3]),
             make_decode(2, 16, 8, 2, 64, 700, seed=92, ctx_lens=[129, 700])]
    results = []
    for inp in cases:
        B, S, Hq, Hkv, D, Lcap = inp.shape
        args = _inputs(inp)
        out = torch.full((B, S, Hq, D), float("nan"), device="cuda")
        lse = torch.full((B, Hq, S), float("nan"), device="cuda")
        status = torch.full((1,), 7, dtype=torch.int32, device="cuda")
        st = ops.block_attn_noalloc(*args, out, lse, status)
        assert st == ops.TT_OK, ops.lib().tt_last_error_detail()
        results.append((inp, args, out, lse, status))
    torch.cuda.synchronize()
    for inp, args, out, lse, status in results:
        assert int(status.item()) == 0
        ref_out, ref_lse = _plan_entry(inp, args)
        assert_parity(out, ref_out.double().cpu().numpy(), "noalloc out vs plan entry")
        assert_parity(lse, ref_lse.double().cpu().numpy(), "noalloc lse vs plan entry")


def test_noalloc_same_problem_twice_is_stable():
    inp = make_decode(2, 16, 32, 2, 128, 2000, seed=93, ctx_lens=[2000, 1111])
    args = _inputs(inp)
    B, S, Hq, Hkv, D, Lcap = inp.shape
    outs = []
    for _ in range(2):
        out = torch.empty((B, S, Hq, D), device="cuda")
        assert ops.block_attn_noalloc(*args, out) == ops.TT_OK
        outs.append(out)
    torch.cuda.synchronize()
    ref_out, _ = _plan_entry(inp, args)
    for out in outs:
        assert_parity(out, ref_out.double().cpu().numpy(), "noalloc repeat")


def test_noalloc_rejects_scratch_beyond_limit():
    inp = make_decode(1, 16, 32, 2, 128, 64, seed=94)
    args = _inputs(inp)
    out = torch.empty((1, 16, 32, 128), device="cuda")
    st = ops.block_attn_noalloc(*args, out, num_ctas=4096)  # 4096 ranges need ~1 GiB of partials
    assert st == ops.TT_ERR_INVALID_ARG
    assert b"scratch" in ops.lib().tt_last_error_detail()


def _oracle(inp):
    from oracle import block_attn as oracle_attn
    from tests.gpu_util import f64
    return oracle_attn(f64(inp.q), f64(inp.k_ctx), f64(inp.v_ctx), f64(inp.k_blk), f64(inp.v_blk), inp.ctx_lens)


@pytest.mark.parametrize("kernel", [ops.KERNEL_AUTO, ops.KERNEL_MMA_SYNC], ids=["tcgen05", "mma_sync"])
@pytest.mark.parametrize("case", ["ragged-gqa16", "no-context", "d64-S5-g3"])
def test_noalloc_matches_oracle(case, kernel):
    """Against the float64 oracle directly, at the parity tests' tolerance: ragged GQA rows
    (context rows past L_n are NaN), a plan shape without any context (ctx_capacity = 0: the
    context maps stand in for the block's), and head_dim 64 with S = 5, g = 3; both kernels."""
    inp = {"ragged-gqa16": lambda: make_decode(3, 16, 32, 2, 128, 900, seed=95, ctx_lens=[900, 0, 129]),
           "no-context": lambda: make_decode(2, 16, 8, 2, 128, 0, seed=96),
           "d64-S5-g3": lambda: make_decode(2, 5, 6, 2, 64, 300, seed=97, ctx_lens=[300, 17])}[case]()
    B, S, Hq, Hkv, D, Lcap = inp.shape
    args = _inputs(inp)
    out = torch.full((B, S, Hq, D), float("nan"), device="cuda")
    lse = torch.full((B, Hq, S), float("nan"), device="cuda")
    status = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    st = ops.block_attn_noalloc(*args, out, lse, status, kernel=kernel)
    assert st == ops.TT_OK, ops.lib().tt_last_error_detail()
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ro, rl = _oracle(inp)
    assert_parity(out, ro, f"{case} noalloc out vs oracle")
    assert_parity(lse, rl, f"{case} noalloc lse vs oracle")


def test_noalloc_reports_out_of_range_ctx_len():
    """A ctx_lens value past ctx_capacity reaches the caller's status word (bit 1), and the
    sequences with valid lengths still match the oracle."""
    inp = make_decode(2, 16, 16, 1, 128, 256, seed=98, ctx_lens=[256, 100])
    args = _inputs(inp)
    bad = torch.tensor([256, 5000], dtype=torch.int32, device="cuda")   # 5000 > ctx_capacity
    out = torch.empty((2, 16, 16, 128), device="cuda")
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    assert ops.block_attn_noalloc(*args[:5], bad, out, None, status) == ops.TT_OK
    torch.cuda.synchronize()
    assert int(status.item()) & 1
    ro, _ = _oracle(inp)
    assert_parity(out[:1], ro[:1], "noalloc out, valid sequence")

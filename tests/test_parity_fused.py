"""The split combine in the attention kernel's tail (one launch per call), against the oracle.

The fused combine keeps per-range arrival counts that only grow: every range adds one per launch,
and the ranges of a cut unit wait for one another's counts before sharing the unit's rows.  These
tests run it the ways a caller would: the default plan for short aligned ranges, calls in a row
whose context lengths change which units are cut, decode and block-causal calls on one plan
(each kind keeps its own counts), and replays of a captured CUDA graph.
"""
import os

import pytest
import torch

from oracle import block_attn as oracle_attn
from oracle import block_causal as oracle_causal
from tests.gpu_util import assert_parity, dev, f64, poison_beyond
from two_tower_block_b200 import ops
from two_tower_block_b200.workloads import make_causal, make_decode

pytestmark = pytest.mark.gpu


def _plan(*args, force=None, **kw):
    old = os.environ.pop("TT_FUSED_COMBINE", None)
    try:
        if force is not None:
            os.environ["TT_FUSED_COMBINE"] = force
        return ops.Plan(*args, **kw)
    finally:
        os.environ.pop("TT_FUSED_COMBINE", None)
        if old is not None:
            os.environ["TT_FUSED_COMBINE"] = old


def _args(inp):
    return [dev(inp.q), dev(poison_beyond(inp.k_ctx, inp.ctx_lens)), dev(poison_beyond(inp.v_ctx, inp.ctx_lens)),
            dev(inp.k_blk), dev(inp.v_blk), torch.from_numpy(inp.ctx_lens).cuda()]


def _oracle(inp):
    return oracle_attn(f64(inp.q), f64(inp.k_ctx), f64(inp.v_ctx), f64(inp.k_blk), f64(inp.v_blk), inp.ctx_lens)


def test_short_aligned_plan_runs_one_launch():
    """B*Hkv = 4 units over 148 SMs and a 1024-key capacity: the plan fuses the combine, a call is
    one kernel launch, and its output matches the oracle."""
    inp = make_decode(2, 16, 32, 2, 128, 1024, seed=121, ctx_lens=[1024, 333])
    B, S, Hq, Hkv, D, Lcap = inp.shape
    plan = _plan(B, Hq, Hkv, D, S, ctx_capacity=Lcap)
    info = plan.info()
    if info.sm_count // (B * Hkv) < 2:
        pytest.skip("fewer than two ranges per unit on this device")
    assert info.fused_combine == 1
    args = _args(inp)
    plan.profile(True)
    for _ in range(3):
        out, lse = plan.block_attn(*args, want_lse=True)
    n_k, _ = plan.profile_read(0)
    n_c, _ = plan.profile_read(1)
    plan.profile(False)
    plan.check()
    assert (n_k, n_c) == (3, 0)
    ro, rl = _oracle(inp)
    assert_parity(out, ro, "fused out")
    assert_parity(lse, rl, "fused lse")


def test_long_capacity_plan_keeps_separate_combine():
    """At a 131072-key capacity a range holds more than 32 key tiles: the separate combine kernel."""
    plan = _plan(4, 32, 2, 128, 16, ctx_capacity=131072)
    assert plan.info().fused_combine == 0


def test_calls_in_a_row_with_changing_cuts():
    """Four calls without a synchronisation between them; each set of context lengths cuts the
    units differently, so the counts of a range are waited for by different peers each time."""
    cases = [[1024, 1024], [17, 1024], [1024, 500], [0, 1]]
    plan = _plan(2, 32, 2, 128, 16, ctx_capacity=1024, force="1")
    runs = []
    for i, lens in enumerate(cases):
        inp = make_decode(2, 16, 32, 2, 128, 1024, seed=130 + i, ctx_lens=lens)
        out, lse = plan.block_attn(*_args(inp), want_lse=True)
        runs.append((inp, out, lse))
    plan.check()
    for inp, out, lse in runs:
        ro, rl = _oracle(inp)
        assert_parity(out, ro, f"lens {list(inp.ctx_lens)} out")
        assert_parity(lse, rl, f"lens {list(inp.ctx_lens)} lse")


def test_decode_and_block_causal_on_one_plan():
    """Decode, block-causal, decode on one fused plan: each kind of call keeps its own counts."""
    B, N, S, Hq, Hkv, D = 2, 256, 16, 16, 2, 128
    plan = _plan(B, Hq, Hkv, D, S, ctx_capacity=N, seq_len=N, force="1")
    dec = [make_decode(B, S, Hq, Hkv, D, N, seed=140 + i, ctx_lens=[N - 7 * i, 100 + i]) for i in range(2)]
    cau = make_causal(B, N, S, Hq, Hkv, D, seed=150)
    o0 = plan.block_attn(*_args(dec[0]))
    oc, lc = plan.block_attn_block_causal(dev(cau.q), dev(cau.k_ctx), dev(cau.v_ctx), dev(cau.k_blk),
                                          dev(cau.v_blk), want_lse=True)
    o1 = plan.block_attn(*_args(dec[1]))
    plan.check()
    for inp, out in ((dec[0], o0), (dec[1], o1)):
        assert_parity(out, _oracle(inp)[0], "decode out")
    ro, rl = oracle_causal(f64(cau.q), f64(cau.k_ctx), f64(cau.v_ctx), f64(cau.k_blk), f64(cau.v_blk), S)
    assert_parity(oc, ro, "causal out")
    assert_parity(lc, rl, "causal lse")


def test_graph_replays():
    """Three calls captured in one CUDA graph and the graph replayed twice: the counts keep
    growing across replays, and every replay gives the oracle's output."""
    inp = make_decode(2, 16, 32, 2, 128, 1024, seed=160, ragged=(64, 1024))
    B, S, Hq, Hkv, D, Lcap = inp.shape
    plan = _plan(B, Hq, Hkv, D, S, ctx_capacity=Lcap, force="1")
    args = _args(inp)
    outs = [torch.empty((B, S, Hq, D), dtype=torch.float32, device="cuda") for _ in range(3)]
    plan.block_attn(*args, out=outs[0])   # warm-up outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for o in outs:
            plan.block_attn(*args, out=o)
    ro, _ = _oracle(inp)
    for _ in range(2):
        for o in outs:
            o.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        plan.check()
        for o in outs:
            assert_parity(o, ro, "graph replay out")
    del g

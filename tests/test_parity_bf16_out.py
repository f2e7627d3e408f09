"""bf16 output (plans made with TT_PLAN_OUT_BF16) through the C ABI.

The kernels compute the same fp32 rows and round them once, to nearest even, when they store
the final output (the split partials and lse stay fp32).  So a bf16-output call must equal the
fp32 call of the same plan shape rounded to bf16, bit for bit, and it must meet the oracle at the
parity tolerances.  Covered: decode on the default kernel (combine in the kernel's tail and as a
separate kernel), on the mma.sync kernel, over a paged cache, from host buffers, and the
block-causal form; the backward refuses such a plan.
"""
import os

import numpy as np
import pytest
import torch

from oracle import block_attn as oracle_attn
from oracle import block_causal as oracle_causal
from tests.gpu_util import assert_parity, dev, f64, poison_beyond
from two_tower_block_b200 import ops
from two_tower_block_b200.workloads import make_causal, make_decode, make_paged

pytestmark = pytest.mark.gpu

FORMS = [pytest.param((ops.KERNEL_AUTO, None, 0), id="tcgen05"),
         pytest.param((ops.KERNEL_AUTO, "0", 0), id="tcgen05_sep_combine"),
         pytest.param((ops.KERNEL_AUTO, None, 37), id="tcgen05_37_ranges"),
         pytest.param((ops.KERNEL_MMA_SYNC, None, 0), id="mma_sync")]


def _plan(form, *args, out_bf16, **kw):
    kernel, fused, num_ctas = form
    old = os.environ.pop("TT_FUSED_COMBINE", None)
    try:
        if fused is not None:
            os.environ["TT_FUSED_COMBINE"] = fused
        return ops.Plan(*args, kernel=kernel, num_ctas=num_ctas, out_bf16=out_bf16, **kw)
    finally:
        os.environ.pop("TT_FUSED_COMBINE", None)
        if old is not None:
            os.environ["TT_FUSED_COMBINE"] = old


def _args(inp):
    return [dev(inp.q), dev(poison_beyond(inp.k_ctx, inp.ctx_lens)), dev(poison_beyond(inp.v_ctx, inp.ctx_lens)),
            dev(inp.k_blk), dev(inp.v_blk), torch.from_numpy(inp.ctx_lens).cuda()]


@pytest.mark.parametrize("form", FORMS)
def test_decode_bf16_out(form):
    inp = make_decode(3, 16, 32, 2, 128, 900, seed=171, ctx_lens=[900, 0, 257])
    B, S, Hq, Hkv, D, Lcap = inp.shape
    args = _args(inp)
    p32 = _plan(form, B, Hq, Hkv, D, S, ctx_capacity=Lcap, out_bf16=False)
    p16 = _plan(form, B, Hq, Hkv, D, S, ctx_capacity=Lcap, out_bf16=True)
    o32, l32 = p32.block_attn(*args, want_lse=True)
    o16, l16 = p16.block_attn(*args, want_lse=True)
    p32.check()
    p16.check()
    assert o16.dtype == torch.bfloat16
    assert torch.equal(o16, o32.to(torch.bfloat16))
    assert torch.equal(l16, l32)
    ro, rl = oracle_attn(f64(inp.q), f64(inp.k_ctx), f64(inp.v_ctx), f64(inp.k_blk), f64(inp.v_blk), inp.ctx_lens)
    assert_parity(o16.float(), ro, "bf16 out")
    assert_parity(l16, rl, "lse")


def test_paged_and_host_bf16_out():
    inp = make_decode(2, 16, 32, 2, 128, 512, seed=172, ctx_lens=[512, 77])
    B, S, Hq, Hkv, D, Lcap = inp.shape
    ro, _ = oracle_attn(f64(inp.q), f64(inp.k_ctx), f64(inp.v_ctx), f64(inp.k_blk), f64(inp.v_blk), inp.ctx_lens)
    pin = make_paged(inp, page_size=32, seed=173)
    plan = ops.Plan(B, Hq, Hkv, D, S, ctx_capacity=Lcap, out_bf16=True, host_io=True)
    out = plan.block_attn_paged(dev(inp.q), dev(pin.k_pages), dev(pin.v_pages), torch.from_numpy(pin.page_table).cuda(),
                                dev(inp.k_blk), dev(inp.v_blk), torch.from_numpy(inp.ctx_lens).cuda())
    host_out = torch.empty((B, S, Hq, D), dtype=torch.bfloat16).pin_memory()
    bits = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).pin_memory()
    plan.block_attn_host(bits(inp.q), bits(inp.k_ctx), bits(inp.v_ctx), bits(inp.k_blk), bits(inp.v_blk),
                         torch.from_numpy(inp.ctx_lens).pin_memory(), host_out)
    torch.cuda.synchronize()
    plan.check()
    assert out.dtype == torch.bfloat16
    assert_parity(out.float(), ro, "paged bf16 out")
    assert_parity(host_out.float(), ro, "host bf16 out")


def test_block_causal_bf16_out_and_backward_refused():
    B, N, S, Hq, Hkv, D = 2, 128, 16, 16, 2, 128
    cau = make_causal(B, N, S, Hq, Hkv, D, seed=174)
    a = [dev(cau.q), dev(cau.k_ctx), dev(cau.v_ctx), dev(cau.k_blk), dev(cau.v_blk)]
    p16 = ops.Plan(B, Hq, Hkv, D, S, seq_len=N, out_bf16=True)
    p32 = ops.Plan(B, Hq, Hkv, D, S, seq_len=N)
    o16, l16 = p16.block_attn_block_causal(*a, want_lse=True)
    o32 = p32.block_attn_block_causal(*a)
    p16.check()
    p32.check()
    assert torch.equal(o16, o32.to(torch.bfloat16))
    ro, rl = oracle_causal(f64(cau.q), f64(cau.k_ctx), f64(cau.v_ctx), f64(cau.k_blk), f64(cau.v_blk), S)
    assert_parity(o16.float(), ro, "causal bf16 out")
    dout = torch.zeros((B, N, Hq, D), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ops.TTError) as e:
        p16.block_causal_backward(*a, o32, l16, dout)
    assert e.value.status == ops.TT_ERR_UNSUPPORTED

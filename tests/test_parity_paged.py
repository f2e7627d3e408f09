"""GPU parity of decode over a paged context cache (tt_block_attn_paged) against the
float64 oracle, which gathers the pages back into a contiguous cache.

Pools are shuffled, rows past L_n in a last page and pages no sequence owns are NaN,
and table entries past a sequence's last page are -1, so a read of any of them shows
(as a non-finite output or a device argument error)."""
import numpy as np
import pytest
import torch

from oracle import block_attn_paged as oracle_paged
from tests.gpu_util import assert_parity, dev, f64
from tests.test_parity import KERNELS, make_plan
from two_tower_block_b200 import ops
from two_tower_block_b200.workloads import make_decode, make_paged, make_workload

pytestmark = pytest.mark.gpu

# Plans made for the transposed-PV or 2-SM forms run paged calls on the default tcgen05
# kernel: they are covered by the full-size cases only.
PAGED_KERNELS = [k for k in KERNELS if k.id not in ("tcgen05_pt", "tcgen05_2sm")]


def run_paged(inp, pc, kernel, num_ctas=0):
    B, S, Hq, Hkv, D, _ = inp.shape
    plan = make_plan(kernel, B, Hq, Hkv, D, S, ctx_capacity=0, num_ctas=num_ctas)
    table = torch.from_numpy(pc.page_table).cuda() if pc.page_table.shape[1] else None
    out, lse = plan.block_attn_paged(dev(inp.q), dev(pc.k_pages), dev(pc.v_pages), table, dev(inp.k_blk),
                                     dev(inp.v_blk), torch.from_numpy(inp.ctx_lens).cuda(), want_lse=True)
    plan.check()
    return out, lse


def oracle_of(inp, pc, idx=slice(None)):
    """Oracle over the sequences ``idx``: the pages they own are copied (in table order)
    into a compact pool, so only those are converted to float64."""
    table = pc.page_table[idx]
    owned = table[table >= 0]
    sub = np.full(table.shape, -1, dtype=np.int32)
    sub[table >= 0] = np.arange(owned.size, dtype=np.int32)
    return oracle_paged(f64(inp.q[idx]), f64(pc.k_pages[owned]), f64(pc.v_pages[owned]), sub,
                        f64(inp.k_blk[idx]), f64(inp.v_blk[idx]), inp.ctx_lens[idx], inp.k_ctx.shape[2])


CASES = {
    "gqa16-ragged": lambda: make_decode(3, 16, 32, 2, 128, 777, seed=31, ctx_lens=[0, 300, 777]),
    "page-boundaries": lambda: make_decode(4, 16, 16, 1, 128, 512, seed=32, ctx_lens=[256, 128, 257, 1]),
    "d64-g4": lambda: make_decode(2, 16, 8, 2, 64, 200, seed=33, ctx_lens=[129, 64]),
    "odd-block-S5-g3": lambda: make_decode(2, 5, 6, 2, 128, 150, seed=34, ctx_lens=[150, 17]),
    "S1-g16": lambda: make_decode(4, 1, 16, 1, 128, 513, seed=35, ctx_lens=[513, 0, 1, 255]),
}


@pytest.mark.parametrize("kernel", PAGED_KERNELS)
@pytest.mark.parametrize("page_size", [16, 32, 64, 128, 256])
@pytest.mark.parametrize("case", list(CASES))
def test_paged_small(case, page_size, kernel):
    inp = CASES[case]()
    pc = make_paged(inp, page_size, seed=page_size)
    out, lse = run_paged(inp, pc, kernel)
    ro, rl = oracle_of(inp, pc)
    assert_parity(out, ro, f"{case} P={page_size} out")
    assert_parity(lse, rl, f"{case} P={page_size} lse")


@pytest.mark.parametrize("kernel", PAGED_KERNELS)
@pytest.mark.parametrize("num_ctas", [1, 37, 300])
def test_paged_split_count_invariance(kernel, num_ctas):
    inp = make_decode(3, 16, 32, 2, 128, 1000, seed=36, ctx_lens=[1000, 517, 3])
    pc = make_paged(inp, 64, seed=5)
    out, lse = run_paged(inp, pc, kernel, num_ctas=num_ctas)
    ro, rl = oracle_of(inp, pc)
    assert_parity(out, ro, f"C={num_ctas} out")
    assert_parity(lse, rl, f"C={num_ctas} lse")


@pytest.fixture(scope="module")
def wl2_paged():
    inp = make_workload(2)
    pc = make_paged(inp, 64, seed=2)
    return inp, pc, oracle_of(inp, pc)


@pytest.mark.parametrize("kernel", KERNELS)
def test_paged_L4096_full(wl2_paged, kernel):
    """Decode B=8, Hq=32, Hkv=2, D=128, L=4096 (1% of keys x8) from 64-row pages: every output."""
    inp, pc, (ro, rl) = wl2_paged
    out, lse = run_paged(inp, pc, kernel)
    assert_parity(out, ro, "paged L4096 out")
    assert_parity(lse, rl, "paged L4096 lse")


@pytest.fixture(scope="module")
def wl3_paged():
    inp = make_workload(3)
    return inp, make_paged(inp, 16, seed=3)


@pytest.mark.parametrize("kernel", KERNELS)
def test_paged_ragged_B64_sampled(wl3_paged, kernel):
    """Ragged B=64 workload from 16-row pages; oracle on sampled sequences."""
    inp, pc = wl3_paged
    out, lse = run_paged(inp, pc, kernel)
    lens = inp.ctx_lens
    for n in sorted({int(np.argmin(lens)), int(np.argmax(lens)), 0, 33}):
        ro, rl = oracle_of(inp, pc, slice(n, n + 1))
        assert_parity(out[n:n + 1], ro, f"paged ragged n={n} out")
        assert_parity(lse[n:n + 1], rl, f"paged ragged n={n} lse")


@pytest.mark.parametrize("kernel", PAGED_KERNELS)
def test_paged_bad_page_is_flagged(kernel):
    """A table entry outside the pool reads as zeros and raises the device argument error."""
    inp = make_decode(2, 16, 8, 2, 128, 300, seed=37, ctx_lens=[300, 100])
    pc = make_paged(inp, 64, seed=7)
    num_pages = pc.k_pages.shape[0]
    pc.page_table[0, 1] = num_pages + 5
    pc.page_table[1, 0] = -3
    with pytest.raises(ops.TTError) as e:
        run_paged(inp, pc, kernel)
    assert e.value.status == ops.TT_ERR_DEVICE_ARG


def test_paged_host_checks():
    inp = make_decode(1, 16, 8, 2, 128, 64, seed=38)
    pc = make_paged(inp, 64, seed=8)
    plan = ops.Plan(1, 8, 2, 128, 16, ctx_capacity=0)
    args = dict(q=dev(inp.q), k_blk=dev(inp.k_blk), v_blk=dev(inp.v_blk),
                ctx_lens=torch.from_numpy(inp.ctx_lens).cuda())
    kp, vp = dev(pc.k_pages), dev(pc.v_pages)
    table = torch.from_numpy(pc.page_table).cuda()
    L = ops.lib()
    for P in (0, 8, 48, 1 << 17):   # not a power of two in [16, 65536]
        st = L.tt_block_attn_paged(plan._h, ops._ptr(args["q"]), ops._ptr(kp), ops._ptr(vp), ops._ptr(table),
                                   kp.shape[0], P, 1, ops._ptr(args["k_blk"]), ops._ptr(args["v_blk"]),
                                   ops._ptr(args["ctx_lens"]), ops._ptr(torch.empty(1, 16, 8, 128, device="cuda")),
                                   None, None)
        assert st == ops.TT_ERR_INVALID_ARG, P
    with pytest.raises(ops.TTError) as e:   # pages_per_seq > 0 without a table
        out = torch.empty(1, 16, 8, 128, device="cuda")
        st = L.tt_block_attn_paged(plan._h, ops._ptr(args["q"]), ops._ptr(kp), ops._ptr(vp), None, kp.shape[0],
                                   64, 1, ops._ptr(args["k_blk"]), ops._ptr(args["v_blk"]),
                                   ops._ptr(args["ctx_lens"]), ops._ptr(out), None, None)
        ops._check(st, "paged")
    assert e.value.status == ops.TT_ERR_INVALID_ARG

"""Pins of the block-causal backward oracle (CPU only): central finite differences of
the forward oracle, and torch float64 autograd through scaled_dot_product_attention
with the block-causal mask (an independent library routine)."""
import numpy as np
import pytest
import torch

from oracle import block_causal, block_causal_backward


def _case(seed, B=2, N=6, S=3, Hq=4, Hkv=2, D=5):
    rng = np.random.default_rng(seed)
    f = lambda *sh: rng.standard_normal(sh)
    return dict(q=f(B, N, Hq, D), k_ctx=f(B, Hkv, N, D), v_ctx=f(B, Hkv, N, D), k_blk=f(B, N, Hkv, D),
                v_blk=f(B, N, Hkv, D), dout=f(B, N, Hq, D), S=S)


def _loss(c, **over):
    a = dict(c)
    a.update(over)
    out, _ = block_causal(a["q"], a["k_ctx"], a["v_ctx"], a["k_blk"], a["v_blk"], a["S"])
    return float((out * c["dout"]).sum())


@pytest.mark.parametrize("name", ["q", "k_blk", "v_blk"])
def test_central_differences(name):
    c = _case(1)
    dq, dk, dv = block_causal_backward(c["q"], c["k_ctx"], c["v_ctx"], c["k_blk"], c["v_blk"], c["dout"], c["S"])
    grad = {"q": dq, "k_blk": dk, "v_blk": dv}[name]
    rng = np.random.default_rng(2)
    h = 1e-6
    for _ in range(12):
        idx = tuple(rng.integers(0, n) for n in c[name].shape)
        xp = c[name].copy(); xp[idx] += h
        xm = c[name].copy(); xm[idx] -= h
        fd = (_loss(c, **{name: xp}) - _loss(c, **{name: xm})) / (2 * h)
        assert abs(fd - grad[idx]) < 1e-6 * max(1.0, abs(fd)), (name, idx, fd, grad[idx])


def test_block_keys_are_seen_by_their_own_block_only():
    """Why dk_blk / dv_blk of block b sum over block b's rows alone: perturbing block b's
    own keys changes the output of block b's rows and of no other row."""
    c = _case(3)
    S = c["S"]
    out0, _ = block_causal(c["q"], c["k_ctx"], c["v_ctx"], c["k_blk"], c["v_blk"], S)
    kb = c["k_blk"].copy()
    kb[:, S:2 * S] += 0.5                      # block 1's own keys
    out1, _ = block_causal(c["q"], c["k_ctx"], c["v_ctx"], kb, c["v_blk"], S)
    changed = np.abs(out1 - out0).max(axis=(0, 2, 3)) > 0
    assert list(np.nonzero(changed)[0]) == list(range(S, 2 * S))


def test_matches_torch_autograd_through_sdpa_with_the_block_mask():
    c = _case(4, B=1, N=8, S=4, Hq=4, Hkv=2, D=6)
    B, N, Hq, D = c["q"].shape
    Hkv, S = c["k_ctx"].shape[1], c["S"]
    g = Hq // Hkv
    q = torch.tensor(c["q"], requires_grad=True)
    kb = torch.tensor(c["k_blk"], requires_grad=True)
    vb = torch.tensor(c["v_blk"], requires_grad=True)
    kc = torch.tensor(c["k_ctx"])
    vc = torch.tensor(c["v_ctx"])
    # keys: context positions 0..N-1 then block positions 0..N-1; query t of block b sees
    # context positions < S*b and block positions in [S*b, S*b + S)
    t = torch.arange(N)
    blk = t // S
    ctx_ok = torch.arange(N)[None, :] < (S * blk)[:, None]
    blk_ok = (torch.arange(N)[None, :] // S) == blk[:, None]
    mask = torch.cat([ctx_ok, blk_ok], dim=1)                      # [N, 2N]
    outs = []
    for j in range(Hq):
        h = j // g
        keys = torch.cat([kc[0, h], kb[0, :, h]], dim=0)
        vals = torch.cat([vc[0, h], vb[0, :, h]], dim=0)
        o = torch.nn.functional.scaled_dot_product_attention(q[0, :, j][None], keys[None], vals[None],
                                                            attn_mask=mask[None])
        outs.append(o[0])
    out = torch.stack(outs, dim=1)[None]                            # [1, N, Hq, D]
    (out * torch.tensor(c["dout"])).sum().backward()
    dq, dk, dv = block_causal_backward(c["q"], c["k_ctx"], c["v_ctx"], c["k_blk"], c["v_blk"], c["dout"], S)
    assert np.allclose(dq, q.grad.numpy(), atol=1e-12)
    assert np.allclose(dk, kb.grad.numpy(), atol=1e-12)
    assert np.allclose(dv, vb.grad.numpy(), atol=1e-12)

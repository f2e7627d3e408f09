"""The float64 oracle against facts outside itself (CPU only)."""
import math

import numpy as np
import pytest
import torch

from oracle import block_attn, block_causal
from oracle.brute import brute_block_causal
from tests import pins
from two_tower_block_b200.workloads import bf16_to_f64, make_decode


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_decode_pins(pin):
    pin(block_attn)


def _causal_case(seed, B=2, N=6, S=2, Hq=4, Hkv=2, D=3):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, N, Hq, D)), rng.standard_normal((B, Hkv, N, D)),
            rng.standard_normal((B, Hkv, N, D)), rng.standard_normal((B, N, Hkv, D)),
            rng.standard_normal((B, N, Hkv, D)), S)


def test_block_causal_vs_brute_predicate():
    for seed, kw in [(101, {}), (102, dict(B=1, N=8, S=4, Hq=2, Hkv=1, D=2)),
                     (103, dict(B=1, N=5, S=1, Hq=3, Hkv=1, D=4))]:
        case = _causal_case(seed, **kw)
        o, l = block_causal(*case)
        bo, bl = brute_block_causal(*case)
        pins._close(o, bo, 1e-12, "causal brute out")
        pins._close(l, bl, 1e-12, "causal brute lse")


def test_block_causal_vs_sdpa_mask():
    """torch SDPA over the [context ; block] key axis with the boolean mask the
    method implies: query position p of block b sees context c < S*b and block
    position u with u // S == b."""
    q, kc, vc, kb, vb, S = _causal_case(104, B=2, N=12, S=4, Hq=4, Hkv=2, D=8)
    B, N, Hq, D = q.shape
    g = 2
    o, l = block_causal(q, kc, vc, kb, vb, S)
    p = np.arange(N)
    ctx_vis = np.arange(N)[None, :] < (S * (p // S))[:, None]
    blk_vis = (np.arange(N)[None, :] // S) == (p // S)[:, None]
    mask = torch.from_numpy(np.concatenate([ctx_vis, blk_vis], axis=1))
    for n in range(B):
        K = torch.cat([torch.from_numpy(kc[n]), torch.from_numpy(kb[n].transpose(1, 0, 2))], 1)
        V = torch.cat([torch.from_numpy(vc[n]), torch.from_numpy(vb[n].transpose(1, 0, 2))], 1)
        K = K.repeat_interleave(g, 0)
        V = V.repeat_interleave(g, 0)
        Q = torch.from_numpy(np.ascontiguousarray(q[n].transpose(1, 0, 2)))
        ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=mask)
        pins._close(o[n], ref.permute(1, 0, 2).numpy(), 1e-12, "causal sdpa")
        s = (Q @ K.transpose(1, 2)) / math.sqrt(D)
        s = s.masked_fill(~mask, -math.inf)
        pins._close(l[n], torch.logsumexp(s, -1).numpy(), 1e-12, "causal lse")


def test_block_causal_first_block_is_self_attention():
    q, kc, vc, kb, vb, S = _causal_case(105, B=1, N=4, S=2, Hq=2, Hkv=1, D=3)
    kc[:] = np.nan   # block 0 reads no context at all
    vc[:] = np.nan
    o, _ = block_causal(q, kc, vc, kb, vb, S, blocks=[0])
    Q = torch.from_numpy(np.ascontiguousarray(q[0, :2].transpose(1, 0, 2)))
    K = torch.from_numpy(np.ascontiguousarray(kb[0, :2].transpose(1, 0, 2))).repeat_interleave(2, 0)
    V = torch.from_numpy(np.ascontiguousarray(vb[0, :2].transpose(1, 0, 2))).repeat_interleave(2, 0)
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V).permute(1, 0, 2).numpy()
    pins._close(o[0, :2], ref, 1e-12, "first block")


def test_block_causal_rejects_ragged_length():
    q, kc, vc, kb, vb, _ = _causal_case(106, N=6)
    with pytest.raises(ValueError):
        block_causal(q, kc, vc, kb, vb, 4)


def test_rejects_bad_ctx_len():
    case = list(pins.rand_case(107, Lcap=4))
    case[5] = np.array([5, 1])
    with pytest.raises(ValueError):
        block_attn(*case)


def test_lse_matches_scipy_logsumexp():
    from scipy.special import logsumexp
    q, kc, vc, kb, vb, lens = pins.rand_case(108, B=1, S=2, Hq=2, Hkv=1, D=4, Lcap=5, lens=[5])
    _, l = block_attn(q, kc, vc, kb, vb, lens)
    for j in range(2):
        for t in range(2):
            keys = np.concatenate([kc[0, 0], kb[0, :, 0]])
            s = [float(q[0, t, j] @ k) / 2.0 for k in keys]
            assert abs(l[0, j, t] - logsumexp(s)) < 1e-12


def test_golden_closed_form_fixture():
    """tests/golden/closed_form_d4.txt: a hand-derived problem (weights 1:2:4:1 by
    construction) whose exact output is written in the file."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "closed_form_d4.txt")
    sec = {}
    cur = None
    for line in open(path):
        line = line.split("#", 1)[0].strip()
        if not line:
            continue
        if line.startswith("["):
            cur = line.strip("[]")
            sec[cur] = []
        else:
            sec[cur].append([float(x) for x in line.split()])
    q = np.array(sec["q"]).reshape(1, 1, 1, 4)
    kc = np.array(sec["k_ctx"]).reshape(1, 1, -1, 4)
    vc = np.array(sec["v_ctx"]).reshape(1, 1, -1, 4)
    kb = np.array(sec["k_blk"]).reshape(1, 1, 1, 4)
    vb = np.array(sec["v_blk"]).reshape(1, 1, 1, 4)
    L = int(sec["ctx_len"][0][0])
    scale = sec["scale"][0][0]
    o, l = block_attn(q, kc, vc, kb, vb, np.array([L]), scale=scale)
    pins._close(o[0, 0, 0], np.array(sec["out"][0]), 1e-13, "golden out")
    pins._close(l[0, 0, 0], sec["lse"][0][0], 1e-13, "golden lse")


def test_bf16_inputs_are_exact_upcasts():
    """The oracle consumes the exact bf16 values: every upcast value has at most
    8 significant bits and the draw is reproducible from the seed."""
    a = make_decode(1, 4, 2, 1, 8, 16, seed=5)
    b = make_decode(1, 4, 2, 1, 8, 16, seed=5)
    assert np.array_equal(a.q, b.q) and np.array_equal(a.k_ctx, b.k_ctx)
    x = bf16_to_f64(a.k_ctx)
    m, _ = np.frexp(x)
    assert np.all((m * 256) == np.round(m * 256))

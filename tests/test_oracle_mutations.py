"""Plant plausible mistakes in a copy of the oracle (CPU only) and require the pins
to catch every one.  This shows the pins in tests/pins.py constrain each part of
the definition: the key set, the GQA mapping, the scale, the single joint
softmax, the bidirectional block, and the log-sum-exp."""
import math

import numpy as np
import pytest

from tests import pins


def mutant_attn(mut):
    def attn(q, k_ctx, v_ctx, k_blk, v_blk, ctx_lens, scale=None):
        B, S, Hq, D = q.shape
        Hkv = k_ctx.shape[1]
        g = Hq // Hkv
        if scale is None:
            scale = 1.0 / math.sqrt(D) if mut != "scale_1_over_D" else 1.0 / D
        if mut == "no_scale":
            scale = 1.0
        out = np.empty((B, S, Hq, D))
        lse = np.empty((B, Hq, S))
        for n in range(B):
            L = int(ctx_lens[n])
            if mut == "len_plus_one":
                L = min(L + 1, k_ctx.shape[2])
            if mut == "len_minus_one":
                L = max(L - 1, 0)
            for j in range(Hq):
                h = j % Hkv if mut == "gqa_modulo" else j // g
                kc, vc = k_ctx[n, h, :L], v_ctx[n, h, :L]
                kb, vb = k_blk[n, :, h], v_blk[n, :, h]
                if mut == "drop_block":
                    keys, vals = kc, vc
                elif mut == "drop_ctx":
                    keys, vals = kb, vb
                elif mut == "values_from_keys":
                    keys, vals = np.concatenate([kc, kb]), np.concatenate([kc, kb])
                else:
                    keys, vals = np.concatenate([kc, kb]), np.concatenate([vc, vb])
                qr = q[n, :, j]
                s = scale * qr @ keys.T
                if mut == "causal_in_block":
                    s[:, L:] = np.where(np.tril(np.ones((S, S), bool)), s[:, L:], -np.inf)
                if mut == "negated_scores":
                    s = -s
                if mut == "two_softmaxes" and L > 0:
                    def sm(x, v):
                        e = np.exp(x - x.max(1, keepdims=True))
                        return (e @ v) / e.sum(1, keepdims=True)
                    o = 0.5 * (sm(s[:, :L], vc) + sm(s[:, L:], vb))
                    m = s.max(1)
                    lse_row = m + np.log(np.exp(s - m[:, None]).sum(1))
                else:
                    m = s.max(1, keepdims=True)
                    e = np.exp(s - m)
                    z = e.sum(1, keepdims=True)
                    o = (e @ vals) / z
                    if mut == "unnormalised":
                        o = e @ vals
                    lse_row = m[:, 0] + np.log(z[:, 0])
                    if mut == "lse_log2":
                        lse_row = (m[:, 0] + np.log(z[:, 0])) / math.log(2.0)
                    if mut == "lse_drop_max":
                        lse_row = np.log(z[:, 0])
                out[n, :, j] = o
                lse[n, j] = lse_row
        return out, lse
    return attn


MUTANTS = ["scale_1_over_D", "no_scale", "len_plus_one", "len_minus_one", "gqa_modulo",
           "drop_block", "drop_ctx", "values_from_keys", "causal_in_block", "negated_scores",
           "two_softmaxes", "unnormalised", "lse_log2", "lse_drop_max"]


def test_unmutated_copy_passes():
    attn = mutant_attn(None)
    for pin in pins.ALL_PINS:
        pin(attn)


@pytest.mark.parametrize("mut", MUTANTS)
def test_mutant_is_caught(mut):
    attn = mutant_attn(mut)
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(attn)
        except (AssertionError, ValueError, IndexError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"mutant {mut} passed every pin"

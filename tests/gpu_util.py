"""Helpers shared by the GPU tests: device copies of the seeded bf16 inputs,
NaN poisoning of unread cache rows, and the parity metric of the method's
tolerance (max-abs <= 1e-2 and relative L2 <= 5e-3 against the float64
oracle, bf16 inputs and fp32 accumulation)."""
from __future__ import annotations

import numpy as np
import torch

from two_tower_block_b200.workloads import bf16_to_f64

MAX_ABS = 1e-2
REL_L2 = 5e-3
BF16_NAN = 0x7FC0


def dev(bits: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bf16 bit patterns -> torch bf16 tensor on the GPU."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).to(device)


def poison_beyond(k_ctx_bits: np.ndarray, lens) -> np.ndarray:
    """Copy of a [B, Hkv, Lcap, D] cache with every row at or beyond L_n set to NaN."""
    k = k_ctx_bits.copy()
    for n, L in enumerate(lens):
        k[n, :, int(L):, :] = BF16_NAN
    return k


def errors(gpu: torch.Tensor, ref: np.ndarray):
    g = gpu.detach().double().cpu().numpy()
    d = g - ref
    max_abs = float(np.max(np.abs(d))) if d.size else 0.0
    rel = float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-30)) if d.size else 0.0
    return max_abs, rel, bool(np.all(np.isfinite(g)))


def assert_parity(gpu, ref, what="", max_abs=MAX_ABS, rel_l2=REL_L2):
    ma, rl, finite = errors(gpu, ref)
    assert finite, f"{what}: non-finite values in GPU output"
    assert ma <= max_abs and rl <= rel_l2, f"{what}: max_abs {ma:.3e} rel_l2 {rl:.3e}"
    return ma, rl


def f64(bits):
    return bf16_to_f64(bits)

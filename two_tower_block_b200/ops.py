"""ctypes binding of libtt_block_attn.so (argument marshalling only).

Every entry point here forwards to the C function of the same name in
``include/tt_block_attn.h``.  torch supplies device memory and streams; all
computation happens in the library's CUDA kernels.  If the library is
missing, or a call is made without a CUDA device, the call raises: there is
no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

__all__ = ["TTError", "Plan", "lib", "library_path", "block_attn", "block_attn_block_causal", "confidence_unmask",
           "selftest_wait_timeout", "work_split", "KERNEL_AUTO", "KERNEL_TCGEN05", "KERNEL_MMA_SYNC",
           "TT_OK", "TT_ERR_INVALID_ARG", "TT_ERR_UNSUPPORTED", "TT_ERR_CUDA", "TT_ERR_DEVICE_ARG",
           "TT_ERR_TIMEOUT", "EXPORTED_SYMBOLS"]

TT_OK, TT_ERR_INVALID_ARG, TT_ERR_UNSUPPORTED, TT_ERR_CUDA, TT_ERR_DEVICE_ARG, TT_ERR_TIMEOUT = range(6)
KERNEL_AUTO, KERNEL_TCGEN05, KERNEL_MMA_SYNC = 0, 1, 2
PLAN_HOST_IO = 1
PLAN_OUT_BF16 = 2

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libtt_block_attn.so")

# Every symbol the header declares (checked by the CPU test suite).
EXPORTED_SYMBOLS = [
    "tt_block_attn_plan", "tt_block_attn_plan_destroy", "tt_block_attn_plan_get_info", "tt_block_attn",
    "tt_block_attn_block_causal", "tt_block_attn_host", "tt_block_attn_check", "tt_block_attn_profile",
    "tt_block_attn_profile_read", "tt_selftest_wait_timeout", "tt_debug_work_split", "tt_status_string",
    "tt_last_error_detail", "tt_block_attn_noalloc", "tt_selftest_exp2", "tt_kv_append",
    "tt_block_attn_block_causal_backward", "tt_confidence_unmask", "tt_block_attn_paged",
    "tt_debug_causal_split",
]


class Desc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("num_q_heads", ctypes.c_int), ("num_kv_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("block_size", ctypes.c_int), ("ctx_capacity", ctypes.c_int),
                ("seq_len", ctypes.c_int), ("scale", ctypes.c_float), ("kernel", ctypes.c_int),
                ("num_ctas", ctypes.c_int), ("flags", ctypes.c_int), ("wait_timeout_us", ctypes.c_int)]


class PlanInfo(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_int), ("num_ctas", ctypes.c_int), ("key_tile", ctypes.c_int),
                ("rows_per_unit", ctypes.c_int), ("workspace_bytes", ctypes.c_size_t),
                ("sm_count", ctypes.c_int), ("variant", ctypes.c_int), ("fused_combine", ctypes.c_int)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load the library once; raise (never fall back) if it is absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(library_path):
        raise RuntimeError(f"{library_path} is missing: build it with `python -m two_tower_block_b200.build`")
    L = ctypes.CDLL(library_path)
    vp, ip, i, f = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int), ctypes.c_int, ctypes.c_float
    L.tt_block_attn_plan.argtypes = [ctypes.POINTER(Desc), i, ctypes.POINTER(vp)]
    L.tt_block_attn_plan_destroy.argtypes = [vp]
    L.tt_block_attn_plan_destroy.restype = None
    L.tt_block_attn_plan_get_info.argtypes = [vp, ctypes.POINTER(PlanInfo)]
    L.tt_block_attn.argtypes = [vp] * 10
    L.tt_block_attn_block_causal.argtypes = [vp] * 9
    L.tt_block_attn_paged.argtypes = [vp, vp, vp, vp, vp, i, i, i, vp, vp, vp, vp, vp, vp]
    L.tt_block_attn_host.argtypes = [vp] * 10
    L.tt_block_attn_check.argtypes = [vp, vp]
    L.tt_block_attn_profile.argtypes = [vp, i]
    L.tt_block_attn_profile_read.argtypes = [vp, i, ip, ctypes.POINTER(ctypes.c_double)]
    L.tt_selftest_wait_timeout.argtypes = [i, i, vp]
    L.tt_debug_work_split.argtypes = [i, ip, i, ctypes.POINTER(ctypes.c_longlong), ip, ip]
    L.tt_debug_causal_split.argtypes = [i, i, i, i, i, i, i, ctypes.POINTER(ctypes.c_longlong)]
    L.tt_block_attn_noalloc.argtypes = [ctypes.POINTER(Desc)] + [vp] * 10
    L.tt_selftest_exp2.argtypes = [i, vp, vp, i]
    L.tt_status_string.argtypes = [i]
    L.tt_status_string.restype = ctypes.c_char_p
    L.tt_last_error_detail.argtypes = []
    L.tt_last_error_detail.restype = ctypes.c_char_p
    for name in EXPORTED_SYMBOLS:
        if name not in ("tt_block_attn_plan_destroy", "tt_status_string", "tt_last_error_detail"):
            getattr(L, name).restype = ctypes.c_int
    _lib = L
    return L


class TTError(RuntimeError):
    def __init__(self, status: int, where: str):
        L = lib()
        self.status = status
        msg = L.tt_status_string(status).decode()
        detail = L.tt_last_error_detail().decode()
        super().__init__(f"{where}: {msg}" + (f" ({detail})" if detail else ""))


def _check(status: int, where: str):
    if status != TT_OK:
        raise TTError(status, where)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
        return ctypes.c_void_p(t.data_ptr())
    return ctypes.c_void_p(int(t))


def _arg(t, name, numel, kind, device):
    """Check one tensor argument before its address reaches the library, whose kernels
    trust every size: ``kind`` "bf16" (any 2-byte type: bf16 values or their bit
    patterns), "f32", "i32", "w32" (any 4-byte integer) or "u8" (any 1-byte type); ``numel`` the element count the
    layout needs; ``device`` a CUDA ordinal, "host", or None (not checked).  None and raw integer addresses
    are passed through (the library rejects a null pointer it needs)."""
    if not isinstance(t, torch.Tensor):
        return
    ok = {"bf16": t.element_size() == 2 and not t.is_floating_point() or t.dtype == torch.bfloat16,
          "f32": t.dtype == torch.float32, "i32": t.dtype == torch.int32,
          "w32": t.element_size() == 4 and not t.is_floating_point(),
          "u8": t.element_size() == 1}[kind]
    if not ok:
        raise TypeError(f"{name}: dtype {t.dtype} where {kind} is expected")
    if t.numel() != numel:
        raise ValueError(f"{name}: {t.numel()} elements where the plan's shape needs {numel}")
    if device == "host":
        if t.is_cuda:
            raise ValueError(f"{name}: a host tensor is expected")
    elif device is not None and (not t.is_cuda or t.device.index != device):
        raise ValueError(f"{name}: expected on cuda:{device}, got {t.device}")


def _args(device, *items):
    """_arg over (tensor, name, numel, kind) items: every dtype and size first, then
    every device, so a wrong shape is reported before where a tensor lives."""
    for t, name, numel, kind in items:
        _arg(t, name, numel, kind, None)
    for t, name, numel, kind in items:
        _arg(t, name, numel, kind, device)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


@dataclass
class Shape:
    batch: int
    q_heads: int
    kv_heads: int
    head_dim: int
    block: int
    ctx_capacity: int = 0
    seq_len: int = 0


class Plan:
    """Owns a tt_plan_t (device scratch, work split) for one shape on one device."""

    out_dtype = torch.float32   # torch.bfloat16 for a plan made with out_bf16=True

    def __init__(self, batch, q_heads, kv_heads, head_dim, block, ctx_capacity=0, seq_len=0, scale=0.0,
                 kernel=KERNEL_AUTO, num_ctas=0, host_io=False, wait_timeout_us=0, device=None, out_bf16=False):
        if device is None:
            device = torch.cuda.current_device()
        self.shape = Shape(batch, q_heads, kv_heads, head_dim, block, ctx_capacity, seq_len)
        self.device = int(device)
        self.out_dtype = torch.bfloat16 if out_bf16 else torch.float32
        d = Desc(batch, q_heads, kv_heads, head_dim, block, ctx_capacity, seq_len, float(scale), kernel,
                 num_ctas, (PLAN_HOST_IO if host_io else 0) | (PLAN_OUT_BF16 if out_bf16 else 0), wait_timeout_us)
        h = ctypes.c_void_p()
        _check(lib().tt_block_attn_plan(ctypes.byref(d), self.device, ctypes.byref(h)), "tt_block_attn_plan")
        self._h = h

    def close(self):
        if getattr(self, "_h", None):
            lib().tt_block_attn_plan_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def info(self) -> PlanInfo:
        inf = PlanInfo()
        _check(lib().tt_block_attn_plan_get_info(self._h, ctypes.byref(inf)), "tt_block_attn_plan_get_info")
        return inf

    # --- decode ------------------------------------------------------------
    def block_attn(self, q, k_ctx, v_ctx, k_blk, v_blk, ctx_lens, out=None, lse=None, stream=None,
                   want_lse=False):
        s = self.shape
        if out is None:
            out = torch.empty((s.batch, s.block, s.q_heads, s.head_dim), dtype=self.out_dtype, device=q.device)
        if lse is None and want_lse:
            lse = torch.empty((s.batch, s.q_heads, s.block), dtype=torch.float32, device=q.device)
        nc = s.batch * s.kv_heads * s.ctx_capacity * s.head_dim
        _args(self.device, *self._decode_items(q, k_blk, v_blk, ctx_lens, out, lse),
              (k_ctx, "k_ctx", nc, "bf16"), (v_ctx, "v_ctx", nc, "bf16"))
        _check(lib().tt_block_attn(self._h, _ptr(q), _ptr(k_ctx), _ptr(v_ctx), _ptr(k_blk), _ptr(v_blk),
                                   _ptr(ctx_lens), _ptr(out), _ptr(lse), _stream(stream)), "tt_block_attn")
        return (out, lse) if want_lse or lse is not None else out

    def _decode_items(self, q, k_blk, v_blk, ctx_lens, out, lse):
        s = self.shape
        nq = s.batch * s.block * s.q_heads * s.head_dim
        nb = s.batch * s.block * s.kv_heads * s.head_dim
        return [(q, "q", nq, "bf16"), (k_blk, "k_blk", nb, "bf16"), (v_blk, "v_blk", nb, "bf16"),
                (ctx_lens, "ctx_lens", s.batch, "i32"), (out, "out", nq, self._out_kind()),
                (lse, "lse", s.batch * s.q_heads * s.block, "f32")]

    def _out_kind(self):
        return "bf16" if self.out_dtype == torch.bfloat16 else "f32"

    def block_attn_paged(self, q, k_pages, v_pages, page_table, k_blk, v_blk, ctx_lens, out=None, lse=None,
                         stream=None, want_lse=False):
        """Decode over a paged context cache: k_pages / v_pages [num_pages, Hkv, P, D] bf16
        pools, page_table [B, pages_per_seq] int32 (device); P = k_pages.shape[2].  With no
        context at all, the pools and the table may be None."""
        s = self.shape
        if out is None:
            out = torch.empty((s.batch, s.block, s.q_heads, s.head_dim), dtype=self.out_dtype, device=q.device)
        if lse is None and want_lse:
            lse = torch.empty((s.batch, s.q_heads, s.block), dtype=torch.float32, device=q.device)
        if k_pages is None:
            num_pages, page_size = 0, 16      # no pool: valid only without context (the library checks)
        else:
            if k_pages.dim() != 4 or k_pages.shape[1] != s.kv_heads or k_pages.shape[3] != s.head_dim:
                raise ValueError(f"k_pages: shape {tuple(k_pages.shape)}, expected [num_pages, {s.kv_heads}, P, "
                                 f"{s.head_dim}]")
            num_pages, _, page_size, _ = k_pages.shape
        pool_numel = k_pages.numel() if k_pages is not None else 0
        pages_per_seq = 0
        if page_table is not None:
            if page_table.dim() != 2 or page_table.shape[0] != s.batch:
                raise ValueError(f"page_table: shape {tuple(page_table.shape)}, expected [{s.batch}, pages_per_seq]")
            pages_per_seq = page_table.shape[1]
        _args(self.device, *self._decode_items(q, k_blk, v_blk, ctx_lens, out, lse),
              (k_pages, "k_pages", pool_numel, "bf16"), (v_pages, "v_pages", pool_numel, "bf16"),
              (page_table, "page_table", s.batch * pages_per_seq, "i32"))
        _check(lib().tt_block_attn_paged(self._h, _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(page_table),
                                         int(num_pages), int(page_size), int(pages_per_seq), _ptr(k_blk),
                                         _ptr(v_blk), _ptr(ctx_lens), _ptr(out), _ptr(lse), _stream(stream)),
               "tt_block_attn_paged")
        return (out, lse) if want_lse or lse is not None else out

    def block_attn_host(self, q, k_ctx, v_ctx, k_blk, v_blk, ctx_lens, out, lse=None, stream=None):
        """Host (ideally pinned) CPU tensors in and out; copies happen inside the library."""
        s = self.shape
        nc = s.batch * s.kv_heads * s.ctx_capacity * s.head_dim
        _args("host", *self._decode_items(q, k_blk, v_blk, ctx_lens, out, lse),
              (k_ctx, "k_ctx", nc, "bf16"), (v_ctx, "v_ctx", nc, "bf16"))
        _check(lib().tt_block_attn_host(self._h, _ptr(q), _ptr(k_ctx), _ptr(v_ctx), _ptr(k_blk), _ptr(v_blk),
                                        _ptr(ctx_lens), _ptr(out), _ptr(lse), _stream(stream)),
               "tt_block_attn_host")
        return out

    # --- block-causal ------------------------------------------------------
    def block_attn_block_causal(self, q, k_ctx, v_ctx, k_blk, v_blk, out=None, lse=None, stream=None,
                                want_lse=False):
        s = self.shape
        if out is None:
            out = torch.empty((s.batch, s.seq_len, s.q_heads, s.head_dim), dtype=self.out_dtype, device=q.device)
        if lse is None and want_lse:
            lse = torch.empty((s.batch, s.q_heads, s.seq_len), dtype=torch.float32, device=q.device)
        _args(self.device, *self._causal_items(q, k_ctx, v_ctx, k_blk, v_blk, out, lse, self._out_kind()))
        _check(lib().tt_block_attn_block_causal(self._h, _ptr(q), _ptr(k_ctx), _ptr(v_ctx), _ptr(k_blk),
                                                _ptr(v_blk), _ptr(out), _ptr(lse), _stream(stream)),
               "tt_block_attn_block_causal")
        return (out, lse) if want_lse or lse is not None else out

    def _causal_items(self, q, k_ctx, v_ctx, k_blk, v_blk, out, lse, out_kind="f32"):
        s = self.shape
        nq = s.batch * s.seq_len * s.q_heads * s.head_dim
        nk = s.batch * s.seq_len * s.kv_heads * s.head_dim
        return [(q, "q", nq, "bf16"), (k_ctx, "k_ctx", nk, "bf16"), (v_ctx, "v_ctx", nk, "bf16"),
                (k_blk, "k_blk", nk, "bf16"), (v_blk, "v_blk", nk, "bf16"), (out, "out", nq, out_kind),
                (lse, "lse", s.batch * s.q_heads * s.seq_len, "f32")]

    def block_causal_backward(self, q, k_ctx, v_ctx, k_blk, v_blk, out, lse, dout, dq=None, dk_blk=None,
                              dv_blk=None, stream=None):
        """Gradients (dq, dk_blk, dv_blk) of sum(dout * out) for the block-causal attention;
        out and lse are the forward's outputs (fp32), dout is bf16."""
        s = self.shape
        if dq is None:
            dq = torch.empty((s.batch, s.seq_len, s.q_heads, s.head_dim), dtype=torch.float32, device=q.device)
        if dk_blk is None:
            dk_blk = torch.empty((s.batch, s.seq_len, s.kv_heads, s.head_dim), dtype=torch.float32,
                                 device=q.device)
        if dv_blk is None:
            dv_blk = torch.empty_like(dk_blk)
        nq = s.batch * s.seq_len * s.q_heads * s.head_dim
        nk = s.batch * s.seq_len * s.kv_heads * s.head_dim
        _args(self.device, *self._causal_items(q, k_ctx, v_ctx, k_blk, v_blk, out, lse),
              (dout, "dout", nq, "bf16"), (dq, "dq", nq, "f32"), (dk_blk, "dk_blk", nk, "f32"),
              (dv_blk, "dv_blk", nk, "f32"))
        _check(lib().tt_block_attn_block_causal_backward(
            self._h, _ptr(q), _ptr(k_ctx), _ptr(v_ctx), _ptr(k_blk), _ptr(v_blk), _ptr(out), _ptr(lse), _ptr(dout),
            _ptr(dq), _ptr(dk_blk), _ptr(dv_blk), _stream(stream)), "tt_block_attn_block_causal_backward")
        return dq, dk_blk, dv_blk

    # --- committed-block cache update ------------------------------------------
    def kv_append(self, k_new, v_new, k_ctx, v_ctx, ctx_lens, advance=True, stream=None):
        """Write k_new/v_new [B,S,Hkv,D] into k_ctx/v_ctx [B,Hkv,Lcap,D] at [L_n, L_n+S) in
        place; advance ctx_lens (device int32) by S when `advance`."""
        s = self.shape
        nb = s.batch * s.block * s.kv_heads * s.head_dim
        nc = s.batch * s.kv_heads * s.ctx_capacity * s.head_dim
        _args(self.device, (k_new, "k_new", nb, "bf16"), (v_new, "v_new", nb, "bf16"), (k_ctx, "k_ctx", nc, "bf16"),
              (v_ctx, "v_ctx", nc, "bf16"), (ctx_lens, "ctx_lens", s.batch, "i32"))
        _check(lib().tt_kv_append(self._h, _ptr(k_new), _ptr(v_new), _ptr(k_ctx), _ptr(v_ctx), _ptr(ctx_lens),
                                  int(bool(advance)), _stream(stream)), "tt_kv_append")

    # --- status / timing ---------------------------------------------------
    def check(self, stream=None):
        """Synchronise and read the device error word; raise TTError on a device-side error."""
        _check(lib().tt_block_attn_check(self._h, _stream(stream)), "tt_block_attn_check")

    def check_status(self, stream=None) -> int:
        return lib().tt_block_attn_check(self._h, _stream(stream))

    def profile(self, enable: bool):
        _check(lib().tt_block_attn_profile(self._h, int(enable)), "tt_block_attn_profile")

    def profile_read(self, kernel_id: int):
        n = ctypes.c_int()
        ms = ctypes.c_double()
        _check(lib().tt_block_attn_profile_read(self._h, kernel_id, ctypes.byref(n), ctypes.byref(ms)),
               "tt_block_attn_profile_read")
        return n.value, ms.value


def confidence_unmask(logits, tokens, masked, gamma=0.8, min_one=True, stream=None):
    """One unmasking step on CUDA tensors: logits [B,S,V] bf16, tokens [B,S] int32 and
    masked [B,S] uint8 (updated in place).  Returns (p_max [B,S] fp32, argmax [B,S] int32,
    n_committed [B] int32)."""
    B, S, V = logits.shape
    dev = logits.device.index if logits.device.index is not None else torch.cuda.current_device()
    _args(dev, (logits, "logits", B * S * V, "bf16"), (tokens, "tokens", B * S, "i32"),
          (masked, "masked", B * S, "u8"))
    p_max = torch.empty((B, S), dtype=torch.float32, device=logits.device)
    arg = torch.empty((B, S), dtype=torch.int32, device=logits.device)
    n_c = torch.empty((B,), dtype=torch.int32, device=logits.device)
    lib().tt_confidence_unmask.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                                           ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    _check(lib().tt_confidence_unmask(_ptr(logits), B, S, V, float(gamma), int(bool(min_one)), _ptr(tokens),
                                      _ptr(masked), _ptr(p_max), _ptr(arg), _ptr(n_c), _stream(stream)),
           "tt_confidence_unmask")
    return p_max, arg, n_c


_plans = {}


def _cached_plan(key, **kw):
    p = _plans.get(key)
    if p is None:
        p = Plan(**kw)
        _plans[key] = p
    return p


def block_attn(q, k_ctx, v_ctx, k_blk, v_blk, ctx_lens, scale=0.0, kernel=KERNEL_AUTO, want_lse=False):
    """Decode block attention on torch CUDA tensors (shapes as in the C header)."""
    B, S, Hq, D = q.shape
    Hkv, Lcap = k_ctx.shape[1], k_ctx.shape[2]
    dev = q.device.index if q.device.index is not None else torch.cuda.current_device()
    key = ("dec", B, S, Hq, Hkv, D, Lcap, float(scale), kernel, dev)
    plan = _cached_plan(key, batch=B, q_heads=Hq, kv_heads=Hkv, head_dim=D, block=S, ctx_capacity=Lcap,
                        scale=scale, kernel=kernel, device=dev)
    return plan.block_attn(q, k_ctx, v_ctx, k_blk, v_blk, ctx_lens, want_lse=want_lse)


def block_attn_block_causal(q, k_ctx, v_ctx, k_blk, v_blk, block_size, scale=0.0, kernel=KERNEL_AUTO,
                            want_lse=False):
    B, N, Hq, D = q.shape
    Hkv = k_ctx.shape[1]
    dev = q.device.index if q.device.index is not None else torch.cuda.current_device()
    key = ("bc", B, N, block_size, Hq, Hkv, D, float(scale), kernel, dev)
    plan = _cached_plan(key, batch=B, q_heads=Hq, kv_heads=Hkv, head_dim=D, block=block_size, seq_len=N,
                        scale=scale, kernel=kernel, device=dev)
    return plan.block_attn_block_causal(q, k_ctx, v_ctx, k_blk, v_blk, want_lse=want_lse)


def selftest_wait_timeout(device=0, timeout_us=20000, stream=None) -> int:
    return lib().tt_selftest_wait_timeout(int(device), int(timeout_us), _stream(stream))


def selftest_exp2(x, device=0):
    """The softmax's FMA-pipe exp2 evaluated on the device for float32 values x."""
    import numpy as np
    x = np.ascontiguousarray(x, dtype=np.float32)
    y = np.empty_like(x)
    _check(lib().tt_selftest_exp2(int(device), x.ctypes.data, y.ctypes.data, x.size), "tt_selftest_exp2")
    return y


def work_split(tiles_per_unit, num_ctas):
    """Host-only: the library's range split for the given per-unit tile counts."""
    n = len(tiles_per_unit)
    tiles = (ctypes.c_int * max(n, 1))(*tiles_per_unit)
    starts = (ctypes.c_longlong * (num_ctas + 1))()
    first = (ctypes.c_int * max(n, 1))()
    last = (ctypes.c_int * max(n, 1))()
    _check(lib().tt_debug_work_split(n, tiles, num_ctas, starts, first, last), "tt_debug_work_split")
    return list(starts), list(first)[:n], list(last)[:n]


def causal_split(batch, num_kv_heads, seq_len, block_size, key_tile, num_ctas, unit_cost=-1):
    """Host-only: the range boundaries of a block-causal call on the default tcgen05 kernel
    (unit_cost -1: the library's default fixed cost per unit; 0: the even split)."""
    starts = (ctypes.c_longlong * (num_ctas + 1))()
    _check(lib().tt_debug_causal_split(batch, num_kv_heads, seq_len, block_size, key_tile, num_ctas, unit_cost,
                                       starts), "tt_debug_causal_split")
    return list(starts)


def block_attn_noalloc(q, k_ctx, v_ctx, k_blk, v_blk, ctx_lens, out, lse=None, status=None, scale=0.0,
                       kernel=KERNEL_AUTO, num_ctas=0, stream=None):
    """Decode through tt_block_attn_noalloc: no plan, no device allocation inside the
    library (its scratch is a fixed 40 MiB device array).  Outputs are caller-owned;
    `status` is an optional one-element uint32/int32 device tensor for the error bits."""
    B, S, Hq, D = q.shape
    Hkv, Lcap = k_ctx.shape[1], k_ctx.shape[2]
    dev = q.device.index if q.device.index is not None else torch.cuda.current_device()
    _args(dev, (q, "q", B * S * Hq * D, "bf16"), (k_ctx, "k_ctx", B * Hkv * Lcap * D, "bf16"),
          (v_ctx, "v_ctx", B * Hkv * Lcap * D, "bf16"), (k_blk, "k_blk", B * S * Hkv * D, "bf16"),
          (v_blk, "v_blk", B * S * Hkv * D, "bf16"), (ctx_lens, "ctx_lens", B, "i32"),
          (out, "out", B * S * Hq * D, "f32"), (lse, "lse", B * Hq * S, "f32"), (status, "status", 1, "w32"))
    d = Desc(B, Hq, Hkv, D, S, Lcap, 0, float(scale), kernel, num_ctas, 0, 0)
    return lib().tt_block_attn_noalloc(ctypes.byref(d), _ptr(q), _ptr(k_ctx), _ptr(v_ctx), _ptr(k_blk),
                                       _ptr(v_blk), _ptr(ctx_lens), _ptr(out), _ptr(lse), _ptr(status),
                                       _stream(stream))

"""WavePrune causal attention for NVIDIA B200 (sm_100a).

Thin ctypes binding of ``libwaveprune.so`` (C ABI in ``include/waveprune.h``).
Every function here only marshals arguments: tensors must already be
contiguous, correctly typed and on the GPU; all arithmetic runs in the
library's CUDA kernels (or, for the cutoff tables and tile schedule, in the
library's host code). PyTorch supplies device memory and the current stream.
There is no fallback: if the library is missing, importing a function raises.

WavePrune (arXiv:2610.06963; reading notes "WavePrune：RoPE 通常只需一个旋转
周期", §2.1 Eq. (6) and §2.3 Eq. (8)) keeps RoPE channel c's contribution to
the logit of pair (i, j) only while i - j <= floor(2*pi/f_c); a dropped
channel adds 0 and the pair stays in the softmax.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

__all__ = [
    "ROPE_INTERLEAVED", "ROPE_HALF_SPLIT", "ROPE_HALF_SPLIT_PAIRED", "MODE_GROUPED", "MODE_CHANNEL", "CUTOFF_INF",
    "WavePruneError", "library_path", "load_library",
    "wp_cutoffs", "wp_schedule", "wp_rope_apply", "wp_prefill", "wp_prefill_backward", "wp_decode",
    "wp_decode_workspace_bytes",
    "wp_decode_static", "DECODE_STATIC_SCRATCH_BYTES", "wp_kcache_group_major", "KCACHE_ROWS", "KCACHE_GROUP_MAJOR",
    "KCACHE_WINDOWED", "wp_kcache_windowed_elems", "wp_kcache_windowed", "wp_kcache_windowed_append",
    "wp_decode_paged",
    "wp_device_status", "wp_set_wait_limit", "wp_wait_probe", "wp_status_str",
]

ROPE_INTERLEAVED = 0
ROPE_HALF_SPLIT = 1
ROPE_HALF_SPLIT_PAIRED = 2  # wp_rope_apply only: half-split rotation written in the interleaved order
MODE_GROUPED = 0
MODE_CHANNEL = 1
CUTOFF_INF = 2 ** 31 - 1
DECODE_STATIC_SCRATCH_BYTES = 16 << 20

WP_OK, WP_ERR_ARG, WP_ERR_UNSUPPORTED, WP_ERR_CUDA, WP_ERR_TIMEOUT = range(5)
KCACHE_ROWS, KCACHE_GROUP_MAJOR, KCACHE_WINDOWED = 0, 1, 2  # wp_kcache_layout

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libwaveprune.so")
_lib = None


class WavePruneError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn}: {wp_status_str(code)} (status {code})")


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libwaveprune.so (build it first with ``python -m
    rope_period_truncated_b200.build``). Raises if it is absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"libwaveprune.so not built ({_LIB_PATH}); run python -m rope_period_truncated_b200.build")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I, D, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_float
    lib.wp_cutoffs.restype = I
    lib.wp_cutoffs.argtypes = [I, D, P, D, D, I, P, P]
    lib.wp_rope_apply.restype = I
    lib.wp_rope_apply.argtypes = [P, P, I, I, I, I, P, I, D, P, D, I, P]
    lib.wp_schedule.restype = I
    lib.wp_schedule.argtypes = [I, I, I, P, I, P, P]
    lib.wp_prefill.restype = I
    lib.wp_prefill.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P, I, F, P]
    lib.wp_prefill_ex.restype = I
    lib.wp_prefill_ex.argtypes = [P, P, P, P, P, P, I, I, ctypes.c_int64, I, I, I, I, P, I, I, F, P]
    lib.wp_prefill_backward_workspace_bytes.restype = ctypes.c_size_t
    lib.wp_prefill_backward_workspace_bytes.argtypes = [I, I, I]
    lib.wp_prefill_backward.restype = I
    lib.wp_prefill_backward.argtypes = [P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, I, I, I, I, I, P, I, F, P]
    lib.wp_decode_workspace_bytes.restype = ctypes.c_size_t
    lib.wp_decode_workspace_bytes.argtypes = [I, I, I, I]
    lib.wp_decode.restype = I
    lib.wp_decode.argtypes = [P, P, P, P, I, I, I, I, I, P, F, P, P, P, ctypes.c_size_t, P]
    lib.wp_decode_static.restype = I
    lib.wp_decode_static.argtypes = [P, P, P, P, I, I, I, I, I, P, F, P, P, P]
    lib.wp_decode_kl.restype = I
    lib.wp_decode_kl.argtypes = [P, P, I, P, P, I, I, I, I, I, P, F, P, P, P, ctypes.c_size_t, P]
    lib.wp_decode_ex.restype = I
    lib.wp_decode_ex.argtypes = [P, P, I, P, P, I, I, I, I, I, I, P, I, I, F, P, P, P, ctypes.c_size_t, P]
    lib.wp_decode_paged.restype = I
    lib.wp_decode_paged.argtypes = [P, P, I, P, I, I, P, I, P, I, I, I, I, P, F, P, P, P, ctypes.c_size_t, P]
    lib.wp_kcache_group_major.restype = I
    lib.wp_kcache_group_major.argtypes = [P, P, I, I, I, I, P]
    lib.wp_kcache_windowed_elems.restype = ctypes.c_size_t
    lib.wp_kcache_windowed_elems.argtypes = [I, I, P]
    lib.wp_kcache_windowed_from_rows.restype = I
    lib.wp_kcache_windowed_from_rows.argtypes = [P, P, P, I, I, I, I, P, P]
    lib.wp_kcache_windowed_append.restype = I
    lib.wp_kcache_windowed_append.argtypes = [P, P, P, I, I, I, I, P, P]
    lib.wp_device_status.restype = I
    lib.wp_device_status.argtypes = [P]
    lib.wp_set_wait_limit.restype = ctypes.c_longlong
    lib.wp_set_wait_limit.argtypes = [ctypes.c_longlong]
    lib.wp_wait_probe.restype = I
    lib.wp_wait_probe.argtypes = [P]
    lib.wp_status_str.restype = ctypes.c_char_p
    lib.wp_status_str.argtypes = [I]
    _lib = lib
    return lib


def wp_status_str(code: int) -> str:
    return load_library().wp_status_str(int(code)).decode()


def _check(fn: str, code: int):
    if code != WP_OK:
        raise WavePruneError(fn, code)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _host_i32(a, n: int | None = None):
    if a is None:
        return None, None
    arr = np.ascontiguousarray(np.asarray(a), dtype=np.int32)
    if n is not None and arr.size != n:
        raise ValueError(f"expected {n} cutoffs, got {arr.size}")
    return arr, arr.ctypes.data_as(ctypes.c_void_p)


def _host_f64(a):
    if a is None:
        return None, None
    arr = np.ascontiguousarray(np.asarray(a), dtype=np.float64)
    return arr, arr.ctypes.data_as(ctypes.c_void_p)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype, ndim: int):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


# --------------------------------------------------------------------- host

def wp_cutoffs(d_h: int, theta: float, layout: int, alpha: float = 2.0, freq_scale=None, scale_all: float = 1.0):
    """Integer cutoffs (chan_cut [d_h/2], group_cut [d_h/16]) as numpy int32."""
    fs, fs_p = _host_f64(freq_scale)
    wc = np.zeros(d_h // 2, dtype=np.int32)
    wg = np.zeros(max(d_h // 16, 1), dtype=np.int32)
    _check("wp_cutoffs", load_library().wp_cutoffs(d_h, theta, fs_p, scale_all, alpha, layout,
                                                    wc.ctypes.data_as(ctypes.c_void_p),
                                                    wg.ctypes.data_as(ctypes.c_void_p)))
    return wc, wg


def wp_schedule(N: int, BM: int, BN: int, cut, want_map: bool = True):
    """Tile classes (cls [nqb,nkb,n] uint8 or None, counts [n,3] int64)."""
    cut_a, cut_p = _host_i32(cut)
    n = cut_a.size
    nqb, nkb = -(-N // BM), -(-N // BN)
    cls = np.empty((nqb, nkb, n), dtype=np.uint8) if want_map else None
    counts = np.zeros((n, 3), dtype=np.int64)
    _check("wp_schedule", load_library().wp_schedule(
        N, BM, BN, cut_p, n, None if cls is None else cls.ctypes.data_as(ctypes.c_void_p),
        counts.ctypes.data_as(ctypes.c_void_p)))
    return cls, counts


# ------------------------------------------------------------------- device

def wp_rope_apply(x: torch.Tensor, theta: float, layout: int, pos: torch.Tensor | None = None, pos0: int = 0,
                  freq_scale=None, scale_all: float = 1.0, out: torch.Tensor | None = None, stream=None):
    """Rotate bf16 x [B,N,H,d] by position*f_c; returns ``out`` (x itself if
    out is x; a new tensor if out is None)."""
    _need(x, "x", torch.bfloat16, 4)
    B, N, H, d = x.shape
    if out is None:
        out = torch.empty_like(x)
    _need(out, "out", torch.bfloat16, 4)
    if out.shape != x.shape:
        raise ValueError("out shape mismatch")
    if pos is not None:
        _need(pos, "pos", torch.int32, 2)
        if tuple(pos.shape) != (B, N):
            raise ValueError("pos must be [B, N]")
    fs, fs_p = _host_f64(freq_scale)
    _check("wp_rope_apply", load_library().wp_rope_apply(
        _ptr(x), _ptr(out), B, N, H, d, _ptr(pos), int(pos0), float(theta), fs_p, float(scale_all), int(layout),
        _stream(stream)))
    return out


def wp_prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cut=None, mode: int = MODE_GROUPED,
               layout: int = ROPE_HALF_SPLIT, softmax_scale: float = 0.0, out: torch.Tensor | None = None,
               lse: torch.Tensor | None = None, want_lse: bool = True, stream=None,
               cu_seqlens: torch.Tensor | None = None, max_seqlen: int | None = None):
    """Causal WavePrune prefill (wp_prefill_ex).

    Uniform batch: q [B,N,Hq,d], k/v [B,N,Hkv,d] bf16 (rotated); returns
    (o [B,N,Hq,d] bf16, lse [B,Hq,N] fp32). Packed batch: q [T,Hq,d], k/v
    [T,Hkv,d] with ``cu_seqlens`` (device int32 [B+1]) and ``max_seqlen`` (an
    upper bound of the lengths); returns (o [T,Hq,d], lse [Hq,T]).
    ``cut``: host cutoffs, one row [d/16] (grouped) or [d/2] (channel mode)
    for every head, or one row per query head [Hq, n]; None = dense."""
    packed = cu_seqlens is not None
    nd = 3 if packed else 4
    _need(q, "q", torch.bfloat16, nd)
    _need(k, "k", torch.bfloat16, nd)
    _need(v, "v", torch.bfloat16, nd)
    if packed:
        _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
        T, Hq, d = q.shape
        B = cu_seqlens.numel() - 1
        if B < 1 or max_seqlen is None or int(max_seqlen) < 1:
            raise ValueError("a packed batch needs cu_seqlens [B+1] and max_seqlen >= 1")
        N = int(max_seqlen)
        Hkv = k.shape[1]
        if tuple(k.shape) != (T, Hkv, d) or tuple(v.shape) != (T, Hkv, d):
            raise ValueError("k/v shape mismatch")
        lse_shape = (Hq, T)
    else:
        B, N, Hq, d = q.shape
        T = B * N
        Hkv = k.shape[2]
        if tuple(k.shape) != (B, N, Hkv, d) or tuple(v.shape) != (B, N, Hkv, d):
            raise ValueError("k/v shape mismatch")
        lse_shape = (B, Hq, N)
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, nd)
    if lse is None and want_lse:
        lse = torch.empty(lse_shape, dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", torch.float32, len(lse_shape))
    n_expected = d // 16 if mode == MODE_GROUPED else d // 2
    cut_rows = 1
    if cut is not None:
        arr = np.asarray(cut)
        if arr.ndim == 2:
            if arr.shape != (Hq, n_expected):
                raise ValueError(f"per-head cutoffs must be [{Hq}, {n_expected}], got {arr.shape}")
            cut_rows = Hq
        cut_a, cut_p = _host_i32(arr.reshape(-1), cut_rows * n_expected)
    else:
        cut_a, cut_p = None, None
    _check("wp_prefill", load_library().wp_prefill_ex(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(cu_seqlens), B, N, T, Hq, Hkv, d, int(mode), cut_p,
        cut_rows, int(layout), float(softmax_scale), _stream(stream)))
    return out, lse


def wp_prefill_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor,
                        dout: torch.Tensor, cut=None, softmax_scale: float = 0.0, dq: torch.Tensor | None = None,
                        dk: torch.Tensor | None = None, dv: torch.Tensor | None = None,
                        workspace: torch.Tensor | None = None, stream=None):
    """Gradients (dq, dk, dv) of a grouped-mode wp_prefill: q/o/dout
    [B,N,Hq,d], k/v [B,N,Hkv,d] bf16, lse [B,Hq,N] fp32 from the forward.
    ``cut``: group cutoffs [d/16], per-head [Hq, d/16], or None (dense)."""
    for t, name in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _need(t, name, torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 3)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    if tuple(k.shape) != (B, N, Hkv, d) or tuple(v.shape) != (B, N, Hkv, d):
        raise ValueError("k/v shape mismatch")
    if tuple(o.shape) != tuple(q.shape) or tuple(dout.shape) != tuple(q.shape) or tuple(lse.shape) != (B, Hq, N):
        raise ValueError("o/dout/lse shape mismatch")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for t, ref, name in ((dq, q, "dq"), (dk, k, "dk"), (dv, v, "dv")):
        _need(t, name, torch.bfloat16, 4)
        if t.shape != ref.shape:
            raise ValueError(f"{name} shape mismatch")
    lib = load_library()
    ws_bytes = int(lib.wp_prefill_backward_workspace_bytes(B, N, Hq))
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    cut_rows = 1
    cut_p = None
    if cut is not None:
        arr = np.asarray(cut)
        cut_rows = Hq if arr.ndim == 2 else 1
        cut_a, cut_p = _host_i32(arr.reshape(-1), cut_rows * (d // 16))
    _check("wp_prefill_backward", lib.wp_prefill_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
        workspace.numel() * workspace.element_size(), B, N, Hq, Hkv, d, cut_p, cut_rows, float(softmax_scale),
        _stream(stream)))
    return dq, dk, dv


def wp_decode_workspace_bytes(B: int, Hq: int, d_h: int, Lmax: int) -> int:
    return int(load_library().wp_decode_workspace_bytes(B, Hq, d_h, Lmax))


def wp_kcache_group_major(kcache: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """K cache [B,Hkv,Lmax,d] bf16 (rows) -> [B,Hkv,d/16,Lmax,16] (group-major)."""
    _need(kcache, "kcache", torch.bfloat16, 4)
    B, Hkv, Lmax, d = kcache.shape
    if out is None:
        out = torch.empty((B, Hkv, d // 16, Lmax, 16), dtype=torch.bfloat16, device=kcache.device)
    _need(out, "out", torch.bfloat16, 5)
    if tuple(out.shape) != (B, Hkv, d // 16, Lmax, 16):
        raise ValueError("out shape mismatch")
    _check("wp_kcache_group_major", load_library().wp_kcache_group_major(
        _ptr(kcache), _ptr(out), B, Hkv, Lmax, d, _stream(stream)))
    return out


def wp_kcache_windowed_elems(Lmax: int, d: int, group_cut) -> int:
    """bf16 elements of one (b, hk) of a windowed K cache under ``group_cut`` [d/16]."""
    cut_a, cut_p = _host_i32(group_cut, d // 16)
    n = load_library().wp_kcache_windowed_elems(int(Lmax), int(d), cut_p)
    if n == 0:
        raise WavePruneError(WP_ERR_ARG, "wp_kcache_windowed_elems")
    return int(n)


def wp_kcache_windowed(kcache: torch.Tensor, lens: torch.Tensor, group_cut, out: torch.Tensor | None = None,
                       stream=None) -> torch.Tensor:
    """K cache [B,Hkv,Lmax,d] bf16 (rows) -> windowed [B,Hkv,elems]: every
    group keeps only the keys its cutoff can still reach (rings of
    round_up_16(W_g + 1) keys). ``lens`` int32 [B] (device)."""
    _need(kcache, "kcache", torch.bfloat16, 4)
    _need(lens, "lens", torch.int32, 1)
    B, Hkv, Lmax, d = kcache.shape
    n = wp_kcache_windowed_elems(Lmax, d, group_cut)
    if out is None:
        out = torch.empty((B, Hkv, n), dtype=torch.bfloat16, device=kcache.device)
    _need(out, "out", torch.bfloat16, 3)
    if tuple(out.shape) != (B, Hkv, n):
        raise ValueError("out shape mismatch")
    cut_a, cut_p = _host_i32(group_cut, d // 16)
    _check("wp_kcache_windowed", load_library().wp_kcache_windowed_from_rows(
        _ptr(kcache), _ptr(lens), _ptr(out), B, Hkv, Lmax, d, cut_p, _stream(stream)))
    return out


def wp_kcache_windowed_append(k_new: torch.Tensor, pos: torch.Tensor, kwin: torch.Tensor, Lmax: int, group_cut,
                              stream=None) -> torch.Tensor:
    """Write the keys k_new [B,Hkv,d] (token positions ``pos`` int32 [B],
    device) into a windowed K cache [B,Hkv,elems] in place; returns it."""
    _need(k_new, "k_new", torch.bfloat16, 3)
    _need(pos, "pos", torch.int32, 1)
    _need(kwin, "kwin", torch.bfloat16, 3)
    B, Hkv, d = k_new.shape
    if tuple(kwin.shape) != (B, Hkv, wp_kcache_windowed_elems(Lmax, d, group_cut)):
        raise ValueError("windowed K cache shape mismatch")
    cut_a, cut_p = _host_i32(group_cut, d // 16)
    _check("wp_kcache_windowed_append", load_library().wp_kcache_windowed_append(
        _ptr(k_new), _ptr(pos), _ptr(kwin), B, Hkv, int(Lmax), d, cut_p, _stream(stream)))
    return kwin


def wp_decode(q: torch.Tensor, kcache: torch.Tensor, vcache: torch.Tensor, lens: torch.Tensor, group_cut=None,
              softmax_scale: float = 0.0, out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
              workspace: torch.Tensor | None = None, want_lse: bool = True, stream=None, mode: int = MODE_GROUPED,
              layout: int = ROPE_INTERLEAVED):
    """Split-KV decode. q [B,Hq,d] (rotated), V cache [B,Hkv,Lmax,d] bf16, K
    cache the same (rows), [B,Hkv,d/16,Lmax,16] (group-major, from
    wp_kcache_group_major) or [B,Hkv,elems] (windowed, from
    wp_kcache_windowed with the same ``group_cut``), lens int32 [B] (device). ``group_cut``: group
    cutoffs [d/16], per-head [Hq, d/16], or (mode=MODE_CHANNEL) channel
    cutoffs [d/2] with ``layout``; None = dense. Returns (o [B,Hq,d] bf16,
    lse [B,Hq] fp32)."""
    _need(q, "q", torch.bfloat16, 3)
    _need(vcache, "vcache", torch.bfloat16, 4)
    _need(lens, "lens", torch.int32, 1)
    B, Hq, d = q.shape
    _, Hkv, Lmax, _ = vcache.shape
    if tuple(vcache.shape) != (B, Hkv, Lmax, d):
        raise ValueError("cache shape mismatch")
    if kcache.dim() == 5:
        _need(kcache, "kcache", torch.bfloat16, 5)
        if tuple(kcache.shape) != (B, Hkv, d // 16, Lmax, 16):
            raise ValueError("group-major K cache shape mismatch")
        k_layout = KCACHE_GROUP_MAJOR
    elif kcache.dim() == 3:
        _need(kcache, "kcache", torch.bfloat16, 3)
        if group_cut is None or np.asarray(group_cut).ndim != 1 or mode != MODE_GROUPED:
            raise ValueError("a windowed K cache takes its own group cutoff table")
        if tuple(kcache.shape) != (B, Hkv, wp_kcache_windowed_elems(Lmax, d, group_cut)):
            raise ValueError("windowed K cache shape mismatch")
        k_layout = KCACHE_WINDOWED
    else:
        _need(kcache, "kcache", torch.bfloat16, 4)
        if tuple(kcache.shape) != tuple(vcache.shape):
            raise ValueError("cache shape mismatch")
        k_layout = KCACHE_ROWS
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    ws_bytes = wp_decode_workspace_bytes(B, Hq, d, Lmax)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    if workspace.numel() * workspace.element_size() < ws_bytes:
        raise ValueError("workspace too small")
    cut_rows = 1 if group_cut is None or np.asarray(group_cut).ndim == 1 else Hq
    if mode == MODE_GROUPED and cut_rows == 1:
        cut_a, cut_p = _host_i32(group_cut, d // 16)
        _check("wp_decode", load_library().wp_decode_kl(
            _ptr(q), _ptr(kcache), k_layout, _ptr(vcache), _ptr(lens), Lmax, B, Hq, Hkv, d, cut_p,
            float(softmax_scale), _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel() * workspace.element_size(),
            _stream(stream)))
        return out, lse
    n = (d // 16 if mode == MODE_GROUPED else d // 2) * cut_rows
    cut_a, cut_p = _host_i32(None if group_cut is None else np.asarray(group_cut).reshape(-1), n)
    _check("wp_decode", load_library().wp_decode_ex(
        _ptr(q), _ptr(kcache), k_layout, _ptr(vcache), _ptr(lens), Lmax, B, Hq, Hkv, d, int(mode), cut_p, cut_rows,
        int(layout), float(softmax_scale), _ptr(out), _ptr(lse), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return out, lse


def wp_decode_paged(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor, block_table: torch.Tensor,
                    lens: torch.Tensor, group_cut=None, softmax_scale: float = 0.0, out: torch.Tensor | None = None,
                    lse: torch.Tensor | None = None, workspace: torch.Tensor | None = None, want_lse: bool = True,
                    stream=None):
    """Split-KV decode over a paged cache. q [B,Hq,d]; v_pages [n_pages,Hkv,P,d];
    k_pages the same (rows) or [n_pages,Hkv,d/16,P,16] (group-major);
    block_table int32 [B, max_pages] (device); lens int32 [B] (device)."""
    _need(q, "q", torch.bfloat16, 3)
    _need(v_pages, "v_pages", torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(lens, "lens", torch.int32, 1)
    B, Hq, d = q.shape
    n_pages, Hkv, P, _ = v_pages.shape
    if tuple(v_pages.shape) != (n_pages, Hkv, P, d) or block_table.shape[0] != B:
        raise ValueError("paged cache shape mismatch")
    if k_pages.dim() == 5:
        _need(k_pages, "k_pages", torch.bfloat16, 5)
        if tuple(k_pages.shape) != (n_pages, Hkv, d // 16, P, 16):
            raise ValueError("group-major K pages shape mismatch")
        k_layout = KCACHE_GROUP_MAJOR
    else:
        _need(k_pages, "k_pages", torch.bfloat16, 4)
        if tuple(k_pages.shape) != tuple(v_pages.shape):
            raise ValueError("K pages shape mismatch")
        k_layout = KCACHE_ROWS
    max_pages = block_table.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    ws_bytes = wp_decode_workspace_bytes(B, Hq, d, max_pages * P)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    if workspace.numel() * workspace.element_size() < ws_bytes:
        raise ValueError("workspace too small")
    cut_a, cut_p = _host_i32(group_cut, d // 16)
    _check("wp_decode_paged", load_library().wp_decode_paged(
        _ptr(q), _ptr(k_pages), k_layout, _ptr(v_pages), n_pages, P, _ptr(block_table), max_pages, _ptr(lens), B, Hq,
        Hkv, d, cut_p, float(softmax_scale), _ptr(out), _ptr(lse), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return out, lse


def wp_decode_static(q: torch.Tensor, kcache: torch.Tensor, vcache: torch.Tensor, lens: torch.Tensor,
                     group_cut=None, softmax_scale: float = 0.0, out: torch.Tensor | None = None,
                     lse: torch.Tensor | None = None, want_lse: bool = True, stream=None):
    """wp_decode without a workspace: the library's fixed device scratch holds
    the split partials, so nothing is allocated for them (for callers that
    cannot allocate device memory). Same arguments and results as wp_decode;
    raises WavePruneError (unsupported) when the batch needs more than
    DECODE_STATIC_SCRATCH_BYTES of scratch."""
    _need(q, "q", torch.bfloat16, 3)
    _need(kcache, "kcache", torch.bfloat16, 4)
    _need(vcache, "vcache", torch.bfloat16, 4)
    _need(lens, "lens", torch.int32, 1)
    B, Hq, d = q.shape
    _, Hkv, Lmax, _ = kcache.shape
    if tuple(kcache.shape) != (B, Hkv, Lmax, d) or tuple(vcache.shape) != tuple(kcache.shape):
        raise ValueError("cache shape mismatch")
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    cut_a, cut_p = _host_i32(group_cut, d // 16)
    _check("wp_decode_static", load_library().wp_decode_static(
        _ptr(q), _ptr(kcache), _ptr(vcache), _ptr(lens), Lmax, B, Hq, Hkv, d, cut_p, float(softmax_scale),
        _ptr(out), _ptr(lse), _stream(stream)))
    return out, lse


def wp_device_status(stream=None) -> int:
    """Synchronise the stream, read and clear the device status word."""
    return int(load_library().wp_device_status(_stream(stream)))


def wp_set_wait_limit(cycles: int) -> int:
    return int(load_library().wp_set_wait_limit(int(cycles)))


def wp_wait_probe(stream=None):
    _check("wp_wait_probe", load_library().wp_wait_probe(_stream(stream)))

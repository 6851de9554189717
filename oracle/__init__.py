"""fp64 CPU oracle for WavePrune causal attention.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package. The product path (``rope_period_truncated_b200``) never does, and the
two share no code: the arithmetic lives in ``wp_oracle.c`` (plain loops, fp64),
this module only marshals numpy arrays.

Page tags used in citations:
  [RN] "WavePrune：RoPE 通常只需一个旋转周期" (reading notes of arXiv:2610.06963)
  [KC] "WavePrune：RoPE只用一个旋转周期，长文本性能反而更好"
  [TW] "Guancheng Du @ducatiqwq" (author's thread)

Every function here is pinned by ``tests/test_oracle_pins.py`` to values that
do not come from the oracle itself (the pages' Table 12, closed forms,
independent library routines, brute force).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

INTERLEAVED = 0
HALF_SPLIT = 1
MODE_GROUPED = 0
MODE_CHANNEL = 1

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wp_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile wp_oracle.c to liboracle.so (gcc, -O2, no fast-math, no FMA
    contraction, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-std=c11", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
                               "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        # WP_ORACLE_LIB points the pins at a deliberately broken copy of the
        # oracle (tests/test_oracle_mutations.py), never at anything else.
        path = os.environ.get("WP_ORACLE_LIB")
        if not path:
            path = build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64, i32, f64 = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        lib.wpo_freq.restype = f64
        lib.wpo_freq.argtypes = [i32, i32, f64, P, f64]
        lib.wpo_channel_cutoff.restype = ctypes.c_int32
        lib.wpo_channel_cutoff.argtypes = [f64, f64]
        lib.wpo_cutoffs.restype = i32
        lib.wpo_cutoffs.argtypes = [i32, f64, P, f64, f64, i32, P, P]
        lib.wpo_rope.restype = None
        lib.wpo_rope.argtypes = [P, P, i64, i64, i32, i32, P, i64, f64, P, f64, i32]
        lib.wpo_round_bf16.restype = None
        lib.wpo_round_bf16.argtypes = [P, P, i64]
        lib.wpo_logits.restype = None
        lib.wpo_logits.argtypes = [P, P, i64, i32, i32, i32, P, f64, P]
        lib.wpo_attention_rows.restype = i32
        lib.wpo_attention_rows.argtypes = [P, P, P, P, i64, P, P, i64, i64, i32, i32, i32, i32, i32, P, f64, P, P,
                                           i32]
        lib.wpo_decode.restype = i32
        lib.wpo_decode.argtypes = [P, P, P, P, i64, i32, i32, i32, i64, P, f64, P, P, i32]
        lib.wpo_attention_backward.restype = i32
        lib.wpo_attention_backward.argtypes = [P, P, P, P, i64, i64, i32, i32, i32, i32, i32, P, f64, P, P, P, i32]
        lib.wpo_tile_classes.restype = i32
        lib.wpo_tile_classes.argtypes = [i64, i32, i32, P, i32, P, P]
        _lib = lib
    return _lib


def _p(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _scale_arr(freq_scale):
    return None if freq_scale is None else np.ascontiguousarray(freq_scale, dtype=np.float64)


def freq(c: int, d_h: int, theta: float, freq_scale=None, scale_all: float = 1.0) -> float:
    """f_c = s_c * scale_all * theta^(-2c/d_h) [RN §1.1, Eq. (2)-(5)]."""
    fs = _scale_arr(freq_scale)
    return _load().wpo_freq(c, d_h, theta, _p(fs), scale_all)


def cutoffs(d_h: int, theta: float, layout: int = INTERLEAVED, alpha: float = 2.0, freq_scale=None,
            scale_all: float = 1.0):
    """Integer cutoffs (W_c [d_h/2], W_g [d_h/16]) [RN §2.1 after Eq. (6); §2.3 Eq. (8)]."""
    fs = _scale_arr(freq_scale)
    wc = np.zeros(d_h // 2, dtype=np.int32)
    wg = np.zeros(d_h // 16, dtype=np.int32)
    rc = _load().wpo_cutoffs(d_h, theta, _p(fs), scale_all, alpha, layout, _p(wc), _p(wg))
    if rc:
        raise ValueError(f"oracle cutoffs: bad arguments (code {rc})")
    return wc, wg


def rope(x, theta: float, layout: int, pos=None, pos0: int = 0, freq_scale=None, scale_all: float = 1.0):
    """Rotate x [B,N,H,d] (fp64) by position * f_c [KC RoPE matrix; RN §1.1]."""
    x = _f64(x)
    B, N, H, d = x.shape
    y = np.empty_like(x)
    pos_a = None if pos is None else np.ascontiguousarray(np.asarray(pos).reshape(B, N), dtype=np.int64)
    _load().wpo_rope(_p(x), _p(y), B, N, H, d, _p(pos_a), pos0, theta, _p(_scale_arr(freq_scale)), scale_all,
                     layout)
    return y


def round_bf16_bits(x) -> np.ndarray:
    """fp64 -> bf16 (ties to even) as uint16 bits, same shape."""
    x = _f64(x)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().wpo_round_bf16(_p(x), _p(out), x.size)
    return out


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp64 (exact)."""
    u32 = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u32.view(np.float32).astype(np.float64)


def logits(q, k, cut, mode: int = MODE_GROUPED, layout: int = INTERLEAVED, scale: float | None = None):
    """Logit matrix [N,N] of one head (-inf above the diagonal) [RN §2.1 Eq. (6); §2.3 Eq. (8)]."""
    q, k = _f64(q), _f64(k)
    N, d = q.shape
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    cut = np.ascontiguousarray(cut, dtype=np.int32)
    L = np.empty((N, N), dtype=np.float64)
    _load().wpo_logits(_p(q), _p(k), N, d, mode, layout, _p(cut), scale, _p(L))
    return L


def attention_rows(q_rows, rows, k, v, Hq: int, cut, mode: int = MODE_GROUPED, layout: int = INTERLEAVED,
                   scale: float | None = None, nthreads: int = 0):
    """Causal WavePrune attention for selected rows.

    q_rows [R,d] are the query vectors of rows (b, h, i) = rows; k, v are
    [B,N,Hkv,d]. Returns (o [R,d], lse [R]) in fp64."""
    k, v = _f64(k), _f64(v)
    B, N, Hkv, d = k.shape
    q_rows = _f64(q_rows).reshape(-1, d)
    rb, rh, ri = (np.ascontiguousarray(np.asarray(r), dtype=np.int64) for r in rows)
    R = q_rows.shape[0]
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    cut = np.ascontiguousarray(cut, dtype=np.int32)
    o = np.empty((R, d), dtype=np.float64)
    lse = np.empty(R, dtype=np.float64)
    rc = _load().wpo_attention_rows(_p(q_rows), _p(rb), _p(rh), _p(ri), R, _p(k), _p(v), B, N, Hq, Hkv, d, mode,
                                    layout, _p(cut), scale, _p(o), _p(lse), nthreads)
    if rc:
        raise ValueError(f"oracle attention: bad arguments (code {rc})")
    return o, lse


def attention(q, k, v, cut, mode: int = MODE_GROUPED, layout: int = INTERLEAVED, scale: float | None = None,
              nthreads: int = 0):
    """Every row: q [B,N,Hq,d], k/v [B,N,Hkv,d] -> (o [B,N,Hq,d], lse [B,Hq,N])."""
    q = _f64(q)
    B, N, Hq, d = q.shape
    bb, tt, hh = np.meshgrid(np.arange(B), np.arange(N), np.arange(Hq), indexing="ij")
    rows = (bb.ravel(), hh.ravel(), tt.ravel())
    o, lse = attention_rows(q.reshape(-1, d), rows, k, v, Hq, cut, mode, layout, scale, nthreads)
    return o.reshape(B, N, Hq, d), lse.reshape(B, N, Hq).transpose(0, 2, 1).copy()


def attention_backward(q, k, v, dout, cut, mode: int = MODE_GROUPED, layout: int = INTERLEAVED,
                       scale: float | None = None, nthreads: int = 0):
    """Gradients (dq, dk, dv) of sum(dout * O) for causal prefill, q/dout
    [B,N,Hq,d], k/v [B,N,Hkv,d] (fp64). The chain rule through the forward
    definition [RN §2.1 Eq. (6); §2.3 Eq. (8)]: masked units add 0 to the
    gradients as they add 0 to the logit."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    cut = np.ascontiguousarray(cut, dtype=np.int32)
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    rc = _load().wpo_attention_backward(_p(q), _p(k), _p(v), _p(dout), B, N, Hq, Hkv, d, mode, layout, _p(cut),
                                        scale, _p(dq), _p(dk), _p(dv), nthreads)
    if rc:
        raise ValueError(f"oracle backward: bad arguments (code {rc})")
    return dq, dk, dv


def decode(q, kc, vc, lens, group_cut, scale: float | None = None, nthreads: int = 0):
    """Decode: q [B,Hq,d] at position len-1 against caches [B,Hkv,Lmax,d].
    Returns (o [B,Hq,d], lse [B,Hq])."""
    q, kc, vc = _f64(q), _f64(kc), _f64(vc)
    B, Hq, d = q.shape
    _, Hkv, Lmax, _ = kc.shape
    lens = np.ascontiguousarray(np.asarray(lens), dtype=np.int32)
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    cut = np.ascontiguousarray(group_cut, dtype=np.int32)
    o = np.empty((B, Hq, d), dtype=np.float64)
    lse = np.empty((B, Hq), dtype=np.float64)
    rc = _load().wpo_decode(_p(q), _p(kc), _p(vc), _p(lens), B, Hq, Hkv, d, Lmax, _p(cut), scale, _p(o), _p(lse),
                            nthreads)
    if rc:
        raise ValueError(f"oracle decode: bad arguments (code {rc})")
    return o, lse


def tile_classes(N: int, BM: int, BN: int, cut, want_map: bool = True):
    """Brute-force tile classes [RN §2.3 table; TW (6/7)].

    Returns (cls [nqb,nkb,ncut] uint8 or None, counts [ncut,3] int64) with
    classes 0 skip / 1 full / 2 boundary / 3 no causal pair."""
    cut = np.ascontiguousarray(cut, dtype=np.int32)
    ncut = cut.size
    nqb, nkb = -(-N // BM), -(-N // BN)
    cls = np.empty((nqb, nkb, ncut), dtype=np.uint8) if want_map else None
    counts = np.zeros((ncut, 3), dtype=np.int64)
    rc = _load().wpo_tile_classes(N, BM, BN, _p(cut), ncut, _p(cls), _p(counts))
    if rc:
        raise ValueError(f"oracle tile classes: bad arguments (code {rc})")
    return cls, counts

#!/usr/bin/env python
"""Benchmark of the WavePrune causal-attention hot path on B200.

One step = one pass of the whole path over one batch of synthetic inputs
already resident in HBM:
  * prefill, 32K context (B1, H_q 32 / H_kv 8, N 32768, d 128, theta 1e6,
    half-split): rotate Q and K (wp_rope_apply), then wp_prefill with the
    grouped cutoffs;
  * decode (16 sequences, lengths U[16384, 32768], same heads): rotate the new
    queries at position len-1, then wp_decode (split-KV + LSE combine).
``value`` is the prefill's useful TFLOP/s (non-skipped group QK MMAs plus PV,
counted per 128x128 tile) over the whole step time; the decode's GB/s over
required bytes (K of in-window groups plus all of V) is reported next to it.
Both are also given as fractions of the measured B200 peaks.

``--impl reference`` times the fp64 CPU oracle instead (a bounded sample of
query rows per step) on the host cores, as the slow reference arm.

Run: python bench.py [--gpus N --steps K --warmup W]; for N > 1 under
torch.distributed.run every rank runs an independent replica (the work is
data-parallel over heads and sequences with no exchange step).
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import wp_synthetic as syn  # noqa: E402

METRIC = "prefill useful TFLOP/s & decode GB/s at 32K ctx, % of B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
BM = BN = 128


def parse_args():
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=40)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-dense", action="store_true")
    p.add_argument("--no-backward", action="store_true")
    p.add_argument("--no-exact", action="store_true", help="skip the exact per-channel prefill entry")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    p.add_argument("--kcache", choices=["group-major", "rows"], default="group-major",
                   help="layout of the decode K cache in HBM")
    p.add_argument("--page-size", type=int, default=0,
                   help="decode from a paged KV cache with pages of this many keys (0: contiguous)")
    p.add_argument("--grouping", choices=["half-split", "paired"], default="half-split",
                   help="paired: Q/K of the half-split model rotated into the interleaved order, groups of 8 "
                        "whole channels (the pages' grouping, Table 12 cutoffs)")
    p.add_argument("--only", choices=["all", "prefill", "decode", "backward"], default="all",
                   help="restrict the step (profiling a single kernel)")
    p.add_argument("--prefill-mode", choices=["grouped", "exact"], default="grouped",
                   help="rule of the timed prefill in a restricted profiling case (--only prefill)")
    p.add_argument("--prefill-n", type=int, default=0,
                   help="override the prefill sequence length (smaller profiling case; not a bench line)")
    return p.parse_args()


# ----------------------------------------------------------------------------- setup

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(values, device):
    """Element-wise max of per-rank timings over all ranks (identity when
    torch.distributed is not initialised or there is one rank)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def bench_config(args, world, wg):
    """The workload description both arms print."""
    return {
        "workload": "prefill long_32k (B1 Hq32/Hkv8 N32768 d128 theta1e6 half-split, grouped cutoffs) + "
                    "decode_32k (16 seqs Hq32/Hkv8 d128 L~U[16384,32768]); step = rope Q,K + prefill + "
                    "rope q + split-KV decode",
        "l2": "inputs larger than L2 each step (384 MiB prefill Q/K/V, 2 GiB KV cache); no flush",
        "parallelism": f"replicas x{world} (independent heads/sequences, no collective)",
        "group_cutoffs": [int(x) for x in wg],
        "decode_kcache": ("group-major [B,Hkv,d/16,L,16]" if args.kcache == "group-major"
                          else "rows [B,Hkv,L,d]"),
        "grouping": ("half-split groups (max over channels c and c+64)" if args.grouping == "half-split"
                     else "paired: 8 whole channels per group (interleaved order after rope)"),
        **({"decode_kv_pages": f"{args.page_size} keys per page, pages shuffled in the pool"}
           if args.page_size else {}),
    }


def source_digest(source: str) -> str:
    """sha256 prefix (16 hex digits) of a kernel source's code followed by the
    code of every header it pulls in with #include "..." (looked up beside
    the including file, then in include/), each once, in the order of first
    inclusion. Comments are removed and runs of whitespace collapsed first,
    so a change to the compiled text changes the digest and a change to a
    comment does not."""
    import hashlib
    import re
    h = hashlib.sha256()
    seen = set()

    def code_of(data: bytes) -> bytes:
        data = re.sub(rb"/\*.*?\*/", b" ", data, flags=re.S)
        data = re.sub(rb"//[^\n]*", b" ", data)
        return re.sub(rb"\s+", b" ", data).strip()

    def visit(path):
        if path in seen:
            return
        seen.add(path)
        with open(path, "rb") as f:
            data = f.read()
        h.update(code_of(data) + b"\n")
        for name in re.findall(rb'^[ \t]*#[ \t]*include[ \t]+"([^"]+)"', data, re.M):
            for d in (os.path.dirname(path), os.path.join(ROOT, "include")):
                cand = os.path.join(d, name.decode())
                if os.path.exists(cand):
                    visit(cand)
                    break

    visit(os.path.join(ROOT, source))
    return h.hexdigest()[:16]


def profiled_traffic(summary: str, source: str):
    """DRAM bytes per launch from a committed ncu summary under profiles/, or
    None when the kernel source (with its headers) has changed since it was
    captured."""
    try:
        kv = {}
        with open(os.path.join(ROOT, "profiles", summary)) as f:
            for line in f:
                if ":" in line and not line.startswith("#"):
                    key, val = line.split(":", 1)
                    kv[key.strip()] = val.strip()
        if kv.get("source_sha256_16") != source_digest(source):
            return None
        return int(kv["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def prefill_flops(N, d, Hq, B, wg):
    """(tile-level, pair-exact) useful FLOPs of one causal prefill.

    Tile level: per 128x128 causal tile, one 2*BM*BN*16 MMA per non-skipped
    group plus the 2*BM*BN*d PV MMA. Pair exact: per pair j <= i,
    2*16 per group with i-j <= W_g plus 2*d."""
    import rope_period_truncated_b200 as wp
    _, counts = wp.wp_schedule(N, BM, BN, wg, want_map=False)
    tiles = int(counts[0].sum())
    qk = sum(int(counts[g, 1] + counts[g, 2]) for g in range(len(wg))) * 2 * BM * BN * 16
    pv = tiles * 2 * BM * BN * d
    tile_level = float(qk + pv) * B * Hq
    delta = np.arange(N, dtype=np.int64)
    pairs = (N - delta).astype(np.float64)
    active = (delta[:, None] <= np.asarray(wg, dtype=np.int64)[None, :]).sum(1)
    pair_exact = float((pairs * (2 * 16 * active + 2 * d)).sum()) * B * Hq
    dense_tile = float(tiles * (2 * BM * BN * d * 2)) * B * Hq
    return tile_level, pair_exact, dense_tile


def backward_flops(N, d, Hq, B, wg):
    """Useful FLOPs of one prefill backward, pair exact: per pair j <= i the
    three products over the in-window groups (S = Q K^T, dQ = dS K,
    dK = dS^T Q: 2*16 each per group) and the two full ones (dP = dO V^T,
    dV = P^T dO: 2*d each)."""
    delta = np.arange(N, dtype=np.int64)
    pairs = (N - delta).astype(np.float64)
    active = (delta[:, None] <= np.asarray(wg, dtype=np.int64)[None, :]).sum(1)
    useful = float((pairs * (3 * 2 * 16 * active + 2 * 2 * d)).sum()) * B * Hq
    dense = float((pairs * (3 * 2 * d + 2 * 2 * d)).sum()) * B * Hq
    return useful, dense


def exact_flops(N, d, Hq, B, wc):
    """Useful FLOPs of one exact-rule prefill, pair exact: per pair j <= i,
    2*2 per channel with i-j <= W_c (its two dims) plus 2*d for PV."""
    delta = np.arange(N, dtype=np.int64)
    pairs = (N - delta).astype(np.float64)
    active = (delta[:, None] <= np.asarray(wc, dtype=np.int64)[None, :]).sum(1)
    return float((pairs * (2 * 2 * active + 2 * d)).sum()) * B * Hq


def decode_required_bytes(lens, wg, B, Hq, Hkv, d):
    """K bytes of in-window groups (32 B per group per key) plus all of V,
    plus the query, output and LSE."""
    lens = np.asarray(lens, dtype=np.int64)
    wg = np.asarray(wg, dtype=np.int64)
    per_seq = (32 * np.minimum(wg[None, :] + 1, lens[:, None])).sum(1) + 2 * d * lens
    kv = float(per_seq.sum()) * Hkv
    dense_kv = float((4 * d * lens).sum()) * Hkv
    io = B * Hq * d * 2 * 2 + B * Hq * 4
    return kv + io, dense_kv + io


class ClockSampler:
    """nvidia-smi clock/throttle samples of this process's GPU, taken while the
    timed region runs."""

    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.path = None
        self.uuid = None
        try:
            self.uuid = str(torch.cuda.get_device_properties(device_index).uuid).lower()
        except Exception:
            pass

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(cmd, stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        mine = [r for r in rows if self.uuid and self.uuid in r[0].lower()]
        if mine:
            rows = mine
        elif len({r[0] for r in rows}) > 1:
            first = rows[0][0]
            rows = [r for r in rows if r[0] == first]

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [v for v in (num(r[1]) for r in rows) if v is not None]
        mx = [v for v in (num(r[2]) for r in rows) if v is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- our arm

class Path:
    """Device buffers and launches of one hot-path step."""

    def __init__(self, device, prefill_n=0, kcache_layout="group-major", grouping="half-split", page_size=0,
                 prefill_mode="grouped"):
        import dataclasses
        import rope_period_truncated_b200 as wp
        self.wp = wp
        self.prefill_mode = prefill_mode
        self.pw = syn.workload("long_32k")
        if prefill_n:
            self.pw = dataclasses.replace(self.pw, N=prefill_n)
        self.dw = syn.workload("decode_32k")
        pw, dw = self.pw, self.dw
        q, k, v = syn.prefill_inputs(pw)
        self.host_prefill = (q, k, v)
        self.q, self.k, self.v = q.to(device), k.to(device), v.to(device)
        self.qr, self.kr = torch.empty_like(self.q), torch.empty_like(self.k)
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((pw.B, pw.Hq, pw.N), dtype=torch.float32, device=device)
        # "paired": Q/K rotated half-split but written in the interleaved order, so
        # the groups hold whole channels and take the interleaved cutoffs
        paired = grouping == "paired" and pw.layout == wp.ROPE_HALF_SPLIT
        self.rope_layout = wp.ROPE_HALF_SPLIT_PAIRED if paired else pw.layout
        self.cut_layout = wp.ROPE_INTERLEAVED if paired else pw.layout
        self.wc, self.wg = wp.wp_cutoffs(pw.d, pw.theta, self.cut_layout, scale_all=pw.scale_all)
        dq, kc, vc, lens = syn.decode_inputs(dw)
        self.host_decode = (dq, lens)
        self.dq = dq.to(device).reshape(dw.B, 1, dw.Hq, dw.d)
        self.dqr = torch.empty_like(self.dq)
        # the K cache is stored group-major ([B, Hkv, d/16, L, 16]) unless asked
        # for rows: the keys a group skips are then contiguous and never read
        self.kc = kc.to(device)
        self.kc_rows = self.kc  # [B, Hkv, Lmax, d]: the layout of wp_decode's contract
        if kcache_layout == "group-major":
            self.kc = wp.wp_kcache_group_major(self.kc)
        self.vc = vc.to(device)
        self.page_size = page_size
        if page_size:
            # the same keys in a paged pool: pages shuffled, one block table per sequence
            B_, Hkv_, L_, d_ = vc.shape
            mp = L_ // page_size
            perm = torch.randperm(B_ * mp, generator=torch.Generator().manual_seed(7)).to(device)
            vpg = self.vc.reshape(B_, Hkv_, mp, page_size, d_).permute(0, 2, 1, 3, 4).reshape(B_ * mp, Hkv_,
                                                                                              page_size, d_)
            self.v_pages = torch.empty_like(vpg)
            self.v_pages[perm] = vpg
            if kcache_layout == "group-major":
                G_ = d_ // 16
                kpg = self.kc.reshape(B_, Hkv_, G_, mp, page_size, 16).permute(0, 3, 1, 2, 4, 5).reshape(
                    B_ * mp, Hkv_, G_, page_size, 16)
            else:
                kpg = self.kc.reshape(B_, Hkv_, mp, page_size, d_).permute(0, 2, 1, 3, 4).reshape(
                    B_ * mp, Hkv_, page_size, d_)
            self.k_pages = torch.empty_like(kpg)
            self.k_pages[perm] = kpg
            self.block_table = perm.to(torch.int32).reshape(B_, mp).contiguous()
            del vpg, kpg
        self.lens_host = lens
        self.lens = lens.to(device)
        self.pos = (lens - 1).to(torch.int32).reshape(dw.B, 1).to(device)
        self.do = torch.empty((dw.B, dw.Hq, dw.d), dtype=torch.bfloat16, device=device)
        self.dlse = torch.empty((dw.B, dw.Hq), dtype=torch.float32, device=device)
        self.ws = torch.empty(wp.wp_decode_workspace_bytes(dw.B, dw.Hq, dw.d, dw.Lmax), dtype=torch.uint8,
                              device=device)
        self.d_rope_layout = wp.ROPE_HALF_SPLIT_PAIRED if paired and dw.layout == wp.ROPE_HALF_SPLIT else dw.layout
        _, self.dwg = wp.wp_cutoffs(dw.d, dw.theta, wp.ROPE_INTERLEAVED if paired else dw.layout)
        self.launches_per_step = 6  # rope Q, rope K, prefill, rope q(decode), decode split, combine

    def prefill(self, cut="wave"):
        self.rope_prefill()
        return self.prefill_only(cut)

    def prefill_only(self, cut="wave"):
        if self.prefill_mode == "exact" and cut == "wave":
            return self.prefill_exact_only()
        return self.wp.wp_prefill(self.qr, self.kr, self.v, self.wg if cut == "wave" else None,
                                  self.wp.MODE_GROUPED, self.cut_layout, out=self.o, lse=self.lse)

    def prefill_exact_only(self):
        """The same prefill under the exact per-channel rule."""
        return self.wp.wp_prefill(self.qr, self.kr, self.v, self.wc, self.wp.MODE_CHANNEL, self.cut_layout,
                                  out=self.o, lse=self.lse)

    def decode(self, cut="wave"):
        wp, dw = self.wp, self.dw
        wp.wp_rope_apply(self.dq, dw.theta, self.d_rope_layout, pos=self.pos, out=self.dqr)
        return self.decode_only(cut)

    def decode_rows_only(self):
        """wp_decode on the K cache in rows [B, Hkv, Lmax, d] (its contract layout)."""
        dw = self.dw
        return self.wp.wp_decode(self.dqr.reshape(dw.B, dw.Hq, dw.d), self.kc_rows, self.vc, self.lens, self.dwg,
                                 out=self.do, lse=self.dlse, workspace=self.ws)

    def rope_prefill(self):
        wp, pw = self.wp, self.pw
        wp.wp_rope_apply(self.q, pw.theta, self.rope_layout, scale_all=pw.scale_all, out=self.qr)
        wp.wp_rope_apply(self.k, pw.theta, self.rope_layout, scale_all=pw.scale_all, out=self.kr)

    def decode_only(self, cut="wave"):
        dw = self.dw
        if self.page_size:
            return self.wp.wp_decode_paged(self.dqr.reshape(dw.B, dw.Hq, dw.d), self.k_pages, self.v_pages,
                                           self.block_table, self.lens, self.dwg if cut == "wave" else None,
                                           out=self.do, lse=self.dlse, workspace=self.ws)
        return self.wp.wp_decode(self.dqr.reshape(dw.B, dw.Hq, dw.d), self.kc, self.vc, self.lens,
                                 self.dwg if cut == "wave" else None, out=self.do, lse=self.dlse,
                                 workspace=self.ws)


def time_kernel(fn, iters, warmup):
    """Median per-launch time (ms) of fn() with CUDA events on the current stream."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
    for a, b in evs:
        a.record()
        fn()
        b.record()
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in evs)


def cpu_baseline(path: Path, target_s: float):
    """The fp64 oracle on sampled query rows of the 32K prefill, on this
    host's cores; returns pair-exact useful TFLOP/s of the sample."""
    import oracle
    pw = path.pw
    q, k, v = path.host_prefill
    threads = os.cpu_count() or 1
    kr = oracle.bf16_bits_to_f64(oracle.round_bf16_bits(
        oracle.rope(k.double().numpy(), pw.theta, pw.layout, scale_all=pw.scale_all)))
    vr = v.double().numpy()
    wg = np.asarray(path.wg, dtype=np.int64)

    def sample(nrows, seed):
        g = torch.Generator().manual_seed(seed)
        rh = torch.randint(0, pw.Hq, (nrows,), generator=g)
        ri = torch.randint(0, pw.N, (nrows,), generator=g)
        rb = torch.zeros(nrows, dtype=torch.int64)
        rows = q[rb, ri, rh].unsqueeze(0).unsqueeze(2)
        qrot = oracle.rope(rows.double().numpy(), pw.theta, pw.layout, pos=ri.numpy().reshape(1, -1),
                           scale_all=pw.scale_all)
        qrot = oracle.bf16_bits_to_f64(oracle.round_bf16_bits(qrot))[0, :, 0]
        keys = ri.numpy().astype(np.int64) + 1
        flops = 0.0
        for n in keys:
            delta = np.arange(n)
            flops += float(((delta[:, None] <= wg[None, :]).sum() * 2 * 16) + n * 2 * pw.d)
        t0 = time.perf_counter()
        oracle.attention_rows(qrot, (rb.numpy(), rh.numpy(), ri.numpy()), kr, vr, pw.Hq, path.wg,
                              oracle.MODE_GROUPED, pw.layout, nthreads=threads)
        return flops, time.perf_counter() - t0

    f0, t0 = sample(256, 1)
    nrows = int(min(65536, max(32, 256 * target_s / max(t0, 1e-3))))
    f1, t1 = sample(nrows, 2)
    if t1 < 0.5 * target_s and nrows < 65536:  # the small sample overestimated the per-row time
        nrows = int(min(65536, nrows * target_s / max(t1, 1e-3)))
        f1, t1 = sample(nrows, 3)
    return {"value": f1 / t1 / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"{nrows} random query rows (all heads) of the 32K prefill, fp64, {t1:.1f} s"}


def run_e2e(path: Path, K: int, tile_flops: float, world: int, dev):
    """The step through the public API with every per-step input copied from
    pinned host memory and every result copied back, timed on the device.

    Inputs and outputs are double-buffered on the device and copies run on
    their own streams, ordered by events: step s+1's host-to-device copies
    and step s-1's device-to-host copies overlap step s's kernels, as a
    serving loop would drive the calls."""
    pw, dw = path.pw, path.dw
    qh, kh, vh = (t.pin_memory() for t in path.host_prefill)
    dqh = path.host_decode[0].reshape(dw.B, 1, dw.Hq, dw.d).pin_memory()
    lensh = path.lens_host.pin_memory()
    posh = (path.lens_host - 1).to(torch.int32).reshape(dw.B, 1).pin_memory()
    host_in = (qh, kh, vh, dqh, lensh, posh)
    host_out = [tuple(torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (path.o, path.lse, path.do, path.dlse))
                for _ in range(2)]
    dev_in = [(path.q, path.k, path.v, path.dq, path.lens, path.pos)]
    dev_in.append(tuple(torch.empty_like(t) for t in dev_in[0]))
    dev_out = [(path.o, path.lse, path.do, path.dlse)]
    dev_out.append(tuple(torch.empty_like(t) for t in dev_out[0]))
    comp = torch.cuda.current_stream()
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def run(nsteps):
        in_free = [ev(), ev()]
        out_free = [ev(), ev()]
        for e in in_free + out_free:
            e.record(comp)
        t0, t1 = ev(), ev()
        t0.record(h2d)
        for s in range(nsteps):
            b = s % 2
            with torch.cuda.stream(h2d):
                h2d.wait_event(in_free[b])  # step s-2 no longer reads these buffers
                for d_, h_ in zip(dev_in[b], host_in):
                    d_.copy_(h_, non_blocking=True)
                in_ready = ev()
                in_ready.record(h2d)
            comp.wait_event(in_ready)
            comp.wait_event(out_free[b])  # step s-2's results have left the device
            path.q, path.k, path.v, path.dq, path.lens, path.pos = dev_in[b]
            path.o, path.lse, path.do, path.dlse = dev_out[b]
            path.prefill()
            path.decode()
            in_free[b] = ev()
            in_free[b].record(comp)
            done = ev()
            done.record(comp)
            with torch.cuda.stream(d2h):
                d2h.wait_event(done)
                for h_, d_ in zip(host_out[b], dev_out[b]):
                    h_.copy_(d_, non_blocking=True)
                out_free[b] = ev()
                out_free[b].record(d2h)
        t1.record(d2h)
        torch.cuda.synchronize()
        path.q, path.k, path.v, path.dq, path.lens, path.pos = dev_in[0]
        path.o, path.lse, path.do, path.dlse = dev_out[0]
        return t0.elapsed_time(t1)

    ke = max(3, min(K, 10))
    run(3)
    e_ms = run(ke) / ke
    e_ms = max_over_ranks([e_ms], dev)[0]
    h2d_b = sum(t.numel() * t.element_size() for t in host_in)
    d2h_b = sum(t.numel() * t.element_size() for t in host_out[0])
    return {"value": round(world * tile_flops / (e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "ms_per_step": round(e_ms, 3), "h2d_bytes_per_step": h2d_b, "d2h_bytes_per_step": d2h_b,
            "copies_declared": True,
            "note": "per-step inputs (Q, K, V, decode queries, lengths, positions) cross PCIe host-to-device and "
                    "outputs (O, LSE of prefill and decode) device-to-host every step, on copy streams that "
                    "overlap the neighbouring steps' kernels (double-buffered); the decode KV cache stays "
                    "resident in HBM (serving state)"}


def run_ours(args, rank, world, local):
    import rope_period_truncated_b200 as wp
    from rope_period_truncated_b200 import build as wpbuild
    wpbuild.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.prefill_mode != "grouped" and args.only != "prefill":
        raise SystemExit("--prefill-mode exact is a profiling case of --only prefill")
    path = Path(dev, args.prefill_n, args.kcache, args.grouping, args.page_size, args.prefill_mode)
    peaks, peak_kind = load_peaks()
    do_prefill = args.only in ("all", "prefill")
    do_decode = args.only in ("all", "decode")
    pw, dw = path.pw, path.dw
    tile_flops, pair_flops, dense_tile_flops = prefill_flops(pw.N, pw.d, pw.Hq, pw.B, path.wg)
    dec_bytes, dense_dec_bytes = decode_required_bytes(path.lens_host.numpy(), path.dwg, dw.B, dw.Hq, dw.Hkv, dw.d)

    def step(evp=None, evd=None, evr=None):
        if not do_prefill:
            pass
        elif evp is None:
            path.prefill()
        else:
            evr[0].record()
            path.rope_prefill()
            evr[1].record()
            evp[0].record()
            path.prefill_only()
            evp[1].record()
        if not do_decode:
            pass
        elif evd is None:
            path.decode()
        else:
            wp.wp_rope_apply(path.dq, dw.theta, path.d_rope_layout, pos=path.pos, out=path.dqr)
            evd[0].record()
            path.decode_only()
            evd[1].record()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if wp.wp_device_status() != 0:
        raise RuntimeError("device status word set during warm-up")
    if world > 1:
        torch.distributed.barrier()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    K = args.steps
    evp = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    evd = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    evr = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t_start.record()
    for s in range(K):
        step(evp[s], evd[s], evr[s])
    t_end.record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    total_ms = t_start.elapsed_time(t_end)
    prefill_ms = statistics.mean(a.elapsed_time(b) for a, b in evp) if do_prefill else float("nan")
    decode_ms = statistics.mean(a.elapsed_time(b) for a, b in evd) if do_decode else float("nan")
    rope_ms = statistics.mean(a.elapsed_time(b) for a, b in evr) if do_prefill else float("nan")
    if wp.wp_device_status() != 0:
        raise RuntimeError("device status word set during the timed steps")
    total_ms, prefill_ms, decode_ms, rope_ms = max_over_ranks([total_ms, prefill_ms, decode_ms, rope_ms], dev)
    ms_per_step = total_ms / K
    value = world * tile_flops / (ms_per_step * 1e-3) / 1e12

    # dense comparison: the same kernels with every cutoff infinite
    dense = None
    if not args.no_dense and args.only == "all":
        # dense and wave alternate (A B B A ...) so that the clock drift of the
        # power cap falls on both alike
        dps, wps, dds, wds = [], [], [], []
        for r in range(4):
            order = [("dense", dps, dds), ("wave", wps, wds)]
            for cut, pl, dl in (order if r % 2 == 0 else order[::-1]):
                pl.append(time_kernel(lambda: path.prefill_only(cut), 3, 1))
                dl.append(time_kernel(lambda: path.decode_only(cut), 10, 3))
        dpf, wpf = statistics.median(dps), statistics.median(wps)
        ddc, wdc = statistics.median(dds), statistics.median(wds)
        dense = {"prefill_ms": round(dpf, 4), "decode_ms": round(ddc, 5),
                 "prefill_speedup": round(dpf / wpf, 4), "decode_speedup": round(ddc / wdc, 4),
                 "prefill_dense_tflops": round(dense_tile_flops / (dpf * 1e-3) / 1e12, 2),
                 "decode_dense_gbs": round(dense_dec_bytes / (ddc * 1e-3) / 1e9, 1)}

    # wp_decode on the K cache in rows [B, Hkv, Lmax, d], the layout of its
    # contract (the step itself reads the K cache group-major)
    decode_rows = None
    if args.only == "all" and not args.page_size:
        rows_ms = statistics.median(time_kernel(path.decode_rows_only, 10, 3) for _ in range(3))
        rows_ms = max_over_ranks([rows_ms], dev)[0]
        rows_gbs = dec_bytes / (rows_ms * 1e-3) / 1e9
        decode_rows = {"kernel": "wp_decode, K cache in rows [B,Hkv,Lmax,d]", "bound": "hbm",
                       "value": round(rows_gbs, 1), "unit": "GB/s", "peak": peaks["hbm_gbs"],
                       "frac": round(rows_gbs / peaks["hbm_gbs"], 4), "kernel_ms": round(rows_ms, 5),
                       "required_bytes": dec_bytes}

    # wp_decode on a windowed K cache: every group keeps only the keys its
    # cutoff can still reach (the rest evicted)
    decode_windowed = None
    if args.only == "all" and not args.page_size:
        kwin = wp.wp_kcache_windowed(path.kc_rows, path.lens, path.dwg)
        win_ms = statistics.median(
            time_kernel(lambda: wp.wp_decode(path.dqr.reshape(dw.B, dw.Hq, dw.d), kwin, path.vc, path.lens,
                                             path.dwg, out=path.do, lse=path.dlse, workspace=path.ws), 10, 3)
            for _ in range(3))
        win_ms = max_over_ranks([win_ms], dev)[0]
        win_gbs = dec_bytes / (win_ms * 1e-3) / 1e9
        decode_windowed = {"kernel": "wp_decode, windowed K cache (per-group rings of round_up_16(W_g + 1) keys)",
                           "bound": "hbm", "value": round(win_gbs, 1), "unit": "GB/s", "peak": peaks["hbm_gbs"],
                           "frac": round(win_gbs / peaks["hbm_gbs"], 4), "kernel_ms": round(win_ms, 5),
                           "required_bytes": dec_bytes, "k_cache_bytes": kwin.numel() * 2,
                           "k_cache_bytes_full": path.kc_rows.numel() * 2,
                           "k_cache_kept": round(kwin.numel() / path.kc_rows.numel(), 4)}
        del kwin

    # backward of the 32K prefill (wp_prefill_backward), wave and dense
    backward = None
    if args.only in ("all", "backward") and not args.no_backward:
        dout = torch.randn(path.o.shape, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16).to(dev)
        dq, dk, dv = torch.empty_like(path.qr), torch.empty_like(path.kr), torch.empty_like(path.v)
        bw_useful, bw_dense = backward_flops(pw.N, pw.d, pw.Hq, pw.B, path.wg)
        path.prefill()  # O and LSE of the wave forward for the backward's inputs
        times = {}
        for cut in ("wave", "dense", "wave", "dense"):
            if cut == "dense":
                path.prefill_only("dense")
            else:
                path.prefill_only("wave")
            t = time_kernel(lambda: wp.wp_prefill_backward(path.qr, path.kr, path.v, path.o, path.lse, dout,
                                                           path.wg if cut == "wave" else None, dq=dq, dk=dk,
                                                           dv=dv), 2, 1)
            times.setdefault(cut, []).append(t)
        wave_ms, dense_ms = min(times["wave"]), min(times["dense"])
        wave_ms, dense_ms = max_over_ranks([wave_ms, dense_ms], dev)
        backward = {"kernel": "wp_prefill_backward (delta + dQ + dK/dV on tcgen05)",
                    "ms": round(wave_ms, 3), "dense_ms": round(dense_ms, 3),
                    "useful_tflops": round(bw_useful / (wave_ms * 1e-3) / 1e12, 2),
                    "dense_tflops": round(bw_dense / (dense_ms * 1e-3) / 1e12, 2),
                    "speedup_over_dense": round(dense_ms / wave_ms, 4),
                    "useful_flops": bw_useful, "peak": peaks["bf16_tflops"],
                    "frac": round(bw_useful / (wave_ms * 1e-3) / 1e12 / peaks["bf16_tflops"], 4),
                    "note": "useful FLOPs pair exact: 3 group-masked products (S, dQ, dK) + 2 full (dP, dV); the "
                            "kernels recompute S and dP in both passes (7 products)"}
        del dout, dq, dk, dv
        path.prefill()  # the wave forward's outputs again

    # the same 32K prefill under the exact per-channel rule (wp_prefill, MODE_CHANNEL)
    exact = None
    if args.only == "all" and not args.no_exact:
        path.rope_prefill()
        ex_flops = exact_flops(pw.N, pw.d, pw.Hq, pw.B, path.wc)
        ex_ms = statistics.median(time_kernel(path.prefill_exact_only, 3, 1) for _ in range(3))
        ex_ms = max_over_ranks([ex_ms], dev)[0]
        exact = {"kernel": "wp_prefill, exact per-channel rule (tcgen05 products of full and partially kept "
                           "groups, rank-2 updates of boundary channels)",
                 "ms": round(ex_ms, 3), "grouped_ms": round(prefill_ms, 3),
                 "useful_tflops": round(ex_flops / (ex_ms * 1e-3) / 1e12, 2), "useful_flops": ex_flops,
                 "peak": peaks["bf16_tflops"],
                 "frac": round(ex_flops / (ex_ms * 1e-3) / 1e12 / peaks["bf16_tflops"], 4),
                 "traffic": (profiled_traffic("prefill_exact_kernel_32k_dram.txt",
                                              "rope_period_truncated_b200/csrc/wp_prefill_exact.cu")
                             if args.prefill_n in (0, 32768) and args.grouping == "half-split" else None),
                 "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)",
                 "note": "useful FLOPs pair exact: 4 per kept channel per pair (its two dims) + 2*d for PV"}
        path.prefill()  # the grouped forward's outputs again

    # end to end through the public API with pinned host buffers
    e2e = None
    if not args.no_e2e and args.only == "all":
        e2e = run_e2e(path, K, tile_flops, world, dev)

    # Each prefill launch is timed on its own (a few ms inside a sub-second
    # region), so the denominator is the measured burst GEMM rate; the
    # fraction of the sustained rate is printed beside it.
    peak_t = peaks["bf16_tflops"]
    rope_bytes = 2 * 2 * (path.q.numel() + path.k.numel())  # read + write of Q and K, bf16
    achieved = tile_flops / (prefill_ms * 1e-3) / 1e12
    dec_gbs = dec_bytes / (decode_ms * 1e-3) / 1e9
    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": bench_config(args, world, path.wg),
        "roofline": {
            "kernel": "wp_prefill (grouped, tcgen05)",
            "bound": "tensor",
            "achieved": round(achieved, 2),
            "peak": peak_t,
            "unit": "TFLOP/s",
            "frac": round(achieved / peak_t, 4),
            "peak_kind": f"{peak_kind} bf16 dense burst",
            "frac_of_burst": round(achieved / peaks["bf16_tflops"], 4),
            "frac_of_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4),
            "traffic": (profiled_traffic("prefill_grouped_kernel_32k_dram.txt",
                                         "rope_period_truncated_b200/csrc/wp_prefill.cu")
                        if args.prefill_n in (0, 32768) and args.grouping == "half-split" else None),
            "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)",
            "kernel_ms": round(prefill_ms, 4),
            "flops_per_launch": tile_flops,
            "pair_exact_flops_per_launch": pair_flops,
            "pair_exact_tflops": round(pair_flops / (prefill_ms * 1e-3) / 1e12, 2),
        },
        "decode": {
            "kernel": "wp_decode (split + combine)",
            "bound": "hbm",
            "value": round(dec_gbs, 1),
            "unit": "GB/s",
            "peak": peaks["hbm_gbs"],
            "frac": round(dec_gbs / peaks["hbm_gbs"], 4),
            "kernel_ms": round(decode_ms, 5),
            "required_bytes": dec_bytes,
        },
        "decode_rows": decode_rows,
        "decode_windowed": decode_windowed,
        "rope": ({"kernel": "wp_rope_apply of Q and K (2 launches)", "bound": "hbm",
                  "value": round(rope_bytes / (rope_ms * 1e-3) / 1e9, 1), "unit": "GB/s", "peak": peaks["hbm_gbs"],
                  "frac": round(rope_bytes / (rope_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                  "kernel_ms": round(rope_ms, 5), "bytes_per_step": rope_bytes} if do_prefill else None),
        "dense_comparison": dense,
        "backward": backward,
        "exact": exact,
        "e2e": e2e,
        "gpu_launches": {"all": 6, "prefill": 3, "decode": 3, "backward": 0}[args.only] * K,
        "clocks": clk,
        "paper_context": {"source": "A100 FlashWavePrune vs FlashAttention-2, d128, theta 1e6 (context only)",
                          "prefill_speedup_32k": 1.15, "decode_speedup_32k": 1.24},
    }
    if args.only != "all" or args.prefill_n:
        out["note"] = "restricted profiling case, not a bench line"
    if rank == 0 and not args.no_cpu_baseline and world == 1 and args.only == "all" and args.grouping == "half-split":
        out["cpu_baseline"] = cpu_baseline(path, args.cpu_seconds)
    return out


# ----------------------------------------------------------------------------- reference arm

def run_reference(args, world=1):
    """The fp64 oracle as the reference arm: each step is a bounded sample of
    query rows of the 32K prefill, timed on the host cores."""
    import oracle
    oracle.build()
    pw = syn.workload("long_32k")
    q, k, v = syn.prefill_inputs(pw)
    _, wg = oracle.cutoffs(pw.d, pw.theta, pw.layout, scale_all=pw.scale_all)
    kr = oracle.bf16_bits_to_f64(oracle.round_bf16_bits(
        oracle.rope(k.double().numpy(), pw.theta, pw.layout, scale_all=pw.scale_all)))
    vr = v.double().numpy()
    threads = os.cpu_count() or 1
    rows_per_step = 64
    wgl = np.asarray(wg, dtype=np.int64)

    def one(seed):
        g = torch.Generator().manual_seed(seed)
        rh = torch.randint(0, pw.Hq, (rows_per_step,), generator=g)
        ri = torch.randint(0, pw.N, (rows_per_step,), generator=g)
        rb = torch.zeros(rows_per_step, dtype=torch.int64)
        rows = q[rb, ri, rh].unsqueeze(0).unsqueeze(2)
        qrot = oracle.rope(rows.double().numpy(), pw.theta, pw.layout, pos=ri.numpy().reshape(1, -1))
        qrot = oracle.bf16_bits_to_f64(oracle.round_bf16_bits(qrot))[0, :, 0]
        flops = 0.0
        for n in ri.numpy().astype(np.int64) + 1:
            delta = np.arange(n)
            flops += float(((delta[:, None] <= wgl[None, :]).sum() * 2 * 16) + n * 2 * pw.d)
        t0 = time.perf_counter()
        oracle.attention_rows(qrot, (rb.numpy(), rh.numpy(), ri.numpy()), kr, vr, pw.Hq, wg,
                              oracle.MODE_GROUPED, pw.layout, nthreads=threads)
        return flops, time.perf_counter() - t0

    for s in range(args.warmup):
        one(100 + s)
    tot_f = tot_t = 0.0
    for s in range(args.steps):
        f, t = one(1000 + s)
        tot_f += f
        tot_t += t
    value = tot_f / tot_t / 1e12
    sample = f"{rows_per_step} random query rows of the 32K prefill per step, fp64 oracle, {threads} threads"
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(args, world, wg),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    rank, world, local = dist_env()
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, world)), flush=True)
        return
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                             device_id=torch.device("cuda", local))
    try:
        out = run_ours(args, rank, world, local)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()

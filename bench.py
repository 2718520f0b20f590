#!/usr/bin/env python3
"""Benchmark of the HiLS attention forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--extra/--no-extra] [--no-cpu-baseline]

One step = one pass of the whole prefill hot path over the workload's
synthetic batch: landmark scoring + inter-chunk normaliser + top-k
(hils_select), then the chunk union, intra-chunk attention and fusion
(hils_attn_fwd, which builds each tile's union itself).  Default workload:
the 512K-token 7B-shaped prefill (B=1, 32/8 heads, d=128, k=64, M=128).
The 128K prefill, the B=16 x 512K decode step, the same decode step over a
paged KV cache (hils_decode_fwd_paged, shuffled page pool) and the HoPE
pre-pass over the 512K q and k (hils_hope) are timed as extra lines inside
the same JSON object ("workloads").

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and
cuda synchronize, CUDA events on the launching stream, max over ranks.
Inputs (q alone is 4.3 GB) are larger than the 126 MB L2, so no flush is
needed between steps.  Multi-GPU (torchrun): every rank runs its own
independent batch (different seed); value = all ranks' query tokens / the
slowest rank's time ("weak" scaling, no collective on the data path).

`--impl reference` times the CPU oracle (the reference implementation of
this project, plain fp64 C) on the host cores for the same workload: a
bounded sample of rows per step, scaled to query-tokens/s.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from chunk_wise_hierarchical_landmark_b200 import workloads as W  # noqa: E402

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
CSRC = os.path.join(ROOT, "chunk_wise_hierarchical_landmark_b200", "csrc")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------
# algorithmic work

def prefill_work(w: W.Workload) -> dict:
    """Algorithmic FLOPs of one prefill over all heads (exact sums over t).
    Scoring: 2*d FLOP per (row, completed chunk).  Attention: 4*d FLOP per
    (row, attended key) -- QK^T and PV -- over min(k, n_c) full chunks plus
    the t mod C + 1 causal keys of the own chunk."""
    t = np.arange(w.L, dtype=np.int64)
    n_c = t // w.C
    keys = np.minimum(w.topk, n_c) * w.C + (t % w.C) + 1
    heads = w.B * w.Hq
    return {"score_flop": float(2 * w.d * n_c.sum() * heads),
            "attn_flop": float(4 * w.d * keys.sum() * heads),
            "candidates": float(n_c.sum() * heads)}


def select_executed_flop(w: W.Workload) -> float:
    """Tensor-core FLOPs the scoring kernel executes over all heads: each
    128-row tile multiplies its Q tile [128 x d] by one 64-row tile of seed
    landmarks when n > 0, n = the completed chunks of the tile's last row,
    and, when n > k (some candidate is not a seed), by ceil(n / 64) landmark
    tiles of 64 rows with one extra K = 16 step each (the masking step), the
    rows before the last using a triangle of that."""
    ntiles = -(-w.L // 128)
    t_last = np.minimum(np.arange(ntiles, dtype=np.int64) * 128 + 127, w.L - 1)
    n = np.minimum(t_last // w.C, w.L // w.C)
    seed = (n > 0).astype(np.int64) * w.d
    scan = np.where(n > w.topk, -(-n // 64), 0) * (w.d + 16)
    return float((seed + scan).sum() * 2 * 128 * 64 * w.B * w.Hq)


def attn_executed_flop(w: W.Workload, tile_union_sizes) -> float:
    """Tensor-core FLOPs the attention kernel executes: every 128-row tile
    runs S = Q K^T (2*128*64*d) and O += P V (2*128*64*d) for each chunk of
    its union (own chunks included), whichever of its rows selected it."""
    return float(np.asarray(tile_union_sizes, dtype=np.float64).sum() * 4 * 128 * 64 * w.d)


def near_tie_sample(w: W.Workload, q, lmk, sel, n_rows=384, seed=0) -> dict:
    """Sampled check of the selection of the timed run: for n_rows rows the
    landmark logits of all completed chunks are formed on the host in fp64
    (plain torch matmul, rounded to fp32 where the kernel decides), ranked by
    (logit desc, chunk asc), and compared with the GPU's sel_idx.  A near-tie
    row has its k-th and (k+1)-th logits within 1e-4 * max(1, |s_k|)."""
    G = w.Hq // w.Hkv
    rng = np.random.default_rng(seed)
    rows = rng.integers(0, w.B * w.Hq * w.L, size=n_rows)
    near = mism = outside = 0
    for r in rows.tolist():
        bh, t = divmod(r, w.L)
        b, hq = divmod(bh, w.Hq)
        n_c = min(t // w.C, w.L // w.C)
        got = sel[b, hq, t].cpu().numpy()
        if n_c == 0:
            continue
        qv = q[b, hq, t].double().cpu()
        lk = lmk[b, hq // G, :n_c].double().cpu()
        s = ((lk @ qv) * w.scale).float().double().numpy()
        order = np.lexsort((np.arange(n_c), -s))
        want = np.sort(order[:w.topk])
        is_near = False
        if n_c > w.topk:
            sk, sk1 = s[order[w.topk - 1]], s[order[w.topk]]
            is_near = abs(sk - sk1) < 1e-4 * max(1.0, abs(sk))
        near += int(is_near)
        g = got[got >= 0]
        if not np.array_equal(np.sort(g), want):
            mism += 1
            outside += int(not is_near)
    return {"rows": int(n_rows), "near_ties": near, "index_mismatches": mism,
            "mismatches_outside_near_ties": outside,
            "how": "logits of all completed chunks in fp64 on the host (torch), ranked "
                   "(logit desc, chunk asc); rows sampled uniformly over (b, head, position)"}


def decode_bytes(w: W.Workload, sel: torch.Tensor) -> float:
    """Algorithmic HBM bytes of one decode step: every landmark key of every
    (b, hkv), plus the K and V of the union of chunks the G query heads of a
    KV head attend (selected chunks and the own chunk), each read once."""
    esize = 2 if w.dtype == "bf16" else 4
    G = w.Hq // w.Hkv
    lmk = w.B * w.Hkv * (w.L // w.C) * w.d * esize
    s = sel.reshape(w.B, w.Hkv, G * w.topk).cpu().numpy()
    own = (w.L - 1) // w.C
    chunks = 0
    for b in range(w.B):
        for h in range(w.Hkv):
            u = set(int(c) for c in s[b, h] if c >= 0)
            u.add(own)
            chunks += len(u)
    last = w.L - own * w.C  # keys in the own chunk
    kv = (chunks - w.B * w.Hkv) * w.C + w.B * w.Hkv * last
    return float(lmk + 2 * kv * w.d * esize)


def source_hash(files):
    h = hashlib.sha256()
    for f in sorted(files):
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            return json.load(f), "measured"
    except OSError:
        return FALLBACK_PEAKS, "fallback"


def load_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu capture, or None when the
    kernel's source changed since the capture."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f).get(kernel)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("workload") != workload:
        return None
    if rec.get("source_hash") != source_hash(rec.get("sources", [])):
        return None
    return rec.get("bytes_per_launch")


# ---------------------------------------------------------------------------
# clocks

class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""
    Q = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.uuid = None
        try:
            self.uuid = str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            pass
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "200"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=10)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        rows = []
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 10:
                continue
            if self.uuid and self.uuid.replace("GPU-", "") not in f[1]:
                continue
            rows.append(f)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(rows[0][3]) if rows[0][3].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# distributed helpers

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(x: float, ws: int) -> float:
    """Largest value over all ranks (the slowest rank's time)."""
    if ws == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(tokens_per_rank: int, ms_per_rank: float, ws: int) -> float:
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * ws / (max_over_ranks(ms_per_rank, ws) * 1e-3)


def barrier(ws):
    if ws > 1:
        torch.distributed.barrier()


# ---------------------------------------------------------------------------
# our arm

def bench_prefill(hb, synth, w, steps, warmup, ws, rank, seed_offset, e2e=True, clocks=True):
    dev = torch.device("cuda")
    q, k, v, lmk = synth.make_inputs(w, "cuda", seed=w.seed + seed_offset)
    p = hb.make_params(w.B, w.Hq, w.Hkv, w.L, w.d, w.topk, w.M, w.C, w.scale,
                       q.dtype, False)
    B, Hq, L, K = w.B, w.Hq, w.L, w.topk
    sel = torch.empty((B, Hq, L, K), dtype=torch.int32, device=dev)
    cw = torch.empty((B, Hq, L, K), dtype=torch.float32, device=dev)
    lse_lmk = torch.empty((B, Hq, L), dtype=torch.float32, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty((B, Hq, L), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        hb.hils_select(p, q, lmk, sel, cw, lse_lmk, None, stream)
        if ev is not None:
            ev[1].record(stream)
        hb.hils_attn_fwd(p, q, k, v, sel, cw, out, lse, None, None, stream)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    n0 = hb.launch_count()
    sampler = ClockSampler(torch.cuda.current_device()) if clocks else None
    if sampler:
        sampler.__enter__()
    barrier(ws)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        step(evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    if sampler:
        sampler.__exit__(None, None, None)
    launches = hb.launch_count() - n0
    ms = t0.elapsed_time(t1) / steps
    sel_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    attn_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    res = dict(ms=ms, sel_ms=sel_ms, attn_ms=attn_ms, launches=launches,
               clocks=sampler.summary() if sampler else None)

    if e2e:
        hq, hk, hv, hl = (x.cpu().pin_memory() for x in (q, k, v, lmk))
        ho = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        hlse = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
        # End to end through the public call, pipelined over the (b, kv-head)
        # groups: the inputs of group i+1 cross the host link while group i
        # computes and group i-1's output travels back (three streams).  Each
        # group is one hils_prefill call on its own KV head and G query heads.
        G = Hq // w.Hkv
        sub_p = hb.make_params(1, G, 1, w.L, w.d, w.topk, w.M, w.C, w.scale, q.dtype, False)
        groups = [(bb, h) for bb in range(B) for h in range(w.Hkv)]

        def views(bb, h):
            qs_ = slice(h * G, (h + 1) * G)
            ks_ = slice(h, h + 1)
            return dict(q=(q[bb, qs_], hq[bb, qs_]), k=(k[bb, ks_], hk[bb, ks_]),
                        v=(v[bb, ks_], hv[bb, ks_]), lmk=(lmk[bb, ks_], hl[bb, ks_]),
                        out=(out[bb, qs_], ho[bb, qs_]), lse=(lse[bb, qs_], hlse[bb, qs_]),
                        sel=sel[bb, qs_], cw=cw[bb, qs_], lse_lmk=lse_lmk[bb, qs_])

        gv = [views(bb, h) for bb, h in groups]
        s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        done_prev = [None] * len(groups)

        def e2e_step():
            for i, g in enumerate(gv):
                with torch.cuda.stream(s_in):
                    if done_prev[i] is not None:  # the previous step's compute read these buffers
                        s_in.wait_event(done_prev[i])
                    for key in ("q", "k", "v", "lmk"):
                        g[key][0].copy_(g[key][1], non_blocking=True)
                    ev_in = torch.cuda.Event()
                    ev_in.record(s_in)
                s_cmp.wait_event(ev_in)
                hb.hils_prefill(sub_p, g["q"][0], g["k"][0], g["v"][0], g["lmk"][0], g["sel"],
                                g["cw"], g["lse_lmk"], g["out"][0], g["lse"][0], None, s_cmp)
                ev_c = torch.cuda.Event()
                ev_c.record(s_cmp)
                done_prev[i] = ev_c
                s_out.wait_event(ev_c)
                with torch.cuda.stream(s_out):
                    g["out"][1].copy_(g["out"][0], non_blocking=True)
                    g["lse"][1].copy_(g["lse"][0], non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        barrier(ws)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(s_in)
        s_cmp.wait_stream(s_in)
        s_out.wait_stream(s_in)
        n_e2e = max(1, steps)
        for _ in range(n_e2e):
            e2e_step()
        s_out.wait_stream(s_in)
        s_out.wait_stream(s_cmp)
        b.record(s_out)
        torch.cuda.synchronize()
        barrier(ws)
        res["e2e_ms"] = a.elapsed_time(b) / n_e2e
        res["h2d"] = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hl))
        res["d2h"] = ho.numel() * ho.element_size() + hlse.numel() * hlse.element_size()
        res["host_inputs"] = (hq, hk, hv, hl)
    res["sel"] = sel
    res["inputs"] = (q, lmk)
    return res


def bench_decode(hb, synth, w, steps, warmup, seed_offset, paged=False):
    dev = torch.device("cuda")
    q, k, v, lmk = synth.make_inputs(w, "cuda", seed=w.seed + seed_offset)
    p = hb.make_params(w.B, w.Hq, w.Hkv, w.L, w.d, w.topk, w.M, w.C, w.scale, q.dtype, False)
    sel = torch.empty((w.B, w.Hq, w.topk), dtype=torch.int32, device=dev)
    cw = torch.empty_like(sel, dtype=torch.float32)
    lse_lmk = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)
    ws_t = hb.workspace(p, hb.HILS_OP_DECODE, dev)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        hb.hils_decode_fwd(p, q, k, v, lmk, sel, cw, lse_lmk, out, lse, ws_t, stream)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        hb.hils_decode_fwd(p, q, k, v, lmk, sel, cw, lse_lmk, out, lse, ws_t, stream)
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    nbytes = decode_bytes(w, sel)
    res = dict(ms=ms, bytes=nbytes)
    if paged:
        # the same step over a paged cache: pages of one 64-token chunk of
        # every KV head, the pool in a random order (a fragmented pool)
        dense_out, dense_sel = out.clone(), sel.clone()
        npg = -(-w.L // w.C)
        g = torch.Generator(device=dev).manual_seed(w.seed + 17 + seed_offset)
        perm = torch.randperm(w.B * npg, generator=g, device=dev)
        table = perm.view(w.B, npg).to(torch.int32)
        kp = torch.zeros((w.B * npg, w.Hkv, w.C, w.d), dtype=k.dtype, device=dev)
        vp = torch.zeros_like(kp)
        for bb in range(w.B):
            idx = perm[bb * npg:(bb + 1) * npg]
            full = (w.L // w.C) * w.C
            kb = k[bb, :, :full].reshape(w.Hkv, w.L // w.C, w.C, w.d).transpose(0, 1)
            vb = v[bb, :, :full].reshape(w.Hkv, w.L // w.C, w.C, w.d).transpose(0, 1)
            kp.index_copy_(0, idx[:w.L // w.C], kb)
            vp.index_copy_(0, idx[:w.L // w.C], vb)
            if full < w.L:
                kp[idx[-1], :, :w.L - full] = k[bb, :, full:]
                vp[idx[-1], :, :w.L - full] = v[bb, :, full:]
        del k, v
        torch.cuda.empty_cache()
        for _ in range(warmup):
            hb.hils_decode_fwd_paged(p, q, kp, vp, table, lmk, sel, cw, lse_lmk, out, lse, ws_t,
                                     stream)
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(steps):
            hb.hils_decode_fwd_paged(p, q, kp, vp, table, lmk, sel, cw, lse_lmk, out, lse, ws_t,
                                     stream)
        b.record(stream)
        torch.cuda.synchronize()
        res["paged_ms"] = a.elapsed_time(b) / steps
        res["paged_pages"] = w.B * npg
        res["paged_equal"] = bool(torch.equal(out, dense_out) and torch.equal(sel, dense_sel))
    return res


def bench_hope(hb, w, steps, warmup, train_len=65536, base=500000.0):
    """The HoPE pre-pass (hils_hope) over q and k of workload w, in place:
    the pairs whose wavelength fits train_len are rotated.  HBM-bound; the
    algorithmic bytes are the rotated elements read and written once."""
    dev = torch.device("cuda")
    g = torch.Generator(device=dev).manual_seed(w.seed + 23)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    q = torch.randn((w.B, w.Hq, w.L, w.d), generator=g, device=dev).to(dt)
    k = torch.randn((w.B, w.Hkv, w.L, w.d), generator=g, device=dev).to(dt)
    npairs = hb.rope_pairs_for(w.d, base, train_len)
    stream = torch.cuda.current_stream()

    def step():
        hb.hils_hope(q, npairs, 0, base, stream)
        hb.hils_hope(k, npairs, 0, base, stream)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    nbytes = 2.0 * 2 * npairs * (w.Hq + w.Hkv) * w.B * w.L * q.element_size()
    return dict(ms=ms, bytes=nbytes, npairs=npairs)


def bench_hope_fused(hb, synth, w, steps, warmup, train_len=65536, base=500000.0):
    """Prefill with HoPE on the queries two ways: the query pre-pass
    (hils_hope over q, into a copy) followed by hils_prefill, and
    hils_prefill_hope, which rotates each query tile as the kernels stage
    it.  The keys are rotated once beforehand in both (a cache holds them
    rotated).  The two must agree bit for bit."""
    dev = torch.device("cuda")
    q, k, v, lmk = synth.make_inputs(w, dev)
    npairs = hb.rope_pairs_for(w.d, base, train_len)
    hb.hils_hope(k, npairs, 0, base)
    p = hb.make_params(w.B, w.Hq, w.Hkv, w.L, w.d, w.topk, w.M, w.C, w.scale, q.dtype)
    ws_t = hb.workspace(p, hb.HILS_OP_PREFILL, dev)
    outs = []
    for _ in range(2):
        outs.append(dict(sel=torch.empty((w.B, w.Hq, w.L, w.topk), dtype=torch.int32, device=dev),
                         cw=torch.empty((w.B, w.Hq, w.L, w.topk), dtype=torch.float32,
                                        device=dev),
                         ll=torch.empty((w.B, w.Hq, w.L), dtype=torch.float32, device=dev),
                         out=torch.empty_like(q),
                         lse=torch.empty((w.B, w.Hq, w.L), dtype=torch.float32, device=dev)))
    q_rot = torch.empty_like(q)
    stream = torch.cuda.current_stream()

    def two_step():
        o = outs[0]
        q_rot.copy_(q)
        hb.hils_hope(q_rot, npairs, 0, base, stream)
        hb.hils_prefill(p, q_rot, k, v, lmk, o["sel"], o["cw"], o["ll"], o["out"], o["lse"],
                        ws_t, stream)

    def fused():
        o = outs[1]
        hb.hils_prefill_hope(p, q, k, v, lmk, 0, npairs, base, o["sel"], o["cw"], o["ll"],
                             o["out"], o["lse"], ws_t, stream)

    res = dict(npairs=npairs)
    for name, fn in (("prepass_ms", two_step), ("fused_ms", fused)):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        res[name] = a.elapsed_time(b) / steps
    res["equal"] = all(torch.equal(outs[0][n].view(torch.int32) if outs[0][n].dtype ==
                                   torch.float32 else outs[0][n],
                                   outs[1][n].view(torch.int32) if outs[1][n].dtype ==
                                   torch.float32 else outs[1][n]) for n in outs[0])
    return res


def tile_union_sizes(hb, sel):
    """Union size of every 128-row tile (the unit the attention kernel walks)."""
    u_off, _ = hb.union(sel, M=128)
    return (u_off[1:] - u_off[:-1]).cpu().numpy()


def backward_work(w: W.Workload) -> float:
    """Algorithmic FLOPs of one backward pass over all heads: per (row,
    attended key) the logit recomputed (2d), dP = <dO, v> (2d), and the dq,
    dk and dv updates (2d each) -- 10d, the attention-backward count -- plus
    4d per (row, selected chunk) for the landmark gradients (ds lmk into dq,
    ds q into dlmk)."""
    t = np.arange(w.L, dtype=np.int64)
    n_c = t // w.C
    keys = np.minimum(w.topk, n_c) * w.C + (t % w.C) + 1
    heads = w.B * w.Hq
    return float((10 * w.d * keys.sum() + 4 * w.d * np.minimum(w.topk, n_c).sum()) * heads)


def bench_backward(hb, synth, w, steps, warmup):
    """hils_attn_bwd for the forward's selection on workload w (seeded dout
    and dlse); fp32 arithmetic on the CUDA cores."""
    dev = torch.device("cuda")
    q, k, v, lmk = synth.make_inputs(w, "cuda", seed=w.seed)
    g = torch.Generator(device=dev).manual_seed(w.seed + 41)
    dout = torch.randn(q.shape, generator=g, device=dev).to(q.dtype)
    dlse = torch.randn(q.shape[:3], generator=g, device=dev)
    sel, cw, _ = hb.select(q, lmk, w.topk, w.M)
    _, lse, _ = hb.attn_fwd(q, k, v, sel, cw, w.M)
    p = hb.make_params(w.B, w.Hq, w.Hkv, w.L, w.d, w.topk, w.M, w.C, w.scale, q.dtype, False)
    dq = torch.empty(q.shape, dtype=torch.float32, device=dev)
    dk = torch.empty(k.shape, dtype=torch.float32, device=dev)
    dv = torch.empty(v.shape, dtype=torch.float32, device=dev)
    dl = torch.empty(lmk.shape, dtype=torch.float32, device=dev)
    ws = torch.empty(hb.lib().hils_attn_bwd_workspace_size(ctypes.byref(p)), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream()

    def step():
        hb.hils_attn_bwd(p, q, k, v, lmk, sel, cw, lse, dout, dlse, dq, dk, dv, dl, ws, stream)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    n0 = hb.launch_count()
    a.record(stream)
    for _ in range(steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    launches = hb.launch_count() - n0
    ms = a.elapsed_time(b) / steps
    flop = backward_work(w)
    return {"value": w.B * w.L / (ms * 1e-3), "unit": "query-tokens/s", "ms_per_step": ms,
            "algorithmic_tflops": flop / (ms * 1e-3) / 1e12, "bound": "alu",
            "workspace_bytes": ws.numel(), "launches": launches}


def bench_qcal(hb, synth, w, steps, warmup, r=32):
    """The Q-Cal prefill of workload w: the calibrated scoring query
    (hils_qcal_query: z = W_down h per position, q + W_up z per head) timed
    alone and as part of hils_prefill_qcal.  h [B, L, Hq*d] and the weights
    are seeded random data of the model's shapes (no trained weights)."""
    dev = torch.device("cuda")
    q, k, v, lmk = synth.make_inputs(w, "cuda", seed=w.seed)
    D = w.Hq * w.d
    g = torch.Generator(device=dev).manual_seed(w.seed + 31)
    h = torch.randn((w.B, w.L, D), generator=g, device=dev).to(q.dtype)
    wd = (torch.randn((r, D), generator=g, device=dev) / D ** 0.5).to(q.dtype)
    # a calibration: the offset is about a tenth of the query (|z| ~ 1 per rank)
    wu = (torch.randn((w.Hq, w.d, r), generator=g, device=dev) * (0.1 / r ** 0.5)).to(q.dtype)
    p = hb.make_params(w.B, w.Hq, w.Hkv, w.L, w.d, w.topk, w.M, w.C, w.scale, q.dtype, False)
    B, Hq, L, K = w.B, w.Hq, w.L, w.topk
    sel = torch.empty((B, Hq, L, K), dtype=torch.int32, device=dev)
    cw = torch.empty((B, Hq, L, K), dtype=torch.float32, device=dev)
    lse_lmk = torch.empty((B, Hq, L), dtype=torch.float32, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty((B, Hq, L), dtype=torch.float32, device=dev)
    q_cal = torch.empty_like(q)
    ws = hb.qcal_workspace(p, r, dev)
    stream = torch.cuda.current_stream()

    def timed(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / steps

    ms_q = timed(lambda: hb.hils_qcal_query(p, q, h, wd, wu, q_cal, ws, stream))
    ms_all = timed(lambda: hb.hils_prefill_qcal(p, q, k, v, lmk, h, wd, wu, q_cal, sel, cw,
                                                lse_lmk, out, lse, ws, stream))
    esz = q.element_size()
    nbytes = float(w.B * L * D * esz + 2 * q.numel() * esz + r * D * esz + Hq * w.d * r * esz)
    return {"value": B * L / (ms_all * 1e-3), "unit": "query-tokens/s", "ms_per_step": ms_all,
            "qcal_query_ms": ms_q, "rank": r, "hidden": D,
            "qcal_query_bytes": nbytes, "qcal_query_gbs": nbytes / (ms_q * 1e-3) / 1e9,
            "inputs": "seeded random h and weights of the model's shapes; offset about 0.1 x the query"}


def union_stats(hb, sel, w):
    """Chunk-union size per group of M rows and adjacent-query overlap."""
    u_off, _ = hb.union(sel, M=w.M)
    sizes = (u_off[1:] - u_off[:-1]).float()
    s = sel.reshape(-1, w.L, w.topk)
    h = min(4, s.shape[0])
    ov = []
    for i in range(h):
        a = s[i, w.topk * w.C + 1:-1].cpu().numpy()
        bb = s[i, w.topk * w.C + 2:].cpu().numpy()
        inter = [(len(set(x) & set(y)) / w.topk) for x, y in zip(a[::97], bb[::97])]
        ov.extend(inter)
    return {"union_mean": round(sizes.mean().item(), 2),
            "union_p50": float(sizes.median().item()),
            "union_p99": float(torch.quantile(sizes, 0.99).item()),
            "adjacent_overlap": round(float(np.mean(ov)) if ov else float("nan"), 4),
            "pages_adjacent_overlap": 0.928}


def alu_peak_tflops(clocks) -> float:
    """fp32 CUDA-core peak: 148 SMs x 128 FMA lanes x 2 FLOP per clock, at the
    median SM clock sampled during the main timed region (the maximum clock
    when none was sampled)."""
    mhz = None
    if clocks:
        mhz = clocks.get("sm_mhz") or clocks.get("sm_max_mhz")
    return 148 * 128 * 2 * (mhz or 1965.0) * 1e6 / 1e12


def cpu_baseline(w, host_inputs, budget_s=15.0):
    """The oracle, as it stands, on all host cores over a bounded sample of
    rows of the same workload; scaled to query-tokens/s."""
    import oracle
    q, k, v, lmk = host_inputs
    p = oracle.Problem(w.B, w.Hq, w.Hkv, w.L, w.d, w.C, w.topk, w.scale)
    cores = os.cpu_count() or 1
    rng = np.random.default_rng(w.seed)
    rows_per_try = max(cores, 8)
    done = 0
    t_total = 0.0
    while t_total < budget_s and done < 1 << 20:
        rows = rng.integers(0, w.B * w.Hq * w.L, size=rows_per_try)
        t0 = time.perf_counter()
        oracle.rows(p, q, k, v, lmk, rows, nthreads=cores)
        t_total += time.perf_counter() - t0
        done += rows_per_try
        rows_per_try = min(rows_per_try * 2, 4096)
    rows_per_s = done / t_total
    return {"value": rows_per_s / w.Hq, "unit": "query-tokens/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{done} rows drawn uniformly over (b, head, position) of {w.name}; "
                      f"{t_total:.1f} s on {cores} threads; value = rows/s / Hq"}


def run_ours(args):
    ws, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    if ws > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    from chunk_wise_hierarchical_landmark_b200 import binding as hb
    from chunk_wise_hierarchical_landmark_b200 import synth
    hb.lib()
    w = W.BY_NAME[args.workload]
    if w.decode:
        return run_decode_line(hb, synth, w, args, ws, rank)
    if args.backward:
        return run_backward_line(hb, synth, w, args, ws, rank)
    res = bench_prefill(hb, synth, w, args.steps, args.warmup, ws, rank, seed_offset=rank)
    ms = max_over_ranks(res["ms"], ws)
    e2e_ms = max_over_ranks(res["e2e_ms"], ws)
    qtok = w.B * w.L * ws
    work = prefill_work(w)
    peaks, peak_src = load_peaks()
    # dominant kernel by time share
    kernels = {
        "hils_select": {"ms": res["sel_ms"], "flop": work["score_flop"]},
        "hils_attn_fwd": {"ms": res["attn_ms"], "flop": work["attn_flop"]},
    }
    # executed tensor-core work: the scoring kernel's MMA tiles, and the
    # attention kernel's per-tile unions (from the timed run's selection)
    sizes = tile_union_sizes(hb, res["sel"])
    kernels["hils_select"]["exec_flop"] = select_executed_flop(w)
    kernels["hils_attn_fwd"]["exec_flop"] = attn_executed_flop(w, sizes)
    dom = max(kernels, key=lambda kname: kernels[kname]["ms"])
    peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    achieved = kernels[dom]["flop"] / (kernels[dom]["ms"] * 1e-3) / 1e12
    achieved_exec = kernels[dom]["exec_flop"] / (kernels[dom]["ms"] * 1e-3) / 1e12
    alg_total = work["score_flop"] + work["attn_flop"]
    exec_total = kernels["hils_select"]["exec_flop"] + kernels["hils_attn_fwd"]["exec_flop"]
    kstep = res["sel_ms"] + res["attn_ms"]
    line = {
        "metric": "HiLS fwd query-tokens/s (prefill, 512K tokens, 7B-shaped GQA 32/8, d=128)",
        "value": qtok / (ms * 1e-3),
        "unit": "query-tokens/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic (seeded; per-rank seed offset)",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "L": w.L, "d": w.d,
                   "chunk": w.C, "topk": w.topk, "M": w.M,
                   "l2": "inputs larger than L2 (q alone %.1f GB); no flush" %
                         (w.B * w.Hq * w.L * w.d * 2 / 1e9),
                   "parallelism": f"independent batch per GPU x{ws}"},
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved / peak,
                     "achieved_executed": achieved_exec, "frac_executed": achieved_exec / peak,
                     "algorithmic_over_executed": kernels[dom]["flop"] / kernels[dom]["exec_flop"],
                     "peak_source": f"{peak_src} bf16 dense, sustained",
                     "traffic": load_traffic(dom, w.name)},
        "kernels": {kn: {"ms": round(kv["ms"], 3),
                         "algorithmic_tflops": round(kv["flop"] / (kv["ms"] * 1e-3) / 1e12, 3),
                         "executed_tflops": round(kv["exec_flop"] / (kv["ms"] * 1e-3) / 1e12, 3),
                         "frac_algorithmic": round(kv["flop"] / (kv["ms"] * 1e-3) / 1e12 / peak, 4),
                         "frac_executed": round(kv["exec_flop"] / (kv["ms"] * 1e-3) / 1e12 / peak, 4),
                         "algorithmic_over_executed": round(kv["flop"] / kv["exec_flop"], 4),
                         "share": round(kv["ms"] / kstep, 3)}
                    for kn, kv in kernels.items()},
        "step_fraction": {"algorithmic_tflops": alg_total / (kstep * 1e-3) / 1e12,
                          "executed_tflops": exec_total / (kstep * 1e-3) / 1e12,
                          "frac_algorithmic": alg_total / (kstep * 1e-3) / 1e12 / peak,
                          "frac_executed": exec_total / (kstep * 1e-3) / 1e12 / peak,
                          "tile_union_mean": round(float(sizes.mean()), 2)},
        "selection_check": near_tie_sample(w, *res["inputs"], res["sel"], seed=w.seed),
        "e2e": {"value": qtok / (e2e_ms * 1e-3), "unit": "query-tokens/s",
                "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"],
                "pipeline": f"{w.B * w.Hkv} (b, kv-head) groups, one hils_prefill call each; "
                            "host->device, compute and device->host on three streams"},
        "gpu_launches": res["launches"],
        "clocks": res["clocks"],
    }
    if args.extra:
        extra = {}
        try:
            extra["union"] = union_stats(hb, res["sel"], w)
        except Exception as e:  # statistics only
            extra["union"] = {"error": str(e)[:200]}
        del res["sel"], res["inputs"]
        torch.cuda.empty_cache()
        # the other prefill configurations: 128K 7B-shaped, 32K small model,
        # and the tiny fp32 one (CUDA-core kernels: no tensor-core fraction)
        for w2 in (W.PREFILL_128K, W.SMALL_32K, W.TINY_F32):
            r2 = bench_prefill(hb, synth, w2, max(5, args.steps), 3, ws, rank, rank, e2e=False,
                               clocks=False)
            wk2 = prefill_work(w2)
            ent = {"value": w2.B * w2.L * ws / (max_over_ranks(r2["ms"], ws) * 1e-3),
                   "unit": "query-tokens/s", "ms_per_step": r2["ms"],
                   "select_ms": r2["sel_ms"], "attn_ms": r2["attn_ms"],
                   "dtype": w2.dtype,
                   "attn_tflops": wk2["attn_flop"] / (r2["attn_ms"] * 1e-3) / 1e12,
                   "select_tflops": wk2["score_flop"] / (r2["sel_ms"] * 1e-3) / 1e12}
            if w2.dtype == "bf16":
                sz2 = tile_union_sizes(hb, r2["sel"])
                ex_s, ex_a = select_executed_flop(w2), attn_executed_flop(w2, sz2)
                ent["attn_executed_tflops"] = ex_a / (r2["attn_ms"] * 1e-3) / 1e12
                ent["select_executed_tflops"] = ex_s / (r2["sel_ms"] * 1e-3) / 1e12
                ent["frac_algorithmic"] = (wk2["attn_flop"] + wk2["score_flop"]) / (r2["ms"] * 1e-3) / 1e12 / peak
                ent["frac_executed"] = (ex_a + ex_s) / (r2["ms"] * 1e-3) / 1e12 / peak
                ent["tile_union_mean"] = round(float(sz2.mean()), 2)
                ent["selection_check"] = near_tie_sample(w2, *r2["inputs"], r2["sel"], n_rows=128,
                                                         seed=w2.seed)
            extra[w2.name] = ent
            del r2
            torch.cuda.empty_cache()
        w3 = W.DECODE_512K
        r3 = bench_decode(hb, synth, w3, max(5, args.steps), 3, rank, paged=True)
        gbs = r3["bytes"] / (r3["ms"] * 1e-3) / 1e9
        extra[w3.name] = {"value": w3.B * ws / (max_over_ranks(r3["ms"], ws) * 1e-3),
                          "unit": "query-tokens/s", "ms_per_step": r3["ms"],
                          "algorithmic_bytes": r3["bytes"], "achieved_gbs": gbs,
                          "hbm_frac": gbs / peaks["hbm_gbs"]}
        pgbs = r3["bytes"] / (r3["paged_ms"] * 1e-3) / 1e9
        extra["decode_paged_gqa_bf16_B16_N524288"] = {
            "value": w3.B * ws / (max_over_ranks(r3["paged_ms"], ws) * 1e-3),
            "unit": "query-tokens/s", "ms_per_step": r3["paged_ms"],
            "algorithmic_bytes": r3["bytes"], "achieved_gbs": pgbs,
            "hbm_frac": pgbs / peaks["hbm_gbs"],
            "pool": f"{r3['paged_pages']} pages of 64 tokens x {w3.Hkv} KV heads, random order",
            "equal_to_dense": r3["paged_equal"]}
        del r3
        torch.cuda.empty_cache()
        try:
            rb = bench_backward(hb, synth, W.SMALL_32K, max(3, args.steps), 2)
            rb["frac"] = rb["algorithmic_tflops"] / alu_peak_tflops(res["clocks"])
            rb["peak_source"] = "fp32 FMA issue rate of the CUDA cores (148 SMs x 128 lanes x 2 FLOP x SM clock)"
            extra["backward_" + W.SMALL_32K.name] = rb
        except Exception as e:  # an extra entry must not cost the main line
            extra["backward_" + W.SMALL_32K.name] = {"error": str(e)[:200]}
        torch.cuda.empty_cache()
        try:
            extra["qcal_" + W.PREFILL_128K.name] = bench_qcal(hb, synth, W.PREFILL_128K,
                                                              max(3, args.steps), 2)
        except Exception as e:  # an extra entry must not cost the main line
            extra["qcal_" + W.PREFILL_128K.name] = {"error": str(e)[:200]}
        torch.cuda.empty_cache()
        try:
            r4 = bench_hope(hb, w, max(5, args.steps), 3)
            hgbs = r4["bytes"] / (r4["ms"] * 1e-3) / 1e9
            extra["hope_prepass_" + w.name] = {
                "ms_per_step": r4["ms"], "rotated_pairs": r4["npairs"],
                "split": "pairs with wavelength <= 65536 tokens at base 500000 (q and k, in place)",
                "algorithmic_bytes": r4["bytes"], "achieved_gbs": hgbs,
                "hbm_frac": hgbs / peaks["hbm_gbs"]}
        except Exception as e:  # an extra entry must not cost the main line
            extra["hope_prepass_" + w.name] = {"error": str(e)[:200]}
        torch.cuda.empty_cache()
        try:
            r5 = bench_hope_fused(hb, synth, W.PREFILL_128K, max(3, args.steps), 2)
            r5["note"] = ("prefill with HoPE on q: hils_hope pre-pass over a copy of q then "
                          "hils_prefill, against hils_prefill_hope (rotation in the kernels' "
                          "query staging); keys pre-rotated in both")
            extra["hope_fused_" + W.PREFILL_128K.name] = r5
        except Exception as e:  # an extra entry must not cost the main line
            extra["hope_fused_" + W.PREFILL_128K.name] = {"error": str(e)[:200]}
        line["workloads"] = extra
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, res["host_inputs"])
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        torch.distributed.destroy_process_group()


def run_decode_line(hb, synth, w, args, ws, rank):
    """A decode workload as the main line (used for profiler captures of the
    decode kernels on a reduced batch): step = one hils_decode_fwd call."""
    peaks, peak_src = load_peaks()
    n0 = hb.launch_count()
    r = bench_decode(hb, synth, w, args.steps, args.warmup, rank)
    launches = hb.launch_count() - n0
    ms = max_over_ranks(r["ms"], ws)
    gbs = r["bytes"] / (r["ms"] * 1e-3) / 1e9
    line = {"metric": "HiLS decode query-tokens/s", "value": w.B * ws / (ms * 1e-3),
            "unit": "query-tokens/s", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic (seeded; per-rank seed offset)",
            "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.L,
                       "d": w.d, "chunk": w.C, "topk": w.topk},
            "roofline": {"bound": "hbm", "kernel": "hils_decode_fwd", "achieved": gbs,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                         "peak_source": f"{peak_src} HBM copy", "traffic": None},
            "gpu_launches": launches}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        torch.distributed.destroy_process_group()


def run_backward_line(hb, synth, w, args, ws, rank):
    """The backward pass of a prefill workload as the main line (used for
    profiler captures of the backward kernels): step = one hils_attn_bwd call
    on the forward's selection, with dO and dlse seeded."""
    r = bench_backward(hb, synth, w, args.steps, args.warmup)
    launches = r["launches"]
    ms = max_over_ranks(r["ms_per_step"], ws)
    peak = alu_peak_tflops(None)
    tflops = backward_work(w) / (ms * 1e-3) / 1e12
    line = {"metric": "HiLS backward query-tokens/s", "value": w.B * w.L * ws / (ms * 1e-3),
            "unit": "query-tokens/s", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic (seeded; dO and dlse seeded)",
            "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "L": w.L,
                       "d": w.d, "chunk": w.C, "topk": w.topk, "inputs": w.dtype},
            "roofline": {"bound": "alu", "kernel": "hils_attn_bwd", "achieved": tflops,
                         "peak": peak, "unit": "TFLOP/s", "frac": tflops / peak,
                         "peak_source": "fp32 FMA issue rate at the maximum SM clock "
                                        "(148 SMs x 128 lanes x 2 FLOP x 1965 MHz)",
                         "traffic": None},
            "gpu_launches": launches}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        torch.distributed.destroy_process_group()


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    from chunk_wise_hierarchical_landmark_b200 import synth
    w = W.BY_NAME[args.workload]
    host = synth.make_inputs(w, "cuda" if torch.cuda.is_available() else "cpu")
    host = tuple(x.cpu() for x in host)
    p = oracle.Problem(w.B, w.Hq, w.Hkv, w.L, w.d, w.C, w.topk, w.scale)
    cores = os.cpu_count() or 1
    rng = np.random.default_rng(w.seed)
    per_step = max(cores * 4, 64)
    q, k, v, lmk = host
    for _ in range(args.warmup):
        oracle.rows(p, q, k, v, lmk, rng.integers(0, w.B * w.Hq * w.L, size=cores), nthreads=cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.rows(p, q, k, v, lmk, rng.integers(0, w.B * w.Hq * w.L, size=per_step),
                    nthreads=cores)
    dt = (time.perf_counter() - t0) / args.steps
    value = per_step / dt / w.Hq
    sample = (f"{per_step} rows per step drawn uniformly over (b, head, position) of {w.name}; "
              f"value = rows/s / Hq")
    line = {
        "impl": "reference",
        "metric": "HiLS fwd query-tokens/s (prefill, 512K tokens, 7B-shaped GQA 32/8, d=128)",
        "value": value, "unit": "query-tokens/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "L": w.L, "d": w.d,
                   "chunk": w.C, "topk": w.topk, "M": w.M},
        "cpu_baseline": {"value": value, "unit": "query-tokens/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "query-tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=W.PREFILL_512K.name, choices=sorted(W.BY_NAME))
    ap.add_argument("--extra", dest="extra", action="store_true", default=True)
    ap.add_argument("--no-extra", dest="extra", action="store_false")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass of the (prefill) workload instead")
    ap.add_argument("--hq", type=int, default=None,
                    help="override the query-head count (smaller cases for profiler captures)")
    ap.add_argument("--hkv", type=int, default=None, help="override the KV-head count")
    ap.add_argument("--batch", type=int, default=None, help="override the batch size")
    args = ap.parse_args()
    if args.hq or args.hkv or args.batch:
        base = W.BY_NAME[args.workload]
        w = base.with_(Hq=args.hq or base.Hq, Hkv=args.hkv or base.Hkv, B=args.batch or base.B)
        w = w.with_(name=f"{base.name}_b{w.B}_hq{w.Hq}_hkv{w.Hkv}")
        W.BY_NAME[w.name] = w
        args.workload = w.name
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

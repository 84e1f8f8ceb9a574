"""Measurement suite over the workload shapes (used by ``bench.py --suite``).

Each record is one JSON object: the shape, the sparse decode-attention time per launch, its
algorithmic bytes and GB/s as a fraction of the HBM peak, the dense fp16 baseline on the same
inputs, or the compress kernel's throughput and compressed size.  Times are the median of
CUDA-event-timed launches with the 126 MB L2 flushed (a 256 MiB read) before each launch.
"""
from __future__ import annotations

import json
import math
import time

import torch

import unstructured_sparse_kv_b200 as M
from unstructured_sparse_kv_b200 import synth

D = 128
FLUSH_BYTES = 256 << 20


class Timer:
    """Median of single calls, each after a read of a buffer larger than L2.  The flush only reads
    (its lines stay clean), so the timed call pays no write-back of flush data.  A short device
    sleep after the flush keeps the GPU busy while the host enqueues the timed call, so that host
    time spent between the call's launches never shows up as device idle time inside the events."""

    def __init__(self, device):
        self.flush = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=device)

    def median_us(self, fn, reps: int = 15, warmup: int = 3) -> float:
        for _ in range(warmup):
            fn()
        times = []
        for _ in range(reps):
            torch.amax(self.flush)
            torch.cuda._sleep(200_000)  # about 100 us at the B200's clocks
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            e1.synchronize()
            times.append(e0.elapsed_time(e1) * 1000.0)
        times.sort()
        return times[len(times) // 2]


def decode_bytes(B, Hq, Hkv, L, kK, kV):
    """Bitmaps + kept values of K and V for every token-head, plus q and out (fp16); kK and kV are
    keep counts, or lists with one keep count per kv head."""
    kK = kK if isinstance(kK, (list, tuple)) else [kK] * Hkv
    kV = kV if isinstance(kV, (list, tuple)) else [kV] * Hkv
    return B * L * sum(32 + 2 * (a + b) for a, b in zip(kK, kV)) + 4 * B * Hq * D


def dense_bytes(B, Hq, Hkv, L):
    return 4 * B * Hkv * L * D + 4 * B * Hq * D


def fits(B, Hkv, L, s, free_bytes):
    dense = 4 * B * Hkv * L * D
    k = M.mustafar_keep_count(D, s)
    comp = 2 * B * Hkv * L * (16 + 2 * k) + 2 * B * Hkv * (L // 64) * 4
    return dense + comp + (2 << 30) < free_bytes


def decode_point(timer, peak, Hq, Hkv, B, L, sK, sV, seed, with_dense=True, pattern="topk"):
    dev = "cuda"
    cap = ((L + 63) // 64) * 64
    K = synth.keys(B, Hkv, L, D, seed, dev, capacity=cap)
    V = synth.values(B, Hkv, L, D, seed, dev, capacity=cap)
    q = synth.queries(B, Hq, D, seed, dev)
    kc = M.CompressedCache(B, Hkv, cap, sK, pattern=pattern)
    vc = M.CompressedCache(B, Hkv, cap, sV, pattern=pattern)
    M.mustafar_compress(K, L, sK if kc.sparsity is not None else 0.0, kc)  # per-head caches ignore it
    M.mustafar_compress(V, L, sV if vc.sparsity is not None else 0.0, vc)
    seq = torch.full((B,), L, dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    ws = torch.zeros(M.mustafar_decode_workspace_bytes(B, Hq, Hkv, L), dtype=torch.uint8, device=dev)
    t_sparse = timer.median_us(lambda: M.mustafar_decode_attn(q, kc, vc, seq, L, 1.0, out=out, lse=lse, workspace=ws))
    nb = decode_bytes(B, Hq, Hkv, L, kc.head_keep, vc.head_keep)
    rec = {"kind": "decode", "pattern": pattern, "q_heads": Hq, "kv_heads": Hkv, "batch": B, "context": L,
           "sparsity_k": sK,
           "sparsity_v": sV, "keep_k": kc.head_keep if kc.per_head else kc.keep,
           "keep_v": vc.head_keep if vc.per_head else vc.keep,
           "splits": M.mustafar_decode_plan_splits(B, Hkv, L, kc.keep, vc.keep),
           "sparse_us": t_sparse, "sparse_bytes": nb, "sparse_gbs": nb / t_sparse / 1e3,
           "sparse_frac_of_peak": nb / t_sparse / 1e3 / peak,
           "compressed_fraction_of_dense": (kc.nbytes() + vc.nbytes()) / (4 * B * Hkv * cap * D)}
    if with_dense:
        wsd = torch.zeros(M.mustafar_decode_workspace_bytes(B, Hq, Hkv, L), dtype=torch.uint8, device=dev)
        t_dense = timer.median_us(lambda: M.mustafar_dense_decode_attn(q, K, V, seq, L, 1.0, out=out, lse=lse,
                                                                        workspace=wsd))
        db = dense_bytes(B, Hq, Hkv, L)
        rec.update({"dense_us": t_dense, "dense_gbs": db / t_dense / 1e3, "dense_frac_of_peak": db / t_dense / 1e3 / peak,
                    "sparse_speedup_vs_dense": t_dense / t_sparse})
    del K, V, kc, vc
    torch.cuda.empty_cache()
    return rec


def compress_point(timer, peak, B, L, H, s, seed, pattern="topk"):
    dev = "cuda"
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    x = torch.randn(B, L, H, D, generator=g, device=dev).to(torch.float16)  # [B, L, H, d] storage
    c = M.CompressedCache(B, H, L, s, pattern=pattern)
    view = x.permute(0, 2, 1, 3)
    t = timer.median_us(lambda: M.mustafar_compress(view, L, s, c))
    # dense read + compressed arrays written (a full-window prefill writes no window copy)
    nbytes = 2 * B * L * H * D + c.nbytes() - (c.window.numel() * 2 if c.window is not None else 0)
    rec = {"kind": "compress", "pattern": pattern, "batch": B, "tokens": L, "kv_heads": H, "sparsity": s,
           "keep": c.keep, "us": t,
           "bytes_read_plus_written": nbytes, "gbs": nbytes / t / 1e3, "frac_of_peak": nbytes / t / 1e3 / peak,
           "compressed_bytes": c.nbytes(), "compressed_fraction_of_dense": c.nbytes() / (2 * B * L * H * D)}
    del x, c
    torch.cuda.empty_cache()
    return rec


def step_point(timer, peak, Hq, Hkv, B, L, s, seed, pattern="topk"):
    """One fused decode step (compress the new K/V token into slot L, attend over L + 1 tokens)."""
    dev = "cuda"
    cap = ((L + 1 + 63) // 64) * 64
    K = synth.keys(B, Hkv, L, D, seed, dev, capacity=cap)
    V = synth.values(B, Hkv, L, D, seed, dev, capacity=cap)
    q = synth.queries(B, Hq, D, seed, dev)
    kc = M.CompressedCache(B, Hkv, cap, s, pattern=pattern)
    vc = M.CompressedCache(B, Hkv, cap, s, pattern=pattern)
    M.mustafar_compress(K, L, s, kc)
    M.mustafar_compress(V, L, s, vc)
    kn, vn = synth.step_tokens(B, Hkv, D, seed, 0, dev)
    pos = torch.full((B,), L, dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    ws = torch.zeros(M.mustafar_decode_workspace_bytes(B, Hq, Hkv, L + 1), dtype=torch.uint8, device=dev)
    # the same slot every time: a repeated step writes the same bytes
    t = timer.median_us(lambda: M.mustafar_decode_step(q, kn, vn, pos, kc, vc, L + 1, 1.0, out=out, lse=lse,
                                                       workspace=ws))
    nb = decode_bytes(B, Hq, Hkv, L + 1, kc.keep, vc.keep)
    rec = {"kind": "decode_step", "pattern": pattern, "q_heads": Hq, "kv_heads": Hkv, "batch": B, "context": L + 1,
           "sparsity": s, "keep_k": kc.keep, "keep_v": vc.keep, "step_us": t, "bytes": nb,
           "gbs": nb / t / 1e3, "frac_of_peak": nb / t / 1e3 / peak}
    del K, V, kc, vc
    torch.cuda.empty_cache()
    return rec


def run(out_path: str, peak: float, which=("c1", "c3", "c4", "heads", "p24", "channel", "sweep"), log=print):
    torch.cuda.set_device(0)
    timer = Timer("cuda")
    recs = []

    def emit(r):
        recs.append(r)
        with open(out_path, "a") as f:
            f.write(json.dumps(r) + "\n")
        log(json.dumps(r))

    if "c1" in which:
        emit(dict(decode_point(timer, peak, 32, 8, 1, 1024, 0.5, 0.5, 1001), workload="b1 ctx1024 s0.5"))
    if "c3" in which:
        emit(dict(decode_point(timer, peak, 32, 8, 4, 32768, 0.7, 0.5, 1003), workload="b4 ctx32k sK0.7 sV0.5"))
    if "c4" in which:
        for s in (0.3, 0.5, 0.7):
            emit(dict(compress_point(timer, peak, 8, 16384, 8, s, 1004), workload="compress b8 16k h8"))
    if "heads" in which:
        # a sparsity per kv head around 0.7 (K) and its mirror (V), against uniform 0.7 on the same inputs
        hs = [0.5, 0.6, 0.7, 0.8, 0.9, 0.7, 0.6, 0.8]
        emit(dict(decode_point(timer, peak, 32, 8, 8, 4096, hs, hs[::-1], 1006, with_dense=False),
                  workload="b8 ctx4096 per-head sparsity (mean 0.7)"))
        emit(dict(decode_point(timer, peak, 32, 8, 8, 4096, 0.7, 0.7, 1006, with_dense=False),
                  workload="b8 ctx4096 uniform 0.7 (same inputs)"))
    if "p24" in which:
        # the 2:4 comparison pattern against unstructured pruning at the same sparsity (0.5) and dense
        for B, L in ((8, 4096), (4, 32768)):
            emit(dict(decode_point(timer, peak, 32, 8, B, L, 0.5, 0.5, 1008, pattern="2:4"),
                      workload=f"b{B} ctx{L} 2:4"))
            emit(dict(decode_point(timer, peak, 32, 8, B, L, 0.5, 0.5, 1008, with_dense=False),
                      workload=f"b{B} ctx{L} unstructured s0.5 (same inputs)"))
    if "channel" in which:
        # channel-wise pruning over 16-token windows against token-wise pruning on the same inputs
        # (keep 40 vs 39 values per token at s = 0.7)
        for B, L in ((8, 4096), (4, 32768)):
            emit(dict(decode_point(timer, peak, 32, 8, B, L, 0.7, 0.7, 1010, pattern="channel"),
                      workload=f"b{B} ctx{L} channel-wise s0.7"))
            emit(dict(decode_point(timer, peak, 32, 8, B, L, 0.7, 0.7, 1010, with_dense=False),
                      workload=f"b{B} ctx{L} token-wise s0.7 (same inputs)"))
        for pattern in ("channel", "topk"):
            emit(dict(step_point(timer, peak, 32, 8, 8, 4096, 0.7, 1010, pattern=pattern),
                      workload=f"decode step call b8 ctx4096 s0.7 {pattern}"))
        emit(dict(compress_point(timer, peak, 8, 16384, 8, 0.7, 1004, pattern="channel"),
                  workload="compress b8 16k h8 channel-wise"))
    if "sweep" in which:
        for Hkv in (8, 32):
            for B in (1, 8, 32):
                for L in (4096, 32768, 131072):
                    for s in (0.0, 0.3, 0.5, 0.7, 0.9):
                        free, _ = torch.cuda.mem_get_info()
                        if not fits(B, Hkv, L, s, free):
                            emit({"kind": "decode", "q_heads": 32, "kv_heads": Hkv, "batch": B, "context": L,
                                  "sparsity_k": s, "sparsity_v": s, "skipped": "does not fit in device memory"})
                            continue
                        emit(dict(decode_point(timer, peak, 32, Hkv, B, L, s, s, 2000 + B + Hkv + int(10 * s)),
                                  workload="sweep"))
    return recs

"""Benchmark of the Mustafar hot path on B200.

A step is one decode step of the Llama-3-8B-like GQA workload at batch 8: prune +
compress the new token's K and V into the compressed caches, then sparse decode
attention over the 4097..4160-token compressed context, all in one launch of the
fused decode step (``mustafar_decode_step``).  The same step as three launches (append
K, append V, attend) is timed beside it.
The workload is 4096 prefill tokens plus 64 decode steps at K and V sparsity 0.7; timed
steps cycle through the 64 decode positions.  Inputs are synthetic (seeded; see
``unstructured_sparse_kv_b200/synth.py``).

Timing: the timed region replays CUDA graphs that hold exactly ``--steps`` decode steps (graphs
of 64 steps plus one graph of the remaining ``steps % 64``); warm-up replays exactly
``--warmup`` steps the same way.  Before that, every graph has been launched once (a graph is
uploaded to the device at its first launch) and a ~0.8 s soak of the same step brings the
clocks to their loaded state; a ~100 us device sleep ahead of the start event hides the host's
enqueueing of the timed launches.  Every step reads one of 8 rotating copies of the compressed
caches (8 x 49.5 MB, over twice the 126 MB L2), so no step finds the previous step's cache in
L2.  The timed region is bracketed by a barrier and ``torch.cuda.synchronize()``; the time is
the max over ranks.  SM clocks and throttle reasons are polled through NVML while the GPU runs.
The comparison legs (the same step as three launches, the attention launch alone, dense fp16
attention, and attention at sparsity 0 / 0.3 / 0.5 / 0.7 / 0.9) are all timed the same way:
replays of 64-step graphs over the same rotation.

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse decode-attn µs/step & compressed-KV GB/s (fraction of HBM peak) vs sparsity"
UNIT = "us/step"
WORKLOAD = dict(batch=8, q_heads=32, kv_heads=8, head_dim=128, context=4096, decode_steps=64,
                sparsity_k=0.7, sparsity_v=0.7)
ROTATE = 8
GRAPH_STEPS = 64
SPARSITY_AXIS = (0.0, 0.3, 0.5, 0.7, 0.9)
FALLBACK_HBM_GBS = 6650.0


# ------------------------------------------------------------------------------------------ helpers
def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("LOCAL_RANK", "0"))


def rank_seed(rank: int) -> int:
    """Each rank runs the same workload shape on its own seeded batch (weak scaling, no exchange)."""
    return 1002 + 1000 * rank


def aggregate_us_per_step(max_elapsed_ms: float, steps: int, world: int) -> float:
    """Whole-job time per step: all ranks' steps together took the slowest rank's time."""
    return max_elapsed_ms * 1000.0 / (steps * world)


def max_over_ranks(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def graph_counts(n: int):
    """How exactly n steps are replayed: (replays of the 64-step graph, steps of the one remainder graph)."""
    return divmod(int(n), GRAPH_STEPS)


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def decode_algorithmic_bytes(B, Hq, Hkv, d, lens, kK, kV):
    """Bytes the decode attention must move: every stored token's bitmaps and kept values
    of K and V, plus q in and out (fp16).  Split partials are overhead, not credited."""
    per_tok = 2 * (d // 8) + 2 * (kK + kV)
    return sum(Hkv * L * per_tok for L in lens) + 2 * (2 * B * Hq * d)


def kernel_source_hash() -> str:
    """Hash of the raw text of every source the decode launch is built from (kernel, device helpers,
    the parameter block and the host-side plan / launch code); any edit invalidates the recorded
    DRAM traffic."""
    h = hashlib.sha256()
    for f in ("common.cuh", "select.cuh", "internal.h", "decode_sparse.cu", "abi.cu"):
        with open(os.path.join(ROOT, "unstructured_sparse_kv_b200", "csrc", f), "rb") as fh:
            h.update(f.encode() + b"\0" + fh.read())
    return h.hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per decode launch from the committed ncu summary, if it was taken on this kernel source."""
    path = os.path.join(ROOT, "profiles", "decode_attn_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        if rec.get("kernel_source_sha256_16") == kernel_source_hash():
            return float(rec["dram_bytes_per_launch_full_workload"])
    except Exception:
        pass
    return None


class ClockSampler:
    """SM clock, power and clock-event (throttle) reasons of one GPU, polled through NVML about every
    2 ms in a background thread while the GPU works, so that even a timed region of a millisecond gets
    samples.  ``mark()`` records the host time at which the timed region starts and ends."""
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80))

    def __init__(self, torch_device):
        self.dev = torch_device
        self.samples = []  # (t, sm_mhz, reasons_bitmask, power_w)
        self.marks = []
        self.err = None
        self._stop = None
        self._thread = None

    def _handle(self, nv):
        import torch
        try:
            pr = torch.cuda.get_device_properties(self.dev)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.dev.index or 0)

    def __enter__(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._handle(nv)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        except Exception as e:  # no NVML: the record says so
            self.err = f"nvml unavailable: {e}"
            return self
        self._stop = threading.Event()

        def poll():
            while not self._stop.is_set():
                try:
                    self.samples.append((time.perf_counter(), float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                         int(nv.nvmlDeviceGetCurrentClocksEventReasons(h)),
                                         nv.nvmlDeviceGetPowerUsage(h) / 1000.0))
                except Exception as e:
                    self.err = str(e)
                    return
                time.sleep(0.002)

        self._thread = threading.Thread(target=poll, daemon=True)
        self._thread.start()
        return self

    def mark(self):
        self.marks.append(time.perf_counter())

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
            try:
                import pynvml as nv
                nv.nvmlShutdown()
            except Exception:
                pass

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.err or "no samples"], "samples": 0}
        window = self.samples
        source = "whole run"
        if len(self.marks) >= 2:
            inside = [x for x in self.samples if self.marks[0] <= x[0] <= self.marks[1]]
            if inside:
                window, source = inside, "timed region"
        sm = sorted(x[1] for x in window)
        bits = 0
        for x in window:
            bits |= x[2]
        return {"sm_mhz": sm[len(sm) // 2], "sm_min_mhz": sm[0], "sm_max_mhz": self.max_mhz,
                "reasons": [n for n, b in self.REASONS if bits & b], "samples": len(window),
                "power_w_max": max(x[3] for x in window), "source": f"NVML every ~2 ms, {source}"}


# ------------------------------------------------------------------------------------------ workload
class Workload:
    def __init__(self, seed: int, device):
        import torch
        import unstructured_sparse_kv_b200 as M
        from unstructured_sparse_kv_b200 import synth
        w = WORKLOAD
        self.M, self.torch = M, torch
        self.B, self.Hq, self.Hkv, self.d = w["batch"], w["q_heads"], w["kv_heads"], w["head_dim"]
        self.L0, self.steps = w["context"], w["decode_steps"]
        self.cap = self.L0 + self.steps
        self.sK, self.sV = w["sparsity_k"], w["sparsity_v"]
        self.dev = device
        B, Hq, Hkv, d, cap = self.B, self.Hq, self.Hkv, self.d, self.cap
        # dense caches hold the prefill and the 64 decode tokens; every copy is fully compressed so that
        # each append rewrites a slot with identical bits and every copy stays a valid cache
        self.K = synth.keys(B, Hkv, cap, d, seed, device)
        self.V = synth.values(B, Hkv, cap, d, seed, device)
        self.kc, self.vc = [], []
        for _ in range(ROTATE):
            kc = M.CompressedCache(B, Hkv, cap, self.sK, device=device)
            vc = M.CompressedCache(B, Hkv, cap, self.sV, device=device)
            M.mustafar_compress(self.K, cap, self.sK, kc)
            M.mustafar_compress(self.V, cap, self.sV, vc)
            self.kc.append(kc)
            self.vc.append(vc)
        self.q = torch.stack([synth.queries(B, Hq, d, seed, device, step=i) for i in range(self.steps)])
        self.kn = self.K[:, :, self.L0:].permute(2, 0, 1, 3).contiguous()  # [steps, B, Hkv, d]
        self.vn = self.V[:, :, self.L0:].permute(2, 0, 1, 3).contiguous()
        self.pos = (self.L0 + torch.arange(self.steps, dtype=torch.int32, device=device))[:, None].repeat(1, B)
        self.seq = (self.pos + 1).contiguous()
        self.out = torch.empty(B, Hq, d, dtype=torch.float16, device=device)
        self.lse = torch.empty(B, Hq, dtype=torch.float32, device=device)
        self.ws = torch.zeros(M.mustafar_decode_workspace_bytes(B, Hq, Hkv, cap), dtype=torch.uint8, device=device)
        self.splits = M.mustafar_decode_plan_splits(B, Hkv, cap, self.kc[0].keep, self.vc[0].keep)
        self.compressed_bytes = self.kc[0].nbytes() + self.vc[0].nbytes()
        self.dense_cache_bytes = 2 * self.K.numel() * self.K.element_size()

    def step(self, i: int, mode: str = "fused"):
        """One decode step: "fused" (one launch), "separate" (append K, append V, attend) or
        "attend" (the attention launch alone)."""
        M, r, j = self.M, i % ROTATE, i % self.steps
        if mode == "fused":
            M.mustafar_decode_step(self.q[j], self.kn[j], self.vn[j], self.pos[j], self.kc[r], self.vc[r], self.cap,
                                   1.0, out=self.out, lse=self.lse, workspace=self.ws)
            return
        if mode == "separate":
            M.mustafar_append(self.kn[j], self.pos[j], self.kc[r])
            M.mustafar_append(self.vn[j], self.pos[j], self.vc[r])
        M.mustafar_decode_attn(self.q[j], self.kc[r], self.vc[r], self.seq[j], self.cap, 1.0, out=self.out,
                               lse=self.lse, workspace=self.ws)

    def capture(self, n: int, run=None, mode: str = "fused"):
        """A CUDA graph of n consecutive steps 0 .. n-1 of ``run(i)`` (default: ``self.step(i, mode)``);
        the steps run once eagerly first (plans, kernel attributes) and are then captured."""
        torch = self.torch
        run = run or (lambda i: self.step(i, mode))
        for i in range(n):
            run(i)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(n):
                run(i)
        return g

    def exact(self, n: int, run=None, mode: str = "fused"):
        """Graphs that replay exactly n steps: n // 64 replays of a 64-step graph, then one graph of the
        remaining n % 64 steps.  Returns (replay function, graphs)."""
        full, rest = graph_counts(n)
        g64 = self.capture(GRAPH_STEPS, run, mode) if full else None
        gr = self.capture(rest, run, mode) if rest else None

        def replay():
            for _ in range(full):
                g64.replay()
            if gr is not None:
                gr.replay()
        return replay, [g for g in (g64, gr) if g is not None]


class DenseBaseline:
    """Dense fp16 decode attention over the same (unpruned) caches, 3 rotating copies (> 3x L2)."""

    def __init__(self, wl: Workload):
        import torch
        self.wl, self.M = wl, wl.M
        self.copies = [wl.K] + [wl.K.clone() for _ in range(2)]
        self.vcopies = [wl.V] + [wl.V.clone() for _ in range(2)]
        self.ws = torch.zeros(wl.M.mustafar_decode_workspace_bytes(wl.B, wl.Hq, wl.Hkv, wl.cap), dtype=torch.uint8,
                              device=wl.dev)

    def step(self, i: int):
        wl, r, j = self.wl, i % 3, i % self.wl.steps
        self.M.mustafar_dense_decode_attn(wl.q[j], self.copies[r], self.vcopies[r], wl.seq[j], wl.cap, 1.0,
                                          out=wl.out, lse=wl.lse, workspace=self.ws)

    def release(self):
        self.copies, self.vcopies = self.copies[:1], self.vcopies[:1]


class SparsityPoint:
    """The bench workload's caches compressed at one sparsity (K and V alike), ROTATE copies, and the
    attention launch alone over them (same queries, lengths and rotation as the decode step)."""

    def __init__(self, wl: Workload, sparsity: float):
        M = wl.M
        self.wl, self.M = wl, M
        self.kc, self.vc = [], []
        for _ in range(ROTATE):
            kc = M.CompressedCache(wl.B, wl.Hkv, wl.cap, sparsity, device=wl.dev)
            vc = M.CompressedCache(wl.B, wl.Hkv, wl.cap, sparsity, device=wl.dev)
            M.mustafar_compress(wl.K, wl.cap, sparsity, kc)
            M.mustafar_compress(wl.V, wl.cap, sparsity, vc)
            self.kc.append(kc)
            self.vc.append(vc)
        self.keep = self.kc[0].keep
        self.nbytes = self.kc[0].nbytes() + self.vc[0].nbytes()

    def step(self, i: int):
        wl, r, j = self.wl, i % ROTATE, i % self.wl.steps
        self.M.mustafar_decode_attn(wl.q[j], self.kc[r], self.vc[r], wl.seq[j], wl.cap, 1.0, out=wl.out,
                                    lse=wl.lse, workspace=wl.ws)


def time_graph(g, replays: int, stream) -> float:
    import torch
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda._sleep(200_000)  # device work ahead of the start event hides the host's first enqueue
    e0.record(stream)
    for _ in range(replays):
        g.replay()
    e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1)


# ------------------------------------------------------------------------------------------ CPU oracle
def oracle_decode_sample(budget_s: float = 12.0, seed: int = 1002):
    """Time the CPU oracle (as it stands) on the same decode workload: append K and V, then
    attention over the compressed caches, over all 64 (b, kv head) streams, for as many
    decode steps as fit in ``budget_s``.  BLAS limited to one thread."""
    import numpy as np
    import torch
    from threadpoolctl import threadpool_limits

    import oracle
    from unstructured_sparse_kv_b200 import synth
    w = WORKLOAD
    B, Hq, Hkv, d, L0, steps = w["batch"], w["q_heads"], w["kv_heads"], w["head_dim"], w["context"], w["decode_steps"]
    cap = L0 + steps
    to_bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    K = to_bits(synth.keys(B, Hkv, cap, d, seed, "cpu"))
    V = to_bits(synth.values(B, Hkv, cap, d, seed, "cpu"))
    kK, kV = oracle.keep_count(d, w["sparsity_k"]), oracle.keep_count(d, w["sparsity_v"])
    kc = oracle.compress(K, kK, cap, L0)
    vc = oracle.compress(V, kV, cap, L0)
    done, t_total = 0, 0.0
    with threadpool_limits(limits=1):
        while done < steps:
            q = to_bits(synth.queries(B, Hq, d, seed, "cpu", step=done))
            t0 = time.perf_counter()
            pos = np.full(B, L0 + done)
            oracle.append(kc, K[:, :, L0 + done], pos)
            oracle.append(vc, V[:, :, L0 + done], pos)
            oracle.attention_over_compressed(q, kc, vc, pos + 1, 1.0, d)
            t_total += time.perf_counter() - t0
            done += 1
            if t_total >= budget_s:
                break
    return {"value": t_total / done * 1e6, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{done} of the 64 decode steps (append K, append V, attention over all 64 streams), "
                      f"float64 NumPy, 1 BLAS thread"}


def _oracle_worker(conn, ks, vs, kK, kV, cap, L0, d):
    """One host process of the all-cores oracle timing: owns a fixed set of (b, kv head) streams,
    compresses them once, then per message appends each stream's step token and attends."""
    import numpy as np

    import oracle
    caches = [(oracle.compress(k[None, None], kK, cap, L0), oracle.compress(v[None, None], kV, cap, L0))
              for k, v in zip(ks, vs)]
    conn.send("ready")
    while True:
        msg = conn.recv()
        if msg is None:
            break
        step, qs = msg
        pos = np.array([L0 + step])
        for (kc, vc), k, v, q in zip(caches, ks, vs, qs):
            oracle.append(kc, k[None, None, L0 + step], pos)
            oracle.append(vc, v[None, None, L0 + step], pos)
            oracle.attention_over_compressed(q[None], kc, vc, pos + 1, 1.0, d)
        conn.send("done")


def oracle_decode_all_cores(budget_s: float = 8.0, seed: int = 1002):
    """The same oracle step spread over the host's cores: one spawned process per core, each owning
    a fixed share of the 64 independent (b, kv head) streams (one BLAS thread each); the step time is
    the wall time until every process has finished its streams."""
    import multiprocessing as mp

    import numpy as np
    import torch

    import oracle
    from unstructured_sparse_kv_b200 import synth
    w = WORKLOAD
    B, Hq, Hkv, d, L0, steps = w["batch"], w["q_heads"], w["kv_heads"], w["head_dim"], w["context"], w["decode_steps"]
    G, cap = Hq // Hkv, L0 + steps
    to_bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    K = to_bits(synth.keys(B, Hkv, cap, d, seed, "cpu"))
    V = to_bits(synth.values(B, Hkv, cap, d, seed, "cpu"))
    kK, kV = oracle.keep_count(d, w["sparsity_k"]), oracle.keep_count(d, w["sparsity_v"])
    streams = [(b, g) for b in range(B) for g in range(Hkv)]
    n = max(1, min(len(os.sched_getaffinity(0)), len(streams)))
    saved = {v: os.environ.get(v) for v in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
    for v in saved:
        os.environ[v] = "1"
    ctx = mp.get_context("spawn")
    procs, conns = [], []
    try:
        for i in range(n):
            mine = streams[i::n]
            a, c = ctx.Pipe()
            p = ctx.Process(target=_oracle_worker, args=(c, [K[b, g] for b, g in mine], [V[b, g] for b, g in mine],
                                                         kK, kV, cap, L0, d), daemon=True)
            p.start()
            procs.append((p, mine))
            conns.append(a)
        for a in conns:
            a.recv()
        done, t_total = 0, 0.0
        while done < steps and (t_total < budget_s or done < 2):
            q = to_bits(synth.queries(B, Hq, d, seed, "cpu", step=done))
            msgs = [(done, [q[b, g * G:(g + 1) * G] for b, g in mine]) for _, mine in procs]
            t0 = time.perf_counter()
            for a, m in zip(conns, msgs):
                a.send(m)
            for a in conns:
                a.recv()
            t_total += time.perf_counter() - t0
            done += 1
        for a in conns:
            a.send(None)
    finally:
        for p, _ in procs:
            p.join(timeout=10)
            if p.is_alive():
                p.kill()
        for v, old in saved.items():
            if old is None:
                os.environ.pop(v, None)
            else:
                os.environ[v] = old
    return {"value": t_total / done * 1e6, "unit": UNIT, "cores": n,
            "sample": f"{done} of the 64 decode steps, 64 streams over {n} spawned processes, 1 BLAS thread each"}


def run_reference(args):
    rank, world, _ = dist_env()
    if world > 1 and rank != 0:
        return 0
    base = oracle_decode_sample(budget_s=min(20.0, 4.0 + 2.0 * args.steps))
    line = {"impl": "reference", "metric": METRIC, "value": base["value"], "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": base["value"] / 1000.0,
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(), "cpu_baseline": base,
            "e2e": {"value": base["value"], "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def config_dict():
    w = WORKLOAD
    return {"workload": "Llama-3-8B-like GQA decode (q32/kv8/d128), batch 8, context 4096 + 64 decode steps, "
                        "K/V sparsity 0.7; step = one fused launch: compress the new K and V token + sparse decode "
                        "attention",
            "batch": w["batch"], "context": w["context"], "decode_steps": w["decode_steps"],
            "sparsity_k": w["sparsity_k"], "sparsity_v": w["sparsity_v"],
            "l2": f"{ROTATE} rotating compressed-cache copies (> 2x the 126 MB L2)", "timing": "exactly --steps fused steps replayed from CUDA graphs (64-step graphs + one graph of the remainder), CUDA events on the launching stream"}


# ------------------------------------------------------------------------------------------ main
def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64 * 300)
    ap.add_argument("--warmup", type=int, default=64 * 4)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--suite", default=None, help="write the workload-shape suite (JSONL) to this path and exit")
    ap.add_argument("--suite-parts", default="c1,c3,c4,heads,p24,channel,sweep")
    ap.add_argument("--profile-launches", type=int, default=0,
                    help="ncu case: build the workload, run this many eager fused steps over the rotated "
                         "caches, and exit without timing")
    ap.add_argument("--profile-shape", default=None,
                    help="ncu case: 'B,L,sK,sV' -- GQA 32/8 decode over two rotating compressed-cache copies "
                         "of that shape (larger than L2 for B*L >= 64k), six mustafar_decode_attn launches, no timing")
    ap.add_argument("--profile-compress", default=None,
                    help="ncu case: 'PATTERN,s' (topk or channel) -- prefill compress of one [8, 16384, 8, 128] "
                         "fp16 tensor ([B, L, H, d] storage), three launches, no timing")
    args = ap.parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.suite:
        import unstructured_sparse_kv_b200 as M
        import suite
        M.load()
        suite.run(args.suite, measured_peak()[0], tuple(args.suite_parts.split(",")))
        return 0
    if args.profile_compress:
        import torch
        import unstructured_sparse_kv_b200 as M
        M.load()
        pattern, sp = args.profile_compress.split(",")
        B, L, H, d = 8, 16384, 8, 128
        g = torch.Generator(device="cuda")
        g.manual_seed(5)
        x = torch.randn(B, L, H, d, generator=g, device="cuda").to(torch.float16)
        c = M.CompressedCache(B, H, L, float(sp), pattern=pattern)
        for _ in range(3):
            M.mustafar_compress(x.permute(0, 2, 1, 3), L, float(sp), c)
        torch.cuda.synchronize()
        print(json.dumps({"profile_case": "compress", "pattern": pattern, "sparsity": float(sp), "launches": 3}))
        return 0
    if args.profile_shape:
        import torch
        import unstructured_sparse_kv_b200 as M
        from unstructured_sparse_kv_b200 import synth
        M.load()
        B, L = (int(x) for x in args.profile_shape.split(",")[:2])
        sK, sV = (float(x) for x in args.profile_shape.split(",")[2:4])
        Hq, Hkv, d, dev = 32, 8, 128, torch.device("cuda", 0)
        K, V = synth.keys(B, Hkv, L, d, 5, dev), synth.values(B, Hkv, L, d, 5, dev)
        q = synth.queries(B, Hq, d, 5, dev)
        seq = torch.full((B,), L, dtype=torch.int32, device=dev)
        copies = []
        for _ in range(2):
            kc, vc = M.CompressedCache(B, Hkv, L, sK, device=dev), M.CompressedCache(B, Hkv, L, sV, device=dev)
            M.mustafar_compress(K, L, sK, kc)
            M.mustafar_compress(V, L, sV, vc)
            copies.append((kc, vc))
        del K, V
        out = torch.empty_like(q)
        lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
        ws = torch.zeros(M.mustafar_decode_workspace_bytes(B, Hq, Hkv, L), dtype=torch.uint8, device=dev)
        for i in range(6):
            kc, vc = copies[i % 2]
            M.mustafar_decode_attn(q, kc, vc, seq, L, 1.0, out=out, lse=lse, workspace=ws)
        torch.cuda.synchronize()
        print(json.dumps({"profile_case": "decode_attn", "batch": B, "context": L, "sparsity_k": sK,
                          "sparsity_v": sV, "launches": 6}))
        return 0
    if args.profile_launches > 0:
        import torch
        import unstructured_sparse_kv_b200 as M
        M.load()
        wl = Workload(rank_seed(0), torch.device("cuda", 0))
        for i in range(args.profile_launches):
            wl.step(i)
        torch.cuda.synchronize()
        print(json.dumps({"profile_case": "decode step workload", "steps": args.profile_launches,
                          "compressed_kv_bytes_per_copy": wl.compressed_bytes, "copies": ROTATE}))
        return 0

    import torch
    import torch.distributed as dist

    import unstructured_sparse_kv_b200 as M
    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", init_method="env://", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    M.load()
    wl = Workload(rank_seed(rank), dev)
    stream = torch.cuda.current_stream()

    # ---- the timed region: exactly K fused steps, replayed from CUDA graphs (one launch per step)
    timed, timed_graphs = wl.exact(args.steps)
    warm, warm_graphs = wl.exact(args.warmup) if args.warmup > 0 else (lambda: None, [])
    leg64 = wl.capture(GRAPH_STEPS)  # 64-step graph of the same fused step for the clock soak
    for g in timed_graphs + warm_graphs:  # a graph is uploaded to the device at its first launch: not timed
        g.replay()
    torch.cuda.synchronize()
    with ClockSampler(dev) as clocks:
        # keep the GPU under load for about a second before the timed region, so that its clocks are
        # the loaded ones and the sampler has a record around the timed region
        soak_reps = max(1, int(0.8e6 / (GRAPH_STEPS * 40.0)))
        for _ in range(soak_reps):
            leg64.replay()
        warm()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        clocks.mark()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        # ~100 us of device work ahead of the start event, so that the host's enqueueing of the timed
        # graph launches overlaps it and never shows up as device idle time inside the region
        torch.cuda._sleep(200_000)
        e0.record(stream)
        timed()
        e1.record(stream)
        torch.cuda.synchronize()
        clocks.mark()
        barrier()
    elapsed_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    us_per_step = aggregate_us_per_step(elapsed_ms, args.steps, world)
    clk = clocks.summary()
    del timed_graphs, warm_graphs

    # ---- the dominant (and only) kernel of the step is the fused decode kernel: one launch per
    # step, so its average launch duration is the timed region's time per step
    lens = [wl.L0 + 1 + i for i in range(wl.steps)]
    avg_bytes = sum(decode_algorithmic_bytes(wl.B, wl.Hq, wl.Hkv, wl.d, [L] * wl.B, wl.kc[0].keep, wl.vc[0].keep)
                    for L in lens) / len(lens)
    peak, peak_kind = measured_peak()
    achieved = avg_bytes / (us_per_step * world * 1e-6) / 1e9  # per launch on one GPU

    # ---- comparison legs, all timed alike: replays of 64-step graphs over the same rotation
    leg_steps = GRAPH_STEPS * max(8, min(100, args.steps // GRAPH_STEPS))

    def time_leg(g):
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        return time_graph(g, leg_steps // GRAPH_STEPS, stream) * 1000.0 / leg_steps

    legs = {"fused": time_leg(leg64)}
    del leg64
    for mode in ("separate", "attend"):
        g = wl.capture(GRAPH_STEPS, mode=mode)
        legs[mode] = time_leg(g)
        del g
    dense = DenseBaseline(wl)
    g = wl.capture(GRAPH_STEPS, run=dense.step)
    legs["dense"] = time_leg(g)
    del g
    att_us, dense_us = legs["attend"], legs["dense"]
    dense_bytes = sum(4 * wl.B * wl.Hkv * L * wl.d for L in lens) / len(lens) + 4 * wl.B * wl.Hq * wl.d

    # ---- the sparsity axis: attention alone over caches compressed at each sparsity (K and V alike),
    # the same inputs, rotation and timing; dense fp16 on the same inputs is the leg above
    by_sparsity = []
    for sp in SPARSITY_AXIS:
        pt = SparsityPoint(wl, sp)
        g = wl.capture(GRAPH_STEPS, run=pt.step)
        us = time_leg(g)
        del g
        b = sum(decode_algorithmic_bytes(wl.B, wl.Hq, wl.Hkv, wl.d, [L] * wl.B, pt.keep, pt.keep)
                for L in lens) / len(lens)
        by_sparsity.append({"sparsity": sp, "keep": pt.keep, "attend_us": us, "gbs": b / (us * 1e-6) / 1e9,
                            "frac": b / (us * 1e-6) / 1e9 / peak, "algorithmic_bytes_per_launch": b,
                            "dense_us": dense_us, "speedup_vs_dense": dense_us / us,
                            "compressed_over_dense_bytes": pt.nbytes / wl.dense_cache_bytes})
        del pt
    dense.release()

    # ---- end to end through the public API with host buffers (eager calls)
    e2e = None
    if True:  # end-to-end leg
        # one pinned host record per step (q | k_new | v_new | pos, each 16-byte aligned), one H2D copy
        # into a device twin, one prepared library call, one D2H copy of out
        parts = [wl.q[0], wl.kn[0], wl.vn[0], wl.pos[0]]
        sizes = [t.numel() * t.element_size() for t in parts]
        offs = [sum(sizes[:i]) for i in range(len(sizes))]
        rec = sum(sizes)
        hin = torch.empty((wl.steps, rec), dtype=torch.uint8).pin_memory()
        for j in range(wl.steps):
            for t, o, n in zip((wl.q[j], wl.kn[j], wl.vn[j], wl.pos[j]), offs, sizes):
                hin[j, o:o + n].copy_(t.contiguous().view(torch.uint8).reshape(-1).cpu())
        outh = torch.empty((wl.steps,) + tuple(wl.out.shape), dtype=torch.float16).pin_memory()
        # two device buffer sets, so that the H2D copy of step i+1 and the D2H copy of step i overlap the
        # attention of their neighbours (copies on two side streams, ordered by events)
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        din = [torch.empty(rec, dtype=torch.uint8, device=dev) for _ in range(2)]
        dout, dlse = [torch.empty_like(wl.out) for _ in range(2)], [torch.empty_like(wl.lse) for _ in range(2)]
        cs = torch.cuda.Stream(dev)  # the graph below is captured on a stream of its own

        def prepared(st):
            # per buffer set and cache copy, the prepared library call launching on stream st
            table = []
            for b in range(2):
                v = [din[b][o:o + n].view(t.dtype).view(t.shape) for t, o, n in zip(parts, offs, sizes)]
                table.append([M.prepare_decode_step(v[0], v[1], v[2], v[3], wl.kc[r], wl.vc[r], wl.cap, 1.0,
                                                    out=dout[b], lse=dlse[b], workspace=wl.ws, stream=st)[0]
                              for r in range(ROTATE)])
            return table

        calls = {stream: prepared(stream), cs: prepared(cs)}
        ev_in, ev_k, ev_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))
        n_e2e = 64 * 10

        def e2e_step(i, st=stream):
            j, r, b = i % wl.steps, i % ROTATE, i % 2
            s_in.wait_event(ev_k[b])  # the attention that last read din[b] has finished
            with torch.cuda.stream(s_in):
                din[b].copy_(hin[j], non_blocking=True)
            ev_in[b].record(s_in)
            st.wait_event(ev_in[b])
            st.wait_event(ev_out[b])  # the D2H copy that last read dout[b] has finished
            calls[st][b][r]()
            ev_k[b].record(st)
            s_out.wait_event(ev_k[b])
            with torch.cuda.stream(s_out):
                outh[j].copy_(dout[b], non_blocking=True)
            ev_out[b].record(s_out)

        for i in range(64):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        s_in.wait_event(f0)  # no copy of the timed steps starts before the clock does
        s_out.wait_event(f0)
        for i in range(n_e2e):
            e2e_step(i)
        stream.wait_event(ev_out[(n_e2e - 1) % 2])  # the last result is on the host
        f1.record(stream)
        torch.cuda.synchronize()
        barrier()
        eager_ms = max_over_ranks(f0.elapsed_time(f1), dev)

        # the same steps, copies included, recorded once as a CUDA graph of the workload's decode steps
        # and replayed (a serving loop's usual form): per step the same H2D copy from the step's pinned
        # record, the same library call and the same D2H copy, with the same stream and event order
        g = torch.cuda.CUDAGraph()
        cs.wait_stream(stream)
        with torch.cuda.graph(g, stream=cs):
            for e in ev_k + ev_out:  # the first steps wait on events recorded inside the capture
                e.record(cs)
            s_in.wait_stream(cs)
            s_out.wait_stream(cs)
            for i in range(wl.steps):
                e2e_step(i, cs)
            cs.wait_stream(s_in)
            cs.wait_stream(s_out)
        stream.wait_stream(cs)
        reps = n_e2e // wl.steps
        g.replay()
        torch.cuda.synchronize()
        barrier()
        torch.cuda._sleep(200_000)  # the timed replays queue behind a short device sleep
        f0.record(stream)
        for _ in range(reps):
            g.replay()
        f1.record(stream)  # every replay ends with its last D2H copy joined into the stream
        torch.cuda.synchronize()
        barrier()
        graph_ms = max_over_ranks(f0.elapsed_time(f1), dev)
        del g
        bi = (wl.q[0].numel() + wl.kn[0].numel() + wl.vn[0].numel()) * 2 + wl.pos[0].numel() * 4
        e2e = {"value": aggregate_us_per_step(graph_ms, reps * wl.steps, world), "unit": UNIT,
               "h2d_bytes_per_step": bi, "d2h_bytes_per_step": wl.out.numel() * 2, "steps": reps * wl.steps,
               "how": "public API, every step: one H2D copy of the step's q/k_new/v_new/pos record from pinned "
                      "host memory, one prepared mustafar_decode_step call (one fused launch), one D2H copy of "
                      "out into pinned host memory; copies on side streams into two buffer sets, so they overlap "
                      "the neighbouring steps; the workload's 64 steps recorded as one CUDA graph and replayed",
               "eager": {"value": aggregate_us_per_step(eager_ms, n_e2e, world), "unit": UNIT, "steps": n_e2e,
                         "how": "the same steps issued one by one from Python"}}

    line = {"metric": METRIC, "value": us_per_step, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": us_per_step / 1000.0, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic", "config": config_dict(),
            "gpu_launches": args.steps,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                         "peak_kind": peak_kind, "traffic": recorded_traffic(),
                         "kernel": "sparse_decode_kernel (fused append)", "algorithmic_bytes_per_launch": avg_bytes,
                         "us_per_launch": us_per_step * world, "splits": wl.splits},
            "legs": {"how": f"replays of 64-step CUDA graphs, {leg_steps} steps each, same rotation",
                     "fused_us": legs["fused"], "separate_us": legs["separate"], "attend_us": att_us,
                     "dense_us": dense_us, "attend_frac": avg_bytes / (att_us * 1e-6) / 1e9 / peak,
                     "dense_frac": dense_bytes / (dense_us * 1e-6) / 1e9 / peak,
                     "sparse_speedup": dense_us / att_us, "fused_step_speedup": dense_us / legs["fused"],
                     "fused_over_separate": legs["separate"] / legs["fused"],
                     "separate": "append K + append V + decode_attn, 3 launches per step",
                     "dense_bytes_per_launch": dense_bytes},
            "by_sparsity": by_sparsity,
            "compressed_kv_bytes": wl.compressed_bytes,
            "clocks": clk, "e2e": e2e}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_decode_sample()
        line["cpu_baseline"]["all_cores"] = oracle_decode_all_cores()
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

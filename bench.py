#!/usr/bin/env python
"""Decode-attention benchmark over a paged KV cache (one JSON line on rank 0).

A step is one call of the library's decode entry point (device-side split
planning, the decode kernel and the LSE-combine kernel) over one batch of the
synthetic workload.  Default workload: GLA-2 decode (the largest configuration
that fits one GPU), batch 128, q_len 1, h_q 128 over two 256-wide latent heads
plus one shared 64-wide RoPE key, lognormal contexts (median 8192, capped at
65536), page size 64, shuffled block table.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload W] [--qlen L] [--page-size S]
  python bench.py --workload gta_prefix|gta_prefix_long [--cascade]   # shared-prefix decode
  python bench.py --workload append_gta|append_gqa|append_mla|append_gla2 [--tokens N]   # cache append + RoPE
  python bench.py --impl reference ...   # the fp64 CPU oracle timed on this host

Decode workloads W: gla2 (default), gta, gqa, mla, gla8, gta_tiny, gta_prefix, gta_prefix_long.

Multi-GPU: the path has no exchange step (sequences are independent), so N GPUs
run N independent replicas of the step (weak scaling, no collective on the data
path); the reported time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from kv_cache_paged_b200 import accounting, workload as wl  # noqa: E402

METRIC = "decode-attention µs/step and KV-cache GB/s as % of B200 HBM peak (1 GPU)"
UNIT = "us/step"
FALLBACK_HBM_GBS, FALLBACK_TFLOPS = 6650.0, 1590.0
L2_FLUSH_BYTES = 256 << 20  # > 126 MB L2
KERNEL_SOURCES = {"group": ["kv_cache_paged_b200/csrc/group_decode.cu", "kv_cache_paged_b200/csrc/common.cuh"],
                  "narrow": ["kv_cache_paged_b200/csrc/latent_narrow.cu", "kv_cache_paged_b200/csrc/common.cuh"],
                  "m128": ["kv_cache_paged_b200/csrc/latent_m128.cu", "kv_cache_paged_b200/csrc/common.cuh"],
                  "pair": ["kv_cache_paged_b200/csrc/latent_pair.cu", "kv_cache_paged_b200/csrc/common.cuh"],
                  "append": ["kv_cache_paged_b200/csrc/append.cu", "kv_cache_paged_b200/csrc/common.cuh"]}
KERNEL_NAMES = {"group": "group_decode_kernel", "narrow": "gla_narrow_kernel",
                "m128": "gla_m128_kernel",
                "pair": "mla_pair_kernel"}


def kernel_kind(inp):
    """Which decode kernel the library runs for these inputs (mirrors the dispatch in csrc/api.cu)."""
    if inp.variant != "gla":
        return "group"
    if inp.d == 512:
        return "pair"
    return "narrow" if (inp.h_q // inp.h_kv) * inp.L <= 64 else "m128"  # query rows per latent head


def describe(inp):
    sl = inp.seqlens
    if inp.variant == "gla":
        kind = "MLA" if inp.h_kv == 1 else f"GLA-{inp.h_kv}"
        shape = f"h_q {inp.h_q}, h_c {inp.h_kv}, d_c {inp.d}, d_r {inp.d_r}"
    elif inp.variant == "gta":
        kind, shape = "GTA", f"h_q {inp.h_q}, h_kv {inp.h_kv}, d_h {inp.d}, d_r {inp.d_r}"
    else:
        kind, shape = "GQA", f"h_q {inp.h_q}, h_kv {inp.h_kv}, d {inp.d}"
    pre = (f", the first {inp.shared_prefix} tokens a prefix shared by the batch (stored once; "
           f"algorithmic bytes count it once)") if getattr(inp, "shared_prefix", 0) else ""
    return (f"{kind} paged decode: B {inp.B}, q_len {inp.L}, {shape}, page {inp.page_size}, "
            f"contexts {int(sl.min())}..{int(sl.max())} (mean {float(sl.mean()):.0f}){pre}")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_TFLOPS, "fallback"


def kernel_hash(kind):
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kind]:
        p = os.path.join(ROOT, rel)
        if os.path.exists(p):
            h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


def committed_traffic(kind, workload, qlen):
    """DRAM bytes per launch from a committed ncu summary, if taken on the current kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        e = d.get(f"{workload}_L{qlen}")
        if e and e.get("kernel_sha") == kernel_hash(kind):
            return float(e["dram_bytes_per_launch"])
    except Exception:
        return None
    return None


# ----------------------------------------------------------------------------- ranks
def max_over_ranks(vals, dist=None, device="cpu"):
    """Each value's maximum over all ranks: a replica step is as slow as the slowest GPU."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return [float(v) for v in vals]
    import torch
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def aggregate(step_us, kv_bytes, world):
    """Whole-job KV throughput of `world` replicas that each moved kv_bytes in step_us (max over ranks)."""
    return world * kv_bytes / (step_us * 1e-6) / 1e9


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock/throttle samples for one GPU while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.rows = []
        self.proc = None
        self.t_on = self.t_off = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu_id), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.th = threading.Thread(target=self._read, daemon=True)
        self.th.start()
        time.sleep(0.5)

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), line.strip()))

    def mark_on(self):
        self.t_on = time.time()

    def mark_off(self):
        self.t_off = time.time()

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = [r for t, r in self.rows if self.t_on is not None and self.t_on - 0.1 <= t <= self.t_off + 0.15]
        if not rows:
            rows = [r for _, r in self.rows]
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            f = [x.strip() for x in r.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- oracle timing
def oracle_sample(inp, budget_s, threads=0):
    """Time the fp64 oracle on a prefix of the batch sized to about budget_s seconds of CPU work
    (threads 0: every core).  Returns (seconds, fraction of the step's work, threads, sequences)."""
    from oracle import oracle as orc
    work = np.maximum(inp.seqlens.astype(np.float64), 0)
    total = work.sum()
    t0 = time.perf_counter()
    _, _, threads = orc.decode_inputs(inp, b_list=np.array([0], np.int32), threads=threads)
    t1 = time.perf_counter() - t0
    per_tok = t1 / max(work[0], 1)
    n, acc = 0, 0.0
    while n < inp.B and (acc + work[n]) * per_tok <= budget_s:
        acc += work[n]
        n += 1
    n = max(n, 1)
    bl = np.arange(n, dtype=np.int32)
    t0 = time.perf_counter()
    _, _, threads = orc.decode_inputs(inp, b_list=bl, threads=threads)
    dt = time.perf_counter() - t0
    return dt, float(work[:n].sum() / total), threads, n


def run_reference(args, inp, cfg, rank):
    """The reference arm: the fp64 CPU oracle, timed as it stands on this host."""
    if rank != 0:
        return
    K, W = args.steps, args.warmup
    budget = max(0.02, min(2.0, 150.0 / max(1, K + W)))
    for _ in range(W):
        oracle_sample(inp, budget)
    per_step = []
    frac = threads = n = None
    for _ in range(K):
        dt, frac, threads, n = oracle_sample(inp, budget)
        per_step.append(dt / frac * 1e6)
    v = float(statistics.mean(per_step))
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus, "steps": K,
            "warmup": W, "ms_per_step": v / 1e3, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": f"first {n} of {inp.B} sequences per step ({frac:.3f} of the step's "
                                       f"work), time scaled to the whole step"},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- cache append
APPEND_SHAPES = {  # per new token, GTA/GLA: `heads` state rows of `dim` and one d_r rope slice;
    # GQA: `heads` K rows (the last d_r dims of each rotated) and `heads` V rows of `dim`
    "append_gta": dict(kind="gta", heads=8, dim=128, d_r=64),
    "append_gqa": dict(kind="gqa", heads=8, dim=128, d_r=128),
    "append_mla": dict(kind="gla", heads=1, dim=512, d_r=64),
    "append_gla2": dict(kind="gla", heads=2, dim=256, d_r=64),
}
APPEND_METRIC = "cache append (state copy + RoPE) us/call and GB/s as % of B200 HBM peak (1 GPU)"


def append_bytes(sh, n):
    """Algorithmic bytes of one append of n tokens: every stored element read once and written once,
    plus the positions and slot indices."""
    if sh["kind"] == "gqa":
        elems = 2 * sh["heads"] * sh["dim"]
    else:
        elems = sh["heads"] * sh["dim"] + sh["d_r"]
    return n * (elems * 2 * 2 + 8)


def append_inputs(sh, n, seed=31):
    rng = np.random.default_rng(seed)
    rows = ((n + 63) // 64 + 8) * 64
    f = lambda shape: wl.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))
    if sh["kind"] == "gqa":
        srcs = [f((n, sh["heads"], sh["dim"])), f((n, sh["heads"], sh["dim"]))]
        dsts = [(rows // 64, 64, sh["heads"], sh["dim"])] * 2
    else:
        srcs = [f((n, sh["heads"], sh["dim"])), f((n, sh["d_r"]))]
        dsts = [(rows // 64, 64, sh["heads"], sh["dim"]), (rows // 64, 64, sh["d_r"])]
    pos = rng.integers(0, 65536, n).astype(np.int32)
    slot = rng.permutation(rows)[:n].astype(np.int32)
    return srcs, dsts, pos, slot


def oracle_append(sh, srcs, pos, n):
    """The reference arm for the append: the oracle's fp64 rotation of every RoPE slice plus a copy."""
    from oracle import oracle as orc
    x = wl.bf16_bits_to_f32(srcs[0][:n] if sh["kind"] == "gqa" else srcs[1][:n]).astype(np.float64)
    for t in range(n):
        if sh["kind"] == "gqa":
            for h in range(sh["heads"]):
                orc.rope(x[t, h, sh["dim"] - sh["d_r"]:], float(pos[t]))
        else:
            orc.rope(x[t], float(pos[t]))
    return [np.copy(a[:n]) for a in srcs]


def run_append(args, rank):
    sh = APPEND_SHAPES[args.workload]
    n = args.tokens
    nbytes = append_bytes(sh, n)
    cfg = {"workload": f"{sh['kind'].upper()} cache append of {n} tokens into a paged cache (page 64, random "
                       f"slot_mapping, positions in [0, 65536)), heads {sh['heads']} x {sh['dim']}, d_r {sh['d_r']}",
           "tokens": n, "algorithmic_bytes_per_call": int(nbytes), "parallelism": "replicas1",
           "l2": "a 256 MiB read evicts L2 before every timed call"}
    srcs, dsts, pos, slot = append_inputs(sh, n)
    # the oracle on a bounded sample, scaled to the call (rank 0, N = 1 only)
    t_cpu = None
    if rank == 0 and (args.impl == "reference" or not args.no_cpu_baseline):
        m = min(n, 2048)
        t0 = time.perf_counter()
        oracle_append(sh, srcs, pos, m)
        t_cpu = (time.perf_counter() - t0) / m * n * 1e6
        cpu = {"value": t_cpu, "unit": "us/call", "cores": 1, "kind": "oracle",
               "sample": f"{m} of {n} tokens, time scaled to the call"}
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps({"impl": "reference", "metric": APPEND_METRIC, "value": t_cpu, "unit": "us/call",
                              "n_gpus": args.gpus, "steps": 1, "warmup": 0, "ms_per_step": t_cpu / 1e3,
                              "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                              "data": "synthetic", "config": cfg, "cpu_baseline": cpu,
                              "e2e": {"value": t_cpu, "unit": "us/call", "h2d_bytes_per_step": 0,
                                      "d2h_bytes_per_step": 0}}), flush=True)
        return
    import torch
    from kv_cache_paged_b200 import binding
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    s0, s1 = bf(srcs[0]), bf(srcs[1])
    c0 = torch.zeros(dsts[0], dtype=torch.bfloat16, device=dev)
    c1 = torch.zeros(dsts[1], dtype=torch.bfloat16, device=dev)
    dpos, dslot = torch.from_numpy(pos).to(dev), torch.from_numpy(slot).to(dev)
    flush = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    st = torch.cuda.Stream(device=dev)

    def call():
        if sh["kind"] == "gqa":
            binding.gqa_append(s0, s1, dpos, dslot, c0, c1, sh["d_r"], stream=st)
        elif sh["kind"] == "gta":
            binding.gta_append(s0, s1, dpos, dslot, c0, c1, stream=st)
        else:
            binding.gla_append(s0, s1, dpos, dslot, c0, c1, stream=st)

    with torch.cuda.stream(st):
        for _ in range(args.warmup):
            flush.max()
            call()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        torch.cuda.synchronize()
        clk = ClockSampler(dev.index)
        clk.start()
        clk.mark_on()
        for a, b in ev:
            flush.max()
            a.record(st)
            call()
            b.record(st)
        torch.cuda.synchronize()
        clk.mark_off()
        clocks = clk.stop()
        us = statistics.mean(a.elapsed_time(b) for a, b in ev) * 1e3
        # end to end: the new tokens' inputs from pinned host memory, the call, one word back
        hs = [torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).pin_memory() for x in srcs]
        hp, hsl = torch.from_numpy(pos).pin_memory(), torch.from_numpy(slot).pin_memory()
        e2e = []
        for _ in range(max(3, args.steps // 4)):
            flush.max()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(st)
            s0.view(torch.int16).copy_(hs[0], non_blocking=True)
            s1.view(torch.int16).copy_(hs[1], non_blocking=True)
            dpos.copy_(hp, non_blocking=True)
            dslot.copy_(hsl, non_blocking=True)
            call()
            word = c1.view(-1)[:1].cpu()
            b.record(st)
            torch.cuda.synchronize()
            e2e.append(a.elapsed_time(b) * 1e3)
    hbm, _, src = load_peaks()
    ach = nbytes / (us * 1e-6) / 1e9
    h2d = sum(x.nbytes for x in srcs) + pos.nbytes + slot.nbytes
    line = {"metric": APPEND_METRIC, "value": us, "unit": "us/call", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": us / 1e3, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16 copy, f64 rotation", "data": "synthetic", "config": cfg,
            "roofline": {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                         "traffic": committed_traffic("append", args.workload, 1) if n == 65536 else None,
                         "peak_source": src, "kernel": "append_kernel", "kernel_us": us},
            "e2e": {"value": statistics.mean(e2e), "unit": "us/call", "h2d_bytes_per_step": int(h2d),
                    "d2h_bytes_per_step": 2},
            "gpu_launches": args.steps, "clocks": clocks}
    if t_cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="kvd", choices=["kvd", "reference"])
    ap.add_argument("--workload", default="gla2", choices=["gta", "gqa", "mla", "gla2", "gta_tiny", "gta_prefix", "gta_prefix_long", "gla8"] + list(APPEND_SHAPES))
    ap.add_argument("--tokens", type=int, default=65536, help="new tokens per call (append workloads)")
    ap.add_argument("--qlen", type=int, default=1)
    ap.add_argument("--page-size", type=int, default=0, help="override the workload's page size (tokens per page)")
    ap.add_argument("--cascade", action="store_true",
                    help="gta_prefix: batched shared-prefix decode + continuation decode + merge per step")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))

    if args.workload in APPEND_SHAPES:
        run_append(args, rank)
        return
    over = {"page_size": args.page_size} if args.page_size > 0 else {}
    inp = wl.make_workload(args.workload, L=args.qlen, **over)
    nbytes, flops, kvb = accounting.of_inputs(inp)
    cfg = {"workload": describe(inp), "global_batch": inp.B * world, "seq_len": int(inp.seqlens.max()),
           "q_len": inp.L, "seed": wl.SEEDS[args.workload], "parallelism": f"replicas{world}",
           "l2": "inputs larger than L2 (KV stream vs 126 MB L2) and, before every timed step, a 256 MiB "
                 "read that evicts the previous step's lines without leaving dirty ones",
           "kv_bytes_per_step": int(kvb), "algorithmic_bytes_per_step": int(nbytes),
           "flops_per_step": int(flops)}

    if args.impl == "reference":
        run_reference(args, inp, cfg, rank)
        return

    import torch
    from kv_cache_paged_b200 import binding

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist

    def barrier():
        if pg is not None:
            pg.barrier()

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)

    caches = {k: bf(v).to(dev) for k, v in inp.caches.items()}

    def packed(arrays):
        """One pinned host buffer and one device buffer holding the given arrays (256-byte
        aligned segments), so that a step's inputs cross PCIe in one copy; returns the host
        buffer, the device buffer and device tensor views of each array."""
        offs, n = [], 0
        for a in arrays:
            offs.append(n)
            n += (a.nbytes + 255) // 256 * 256
        host = torch.empty(max(n, 256), dtype=torch.uint8).pin_memory()
        for a, o in zip(arrays, offs):
            host[o:o + a.nbytes].numpy()[:] = np.ascontiguousarray(a).view(np.uint8).reshape(-1)
        devbuf = host.to(dev)
        views = [devbuf[o:o + a.nbytes].view(torch.int16 if a.dtype == np.uint16 else torch.int32).view(
            torch.bfloat16 if a.dtype == np.uint16 else torch.int32).reshape(a.shape) for a, o in zip(arrays, offs)]
        return host, devbuf, views

    in_h, in_d, (q, bt, sl) = packed([inp.q, inp.block_table, inp.seqlens])
    d_v = inp.d
    rows_out = inp.B * inp.L * inp.h_q
    out_bytes = (rows_out * d_v * 2 + 255) // 256 * 256
    res_d = torch.empty(out_bytes + rows_out * 4, dtype=torch.uint8, device=dev)
    out = res_d[:rows_out * d_v * 2].view(torch.bfloat16).view(inp.B, inp.L, inp.h_q, d_v)
    lse = res_d[out_bytes:].view(torch.float32).view(inp.B, inp.L, inp.h_q)
    res_h = torch.empty(res_d.numel(), dtype=torch.uint8).pin_memory()
    ws = torch.zeros(1 << 30 if inp.variant == "gla" else 1 << 26, dtype=torch.uint8, device=dev)
    flush = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)

    def evict_l2():
        # A read of a buffer twice the size of L2 evicts every line of the previous step.  A
        # write would do the same but leave ~126 MB of dirty lines whose write-back then
        # competes with the timed step for HBM bandwidth.
        flush.max()
    stream = torch.cuda.Stream(device=dev)
    names = {"gqa": ("k_cache", "v_cache"), "gta": ("tied_cache", "rope_cache"),
             "gla": ("latent_cache", "rope_cache")}[inp.variant]
    fn = {"gqa": binding.gqa_decode, "gta": binding.gta_decode, "gla": binding.gla_decode}[inp.variant]
    c0, c1 = caches[names[0]], caches[names[1]]
    launches_per_step = 2  # decode kernel (planning fused in) + LSE combine

    def step(qq, btt, sll, oo=None, ll=None):
        fn(qq, c0, c1, btt, sll, inp.scale, out=out if oo is None else oo, lse=lse if ll is None else ll,
           workspace=ws, stream=stream)

    if args.cascade:
        # cascade decoding of a batch-shared prefix: the prefix once for all rows of a KV group
        # (kvd_gta_prefix_decode), each sequence's own tokens (kvd_gta_decode over its own
        # pages), then kvd_merge_states.  The block table and seqlens a step uploads are the
        # continuation's; the prefix's pages are cached state like the KV cache.
        if inp.variant != "gta" or not getattr(inp, "shared_prefix", 0):
            raise SystemExit("--cascade needs a GTA workload with a shared prefix (gta_prefix)")
        P = inp.shared_prefix
        pp = P // inp.page_size
        suf = np.full_like(inp.block_table, -1)
        suf[:, : inp.max_pages - pp] = inp.block_table[:, pp:]
        in_h, in_d, (q, bt, sl) = packed([inp.q, suf, (inp.seqlens - P).astype(np.int32)])
        pre_bt = torch.from_numpy(np.ascontiguousarray(inp.block_table[:1, :pp])).to(dev)
        pre_len = torch.tensor([P], dtype=torch.int32, device=dev)
        out_p, lse_p = torch.empty_like(out), torch.empty_like(lse)
        out_s, lse_s = torch.empty_like(out), torch.empty_like(lse)
        ws_p = torch.zeros(1 << 28, dtype=torch.uint8, device=dev)
        launches_per_step = 5  # prefix kernel + combine, continuation kernel + combine, merge

        def step(qq, btt, sll, oo=None, ll=None):
            binding.gta_prefix_decode(qq, c0, c1, pre_bt, pre_len, inp.scale, out=out_p, lse=lse_p, workspace=ws_p,
                                      stream=stream)
            binding.gta_decode(qq, c0, c1, btt, sll, inp.scale, out=out_s, lse=lse_s, workspace=ws, stream=stream)
            binding.merge_states(out_p, lse_p, out_s, lse_s, out=out if oo is None else oo,
                                 lse=lse if ll is None else ll, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            evict_l2()
            step(q, bt, sl)
    err = binding.read_device_error(ws, stream)
    if err:
        raise SystemExit(f"device error flags after warm-up: {err}")

    gpu_index = torch.cuda.get_device_properties(dev).uuid if hasattr(torch.cuda.get_device_properties(dev), "uuid") else local
    sampler = ClockSampler(f"GPU-{gpu_index}" if not isinstance(gpu_index, int) else gpu_index)
    sampler.start()

    K = args.steps
    # (1) the timed steps: events around each whole call, nothing between its kernels
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    barrier()
    torch.cuda.synchronize(dev)
    sampler.mark_on()
    t_wall = time.perf_counter()
    with torch.cuda.stream(stream):
        for k in range(K):
            evict_l2()
            ev[k][0].record(stream)
            step(q, bt, sl)
            ev[k][1].record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    t_wall = time.perf_counter() - t_wall
    step_ms = [ev[k][0].elapsed_time(ev[k][1]) for k in range(K)]
    # (2) the same K steps again with events recorded by the library just before and after
    # its main decode kernel on the launching stream (the roofline's kernel time)
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    with torch.cuda.stream(stream):
        for k in range(K):          # create the events (torch creates them lazily on record)
            kev[k][0].record(stream)
            kev[k][1].record(stream)
        for k in range(K):
            evict_l2()
            binding.profile_events(kev[k][0], kev[k][1])
            step(q, bt, sl)
    torch.cuda.synchronize(dev)
    sampler.mark_off()
    binding.profile_events(None, None)
    kern_ms = [kev[k][0].elapsed_time(kev[k][1]) for k in range(K)]
    if args.cascade:
        kern_ms = step_ms  # several decode launches per step: the roofline takes the whole step
    clocks = sampler.stop()

    # end to end through the public API with host buffers: H2D of the step's inputs
    # (q, seqlens, block table) from pinned memory, the call, D2H of out and lse.
    KE = max(1, min(args.e2e_steps, K))
    ee = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(KE)]
    with torch.cuda.stream(stream):
        for k in range(KE):
            evict_l2()
            ee[k][0].record(stream)
            in_d.copy_(in_h, non_blocking=True)    # q, block table and seqlens: one copy
            step(q, bt, sl)
            res_h.copy_(res_d, non_blocking=True)  # out and lse: one copy
            ee[k][1].record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = [ee[k][0].elapsed_time(ee[k][1]) for k in range(KE)]

    # the same KE steps as a serving loop runs them: two sets of input and result buffers, the
    # H2D of step k + 1 and the D2H of step k - 1 on their own streams overlapping step k's
    # kernels; every step still moves its inputs in and its result out.  Per-step time = the
    # whole loop (first H2D issued to last D2H done) / KE.  No L2-eviction read between the steps
    # here (its time would count in the loop): each step's KV stream is larger than L2.
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    in_d2 = [in_d, torch.empty_like(in_d)]
    views2 = [(q, bt, sl), tuple(in_d2[1][t.data_ptr() - in_d.data_ptr():][:t.numel() * t.element_size()]
                                 .view(t.dtype).view(t.shape) for t in (q, bt, sl))]
    res_d2 = [res_d, torch.empty_like(res_d)]
    outs2 = [(out, lse), (res_d2[1][:rows_out * d_v * 2].view(torch.bfloat16).view(out.shape),
                          res_d2[1][out_bytes:].view(torch.float32).view(lse.shape))]
    res_h2 = [res_h, torch.empty_like(res_h).pin_memory()]
    ev_in, ev_c, ev_out = ([torch.cuda.Event() for _ in range(KE)] for _ in range(3))

    def enqueue_loop(origin):
        """The KE steps on s_in / stream / s_out, forked from and joined back into `origin`."""
        fork = torch.cuda.Event()
        fork.record(origin)
        for s_ in (s_in, stream, s_out):
            s_.wait_event(fork)
        for k in range(KE):
            i = k % 2
            if k >= 2:
                s_in.wait_event(ev_c[k - 2])     # input buffer i: step k - 2 has read it
            with torch.cuda.stream(s_in):
                in_d2[i].copy_(in_h, non_blocking=True)
            ev_in[k].record(s_in)
            stream.wait_event(ev_in[k])
            if k >= 2:
                stream.wait_event(ev_out[k - 2])  # result buffer i: step k - 2's result is out
            with torch.cuda.stream(stream):
                step(*views2[i], *outs2[i])
            ev_c[k].record(stream)
            s_out.wait_event(ev_c[k])
            with torch.cuda.stream(s_out):
                res_h2[i].copy_(res_d2[i], non_blocking=True)
            ev_out[k].record(s_out)
        for e_ in (ev_in[KE - 1], ev_c[KE - 1], ev_out[KE - 1]):
            origin.wait_event(e_)

    # the loop as a serving engine runs it, captured once in a CUDA graph so that the host does
    # not pace the short steps; timed over one replay.  If capture fails, the same loop enqueued
    # from the host is timed instead (and the line says so).
    origin = torch.cuda.Stream(device=dev)
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e2e_mode = "cuda graph of the steps, one replay timed"
    try:
        graph = torch.cuda.CUDAGraph()
        # thread-local capture: CUDA calls of other threads (NCCL's watchdog under torchrun) do not
        # invalidate it
        with torch.cuda.graph(graph, stream=origin, capture_error_mode="thread_local"):
            enqueue_loop(origin)
        with torch.cuda.stream(origin):
            graph.replay()              # warm
            p0.record(origin)
            graph.replay()
            p1.record(origin)
        torch.cuda.synchronize(dev)
        del graph
    except Exception as ex:  # noqa: BLE001 - measurement method only; the step itself is unchanged
        torch.cuda.synchronize(dev)
        e2e_mode = f"host-enqueued loop (graph capture failed: {type(ex).__name__})"
        p0.record(origin)
        enqueue_loop(origin)
        p1.record(origin)
        torch.cuda.synchronize(dev)
    e2e_pipe_ms = p0.elapsed_time(p1) / KE
    if not (torch.equal(res_h2[0], res_h2[1]) if KE >= 2 else True):
        raise SystemExit("the two result buffers of the pipelined e2e loop differ")
    err = binding.read_device_error(ws, stream)
    if err:
        raise SystemExit(f"device error flags after timing: {err}")

    # read-only calibration of device memory (kvd_read_stream, outside the timed regions): the
    # best rate at which a stream that only reads can arrive, reported beside the copy peak
    rbuf = torch.empty(2 << 30, dtype=torch.uint8, device=dev)
    sink = torch.zeros(1, dtype=torch.int64, device=dev)
    rd_ms = []
    with torch.cuda.stream(stream):
        for i in range(8):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            binding.read_stream(rbuf, sink, stream=stream)
            b.record(stream)
            b.synchronize()
            if i >= 3:
                rd_ms.append(a.elapsed_time(b))
    read_gbs = rbuf.numel() / (min(rd_ms) * 1e-3) / 1e9
    del rbuf

    t_step = statistics.mean(step_ms)
    t_kern = statistics.mean(kern_ms)
    t_e2e_serial = statistics.mean(e2e_ms)
    t_step, t_kern, t_e2e, t_e2e_serial = max_over_ranks([t_step, t_kern, e2e_pipe_ms, t_e2e_serial], pg,
                                                         device=dev)

    hbm, tfl, peak_src = load_peaks()
    variant_kind = kernel_kind(inp)
    tensor_bound = flops / (tfl * 1e12) > nbytes / (hbm * 1e9)
    if tensor_bound:
        achieved = flops / (t_kern * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tfl, "unit": "TFLOP/s", "frac": achieved / tfl}
    else:
        achieved = nbytes / (t_kern * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm}
    roof["peak_source"] = f"{peak_src} (MEASURED_PEAKS.json)" if peak_src == "measured" else "fallback"
    roof["peak_read"] = read_gbs
    roof["peak_read_source"] = "kvd_read_stream: best of 5 streaming reads of 2 GiB in this process (GB/s)"
    if not tensor_bound:
        roof["frac_read"] = achieved / read_gbs
    roof["kernel"] = KERNEL_NAMES[variant_kind]
    roof["kernel_us"] = t_kern * 1e3
    # the committed ncu traffic was taken on the workload's own page size
    roof["traffic"] = committed_traffic(variant_kind, args.workload, inp.L) if args.page_size <= 0 else None
    roof["roofline_us"] = accounting.roofline_us(nbytes, flops, hbm, tfl)

    kv_gbs = aggregate(t_step * 1e3, kvb, 1)
    line = {"metric": METRIC, "value": t_step * 1e3, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": t_step, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
            "kv_gbs": kv_gbs * world, "kv_gbs_per_gpu": kv_gbs, "kv_frac_of_hbm_peak": kv_gbs / hbm,
            "step_us_p10_p50_p90": [float(np.percentile(step_ms, p) * 1e3) for p in (10, 50, 90)],
            "roofline_frac_of_step": roof["roofline_us"] / (t_step * 1e3),
            "roofline": roof,
            "e2e": {"value": t_e2e * 1e3, "unit": UNIT,
                    "h2d_bytes_per_step": int(in_h.numel()), "d2h_bytes_per_step": int(res_h.numel()),
                    "schedule": "two buffer sets; step k+1's H2D and step k-1's D2H overlap step k on their "
                                "own streams; per step = whole loop / steps; no L2 eviction between steps (the "
                                "KV stream of a step exceeds L2); " + e2e_mode,
                    "serial_value": t_e2e_serial * 1e3,
                    "serial_schedule": "H2D, the call, D2H on one stream, mean of per-step events"},
            "gpu_launches": K * launches_per_step, "timed_region_wall_s": t_wall,
            "kernel_timing": ("whole steps (cascade: several decode launches per step)" if args.cascade else
                              "second pass of K steps with events around the decode kernel"),
            "clocks": clocks}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # a bounded sample of about cpu_budget seconds: a prefix of the batch, repeated when
        # the whole step takes the oracle much less than the budget
        dt, frac, threads, n = oracle_sample(inp, args.cpu_budget)
        reps, total = 1, dt
        while total < 0.5 * args.cpu_budget and reps < 1000:
            d2, _, _, _ = oracle_sample(inp, args.cpu_budget)
            total += d2
            reps += 1
        line["cpu_baseline"] = {"value": total / reps / frac * 1e6, "unit": UNIT, "cores": threads,
                                "kind": "oracle",
                                "sample": f"first {n} of {inp.B} sequences ({frac:.3f} of the step's work), "
                                          f"{reps} run(s) in {total:.1f} s, mean scaled to the whole step"}
        # the same oracle on one thread, on a smaller sample
        dt1, frac1, _, n1 = oracle_sample(inp, args.cpu_budget / 3, threads=1)
        line["cpu_baseline"]["single_thread"] = {
            "value": dt1 / frac1 * 1e6, "unit": UNIT, "cores": 1,
            "sample": f"first {n1} of {inp.B} sequences ({frac1:.4f} of the step's work) in {dt1:.1f} s, "
                      f"scaled to the whole step"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()


if __name__ == "__main__":
    main()

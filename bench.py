"""Benchmark of the MLA absorb decode step on B200.

One step = the whole hot path on one batch: mla_absorb_q -> mla_attn_decode
(split-t + combine) -> mla_out_proj, for the DeepSeek-V3 decode workload
(batch 8, 128 heads, kv_lora_rank 512, rope 64, one query per sequence,
4096 cached tokens each), seeded synthetic inputs resident in HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line.  `value` is microseconds per step (lower is better),
the max over ranks; with N > 1 every rank runs an independent replica (the
path has no cross-GPU exchange).  Inputs are larger than L2: every per-step
input (q, kv and pe caches, wkv_b) exists in several copies, step i uses copy
i mod copies, and between two uses of one copy the other copies move more than
twice the L2 size, so each step reads its inputs from HBM.  The K timed steps
run back to back (CUDA-graph replays of the public calls) between two CUDA
events.  `--impl reference` times the fp64 CPU oracle on the host cores
instead, one (sequence, head) pair per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MLA absorb decode µs/step & cache GB/s, TFLOP/s as % of roofline (1×B200)"
UNIT = "us/step"
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS = 6650.0, 1590.0
KV_BYTES_PER_TOKEN = (512 + 64) * 2            # latent + rotary key, bf16
FLOP_PER_TOKEN_PER_HEAD = 2 * (576 + 512)      # score and value products
L2_BYTES = 126 << 20                           # B200 L2
ROTATE_MIN_BYTES = 2 * L2_BYTES                # traffic between two uses of one input copy


MIN_TIMED_MS = 200.0                           # least total length of a repeated timed region
CHAIN = 8                                      # steps per graph for the chained-step time


def decode_algorithmic(w):
    """Algorithmic bytes and flop of one decode attention call: the cache rows (kv + pe) of every
    visible key, and per query row q_abs, q_pe in and o_lat out; 2 * H * (576 + 512) flop per key."""
    B, H, C = w.batch, w.dims.heads, w.dims.kv_lora_rank
    alg_bytes = w.total_k * KV_BYTES_PER_TOKEN + B * H * (C + w.dims.qk_rope + C) * 2
    return alg_bytes, w.total_k * H * FLOP_PER_TOKEN_PER_HEAD


class DecodeBench:
    """A decode workload resident on the GPU in rotating copies (together larger than twice L2),
    with CUDA graphs of the public calls: the whole step (absorb, attention, merge fused into the
    output projection), the attention call (attention kernel + split merge) and the attention
    kernel alone (split partials left in the workspace)."""

    def __init__(self, w, dev, warmup):
        import torch
        from deepseek_mla_latent_b200 import mla
        self.w, self.dev = w, dev
        self.d = d = mla.dims_from(w.dims)
        self.dt = dt = torch.bfloat16 if w.dims.dtype == "bf16" else torch.float32
        B, H, C, Dv = w.batch, w.dims.heads, w.dims.kv_lora_rank, w.dims.v_head
        max_k = max(w.seqlens_k)
        cu_k = torch.from_numpy(w.cu_seqlens_k).to(dev)
        host = [torch.from_numpy(a).to(dtype=dt) for a in (w.q, w.kv, w.pe, w.wkv_b)]
        self.per_copy = sum(t.numel() * t.element_size() for t in host)
        self.copies = min(16, max(2, math.ceil(ROTATE_MIN_BYTES / self.per_copy) + 1))
        self.inputs = [[t.to(dev) for t in host] for _ in range(self.copies)]   # (q, kv, pe, wkv_b) per copy
        del host
        bufs = {"q_abs": torch.empty((B, H, C), dtype=dt, device=dev),
                "o_lat": torch.empty((B, H, C), dtype=dt, device=dev),
                "out": torch.empty((B, H, Dv), dtype=dt, device=dev),
                "ws": mla.workspace(d, B, B, max_k, 0, device=dev),
                "ws_out": mla.decode_out_workspace(d, B, max_k, 0, device=dev),
                "ws_fused": mla.decode_fused_workspace(d, B, max_k, 0, device=dev)}
        tensor_cores = mla.kernel_family(d) == 1   # the partial form and its merge exist there only
        # the split partials of the attention kernel alone (also for one split)
        bufs["ws_part"] = mla.partials_workspace(d, B, max_k, 0, device=dev) if tensor_cores else None
        self.stream = torch.cuda.current_stream()
        inputs = self.inputs

        def step(k):
            # the whole hot path through the public calls: absorb, then attention (+ split merge
            # fused into the output projection) in one call
            q, kv, pe, wkv_b = inputs[k]
            q_abs = mla.absorb_q(d, q, wkv_b, bufs["q_abs"])
            return mla.attn_decode_out(d, q_abs, q, kv, pe, cu_k, max_k, wkv_b, bufs["out"], bufs["ws_out"])

        def step_one_kernel(k):
            # the same step with attention, merge and projection in one kernel (mla_attn_decode_fused)
            q, kv, pe, wkv_b = inputs[k]
            q_abs = mla.absorb_q(d, q, wkv_b, bufs["q_abs"])
            return mla.attn_decode_fused(d, q_abs, q, kv, pe, cu_k, max_k, wkv_b, bufs["out"], bufs["ws_fused"])

        def attention_call(k):
            q, kv, pe, _ = inputs[k]
            mla.attn_decode(d, bufs["q_abs"], q, kv, pe, cu_k, max_k, bufs["o_lat"], bufs["ws"])

        def attention_kernel(k):
            q, kv, pe, _ = inputs[k]
            mla.attn_decode_partials(d, bufs["q_abs"], q, kv, pe, cu_k, max_k, bufs["ws_part"])

        # the absorb kernel alone, and the merge fused into the output projection alone (over the
        # partials attention_kernel leaves in the workspace)
        self.splits = mla.decode_num_splits(d, B, max_k, 0)
        part_o, part_ml = mla.split_partials(d, bufs["ws_part"], B, self.splits) if tensor_cores else (None, None)

        def absorb_kernel(k):
            q, _, _, wkv_b = inputs[k]
            mla.absorb_q(d, q, wkv_b, bufs["q_abs"])

        def merge_proj_kernel(k):
            mla.merge_partials_out(d, part_o, part_ml, inputs[k][3], bufs["out"])

        self.step = step
        for i in range(max(3, warmup)):
            step(i % self.copies)
        mla.device_status()

        def capture(fn):
            side = torch.cuda.Stream()
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                fn()
            torch.cuda.current_stream().wait_stream(side)
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                fn()
            return graph

        # The timed steps replay CUDA graphs captured from the same calls, so host-side launch
        # work does not leave the GPU idle inside the timed region.
        self.g_step = [capture(lambda k=k: step(k)) for k in range(self.copies)]
        self.g_step2 = [capture(lambda k=k: step_one_kernel(k)) for k in range(self.copies)]
        self.g_attn = [capture(lambda k=k: attention_call(k)) for k in range(self.copies)]
        self.g_kern = [capture(lambda k=k: attention_kernel(k)) for k in range(self.copies)]
        self.g_absorb = [capture(lambda k=k: absorb_kernel(k)) for k in range(self.copies)]
        self.g_mproj = [capture(lambda k=k: merge_proj_kernel(k)) for k in range(self.copies)] if tensor_cores else None
        # CHAIN steps in one graph, as the attention of consecutive layers of a model: each step's
        # first kernel may start (programmatic dependent launch) during the previous step's last
        self.g_chain = [capture(lambda k=k: [step((k + i) % self.copies) for i in range(CHAIN)])
                        for k in range(self.copies)]
        for i in range(max(3, warmup)):
            for g in (self.g_step, self.g_step2, self.g_attn, self.g_kern, self.g_chain, self.g_absorb,
                      self.g_mproj or self.g_absorb):
                g[i % self.copies].replay()
        mla.device_status()

    def timed(self, graphs, n, world=1):
        """Milliseconds for exactly n replays, back to back between two events on the stream."""
        import torch
        import torch.distributed as dist
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(self.stream)
        for i in range(n):
            graphs[i % self.copies].replay()
        e1.record(self.stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        return e0.elapsed_time(e1)


def other_configs(args, dev, hbm, tf):
    """The ragged, long-context and chunked-prefill workloads, each timed on its own, for the
    same JSON line: step and attention times and the fraction of the roofline that binds."""
    import torch
    from deepseek_mla_latent_b200 import workloads as wl
    res = {}
    for idx in (2, 3):
        w = wl.workload(idx)
        b = DecodeBench(w, dev, 3)
        n = 50
        step_ms = statistics.mean(b.timed(b.g_step, n) for _ in range(3))
        attn_ms = statistics.mean(b.timed(b.g_attn, n) for _ in range(3))
        kern_ms = statistics.mean(b.timed(b.g_kern, n) for _ in range(3))
        alg_bytes, alg_flop = decode_algorithmic(w)
        gbs = alg_bytes / (kern_ms / n * 1e-3) / 1e9
        res[w.name] = {"step_us": step_ms / n * 1e3, "attn_call_us": attn_ms / n * 1e3,
                       "attn_kernel_us": kern_ms / n * 1e3, "attn_cache_gbs": gbs, "bound": "hbm",
                       "frac": gbs / hbm, "tensor_frac": alg_flop / (kern_ms / n * 1e-3) / 1e12 / tf,
                       "steps": n, "repeats": 3, "tokens": w.total_k}
        del b
        torch.cuda.empty_cache()
    w = wl.workload(4)
    us_step, us_attn, attn_flop, proj_flop, err = prefill_timings(w, 5, 3, prefill_check_pairs(w))
    tflops = attn_flop / (us_attn * 1e-6) / 1e12
    res[w.name] = {"step_us": us_step, "attn_call_us": us_attn, "attn_tflops": tflops, "bound": "tensor",
                   "frac": tflops / tf, "parity_max_rel_err": err, "steps": 5,
                   "naive_path": naive_path_line(w, 5, 3, tf)}
    torch.cuda.empty_cache()
    return res


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", type=int, default=None,
                   help="workload index (default 1 = DeepSeek-V3 decode b8 t4096; 4 for --op prefill, 3 for --op seqpar)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-extra-configs", action="store_true",
                   help="skip the ragged, long-context and chunked-prefill workloads in the decode line")
    p.add_argument("--cpu-seconds", type=float, default=15.0)
    p.add_argument("--op", choices=["decode", "append", "paged", "expand", "prefill", "sparse", "seqpar"],
                   default="decode",
                   help="decode: the decode step (the benchmark); append: the latent-cache append alone; "
                        "paged: the decode attention call over a paged cache beside the packed one; "
                        "expand: the latent KV expansion; prefill: the chunked-prefill step "
                        "(workload 4 unless --workload names another prefill workload); sparse: decode "
                        "over --topk selected rows per sequence beside the dense call; seqpar: decode with "
                        "every sequence's cache split over the ranks (NCCL all-gather of the split partials), "
                        "workload 3 unless --workload names another decode workload")
    p.add_argument("--batch", type=int, default=4, help="sequences per expansion call (--op expand)")
    p.add_argument("--seq-len", type=int, default=1024, help="tokens per sequence (--op expand)")
    p.add_argument("--tokens", type=int, default=65536, help="new tokens per append call (--op append)")
    p.add_argument("--page-size", type=int, default=64, help="tokens per page (--op paged)")
    p.add_argument("--topk", type=int, default=2048, help="selected rows per sequence (--op sparse)")
    return p.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def reduce_max(values, device):
    """Element-wise max of per-rank float values over all ranks (identity with one rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), float(pk["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


# The sources that define the latent attention kernel (the roofline's dominant kernel): an ncu
# summary of it stays valid while these files are unchanged.
ATTN_KERNEL_SOURCES = ("common.cuh", "sm100_ptx.cuh", "sm100_attn.cuh")


def kernel_source_hash(names=None) -> str:
    """sha256 prefix over the library's CUDA sources (or the named files among them)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "deepseek_mla_latent_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh")) and (names is None or name in names):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def attn_kernel_hash() -> str:
    return kernel_source_hash(ATTN_KERNEL_SOURCES)


def profiled_traffic(workload_name: str):
    """DRAM bytes per launch of the attention kernel from the committed ncu summary,
    if it was taken on the current sources of that kernel; else None."""
    path = os.path.join(ROOT, "profiles", f"attn_decode_{workload_name}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    m_hash = re.search(r"attn_kernel_source_hash:\s*([0-9a-f]+)", text)
    m_bytes = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not m_hash or not m_bytes or m_hash.group(1) != attn_kernel_hash():
        return None
    return float(m_bytes.group(1))


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.proc = None
        self.gpu_id = gpu_id

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) != 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(names, parts[3:]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def host_cores():
    """(cores this process may run on, BLAS threads the oracle's matrix products use)."""
    try:
        cores = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        cores = os.cpu_count() or 1
    try:
        from threadpoolctl import threadpool_info
        blas = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # noqa: BLE001
        blas = cores
    return int(cores), int(blas)


def cpu_baseline_oracle(w, seconds: float):
    """Time the fp64 oracle (naive path) on (sequence, head) pairs of the workload for
    about `seconds`, and scale to one whole step (all sequences x all heads)."""
    import oracle
    cores, blas = host_cores()
    H, B = w.dims.heads, w.batch
    pairs = [(b, h) for h in range(H) for b in range(B)]
    done, t0 = 0, time.perf_counter()
    while done < len(pairs) and (done < 4 or time.perf_counter() - t0 < seconds):
        oracle.workload_naive(w, pairs=[pairs[done]])
        done += 1
    el = time.perf_counter() - t0
    per_pair = el / done
    return {"value": per_pair * len(pairs) * 1e6, "unit": UNIT, "cores": cores, "blas_threads": blas,
            "kind": "oracle", "value_kind": "scaled from a timed sample",
            "sample": f"{done} of {len(pairs)} (sequence, head) pairs of the same workload, naive fp64 path, "
                      f"{el:.1f} s, scaled to the whole step"}


def workload_config(w, world: int) -> dict:
    """The `config` keys both arms report for a workload."""
    return {"workload": w.name, "batch": w.batch, "heads": w.dims.heads, "kv_lora_rank": w.dims.kv_lora_rank,
            "qk_rope": w.dims.qk_rope, "seq_len_k": max(w.seqlens_k), "queries_per_seq": 1,
            "parallelism": "replicas" if world > 1 else "single"}


def run_reference(args, rank, world):
    """The reference arm: the fp64 oracle on the host cores.  Each timed step runs one (sequence,
    head) pair of the workload and is scaled by the number of pairs to one whole step, so
    `value` and `ms_per_step` are scaled from a timed sample (`value_kind` says so)."""
    from deepseek_mla_latent_b200 import workloads as wl
    if rank != 0:
        return
    w = wl.workload(args.workload)
    import oracle
    cores, blas = host_cores()
    H, B = w.dims.heads, w.batch
    pairs = [(b, h) for h in range(H) for b in range(B)]
    for i in range(args.warmup):
        oracle.workload_naive(w, pairs=[pairs[i % len(pairs)]])
    t0 = time.perf_counter()
    for i in range(args.steps):
        oracle.workload_naive(w, pairs=[pairs[i % len(pairs)]])
    el = time.perf_counter() - t0
    us_step = el / args.steps * len(pairs) * 1e6
    line = {"metric": METRIC, "value": us_step, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": us_step / 1e3, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "value_kind": f"scaled from a timed sample: {args.steps} of {len(pairs)} (sequence, head) pairs "
                          f"timed ({el:.2f} s), times {len(pairs)} / {args.steps}",
            "config": workload_config(w, world),
            "cpu_baseline": {"value": us_step, "unit": UNIT, "cores": cores, "blas_threads": blas,
                             "kind": "oracle", "value_kind": "scaled from a timed sample",
                             "sample": f"each step: one (sequence, head) pair of {len(pairs)}, naive fp64 path, "
                                       f"scaled to the whole step ({args.steps} pairs timed, {el:.2f} s)"},
            "e2e": {"value": us_step, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_append(args, rank, world):
    """Time mla_append_latent (RMSNorm of the latent, RoPE of the rotary key, slot writes) on
    `--tokens` new tokens of the DeepSeek-V3 shapes; one JSON line (single GPU)."""
    import torch
    from deepseek_mla_latent_b200 import mla
    from deepseek_mla_latent_b200 import workloads as wl
    torch.cuda.set_device(0)
    n, C, R = args.tokens, 512, 64
    d = mla.dims_from(wl.V3)
    g = torch.Generator(device="cpu").manual_seed(0)
    dev = "cuda"
    copies = 2 if n * (C + R) * 2 * 2 > L2_BYTES else min(16, max(2, math.ceil(2 * L2_BYTES / (n * (C + R) * 4))))
    bufs = []
    for _ in range(copies):
        kv_new = torch.randn(n, C, generator=g).to(dev, torch.bfloat16)
        pe_new = torch.randn(n, R, generator=g).to(dev, torch.bfloat16)
        kvc = torch.empty(n, C, dtype=torch.bfloat16, device=dev)
        pec = torch.empty(n, R, dtype=torch.bfloat16, device=dev)
        bufs.append((kv_new, pe_new, kvc, pec))
    gamma = torch.ones(C, dtype=torch.bfloat16, device=dev)
    pos = (torch.arange(n, dtype=torch.int32) % 4096).to(dev)
    slots = torch.randperm(n, generator=g).to(dev)
    call = lambda k: mla.append_latent(d, bufs[k][0], bufs[k][1], pos, slots, bufs[k][2], bufs[k][3], gamma)
    for i in range(max(3, args.warmup)):
        call(i % copies)
    graphs = []
    for k in range(copies):
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            call(k)
        torch.cuda.current_stream().wait_stream(side)
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            call(k)
        graphs.append(gr)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.steps):
        graphs[i % copies].replay()
    e1.record()
    torch.cuda.synchronize()
    mla.device_status()
    us = e0.elapsed_time(e1) / args.steps * 1e3
    alg_bytes = n * (C + R) * 2 * 2 + C * 2 + n * (4 + 8)
    hbm, _, peak_kind = load_peaks()
    gbs = alg_bytes / (us * 1e-6) / 1e9
    print(json.dumps({
        "metric": "MLA latent-cache append GB/s (1xB200)", "value": gbs, "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "us_per_call": us, "higher_is_better": True,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"append_v3_{n}_tokens", "tokens": n, "kv_lora_rank": C, "qk_rope": R,
                   "l2": f"{copies} rotating input/cache copies"},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                     "peak_kind": peak_kind},
        "gpu_launches": args.steps}), flush=True)


def run_paged(args, rank, world):
    """Time the decode attention call (attention kernel + split merge) over the workload's cache
    scattered into randomly placed pages (mla_attn_paged), and the packed call on the same keys;
    one JSON line (single GPU)."""
    import torch
    from deepseek_mla_latent_b200 import mla
    from deepseek_mla_latent_b200 import workloads as wl
    torch.cuda.set_device(0)
    dev = "cuda"
    w = wl.workload(args.workload)
    if any(s != 1 for s in w.seqlens_q):
        raise SystemExit("--op paged times decode workloads")
    pc = wl.paged_cache(w, args.page_size, seed=0, spare_pages=64, fill=0.0)
    d = mla.dims_from(w.dims)
    dt = torch.bfloat16
    B, H, C = w.batch, w.dims.heads, w.dims.kv_lora_rank
    max_k = max(w.seqlens_k)
    t = lambda a, ty=dt: torch.from_numpy(np.ascontiguousarray(a)).to(device=dev, dtype=ty)
    per_copy = (pc.kv_cache.size + pc.pe_cache.size + w.kv.size + w.pe.size) * 2
    copies = min(16, max(2, math.ceil(ROTATE_MIN_BYTES / per_copy) + 1))
    q, wkv_b = t(w.q), t(w.wkv_b)
    q_abs = mla.absorb_q(d, q, wkv_b)
    table, seqlens, cu_k = t(pc.block_table, torch.int32), t(pc.seqlens_k, torch.int32), t(w.cu_seqlens_k, torch.int32)
    caches = [(t(pc.kv_cache), t(pc.pe_cache), t(w.kv), t(w.pe)) for _ in range(copies)]
    o_lat = torch.empty((B, H, C), dtype=dt, device=dev)
    ws = mla.workspace(d, B, B, max_k, 0, device=dev)
    paged = lambda k: mla.attn_paged(d, q_abs, q, seqlens, max_k, caches[k][0], caches[k][1], table, pc.page_size,
                                     o_lat=o_lat, ws=ws)
    packed = lambda k: mla.attn_decode(d, q_abs, q, caches[k][2], caches[k][3], cu_k, max_k, o_lat, ws)

    def capture(fn):
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            fn()
        torch.cuda.current_stream().wait_stream(side)
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            fn()
        return gr

    for i in range(max(3, args.warmup)):
        paged(i % copies)
        packed(i % copies)
    mla.device_status()
    g_paged = [capture(lambda k=k: paged(k)) for k in range(copies)]
    g_packed = [capture(lambda k=k: packed(k)) for k in range(copies)]
    for i in range(max(3, args.warmup)):
        g_paged[i % copies].replay()
        g_packed[i % copies].replay()
    torch.cuda.synchronize()

    def timed(graphs):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(args.steps):
            graphs[i % copies].replay()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / args.steps * 1e3

    us_paged, us_packed = timed(g_paged), timed(g_packed)
    mla.device_status()
    hbm, _, peak_kind = load_peaks()
    alg_bytes = w.total_k * KV_BYTES_PER_TOKEN + B * H * (C + w.dims.qk_rope + C) * 2
    gbs = alg_bytes / (us_paged * 1e-6) / 1e9
    print(json.dumps({
        "metric": "MLA paged-cache decode attention GB/s (1xB200)", "value": gbs, "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "us_per_call": us_paged, "packed_us_per_call": us_packed,
        "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{w.name}_page{pc.page_size}", "batch": B, "seq_len_k": max_k,
                   "page_size": pc.page_size, "num_pages": pc.num_pages,
                   "num_splits": mla.decode_num_splits(d, B, max_k, 0),
                   "l2": f"{copies} rotating copies of the paged and packed caches"},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                     "peak_kind": peak_kind},
        "gpu_launches": args.steps * (2 if mla.decode_num_splits(d, B, max_k, 0) > 1 else 1)}), flush=True)


def run_sparse(args, rank, world):
    """Time token-granular sparse decode (mla_attn_sparse_decode: the selected rows gathered into
    one page per sequence, then the paged attention and split merge) with `--topk` random rows of
    each sequence's cache, beside the dense decode call on the same cache; one JSON line (single GPU)."""
    if world > 1 and rank != 0:
        return
    import torch
    from deepseek_mla_latent_b200 import mla
    from deepseek_mla_latent_b200 import workloads as wl
    torch.cuda.set_device(0)
    dev = "cuda"
    w = wl.workload(args.workload)
    if any(s != 1 for s in w.seqlens_q):
        raise SystemExit("--op sparse times decode workloads")
    d = mla.dims_from(w.dims)
    dt = torch.bfloat16
    B, H, C = w.batch, w.dims.heads, w.dims.kv_lora_rank
    topk = args.topk
    rng = np.random.default_rng(0)
    idx = np.full((B, topk), -1, dtype=np.int32)
    counts = np.zeros(B, dtype=np.int32)
    cu = w.cu_seqlens_k
    for b in range(B):
        n = min(topk, int(cu[b + 1] - cu[b]))
        idx[b, :n] = rng.choice(np.arange(cu[b], cu[b + 1]), size=n, replace=False)
        counts[b] = n
    t = lambda a, ty=dt: torch.from_numpy(np.ascontiguousarray(a)).to(device=dev, dtype=ty)
    per_copy = (w.kv.size + w.pe.size) * 2
    copies = min(16, max(2, math.ceil(ROTATE_MIN_BYTES / per_copy) + 1))
    q, wkv_b = t(w.q), t(w.wkv_b)
    q_abs = mla.absorb_q(d, q, wkv_b)
    ti, tc, cu_k = t(idx, torch.int32), t(counts, torch.int32), t(cu, torch.int32)
    caches = [(t(w.kv), t(w.pe)) for _ in range(copies)]
    o_lat = torch.empty((B, H, C), dtype=dt, device=dev)
    ws_s = torch.empty(int(mla.LIB.mla_sparse_workspace_size(ctypes_byref(d), B, topk, 0)), dtype=torch.uint8,
                       device=dev)
    ws_d = mla.workspace(d, B, B, max(w.seqlens_k), 0, device=dev)
    sparse = lambda k: mla.attn_sparse_decode(d, q_abs, q, caches[k][0], caches[k][1], ti, tc, o_lat=o_lat, ws=ws_s)
    dense = lambda k: mla.attn_decode(d, q_abs, q, caches[k][0], caches[k][1], cu_k, max(w.seqlens_k), o_lat, ws_d)

    def capture(fn):
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            fn()
        torch.cuda.current_stream().wait_stream(side)
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            fn()
        return gr

    for i in range(max(3, args.warmup)):
        sparse(i % copies)
        dense(i % copies)
    mla.device_status()
    g_s = [capture(lambda k=k: sparse(k)) for k in range(copies)]
    g_d = [capture(lambda k=k: dense(k)) for k in range(copies)]
    torch.cuda.synchronize()

    def timed(graphs):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(args.steps):
            graphs[i % copies].replay()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / args.steps * 1e3

    us_s, us_d = timed(g_s), timed(g_d)
    mla.device_status()
    hbm, _, peak_kind = load_peaks()
    sel = int(counts.sum())
    # the selected rows are read once from the cache, written to and read back from the page scratch
    alg_bytes = sel * KV_BYTES_PER_TOKEN + B * H * (C + w.dims.qk_rope + C) * 2
    gbs = alg_bytes / (us_s * 1e-6) / 1e9
    print(json.dumps({
        "metric": "MLA token-sparse decode attention GB/s (1xB200)", "value": gbs, "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "us_per_call": us_s, "dense_us_per_call": us_d,
        "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{w.name}_top{topk}", "batch": B, "seq_len_k": max(w.seqlens_k), "topk": topk,
                   "selected_rows": sel, "num_splits": mla.decode_num_splits(d, B, topk, 0),
                   "l2": f"{copies} rotating copies of the cache"},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                     "peak_kind": peak_kind, "algorithmic_bytes": "selected rows once (1152 B each) + q_abs, q_pe in, "
                                                                 "o_lat out"},
        "gpu_launches": args.steps * (3 if mla.decode_num_splits(d, B, topk, 0) > 1 else 2)}), flush=True)


def ctypes_byref(x):
    import ctypes
    return ctypes.byref(x)


def prefill_attention_flop(w) -> float:
    """Algorithmic flop of the absorb-form attention of a chunked prefill: 2 * H * (576 + 512)
    per (query, visible key), query i of s new queries over t keys seeing t - s + i + 1."""
    per_pair = 2.0 * w.dims.heads * (w.dims.kv_lora_rank + w.dims.qk_rope + w.dims.kv_lora_rank)
    visible = 0
    for s, t in zip(w.seqlens_q, w.seqlens_k):
        visible += sum(max(0, min(t, t - s + i + 1)) for i in range(s))
    return per_pair * visible


def prefill_timings(w, steps: int, warmup: int, check_pairs=()):
    """Time the chunked-prefill step (mla_absorb_q -> mla_attn_prefill_chunk -> mla_out_proj) and
    the attention call alone on one GPU.  With `check_pairs`, the step's output for those
    (sequence, head) pairs is first compared with the oracle (max error relative to max|oracle|).
    Returns (us_step, us_attn, attention flop, projection flop, max relative error or None)."""
    import torch
    from deepseek_mla_latent_b200 import mla
    d = mla.dims_from(w.dims)
    dt = torch.bfloat16
    t = lambda a, ty=dt: torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=ty)
    q, kv, pe, wkv_b = t(w.q), t(w.kv), t(w.pe), t(w.wkv_b)
    cu_q, cu_k = t(w.cu_seqlens_q, torch.int32), t(w.cu_seqlens_k, torch.int32)
    n, H, C = w.n_q, w.dims.heads, w.dims.kv_lora_rank
    max_q, max_k = max(w.seqlens_q), max(w.seqlens_k)
    q_abs = torch.empty((n, H, C), dtype=dt, device="cuda")
    o_lat = torch.empty((n, H, C), dtype=dt, device="cuda")
    out = torch.empty((n, H, w.dims.v_head), dtype=dt, device="cuda")
    ws = mla.workspace(d, w.batch, n, max_k, 0, device="cuda")

    def attention():
        mla.attn_prefill_chunk(d, q_abs, q, cu_q, cu_k, max_q, max_k, kv, pe, o_lat, ws)

    def step():
        mla.absorb_q(d, q, wkv_b, q_abs)
        attention()
        mla.out_proj(d, o_lat, wkv_b, out)

    err = None
    if check_pairs:
        import oracle
        step()
        mla.device_status()
        got = out.float().cpu().numpy()
        ref = oracle.workload_naive(w, pairs=list(check_pairs))
        cq = w.cu_seqlens_q
        err = 0.0
        for (b, h), r in ref.items():
            e = float(np.max(np.abs(got[cq[b]:cq[b + 1], h, :] - r))) / max(float(np.max(np.abs(r))), 1e-30)
            err = max(err, e)
    for _ in range(max(3, warmup)):
        step()
    mla.device_status()

    def timed(fn):
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps * 1e3

    us_step, us_attn = timed(step), timed(attention)
    mla.device_status()
    attn_flop = prefill_attention_flop(w)
    proj_flop = 2.0 * n * H * C * (w.dims.qk_nope + w.dims.v_head)
    return us_step, us_attn, attn_flop, proj_flop, err


def expanded_prefill_flop(w):
    """Algorithmic flop of the naive-path prefill: the expansion of every cache row
    (2 * H * (Dn + Dv) * C per row) and the per-head attention, 2 * H * (Dn + R + Dv) per
    (query, visible key) pair."""
    dd = w.dims
    expand = 2.0 * w.total_k * dd.heads * (dd.qk_nope + dd.v_head) * dd.kv_lora_rank
    per_pair = 2.0 * dd.heads * (dd.qk_nope + dd.qk_rope + dd.v_head)
    visible = sum(max(0, min(t, t - s + i + 1)) for s, t in zip(w.seqlens_q, w.seqlens_k) for i in range(s))
    return expand, per_pair * visible


def expanded_prefill_timings(w, steps: int, warmup: int, check_pairs=()):
    """Time the naive-path chunked prefill on one GPU: mla_expand_kv over the whole packed cache,
    then mla_attn_prefill_expanded.  Returns (us_step, us_attn, expansion flop, attention flop,
    max relative error against the oracle on `check_pairs` or None)."""
    import torch
    from deepseek_mla_latent_b200 import mla
    d = mla.dims_from(w.dims)
    dt = torch.bfloat16
    t = lambda a, ty=dt: torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=ty)
    q, kv, pe, wkv_b = t(w.q), t(w.kv), t(w.pe), t(w.wkv_b)
    cu_q, cu_k = t(w.cu_seqlens_q, torch.int32), t(w.cu_seqlens_k, torch.int32)
    T, H = kv.shape[0], w.dims.heads
    max_q = max(w.seqlens_q)
    k = torch.empty((1, H, T, w.dims.qk_nope), dtype=dt, device="cuda")
    v = torch.empty((1, H, T, w.dims.v_head), dtype=dt, device="cuda")
    out = torch.empty((w.n_q, H, w.dims.v_head), dtype=dt, device="cuda")

    def attention():
        mla.attn_prefill_expanded(d, q, k[0], v[0], pe, cu_q, cu_k, max_q, out)

    def step():
        mla.expand_kv(d, kv, wkv_b, 1, T, eps=1e-6, k_nope=k, v=v)
        attention()

    err = None
    if check_pairs:
        import oracle
        step()
        mla.device_status()
        got = out.float().cpu().numpy()
        dd = w.dims
        ref = oracle.mla_naive(w.q, oracle.rms_norm(w.kv, None, 1e-6), w.pe, w.wkv_b, w.cu_seqlens_q,
                               w.cu_seqlens_k, dd.heads, dd.qk_nope, dd.qk_rope, dd.v_head, dd.scale,
                               pairs=list(check_pairs))
        cq = w.cu_seqlens_q
        err = 0.0
        for (b, h), r in ref.items():
            e = float(np.max(np.abs(got[cq[b]:cq[b + 1], h, :] - r))) / max(float(np.max(np.abs(r))), 1e-30)
            err = max(err, e)
    for _ in range(max(3, warmup)):
        step()
    mla.device_status()

    def timed(fn):
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps * 1e3

    us_step, us_attn = timed(step), timed(attention)
    mla.device_status()
    ex_flop, at_flop = expanded_prefill_flop(w)
    return us_step, us_attn, ex_flop, at_flop, err


def naive_path_line(w, steps, warmup, tf):
    """The naive path of the same chunked prefill (expansion + per-head attention) for the JSON line."""
    import torch
    x_step, x_attn, ex_flop, at_flop, x_err = expanded_prefill_timings(w, steps, warmup, prefill_check_pairs(w))
    torch.cuda.empty_cache()
    at_tf = at_flop / (x_attn * 1e-6) / 1e12
    return {"us_per_step": x_step, "attn_us_per_call": x_attn, "expand_us": x_step - x_attn,
            "step_tflops": (ex_flop + at_flop) / (x_step * 1e-6) / 1e12, "attn_tflops": at_tf,
            "attn_frac": at_tf / tf, "flop": {"expansion": ex_flop, "attention": at_flop},
            "parity_max_rel_err": x_err}


def prefill_check_pairs(w):
    """(sequence, head) pairs the prefill benchmark checks against the oracle: one head of every
    sequence (all its query rows, first and last included) and heads 0 and 127 of sequence 0."""
    H = w.dims.heads
    return sorted({(b, (37 * b + 5) % H) for b in range(w.batch)} | {(0, 0), (0, H - 1)})


def run_prefill(args, rank, world):
    """Time the chunked-prefill step and the attention call alone on a prefill workload; one
    JSON line.  One GPU: under a multi-rank launch rank 0 alone runs and prints."""
    if world > 1 and rank != 0:
        return
    import torch
    from deepseek_mla_latent_b200 import workloads as wl
    torch.cuda.set_device(0)
    idx = args.workload if any(s > 1 for s in wl.workload_shape(args.workload)[2]) else 4
    w = wl.workload(idx)
    us_step, us_attn, attn_flop, proj_flop, err = prefill_timings(w, args.steps, args.warmup,
                                                                   prefill_check_pairs(w))
    hbm, tf, peak_kind = load_peaks()
    naive = naive_path_line(w, args.steps, args.warmup, tf)
    attn_tf = attn_flop / (us_attn * 1e-6) / 1e12
    line = {
        "metric": "MLA absorb chunked-prefill TFLOP/s (1xB200)", "value": attn_tf, "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "us_per_step": us_step, "attn_us_per_call": us_attn,
        "step_tflops": (attn_flop + proj_flop) / (us_step * 1e-6) / 1e12, "higher_is_better": True,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "queries_per_seq": max(w.seqlens_q),
                   "seq_len_k": max(w.seqlens_k),
                   "l2": "the step moves over 1 GB (q_abs and o_lat of 4096 rows), far above L2"},
        "parity": {"pairs": len(prefill_check_pairs(w)), "max_rel_err": err, "tol": 2e-2},
        "naive_path": naive,
        "roofline": {"bound": "tensor", "achieved": attn_tf, "peak": tf, "unit": "TFLOP/s", "frac": attn_tf / tf,
                     "peak_kind": peak_kind + " (burst)"},
        "gpu_launches": args.steps * 3}
    if not args.no_cpu_baseline:
        cpu = cpu_baseline_oracle(w, args.cpu_seconds)
        # the oracle's time for the whole step, in the line's unit (the same algorithmic flop)
        cpu["value"] = attn_flop / (cpu["value"] * 1e-6) / 1e12
        cpu["unit"] = "TFLOP/s"
        line["cpu_baseline"] = cpu
    print(json.dumps(line), flush=True)


def run_expand(args, rank, world):
    """Time mla_expand_kv (RMSNorm of the compressed KV, projection to all heads, head-major
    split into K_nope and V) at DeepSeek-V3 shapes; one JSON line (single GPU)."""
    import torch
    from deepseek_mla_latent_b200 import mla
    from deepseek_mla_latent_b200 import workloads as wl
    torch.cuda.set_device(0)
    dev = "cuda"
    B, S = args.batch, args.seq_len
    e = wl.expand_inputs(wl.V3, B, S, seed=0)
    d = mla.dims_from(wl.V3)
    H, C = wl.V3.heads, wl.V3.kv_lora_rank
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device=dev, dtype=torch.bfloat16)
    n = B * S
    out_bytes = n * H * 256 * 2
    # outputs above L2 evict the inputs between calls; below it, rotate enough copies
    copies = 2 if out_bytes > L2_BYTES else min(16, max(2, math.ceil(2 * L2_BYTES / out_bytes)))
    sets = [(t(e.kv_c), t(e.wkv_b), torch.empty((B, H, S, 128), dtype=torch.bfloat16, device=dev),
             torch.empty((B, H, S, 128), dtype=torch.bfloat16, device=dev)) for _ in range(copies)]
    gamma = t(e.gamma)
    call = lambda k: mla.expand_kv(d, sets[k][0], sets[k][1], B, S, gamma=gamma, k_nope=sets[k][2], v=sets[k][3])
    for i in range(max(3, args.warmup)):
        call(i % copies)
    mla.device_status()
    graphs = []
    for k in range(copies):
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            call(k)
        torch.cuda.current_stream().wait_stream(side)
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            call(k)
        graphs.append(gr)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.steps):
        graphs[i % copies].replay()
    e1.record()
    torch.cuda.synchronize()
    mla.device_status()
    us = e0.elapsed_time(e1) / args.steps * 1e3
    flop = 2.0 * n * H * 256 * C
    alg_bytes = n * C * 2 + H * 256 * C * 2 + C * 2 + out_bytes
    hbm, tf_burst, peak_kind = load_peaks()   # the burst bf16 figure: a kernel timed alone
    tflops = flop / (us * 1e-6) / 1e12
    print(json.dumps({
        "metric": "MLA latent KV expansion TFLOP/s (1xB200)", "value": tflops, "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "us_per_call": us, "higher_is_better": True,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"expand_v3_b{B}_s{S}", "batch": B, "seq_len": S, "heads": H, "kv_lora_rank": C,
                   "l2": f"{copies} rotating input/output sets ({out_bytes / 2**20:.0f} MiB written per call)"},
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": tf_burst, "unit": "TFLOP/s",
                     "frac": tflops / tf_burst, "peak_kind": peak_kind + " (burst)",
                     "hbm_gbs": alg_bytes / (us * 1e-6) / 1e9, "hbm_frac": alg_bytes / (us * 1e-6) / 1e9 / hbm},
        "gpu_launches": args.steps}), flush=True)


def run_seqpar(args, rank, world, local):
    """Decode with every sequence's cache split along its tokens over the ranks (seqpar): each rank
    attends to its range in the partial form, the ranks all-gather the partials (NCCL) and merge
    them fused into the output projection.  Strong scaling: the same sequences at any N.  One JSON
    line from rank 0 with the time per step (max over ranks) beside the single-GPU decode step."""
    import datetime
    import torch
    import torch.distributed as dist
    from deepseek_mla_latent_b200 import mla, seqpar
    from deepseek_mla_latent_b200 import workloads as wl
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    else:
        import socket
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        store = dist.TCPStore("127.0.0.1", port, 1, True, timeout=datetime.timedelta(seconds=60))
        dist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        w = wl.workload(args.workload)
        if any(s != 1 for s in w.seqlens_q):
            raise SystemExit("--op seqpar times decode workloads")
        d = mla.dims_from(w.dims)
        T = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device=dev, dtype=torch.bfloat16)
        q, kv, pe, wkv_b = T(w.q), T(w.kv), T(w.pe), T(w.wkv_b)
        B, H = w.batch, w.dims.heads
        q_abs = mla.absorb_q(d, q, wkv_b)
        kv_r, pe_r, cu_r, max_r = seqpar.local_cache(kv, pe, w.cu_seqlens_k, world, rank)
        # splits per rank: enough units to fill this GPU with the rank's range
        splits = mla.decode_num_splits(d, B, max_r, 0)
        step = lambda: seqpar.decode_sequence_parallel(d, q_abs, q, kv_r, pe_r, cu_r, max_r, splits, wkv_b=wkv_b)
        for _ in range(max(3, args.warmup)):
            out = step()
        torch.cuda.synchronize()
        dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            out = step()
        e1.record()
        torch.cuda.synchronize()
        dist.barrier()
        us, = reduce_max([e0.elapsed_time(e1) / args.steps * 1e3], dev)
        mla.device_status()
        # the single-GPU decode step on the whole cache, for the result and the time beside it
        cu_k = torch.from_numpy(w.cu_seqlens_k).to(dev)
        dense = mla.attn_decode_out(d, q_abs, q, kv, pe, cu_k, max(w.seqlens_k), wkv_b)
        for _ in range(3):
            mla.attn_decode_out(d, q_abs, q, kv, pe, cu_k, max(w.seqlens_k), wkv_b, dense)
        torch.cuda.synchronize()
        e0.record()
        for _ in range(args.steps):
            mla.attn_decode_out(d, q_abs, q, kv, pe, cu_k, max(w.seqlens_k), wkv_b, dense)
        e1.record()
        torch.cuda.synchronize()
        dense_us = e0.elapsed_time(e1) / args.steps * 1e3
        mla.device_status()
        rel = float((out.float() - dense.float()).abs().max() / dense.float().abs().max())
        exchange = splits * B * H * (w.dims.kv_lora_rank * 2 + 8)
        if rank == 0:
            print(json.dumps({
                "metric": "MLA sequence-parallel decode us/step (cache split over the GPUs, NCCL exchange)",
                "value": us, "unit": "us/step", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "higher_is_better": False, "scaling": "strong", "dtype": "bf16", "data": "synthetic",
                "config": {"workload": w.name, "batch": B, "seq_len_k": int(max(w.seqlens_k)),
                           "parallelism": f"sequence split over {world} GPU(s)", "splits_per_rank": splits},
                "single_gpu_decode_us": dense_us, "exchange_bytes_per_rank": exchange,
                "max_rel_diff_vs_single_gpu": rel,
                "timing": "eager calls between CUDA events, inputs resident (the cache is read once per step)",
                "gpu_launches": args.steps * 2}), flush=True)
    finally:
        dist.destroy_process_group()


def main():
    args = parse_args()
    if args.workload is None:
        args.workload = {"seqpar": 3, "prefill": 4}.get(args.op, 1)
    rank, world, local = dist_env()
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.op == "append":
        run_append(args, rank, world)
        return
    if args.op == "paged":
        run_paged(args, rank, world)
        return
    if args.op == "expand":
        run_expand(args, rank, world)
        return
    if args.op == "prefill":
        run_prefill(args, rank, world)
        return
    if args.op == "sparse":
        run_sparse(args, rank, world)
        return
    if args.op == "seqpar":
        run_seqpar(args, rank, world, local)
        return

    import torch
    import torch.distributed as dist
    from deepseek_mla_latent_b200 import mla
    from deepseek_mla_latent_b200 import workloads as wl

    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    w = wl.workload(args.workload)
    bench = DecodeBench(w, dev, args.warmup)
    d, B, H, C, Dv, dt = bench.d, w.batch, w.dims.heads, w.dims.kv_lora_rank, w.dims.v_head, bench.dt

    sampler = None
    if rank == 0:
        try:
            gpu_id = str(torch.cuda.get_device_properties(dev).uuid)
            gpu_id = gpu_id if gpu_id.startswith("GPU-") else "GPU-" + gpu_id
        except Exception:  # noqa: BLE001
            gpu_id = str(local)
        sampler = ClockSampler(gpu_id)
        sampler.start()
        time.sleep(0.3)

    # Each measurement times exactly K steps between two events (barrier and synchronize on both
    # sides); it is repeated, the same number of times on every rank, until the timed region has
    # lasted at least MIN_TIMED_MS in all, so that the clock samples see the GPU under load.
    def repeated(graphs):
        first = reduce_max([bench.timed(graphs, args.steps, world)], dev)[0]
        reps = max(1, min(1000, math.ceil(MIN_TIMED_MS / max(first, 1e-3))))
        runs = [first] + [bench.timed(graphs, args.steps, world) for _ in range(reps - 1)]
        runs = reduce_max(runs, dev)
        return statistics.mean(runs), len(runs)

    total_ms, reps = repeated(bench.g_step)
    step2_ms, _ = repeated(bench.g_step2)
    chain_ms = statistics.mean(bench.timed(bench.g_chain, max(1, args.steps // CHAIN), world) for _ in range(3))
    absorb_ms, _ = repeated(bench.g_absorb)
    mproj_ms = repeated(bench.g_mproj)[0] if bench.g_mproj else float("nan")
    chain_us = chain_ms / (max(1, args.steps // CHAIN) * CHAIN) * 1e3
    # the attention call alone (attention kernel + split merge) and the attention kernel alone
    # (the split partials left in the workspace, mla_attn_decode_partials)
    attn_total_ms, _ = repeated(bench.g_attn)
    kern_total_ms, _ = repeated(bench.g_kern)
    clocks = sampler.stop() if sampler else None
    mla.device_status()
    us_step = total_ms / args.steps * 1e3
    mean_attn_ms = attn_total_ms / args.steps
    mean_kern_ms = kern_total_ms / args.steps

    # End to end through the same public calls: pinned host q -> device, step, out -> pinned host,
    # the K steps back to back between two events, inputs rotating over the same copies.
    q_pinned = torch.from_numpy(w.q).to(dt).pin_memory()
    out_pinned = torch.empty((B, H, Dv), dtype=dt).pin_memory()
    e2e_steps = min(args.steps, 500)
    for i in range(3):
        bench.inputs[i % bench.copies][0].copy_(q_pinned, non_blocking=True)
        out_pinned.copy_(bench.step(i % bench.copies), non_blocking=True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e2e_s, e2e_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_s.record(bench.stream)
    for i in range(e2e_steps):
        k = i % bench.copies
        bench.inputs[k][0].copy_(q_pinned, non_blocking=True)
        out_pinned.copy_(bench.step(k), non_blocking=True)
    e2e_e.record(bench.stream)
    torch.cuda.synchronize()
    e2e_ms, = reduce_max([e2e_s.elapsed_time(e2e_e)], dev)
    e2e_us = e2e_ms / e2e_steps * 1e3

    if rank == 0:
        hbm, tf, peak_kind = load_peaks()
        alg_bytes, alg_flop = decode_algorithmic(w)
        attn_s, kern_s = mean_attn_ms / 1e3, mean_kern_ms / 1e3
        achieved_gbs = alg_bytes / kern_s / 1e9
        Dn, Cl = w.dims.qk_nope, w.dims.kv_lora_rank
        absorb_bytes = H * Dn * Cl * 2 + B * H * Dn * 2 + B * H * Cl * 2
        mproj_bytes = H * Dv * Cl * 2 + bench.splits * B * H * (Cl * 2 + 8) + B * H * Dv * 2
        traffic = profiled_traffic(w.name)
        line = {
            "metric": METRIC, "value": us_step, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": us_step / 1e3, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if dt == torch.bfloat16 else "f32", "data": "synthetic",
            "config": {**workload_config(w, world),
                       "l2": f"inputs larger than L2: {bench.copies} rotating copies of q, kv, pe and wkv_b "
                             f"({bench.copies * bench.per_copy / 2**20:.0f} MiB), steps back to back between "
                             "two events"},
            "repeats": reps,
            "tokens_per_s": world * B / (us_step / 1e6),
            "step_fused_kernel_us": step2_ms / args.steps * 1e3,
            "step_chained_us": chain_us,
            "step_chained": f"{CHAIN} steps captured in one graph (consecutive layers): each absorb may start "
                            "during the previous step's projection",
            "attn_kernel_us": mean_kern_ms * 1e3,
            "attn_call_us": mean_attn_ms * 1e3,
            "attn_cache_gbs": achieved_gbs,
            "attn_call_gbs": alg_bytes / attn_s / 1e9,
            "attn_tflops": alg_flop / kern_s / 1e12,
            # the other two kernels of the step, each alone: the absorb (W_k 16.8 MB + q in, q_abs
            # out) and the merge fused into the output projection (W_v 16.8 MB + the split partials
            # in, out out; the partials are L2-resident, as after the attention in the step)
            "absorb_kernel_us": absorb_ms / args.steps * 1e3,
            "absorb_gbs": absorb_bytes / (absorb_ms / args.steps * 1e-3) / 1e9,
            "merge_proj_kernel_us": mproj_ms / args.steps * 1e3 if bench.g_mproj else None,
            "merge_proj_gbs": mproj_bytes / (mproj_ms / args.steps * 1e-3) / 1e9 if bench.g_mproj else None,
            "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm, "unit": "GB/s",
                         "frac": achieved_gbs / hbm, "traffic": traffic, "peak_kind": peak_kind,
                         "kernel": "latent attention kernel alone (CUDA events around its launches)",
                         "tensor_frac": alg_flop / kern_s / 1e12 / tf},
            "e2e": {"value": e2e_us, "unit": UNIT, "h2d_bytes_per_step": int(q_pinned.numel() * q_pinned.element_size()),
                    "d2h_bytes_per_step": int(out_pinned.numel() * out_pinned.element_size())},
            "gpu_launches": None,
            "clocks": clocks,
            "kernel_family": mla.kernel_family(d),
            "kernel_source_hash": kernel_source_hash(),
            "attn_kernel_source_hash": attn_kernel_hash(),
        }
        if clocks and clocks.get("sm_mhz"):
            # times x the median sampled SM clock: thousands of SM cycles, comparable across boxes
            # whose clocks differ
            line["sm_kcycles"] = {"step": us_step * clocks["sm_mhz"] / 1e3,
                                  "attn_kernel": mean_kern_ms * 1e3 * clocks["sm_mhz"] / 1e3}
        # absorb_q + attention + output projection (with the split merge fused in), one launch each
        splits = mla.decode_num_splits(d, B, max(w.seqlens_k), 0)
        line["gpu_launches"] = args.steps * reps * 3
        line["config"]["num_splits"] = splits
        if world == 1 and not args.no_extra_configs:
            del bench
            torch.cuda.empty_cache()
            line["other_configs"] = other_configs(args, dev, hbm, tf)
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline_oracle(w, args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

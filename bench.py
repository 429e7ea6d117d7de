"""Benchmark: paged decode attention on B200, KV-read GB/s per decode step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference] [--partition-size P] [--engine auto|core|tensor]

A step is one decode step of the workload's batch: copy-on-write block
copies (when the host manager reports any), the cache write of the step's new
tokens, and decode attention over every sequence.  The host metadata of every
step (slot mapping, copy pairs, block tables, lengths) is produced by the
library's C++ manager before the timed region and sits in HBM with the
queries and new K/V rows, so the timed region holds only the library's
kernels.  Timing: CUDA events on the launching stream around K consecutive
steps after W warm-up steps, synchronised on both sides; every step is a new
token of the same sequences (the KV cache, 0.6-2.7 GB, is larger than the
126 MB L2, so no flush is needed).

value = algorithmic bytes of the K steps / timed span, algorithmic bytes per
step = sum_s L_s * Hkv * D * 2 * e (K and V) + 2 * S * Hq * D * e (q, out)
+ sum_s ceil(L_s / bs) * 4 (block-table entries).

e2e = the same metric through the public API with host buffers: the C++
manager appends the step's tokens live, pinned host buffers are copied to the
device, the kernels run and the output comes back to the host, every step.

Multi-GPU: independent replicas (the decode path has no exchange step); each
rank runs its own copy of the batch; value = bytes of all ranks / max-over-
ranks time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "paged decode attention: KV-read GB/s (% of B200 HBM peak) and seqs/s per step"
DEFAULT_WORKLOAD = "mha7b_f16"


# ----------------------------------------------------------------------------- helpers

def algorithmic_bytes(lens, hq, hkv, d, bs, esize):
    kv = sum(lens) * hkv * d * 2 * esize
    qo = 2 * len(lens) * hq * d * esize
    tab = sum(-(-L // bs) for L in lens) * 4
    return kv + qo + tab


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled while the GPU is busy."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.index), "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def profiled_traffic(workload, algo_bytes):
    """DRAM bytes per decode launch from the committed ncu summary of this
    workload, scaled to this launch's algorithmic bytes; None if there is no
    summary or the decode sources changed since it was captured."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"decode_{workload}.md")
    if not os.path.exists(path):
        return None
    fields = {}
    for line in open(path):
        if ":" in line and line.split(":")[0] in ("traffic_bytes_per_launch",
                                                   "algorithmic_bytes_per_launch",
                                                   "source_sha256_16"):
            k, v = line.split(":", 1)
            fields[k] = v.strip()
    try:
        want = dict(x.split("=") for x in fields["source_sha256_16"].split())
        for name, h in want.items():
            src = os.path.join(ROOT, "paged_kv_cache_426_b200", "csrc", name)
            if hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] != h:
                return None
        t, a = int(fields["traffic_bytes_per_launch"]), int(fields["algorithmic_bytes_per_launch"])
    except (KeyError, ValueError, OSError):
        return None
    return int(round(t * algo_bytes / a))


def profiled_fields(path):
    """The numeric fields of a committed ncu summary, or None if it is missing
    or any source it lists (source_sha256_16) has changed since."""
    import hashlib
    if not os.path.exists(path):
        return None
    fields = {}
    for line in open(path):
        if ":" in line and not line.startswith(" "):
            k, v = line.split(":", 1)
            fields[k.strip()] = v.strip()
    try:
        want = dict(x.split("=") for x in fields["source_sha256_16"].split())
        for name, h in want.items():
            src = os.path.join(ROOT, "paged_kv_cache_426_b200", "csrc", name)
            if hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] != h:
                return None
    except (KeyError, ValueError, OSError):
        return None
    return fields


def prefill_flops(b):
    """Algorithmic FLOPs of causal prefill attention: chunk row i of sequence
    s sees L_s - n_s + i + 1 keys; per query head and key, 2 * head_dim for
    q.k and 2 * head_dim for p.v."""
    keys = sum(n * (L - n) + n * (n + 1) // 2 for L, n in zip(b.context_lens, b.query_lens))
    return 4 * b.head_dim * b.num_q_heads * keys


def tensor_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def prefill_cpu_baseline(b, seconds):
    """The prefill oracle, as it stands, on the host cores: float64 causal
    attention of chunk rows (a few at a time, cycling over sequences and KV
    heads) for about ``seconds``; throughput in algorithmic TFLOP/s."""
    import oracle
    from threadpoolctl import threadpool_info
    rec = oracle.run_prefill(b, compute=False)
    q = oracle.as_storage(b.q, b.dtype)
    cu = b.query_offsets
    G = b.num_q_heads // b.num_kv_heads
    S = len(b.context_lens)
    rows_done, flops, k, t0 = 0, 0, 0, time.perf_counter()
    while time.perf_counter() - t0 < seconds:
        s, j = k % S, (k // S) % b.num_kv_heads
        L, n = b.context_lens[s], b.query_lens[s]
        rows = list(range((k * 7) % n, n, max(1, n // 4)))[:4]
        oracle.prefill_rows(q[cu[s]:cu[s + 1]], rec.key_cache, rec.value_cache, rec.block_tables[s],
                            L, n, b.scale, j, b.dtype, rows=rows)
        flops += sum(4 * b.head_dim * G * (L - n + i + 1) for i in rows)
        rows_done += len(rows)
        k += 1
    dt = time.perf_counter() - t0
    threads = max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{rows_done} chunk rows x {G} query heads ({k} (sequence, KV head) visits "
                      f"over {b.name}), float64 numpy (gather through the block table + causal "
                      f"softmax attention per row), {dt:.1f} s",
            "host_cpus": len(os.sched_getaffinity(0))}


def run_prefill_bench(args):
    """One GPU, one JSON line: a step writes the chunks' K/V into the cache
    (pa_reshape_and_cache) and runs causal prefill attention over the paged
    cache (pa_prefill).  The tokens before each chunk are written once,
    untimed."""
    import paged_kv_cache_426_b200 as pa
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    b = workloads.PREFILL_BUILDERS[args.prefill]()
    td = b.torch_dtype
    mgr = pa.BlockManager(pa.BlockAllocator(b.num_blocks, b.free_order), b.block_size)
    shape = (b.num_blocks, b.num_kv_heads, b.block_size, b.head_dim)
    kc = torch.zeros(shape, dtype=td, device=dev)
    vc = torch.zeros(shape, dtype=td, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    ctx, chunk = [], []
    for s, (L, n) in enumerate(zip(b.context_lens, b.query_lens)):
        mgr.add_seq(s)
        slots = mgr.append(s, L)[0]
        ctx.append((slots[:L - n], b.k[s][:L - n], b.v[s][:L - n]))
        chunk.append((slots[L - n:], b.k[s][L - n:], b.v[s][L - n:]))
    cs = torch.cat([c[0] for c in ctx])
    if cs.numel():
        pa.pa_reshape_and_cache(torch.cat([c[1] for c in ctx]).to(dev),
                                torch.cat([c[2] for c in ctx]).to(dev), kc, vc, cs.to(dev),
                                err_flag=err)
    ch_slots = torch.cat([c[0] for c in chunk]).to(dev)
    ch_k = torch.cat([c[1] for c in chunk]).to(dev)
    ch_v = torch.cat([c[2] for c in chunk]).to(dev)
    mb = max(-(-L // b.block_size) for L in b.context_lens)
    tab, lens = mgr.block_tables(list(range(len(b.context_lens))), mb)
    tab, lens = tab.to(dev), lens.to(dev)
    cu = torch.tensor(b.query_offsets, dtype=torch.int32, device=dev)
    q = b.q.to(dev)
    out = torch.empty_like(q)
    max_q = max(b.query_lens)
    stream = torch.cuda.current_stream()

    def write():
        pa.pa_reshape_and_cache(ch_k, ch_v, kc, vc, ch_slots, err_flag=err)

    def attend():
        pa.pa_prefill(out, q, kc, vc, tab, lens, cu, max_q, b.scale, err_flag=err)

    sampler = ClockSampler(0)
    sampler.start()
    t_end = time.time() + args.soak
    while time.time() < t_end:
        for _ in range(5):
            write()
            attend()
        torch.cuda.synchronize()
    for _ in range(args.warmup):
        write()
        attend()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    for i in range(args.steps):
        ev[i][0].record(stream)
        write()
        ev[i][1].record(stream)
        attend()
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    assert int(err.item()) == 0, f"device error flag {int(err.item())}"
    span_ms = ev[0][0].elapsed_time(ev[-1][2])
    pf_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / args.steps
    flop = prefill_flops(b)
    value = flop * args.steps / (span_ms * 1e-3) / 1e12
    achieved = flop / (pf_ms * 1e-3) / 1e12
    peak, kind = tensor_peak()
    prof = profiled_fields(os.path.join(ROOT, "profiles", f"{b.name}.md"))
    traffic = int(prof["traffic_bytes_per_launch"]) if prof else None
    T = sum(b.query_lens)
    res = {
        "metric": "paged prefill attention: causal TFLOP/s per step (chunk write + attention)",
        "value": round(value, 1), "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(span_ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": b.dtype,
        "data": "synthetic (seeded; see workloads/)",
        "config": {"workload": b.name, "num_seqs": len(b.context_lens), "chunk_tokens": T,
                   "num_q_heads": b.num_q_heads, "num_kv_heads": b.num_kv_heads,
                   "head_dim": b.head_dim, "block_size": b.block_size,
                   "mean_context_len": round(sum(b.context_lens) / len(b.context_lens), 1),
                   "flop_per_step": flop, "parallelism": "one GPU",
                   "l2": "inputs larger than L2 (KV cache, queries and outputs each > 126 MB)"
                   if b.name == "prefill_gqa8b_bf16" else "KV cache larger than L2"},
        "prefill_only": {"tflops": round(achieved, 1), "ms": round(pf_ms, 4),
                         "tokens_per_s": round(T / (pf_ms * 1e-3), 1)},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": traffic,
                     "peak_kind": f"{kind} cuBLAS bf16 GEMM (burst; fp16 has the same nominal peak)",
                     "kernel": "pa_prefill"},
        "gpu_launches": 2 * args.steps,
        "clocks": clocks,
    }
    if args.cpu_baseline:
        res["cpu_baseline"] = prefill_cpu_baseline(b, args.cpu_seconds)
    return res


def dist_setup(n_gpus):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _over_ranks(x, world, op):
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(x, world):
    import torch.distributed as dist
    return _over_ranks(x, world, dist.ReduceOp.MAX if world > 1 else None)


def sum_over_ranks(x, world):
    import torch.distributed as dist
    return _over_ranks(x, world, dist.ReduceOp.SUM if world > 1 else None)


def aggregate(rank_bytes, rank_span_ms, world):
    """Whole-job throughput of `world` replicas: the bytes every rank moved
    over the slowest rank's device time.  Returns (bytes, span_ms, GB/s)."""
    span_ms = max_over_ranks(rank_span_ms, world)
    total = sum_over_ranks(rank_bytes, world)
    return total, span_ms, total / (span_ms * 1e-3) / 1e9


# ----------------------------------------------------------------------------- our path

class Session:
    """One replica: caches, the C++ manager, and per-step device inputs."""

    def __init__(self, w, P, dev, engine="auto"):
        import paged_kv_cache_426_b200 as pa
        self.pa, self.w, self.P, self.dev = pa, w, P, dev
        dt = w.torch_dtype
        self.esize = torch.tensor([], dtype=dt).element_size()
        self.kc = torch.empty((w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim), dtype=dt,
                              device=dev)
        self.vc = torch.empty_like(self.kc)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.max_len = max(w.meta["lens"]) - 1 + w.num_steps
        self.mb = -(-self.max_len // w.block_size)
        steps = [op for op in w.ops if op[0] == "step"]
        self.S = len(steps[0][1])
        self.ws = pa.alloc_workspace(self.S, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                     self.max_len, P, dev)

    def new_manager(self):
        pa = self.pa
        alloc = pa.BlockAllocator(self.w.num_blocks, self.w.free_order)
        return alloc, pa.BlockManager(alloc, self.w.block_size)

    def prefill(self, write=True):
        """Run the script up to the first step; write the prefill K/V (untimed)."""
        w, pa = self.w, self.pa
        alloc, mgr = self.new_manager()
        ks, vs, slots = [], [], []
        for op in w.ops:
            if op[0] == "add":
                mgr.add_seq(op[1])
            elif op[0] == "fork":
                mgr.fork(op[1], op[2])
            elif op[0] == "write":
                sl, cow = mgr.append(op[1], w.kv["k" + op[2]].shape[0])
                if cow and write:     # a write into a shared block copies it first
                    self._flush(ks, vs, slots)
                    pa.pa_copy_blocks(self.kc, self.vc, torch.tensor(cow, device=self.dev))
                ks.append(w.kv["k" + op[2]])
                vs.append(w.kv["v" + op[2]])
                slots.append(sl)
            elif op[0] == "step":
                break
        if write:
            self._flush(ks, vs, slots)
            torch.cuda.synchronize()
        return alloc, mgr

    def _flush(self, ks, vs, slots):
        if not ks:
            return
        k = torch.cat(ks).to(self.dev)
        v = torch.cat(vs).to(self.dev)
        s = torch.cat(slots).to(self.dev)
        self.pa.pa_reshape_and_cache(k, v, self.kc, self.vc, s)
        ks.clear(); vs.clear(); slots.clear()

    def plan_steps(self, mgr, n):
        """Host metadata of steps 0..n-1, uploaded to HBM with the step inputs."""
        w = self.w
        plan = []
        for k in range(n):
            seqs = w.step_seqs(k)
            slots, cow = mgr.append_step(seqs)
            tab, lens = mgr.block_tables(seqs, self.mb)
            plan.append(dict(
                slots=slots.to(self.dev), cow=cow.to(self.dev) if cow.shape[0] else None,
                tab=tab.to(self.dev), lens=lens.to(self.dev), lens_host=lens.tolist(),
                q=w.step_q[k].to(self.dev), k=w.step_k[k].to(self.dev),
                v=w.step_v[k].to(self.dev)))
        return plan

    def run_step(self, st, out):
        pa, w = self.pa, self.w
        n = 0
        if st["cow"] is not None:
            pa.pa_copy_blocks(self.kc, self.vc, st["cow"], err_flag=self.err)
            n += 1
        pa.pa_reshape_and_cache(st["k"], st["v"], self.kc, self.vc, st["slots"], err_flag=self.err)
        return n + 1

    def decode(self, st, out):
        """One pa_decode call: the decode kernel, plus the split-K merge kernel
        when a sequence can span several partitions.  Returns the launches."""
        self.pa.pa_decode(out, st["q"], self.kc, self.vc, st["tab"], st["lens"], self.max_len,
                          self.w.scale, partition_size=self.P, workspace=self.ws,
                          err_flag=self.err)
        n_pmax = -(-self.max_len // self.P) if self.P > 0 else 1
        return 2 if n_pmax > 1 else 1

    def bytes_of(self, lens):
        w = self.w
        return algorithmic_bytes(lens, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size,
                                 self.esize)


def run_ours(args, rank, world, local):
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    n_steps = args.warmup + args.steps
    w = workloads.make(args.workload, steps=n_steps)
    P = w.partition_size if args.partition_size is None else args.partition_size
    import paged_kv_cache_426_b200 as pa
    pa.pa_set_decode_engine({"auto": 0, "core": 1, "tensor": 2}[args.engine])
    sess = Session(w, P, dev, args.engine)
    _, mgr = sess.prefill()
    plan = sess.plan_steps(mgr, n_steps)
    out = torch.empty_like(plan[0]["q"])
    stream = torch.cuda.current_stream()

    # clock soak: step 0 again and again (idempotent writes) while the sampler starts
    sampler = ClockSampler(local)
    sampler.start()
    t_end = time.time() + args.soak
    while time.time() < t_end:
        for _ in range(10):
            sess.run_step(plan[0], out)
            sess.decode(plan[0], out)
        torch.cuda.synchronize()

    for k in range(args.warmup):
        sess.run_step(plan[k], out)
        sess.decode(plan[k], out)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    launches = 0
    for i in range(args.steps):
        st = plan[args.warmup + i]
        ev[i][0].record(stream)
        launches += sess.run_step(st, out)
        ev[i][1].record(stream)
        launches += sess.decode(st, out)
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    assert int(sess.err.item()) == 0, f"device error flag {int(sess.err.item())}"
    span_ms = ev[0][0].elapsed_time(ev[-1][2])
    dec_ms = [ev[i][1].elapsed_time(ev[i][2]) for i in range(args.steps)]
    step_bytes = [sess.bytes_of(plan[args.warmup + i]["lens_host"]) for i in range(args.steps)]
    total_bytes, span_ms, value = aggregate(sum(step_bytes), span_ms, world)
    dec_avg_ms = sum(dec_ms) / len(dec_ms)
    dec_gbs = (sum(step_bytes) / len(step_bytes)) / (dec_avg_ms * 1e-3) / 1e9
    peak, peak_kind = measured_peaks()
    S = sess.S

    e2e = run_e2e(sess, w, args, world) if args.e2e else None

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(span_ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": w.dtype, "data": "synthetic (seeded; see workloads/)",
        "config": {"workload": w.name, "num_seqs": S, "num_q_heads": w.num_q_heads,
                   "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim,
                   "block_size": w.block_size, "partition_size": P,
                   "mean_context_len": round(sum(plan[args.warmup]["lens_host"]) / S, 1),
                   "kv_bytes_per_step": step_bytes[0],
                   "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (KV cache >= 0.6 GB vs 126 MB)",
                   "engine": args.engine},
        "seqs_per_s": round(S * world / (span_ms * 1e-3 / args.steps), 1),
        "decode_only": {"gbs": round(dec_gbs, 1), "ms": round(dec_avg_ms, 4),
                        "seqs_per_s": round(S / (dec_avg_ms * 1e-3), 1)},
        "roofline": {"bound": "hbm", "achieved": round(dec_gbs, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(dec_gbs / peak, 4),
                     "traffic": profiled_traffic(w.name, sum(step_bytes) / len(step_bytes)),
                     "peak_kind": f"{peak_kind} copy bandwidth", "kernel": "pa_decode"},
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if e2e:
        result["e2e"] = e2e
    if rank == 0 and world == 1 and args.cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    return result


def run_e2e(sess, w, args, world):
    """Same metric through the public API with host buffers, every step: the
    live C++ manager's appends and block tables (host), then the step's H2D
    copies from pinned buffers, cache write, decode and the D2H of out.  The
    device part of each timed step is one CUDA graph (captured beforehand from
    the same public calls), so Python launch overhead does not pose as step
    time; the host part runs every step inside the timed region."""
    pa = sess.pa
    dev = sess.dev
    _, mgr = sess.prefill(write=False)       # same script -> same pool state
    S, mb = sess.S, sess.mb
    hq, hkv, d = w.num_q_heads, w.num_kv_heads, w.head_dim

    def pinned_set():
        return dict(slots=torch.empty(S, dtype=torch.int64).pin_memory(),
                    cow=torch.empty((S, 2), dtype=torch.int64).pin_memory(),
                    tab=torch.empty((S, mb), dtype=torch.int32).pin_memory(),
                    lens=torch.empty(S, dtype=torch.int32).pin_memory(),
                    out=torch.empty((S, hq, d), dtype=w.torch_dtype).pin_memory())
    pins = [pinned_set(), pinned_set()]          # alternate steps use alternate sets
    # the batch of each step (which sequences run) is a step input like q/K/V
    seq_ids = [torch.tensor(w.step_seqs(k), dtype=torch.int64) for k in range(w.num_steps)]
    qs = [w.step_q[k].pin_memory() for k in range(w.num_steps)]
    kk = [w.step_k[k].pin_memory() for k in range(w.num_steps)]
    vv = [w.step_v[k].pin_memory() for k in range(w.num_steps)]
    dq = torch.empty((S, hq, d), dtype=w.torch_dtype, device=dev)
    dk = torch.empty((S, hkv, d), dtype=w.torch_dtype, device=dev)
    dvv = torch.empty_like(dk)
    dslots = torch.empty(S, dtype=torch.int64, device=dev)
    dcow = torch.empty((S, 2), dtype=torch.int64, device=dev)
    dtab = torch.empty((S, mb), dtype=torch.int32, device=dev)
    dlens = torch.empty(S, dtype=torch.int32, device=dev)
    dout = torch.empty((S, hq, d), dtype=w.torch_dtype, device=dev)

    def host_part(k, pin):
        seqs = seq_ids[k]
        _, cow = mgr.append_step(seqs, slots_out=pin["slots"], cow_out=pin["cow"])
        _, lens = mgr.block_tables(seqs, mb, tables_out=pin["tab"], lens_out=pin["lens"])
        ncow = cow.shape[0]
        if ncow:                                 # copy-on-write pairs vary: never in a graph
            dcow[:ncow].copy_(pin["cow"][:ncow], non_blocking=True)
            pa.pa_copy_blocks(sess.kc, sess.vc, dcow[:ncow], err_flag=sess.err)
        return ncow, lens

    def device_part(k, pin):
        dq.copy_(qs[k], non_blocking=True)
        dk.copy_(kk[k], non_blocking=True)
        dvv.copy_(vv[k], non_blocking=True)
        dslots.copy_(pin["slots"], non_blocking=True)
        dtab.copy_(pin["tab"], non_blocking=True)
        dlens.copy_(pin["lens"], non_blocking=True)
        pa.pa_reshape_and_cache(dk, dvv, sess.kc, sess.vc, dslots, err_flag=sess.err)
        pa.pa_decode(dout, dq, sess.kc, sess.vc, dtab, dlens, sess.max_len, w.scale,
                     partition_size=sess.P, workspace=sess.ws, err_flag=sess.err)
        pin["out"].copy_(dout, non_blocking=True)

    for k in range(args.warmup):                 # eager: first launches set kernel attributes
        host_part(k, pins[k % 2])
        device_part(k, pins[k % 2])
        torch.cuda.synchronize()
    graphs = {}
    try:
        for k in range(args.warmup, args.warmup + args.steps):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                device_part(k, pins[k % 2])
            graphs[k] = g
    except Exception:                            # capture unavailable: launch eagerly
        graphs = {}
    torch.cuda.synchronize()
    h2d = d2h = 0
    total_bytes = 0
    times = []
    for k in range(args.warmup, args.warmup + args.steps):
        pin = pins[k % 2]
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        ncow, lens = host_part(k, pin)
        if graphs:
            graphs[k].replay()
        else:
            device_part(k, pin)
        torch.cuda.synchronize()                 # out is in host memory
        times.append(time.perf_counter() - t0)
        total_bytes += sess.bytes_of(lens.tolist())
        h2d = sum(t.numel() * t.element_size() for t in (qs[k], kk[k], vv[k], pin["slots"],
                                                          pin["tab"], pin["lens"]))
        h2d += ncow * 16
        d2h = pin["out"].numel() * pin["out"].element_size()
    used_graphs = bool(graphs)
    graphs.clear()
    total_bytes, span_ms, gbs = aggregate(total_bytes, sum(times) * 1e3, world)
    span = span_ms * 1e-3
    return {"value": round(gbs, 1), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(span / args.steps * 1e3, 4),
            "device_part": "cuda graph" if used_graphs else "eager"}


# ----------------------------------------------------------------------------- the oracle on the host

def cpu_baseline(w, seconds):
    """The oracle, as it stands, on the host cores: float64 decode of as many
    whole sequences of the first step's batch as fit in about ``seconds``."""
    import numpy as np
    import oracle
    from threadpoolctl import threadpool_info
    rec = oracle.run(w, decode=False, steps=1)
    st = rec.steps[0]
    q = oracle.as_storage(w.step_q[0], w.dtype)
    esize = torch.tensor([], dtype=w.torch_dtype).element_size()
    done, nbytes, t0 = 0, 0, time.perf_counter()
    S = len(st.seqs)
    while True:                 # whole sequences, cycling over the batch, ~`seconds` of work
        s = done % S
        oracle.paged_decode(q[s:s + 1], rec.key_cache, rec.value_cache, st.block_tables[s:s + 1],
                            st.context_lens[s:s + 1], w.scale, w.dtype)
        nbytes += algorithmic_bytes([int(st.context_lens[s])], w.num_q_heads, w.num_kv_heads,
                                    w.head_dim, w.block_size, esize)
        done += 1
        if time.perf_counter() - t0 > seconds:
            break
    dt = time.perf_counter() - t0
    threads = max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
    return {"value": round(nbytes / dt / 1e9, 4), "unit": "GB/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{done} sequence decodes ({done / S:.2f} passes over the {S} sequences of "
                      f"step 0 of {w.name}), float64 numpy (gather through the block table + "
                      f"softmax attention), {dt:.1f} s",
            "seqs_per_s": round(done / dt, 3), "host_cpus": len(os.sched_getaffinity(0))}


def run_reference(args, rank, world):
    """The oracle timed on the host: each step a bounded sample of the batch."""
    if rank != 0:
        return None
    w = workloads.make(args.workload, steps=1)
    per_step = max(1.0, args.cpu_seconds / max(1, args.steps))
    for _ in range(args.warmup):
        cpu_baseline(w, 0.5)
    vals = []
    base = None
    t0 = time.perf_counter()
    for _ in range(args.steps):
        base = cpu_baseline(w, per_step)
        vals.append(base["value"])
    span = time.perf_counter() - t0
    value = sum(vals) / len(vals)
    base["value"] = round(value, 4)
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(span / args.steps * 1e3, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded; see workloads/)",
            "config": {"workload": w.name, "parallelism": "host cores"},
            "cpu_baseline": base,
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def waste_report(name, lens, block_sizes, max_len, script=None):
    """Memory held per stored token for one batch: paged blocks vs a contiguous
    reservation of ``max_len`` slots per sequence.  The paged figure comes from
    the library's own allocator and manager (blocks they actually hand out);
    ``script`` (a workload's ops) replays adds, forks and writes so that shared
    blocks are counted once.  Host only: no GPU is touched."""
    import paged_kv_cache_426_b200 as pa
    rows = []
    tokens = int(sum(lens))
    for bs in block_sizes:
        need = sum(-(-L // bs) for L in lens) + len(lens)
        alloc = pa.BlockAllocator(need)
        mgr = pa.BlockManager(alloc, bs)
        for s, L in enumerate(lens):
            mgr.add_seq(s)
            if L:
                mgr.append(s, int(L))
        blocks = alloc.num_blocks - alloc.num_free()
        slots = blocks * bs
        rows.append({"waste": name, "block_size": bs, "num_seqs": len(lens), "tokens": tokens,
                     "paged_blocks": blocks, "paged_slots": slots,
                     "paged_waste": round(1 - tokens / slots, 4),
                     "contiguous_max_len": max_len, "contiguous_slots": len(lens) * max_len,
                     "contiguous_waste": round(1 - tokens / (len(lens) * max_len), 4)})
    return rows


def sharing_report(w):
    """Blocks held by a forked/shared-prefix script vs the same sequences with
    every prefix stored once per sequence (the library's manager both times)."""
    import paged_kv_cache_426_b200 as pa

    def held(dup):
        alloc = pa.BlockAllocator(1 << 18)           # host-only pool, ample for either layout
        mgr = pa.BlockManager(alloc, w.block_size)
        lengths = {}
        for op in w.ops:
            if op[0] == "add":
                mgr.add_seq(op[1]); lengths[op[1]] = 0
            elif op[0] == "fork":
                if dup:             # a private copy of everything the parent holds
                    mgr.add_seq(op[2])
                    if lengths[op[1]]:
                        mgr.append(op[2], lengths[op[1]])
                else:
                    mgr.fork(op[1], op[2])
                lengths[op[2]] = lengths[op[1]]
            elif op[0] == "write":
                n = w.kv["k" + op[2]].shape[0]
                mgr.append(op[1], n); lengths[op[1]] += n
            elif op[0] == "step":
                break
        return alloc.num_blocks - alloc.num_free(), sum(lengths.values())
    shared, toks = held(False)
    dup, _ = held(True)
    return {"sharing": w.name, "block_size": w.block_size, "logical_tokens": toks,
            "blocks_shared": shared, "blocks_duplicated": dup,
            "memory_saved": round(1 - shared / dup, 4)}


def run_waste(args):
    """Host-only memory accounting of the decode batches (one JSON line each)."""
    batches = [("gqa8b_bf16", workloads.make("gqa8b_bf16_bs16", steps=1), 8192),
               ("mha7b_f16", workloads.make("mha7b_f16", steps=1), 2048),
               ("long_bf16", workloads.make("long_bf16", steps=1), 131072)]
    for name, w, max_len in batches:
        for row in waste_report(name, w.meta["lens"], (8, 16, 32, 64, 128), max_len):
            print(json.dumps(row), flush=True)
    print(json.dumps(sharing_report(workloads.make("prefix_f16", steps=1))), flush=True)


def run_sweep(args):
    """Block-size and indirection study with the same decode path: the GQA
    batch's lengths and shapes at block sizes 8..128, with physical ids
    shuffled or in allocation order (each sequence's blocks consecutive), and
    batch-1 decodes of growing length.  Decode-only device time over
    ``args.steps`` steps; one JSON line per point."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    import paged_kv_cache_426_b200 as pa
    pa.pa_set_decode_engine({"auto": 0, "core": 1, "tensor": 2}[args.engine])
    n = args.warmup + args.steps
    gqa_lens = workloads.make("gqa8b_bf16_bs16", steps=1).meta["lens"]
    points = [("block_size", bs, layout, gqa_lens) for bs in (8, 16, 32, 64, 128)
              for layout in ("shuffled", "consecutive")]
    points += [("batch1", 16, layout, [L]) for L in (512, 4096, 32768, 131072)
               for layout in ("shuffled", "consecutive")]
    for kind, bs, layout, lens in points:
        w = workloads.custom("bf16", lens, 32, 8, 128, bs, seed=426 + bs, steps=n,
                             partition_size=1024, shuffle=(layout == "shuffled"))
        sess = Session(w, w.partition_size, dev, args.engine)
        _, mgr = sess.prefill()
        plan = sess.plan_steps(mgr, n)
        out = torch.empty_like(plan[0]["q"])
        for k in range(args.warmup):
            sess.run_step(plan[k], out)
            sess.decode(plan[k], out)
        torch.cuda.synchronize()
        total_ms, total_bytes = 0.0, 0
        for k in range(args.warmup, n):
            sess.run_step(plan[k], out)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            sess.decode(plan[k], out)
            b.record()
            torch.cuda.synchronize()
            total_ms += a.elapsed_time(b)
            total_bytes += sess.bytes_of(plan[k]["lens_host"])
        print(json.dumps({"sweep": kind, "block_size": bs, "layout": layout,
                          "num_seqs": len(lens), "max_len": max(lens), "steps": args.steps,
                          "gbs": round(total_bytes / total_ms / 1e6, 1),
                          "ms_per_step": round(total_ms / args.steps, 4),
                          "err": int(sess.err.item())}), flush=True)
        del sess, plan, out
        torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=29)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(workloads.BUILDERS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--partition-size", type=int, default=None)
    ap.add_argument("--engine", default="auto", choices=["auto", "core", "tensor"])
    ap.add_argument("--soak", type=float, default=1.0, help="seconds of clock soak")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--sweep", action="store_true",
                    help="block-size / indirection study instead of the benchmark line")
    ap.add_argument("--waste", action="store_true",
                    help="host-only memory accounting: paged vs contiguous reservation")
    ap.add_argument("--prefill", default=None, choices=sorted(workloads.PREFILL_BUILDERS),
                    help="causal prefill attention over the paged cache on this batch "
                         "(one GPU) instead of the decode line")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")
    rank, world, local = (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
                          int(os.environ.get("LOCAL_RANK", "0")))
    if args.sweep:
        run_sweep(args)
        return
    if args.waste:
        run_waste(args)
        return
    if args.prefill:
        print(json.dumps(run_prefill_bench(args)), flush=True)
        return
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    rank, world, local = dist_setup(args.gpus)
    res = run_ours(args, rank, world, local)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

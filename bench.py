"""Benchmark: paged decode attention on B200, KV-read GB/s per decode step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference] [--partition-size P] [--engine auto|core|tensor]
                    [--only] [--extra-steps K2]

A step is one decode step of the workload's batch: copy-on-write block
copies (when the host manager reports any), the cache write of the step's new
tokens, and decode attention over every sequence (the decode kernel plus the
split-K merge).  The cache write is part of the pa_decode call (its
key_new / value_new / slot_mapping option): the tensor-core decode kernel
stores each new token just before it copies the block that holds it.  The host metadata of every step (slot mapping, copy pairs,
block tables, lengths) is produced by the library's C++ manager before the
timed region and sits in HBM with the queries and new K/V rows.  Each step is
captured once as a CUDA graph from the public calls and replayed; CUDA events
on the launching stream around each replay give per-step device times (and
their percentiles), W warm-up steps run first, everything synchronised on
both sides.  Every step is a new token of the same sequences; the KV cache of
the headline batch (1.1 GB) is larger than the 126 MB L2, so no flush is
needed there; batches whose cache is not several times L2 are flushed (a
256 MB write) before each timed replay and are also reported warm.

value = algorithmic bytes of the K steps / timed span, algorithmic bytes per
step = sum_s L_s * Hkv * D * 2 * e (K and V) + 2 * S * Hq * D * e (q, out)
+ sum_s ceil(L_s / bs) * 4 (block-table entries).  roofline.achieved is the
same bytes over the decode call alone (its own graph replays).  At one GPU the
line also carries per_workload: the other decode batches (GQA at block 16 and
32, long context, shared prefix with logical and unique-physical bytes, the
tiny fp32 batch), each with decode and whole-step GB/s, fractions of the
measured copy peak, of a read peak measured here and of 8 TB/s, p10/p50/p90
step times and ncu traffic over algorithmic bytes.

e2e = the same metric through the public API with host buffers: the C++
manager appends the step's tokens live, pinned host buffers are copied to the
device, the kernels run and the output comes back to the host, every step,
pipelined one step ahead as a serving loop runs.

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
# the other decode batches, measured in the same run (one GPU) and reported under per_workload
GATE_WORKLOADS = ("gqa8b_bf16_bs16", "gqa8b_bf16_bs32", "long_bf16", "prefix_f16", "tiny_f32")
NOMINAL_HBM_GBS = 8000.0


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

    ws = pa.prefill_workspace(dev)

    def attend():
        pa.pa_prefill(out, q, kc, vc, tab, lens, cu, max_q, b.scale, workspace=ws, err_flag=err)

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
    """One replica of one workload: caches, the C++ manager, and per-step
    device inputs."""

    def __init__(self, w, P, dev, engine="auto"):
        import paged_kv_cache_426_b200 as pa
        self.pa, self.w, self.P, self.dev = pa, w, P, dev
        self.engine = None if engine == "auto" else engine     # per-call option
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
                tab_host=tab, q=w.step_q[k].to(self.dev), k=w.step_k[k].to(self.dev),
                v=w.step_v[k].to(self.dev)))
        return plan

    def cow(self, st):
        """Copy-on-write copies of one step, when the manager reported any.
        Returns the launches."""
        if st["cow"] is None:
            return 0
        self.pa.pa_copy_blocks(self.kc, self.vc, st["cow"], err_flag=self.err)
        return 1

    def decode(self, st, out, write=False):
        """One pa_decode call, with the step's cache write when ``write``: the
        decode kernel (which writes the new tokens itself on the tensor-core
        engine; the CUDA-core engine gets a write launch first), plus the
        split-K merge kernel unless the decode kernel merges the splits
        itself.  Returns the launches."""
        self.pa.pa_decode(out, st["q"], self.kc, self.vc, st["tab"], st["lens"], self.max_len,
                          self.w.scale, partition_size=self.P, workspace=self.ws,
                          err_flag=self.err, engine=self.engine,
                          write=(st["k"], st["v"], st["slots"]) if write else None)
        n_pmax = -(-self.max_len // self.P) if self.P > 0 else 1
        tensor = self.w.dtype != "f32" and self.engine not in ("core", 1)
        merged_inside = tensor and n_pmax <= 4
        return 1 + (n_pmax > 1 and not merged_inside) + (write and not tensor)

    def step(self, st, out):
        return self.cow(st) + self.decode(st, out, write=True)

    def bytes_of(self, lens):
        w = self.w
        return algorithmic_bytes(lens, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size,
                                 self.esize)

    def unique_bytes_of(self, st):
        """Like bytes_of, but K/V counted once per physical block (the largest
        number of its rows any sequence reads): blocks shared by reference
        count are stored once and can be read from HBM once."""
        w = self.w
        bs = w.block_size
        rows = {}
        for row, L in zip(st["tab_host"].tolist(), st["lens_host"]):
            for i in range(-(-L // bs)):
                b = row[i]
                rows[b] = max(rows.get(b, 0), min(bs, L - i * bs))
        kv = sum(rows.values()) * w.num_kv_heads * w.head_dim * 2 * self.esize
        S = len(st["lens_host"])
        return (kv + 2 * S * w.num_q_heads * w.head_dim * self.esize
                + sum(-(-L // bs) for L in st["lens_host"]) * 4)


def capture(fn):
    """A CUDA graph of whatever ``fn`` launches on the current stream."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def replay_timed(graphs, flush=None):
    """Replay ``graphs`` in order on the current stream, a CUDA event pair
    around each replay; with ``flush`` (a buffer larger than L2) the buffer
    is overwritten before each replay, outside its event pair.  Returns the
    per-replay device times (ms) and the span from the first start to the
    last end (ms)."""
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in graphs]
    for g, (a, b) in zip(graphs, ev):
        if flush is not None:
            flush.fill_(1)
        a.record(stream)
        g.replay()
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev], ev[0][0].elapsed_time(ev[-1][1])


def pct(xs, q):
    """q-th percentile (0..100) of xs, linear interpolation."""
    xs = sorted(xs)
    if len(xs) == 1:
        return xs[0]
    r = (len(xs) - 1) * q / 100.0
    lo = int(math.floor(r))
    hi = min(lo + 1, len(xs) - 1)
    return xs[lo] + (xs[hi] - xs[lo]) * (r - lo)


def spread(ms):
    return {"p10": round(pct(ms, 10), 4), "p50": round(pct(ms, 50), 4),
            "p90": round(pct(ms, 90), 4)}


def read_peak(dev, gib=4, reps=6):
    """HBM read bandwidth of this GPU, measured here: a plain reduction over
    ``gib`` GiB (torch's sum kernel reads every byte once and writes a
    scalar), best of ``reps``; GB/s.  The buffer is freed afterwards."""
    x = torch.ones((gib << 30) // 4, dtype=torch.float32, device=dev)
    best = 0.0
    for i in range(reps + 1):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        x.sum()
        b.record()
        torch.cuda.synchronize()
        if i:
            best = max(best, x.numel() * 4 / (a.elapsed_time(b) * 1e-3) / 1e9)
    del x
    torch.cuda.empty_cache()
    return round(best, 1)


def workload_config(w, P, S, lens, step_bytes, world, engine, l2):
    return {"workload": w.name, "num_seqs": S, "num_q_heads": w.num_q_heads,
            "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim,
            "block_size": w.block_size, "partition_size": P,
            "mean_context_len": round(sum(lens) / S, 1), "kv_bytes_per_step": step_bytes,
            "parallelism": f"replicas x{world}", "l2": l2, "engine": engine}


L2_BYTES = 126 << 20


def measure(name, args, dev, n_timed, world, engine="auto", flush_buf=None, warm_too=False,
            sampler=None):
    """Device-timed steps of one workload.  Every step (copy-on-write copies,
    decode with the step's cache write, merge) and, separately, its decode
    call alone (no write) are
    captured as CUDA graphs and replayed in step order with CUDA events around
    each replay.  Returns the numbers and the session (for the end-to-end
    leg)."""
    n_steps = args.warmup + n_timed
    w = workloads.make(name, steps=n_steps)
    P = w.partition_size if args.partition_size is None else args.partition_size
    sess = Session(w, P, dev, engine)
    _, mgr = sess.prefill()
    plan = sess.plan_steps(mgr, n_steps)
    out = torch.empty_like(plan[0]["q"])
    # eager warm-up steps (kernel attributes are set on first use), then graphs
    for k in range(args.warmup):
        sess.step(plan[k], out)
    torch.cuda.synchronize()
    timed = plan[args.warmup:]
    launches = 0
    step_graphs, dec_graphs = [], []
    for st in timed:
        n = [0]

        def whole(st=st, n=n):
            n[0] = sess.step(st, out)
        step_graphs.append(capture(whole))
        dec_graphs.append(capture(lambda st=st: sess.decode(st, out)))
        launches += n[0]
    # all timed steps in one graph each: the span (no gap between steps but
    # the kernels' own), and the decode calls alone
    all_steps = capture(lambda: [sess.step(st, out) for st in timed])
    all_decodes = capture(lambda: [sess.decode(st, out) for st in timed])
    # clock soak (the first step again and again: idempotent writes); the
    # sampler sees the soak and the timed replays only
    if sampler is not None:
        sampler.start()
    t_end = time.time() + args.soak
    while time.time() < t_end:
        for _ in range(10):
            step_graphs[0].replay()
        torch.cuda.synchronize()
    step_graphs[0].replay()
    dec_graphs[0].replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    # a batch whose K/V (each physical block once) is not several times the
    # L2 gets the L2 flushed before every timed replay, outside the events
    unique = [sess.unique_bytes_of(st) for st in timed]
    need_flush = flush_buf is not None and min(unique) < 4 * L2_BYTES
    fl = flush_buf if need_flush else None
    if need_flush:
        step_ms, _ = replay_timed(step_graphs, fl)
        dec_ms, _ = replay_timed(dec_graphs, fl)
        span_ms, dec_avg_ms = sum(step_ms), sum(dec_ms) / len(dec_ms)
    else:
        (span_ms,), _ = replay_timed([all_steps])
        (dec_total,), _ = replay_timed([all_decodes])
        dec_avg_ms = dec_total / len(timed)
        step_ms, _ = replay_timed(step_graphs)
        dec_ms, _ = replay_timed(dec_graphs)
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler is not None else None
    barrier(world)
    assert int(sess.err.item()) == 0, f"{name}: device error flag {int(sess.err.item())}"
    step_bytes = [sess.bytes_of(st["lens_host"]) for st in timed]
    res = dict(w=w, sess=sess, P=P, plan=plan, step_bytes=step_bytes, step_ms=step_ms,
               dec_ms=dec_ms, span_ms=span_ms, dec_avg_ms=dec_avg_ms, launches=launches,
               flushed=need_flush, clocks=clocks)
    if name.startswith("prefix"):
        res["unique_bytes"] = unique
    if warm_too and need_flush:
        (ws,), _ = replay_timed([all_steps])
        (wd,), _ = replay_timed([all_decodes])
        res["warm_step_ms"], _ = replay_timed(step_graphs)
        res["warm_dec_ms"], _ = replay_timed(dec_graphs)
        res["warm_span_ms"], res["warm_dec_avg_ms"] = ws, wd / len(timed)
    del step_graphs, dec_graphs, all_steps, all_decodes
    return res


def summarize(m, peak, rpeak):
    """Per-workload summary: GB/s of the decode call and of the whole step,
    their fractions of the measured copy peak, the read peak and 8 TB/s,
    step-time percentiles, and ncu traffic over algorithmic bytes."""
    w, sess = m["w"], m["sess"]
    b = sum(m["step_bytes"]) / len(m["step_bytes"])
    dec = m["dec_avg_ms"]
    stp = m["span_ms"] / len(m["step_ms"])
    dec_gbs = b / (dec * 1e-3) / 1e9
    stp_gbs = b / (stp * 1e-3) / 1e9
    traffic = profiled_traffic(w.name, b)
    r = {"decode_gbs": round(dec_gbs, 1), "step_gbs": round(stp_gbs, 1),
         "decode_frac_measured_copy": round(dec_gbs / peak, 4),
         "decode_frac_read_peak": round(dec_gbs / rpeak, 4) if rpeak else None,
         "decode_frac_8tbs": round(dec_gbs / NOMINAL_HBM_GBS, 4),
         "step_frac_measured_copy": round(stp_gbs / peak, 4),
         "step_frac_8tbs": round(stp_gbs / NOMINAL_HBM_GBS, 4),
         "decode_ms": spread(m["dec_ms"]), "step_ms": spread(m["step_ms"]),
         "algorithmic_bytes_per_step": int(b),
         "traffic_over_algorithmic": round(traffic / b, 4) if traffic else None,
         "seqs_per_s": round(sess.S / (stp * 1e-3), 1),
         "decode_seqs_per_s": round(sess.S / (dec * 1e-3), 1),
         "steps": len(m["step_ms"]), "partition_size": m["P"], "dtype": w.dtype,
         "l2": ("L2 flushed (256 MB write) before every timed replay, steps timed one by one"
                if m["flushed"] else "K/V read per step larger than L2")}
    if "unique_bytes" in m:
        u = sum(m["unique_bytes"]) / len(m["unique_bytes"])
        r["logical_bytes_per_step"] = int(b)
        r["unique_physical_bytes_per_step"] = int(u)
        r["decode_unique_gbs"] = round(u / (dec * 1e-3) / 1e9, 1)
        r["step_unique_gbs"] = round(u / (stp * 1e-3) / 1e9, 1)
    if "warm_step_ms" in m:
        wd = m["warm_dec_avg_ms"]
        ws = m["warm_span_ms"] / len(m["warm_step_ms"])
        r["warm"] = {"decode_gbs": round(b / (wd * 1e-3) / 1e9, 1),
                     "step_gbs": round(b / (ws * 1e-3) / 1e9, 1),
                     "decode_ms": spread(m["warm_dec_ms"]), "step_ms": spread(m["warm_step_ms"])}
    return r


def run_ours(args, rank, world, local):
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peak, peak_kind = measured_peaks()
    rpeak = read_peak(dev) if world == 1 else None
    m = measure(args.workload, args, dev, args.steps, world, args.engine,
                sampler=ClockSampler(local))
    w, sess, P, launches, clocks = m["w"], m["sess"], m["P"], m["launches"], m["clocks"]
    step_bytes = m["step_bytes"]
    total_bytes, span_ms, value = aggregate(sum(step_bytes), m["span_ms"], world)
    dec_avg_ms = m["dec_avg_ms"]
    dec_gbs = (sum(step_bytes) / len(step_bytes)) / (dec_avg_ms * 1e-3) / 1e9
    S = sess.S
    lens0 = m["plan"][args.warmup]["lens_host"]
    e2e = run_e2e(sess, w, args, world) if args.e2e else None
    head = summarize(m, peak, rpeak)
    del m

    per = {}
    if world == 1 and args.all_workloads:
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        for name in GATE_WORKLOADS:
            if name == args.workload:
                continue
            mw = measure(name, args, dev, args.extra_steps, world, args.engine, flush_buf=flush,
                         warm_too=True)
            per[name] = summarize(mw, peak, rpeak)
            if args.e2e and name != "tiny_f32":
                e = run_e2e(mw["sess"], mw["w"], args, world)
                e["frac_of_step"] = round(e["value"] / per[name]["step_gbs"], 4)
                per[name]["e2e"] = e
            del mw
            torch.cuda.empty_cache()
        del flush
    per[args.workload] = head

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(span_ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": w.dtype, "data": "synthetic (seeded; see workloads/)",
        "config": workload_config(w, P, S, lens0, step_bytes[0], world, args.engine,
                                  "inputs larger than L2 (KV cache >= 0.6 GB vs 126 MB)"),
        "timing": "the K steps as one CUDA graph (captured from the public calls) between CUDA "
                  "events; decode_only likewise for the decode calls alone; percentiles from "
                  "one graph per step",
        "seqs_per_s": round(S * world / (span_ms * 1e-3 / args.steps), 1),
        "decode_only": {"gbs": round(dec_gbs, 1), "ms": round(dec_avg_ms, 4),
                        "seqs_per_s": round(S / (dec_avg_ms * 1e-3), 1)},
        "step_ms": head["step_ms"], "decode_ms": head["decode_ms"],
        "frac_of_8tbs": {"step": round(value / world / NOMINAL_HBM_GBS, 4),
                         "decode": round(dec_gbs / NOMINAL_HBM_GBS, 4)},
        "read_peak_gbs": rpeak,
        "roofline": {"bound": "hbm", "achieved": round(dec_gbs, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(dec_gbs / peak, 4),
                     "traffic": profiled_traffic(w.name, sum(step_bytes) / len(step_bytes)),
                     "peak_kind": f"{peak_kind} copy bandwidth (burst, kernel timed alone)",
                     "frac_of_read_peak": round(dec_gbs / rpeak, 4) if rpeak else None,
                     "kernel": "pa_decode"},
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if per and len(per) > 1:
        result["per_workload"] = per
    if e2e:
        e2e["frac_of_step"] = round(e2e["value"] / value, 4)
        result["e2e"] = e2e
    if rank == 0 and world == 1 and args.cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
        result["cpu_baseline"]["one_core"] = cpu_baseline(w, args.cpu_seconds, threads=1)
    return result


def run_e2e(sess, w, args, world):
    """Same metric through the public API with host buffers, every step: the
    live C++ manager's appends and block tables (host), the step's H2D copies
    from pinned buffers, copy-on-write copies, decode with the cache write, and
    the D2H of out.  Steps are pipelined the way a serving loop runs them: step
    k is one CUDA graph of three branches, step k's decode (and write), the H2D
    copies of step k + 1's inputs into the other device set, and the D2H of
    step k - 1's out, captured beforehand from the same public calls; while it
    runs, the host prepares step k + 2 (manager calls into the pinned set step
    k's copies have finished reading).  One graph launch per step: Python
    launch overhead does not pose as step time."""
    pa = sess.pa
    dev = sess.dev
    _, mgr = sess.prefill(write=False)       # same script -> same pool state
    S, mb = sess.S, sess.mb
    hq, hkv, d = w.num_q_heads, w.num_kv_heads, w.head_dim
    dt = w.torch_dtype
    n = w.num_steps

    def pinned_set():
        return dict(slots=torch.empty(S, dtype=torch.int64).pin_memory(),
                    tab=torch.empty((S, mb), dtype=torch.int32).pin_memory(),
                    lens=torch.empty(S, dtype=torch.int32).pin_memory(),
                    out=torch.empty((S, hq, d), dtype=dt).pin_memory())

    def device_set():
        return dict(q=torch.empty((S, hq, d), dtype=dt, device=dev),
                    k=torch.empty((S, hkv, d), dtype=dt, device=dev),
                    v=torch.empty((S, hkv, d), dtype=dt, device=dev),
                    slots=torch.empty(S, dtype=torch.int64, device=dev),
                    cow=torch.empty((S, 2), dtype=torch.int64, device=dev),
                    tab=torch.empty((S, mb), dtype=torch.int32, device=dev),
                    lens=torch.empty(S, dtype=torch.int32, device=dev),
                    out=torch.empty((S, hq, d), dtype=dt, device=dev))
    pins = [pinned_set(), pinned_set()]          # step k uses set k % 2
    devs = [device_set(), device_set()]
    cow_pins = [torch.empty((S, 2), dtype=torch.int64).pin_memory() for _ in range(n)]
    # the batch of each step (which sequences run) is a step input like q/K/V
    seq_ids = [torch.tensor(w.step_seqs(k), dtype=torch.int64) for k in range(n)]
    qs = [w.step_q[k].pin_memory() for k in range(n)]
    kk = [w.step_k[k].pin_memory() for k in range(n)]
    vv = [w.step_v[k].pin_memory() for k in range(n)]
    main = torch.cuda.current_stream()
    copy_s, out_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def h2d(k):
        D, pin = devs[k % 2], pins[k % 2]
        D["q"].copy_(qs[k], non_blocking=True)
        D["k"].copy_(kk[k], non_blocking=True)
        D["v"].copy_(vv[k], non_blocking=True)
        D["slots"].copy_(pin["slots"], non_blocking=True)
        D["tab"].copy_(pin["tab"], non_blocking=True)
        D["lens"].copy_(pin["lens"], non_blocking=True)

    def d2h(k):
        pins[k % 2]["out"].copy_(devs[k % 2]["out"], non_blocking=True)

    def compute(k):
        D = devs[k % 2]
        pa.pa_decode(D["out"], D["q"], sess.kc, sess.vc, D["tab"], D["lens"], sess.max_len,
                     w.scale, partition_size=sess.P, workspace=sess.ws, err_flag=sess.err,
                     engine=sess.engine, write=(D["k"], D["v"], D["slots"]))

    def host_part(k):
        pin = pins[k % 2]
        _, cow = mgr.append_step(seq_ids[k], slots_out=pin["slots"], cow_out=cow_pins[k])
        _, lens = mgr.block_tables(seq_ids[k], mb, tables_out=pin["tab"], lens_out=pin["lens"])
        return cow.shape[0], lens

    def cow_copies(k, ncow):
        # copy-on-write pairs vary: never in a graph; on the stream before step k
        dcow = devs[k % 2]["cow"][:ncow]
        dcow.copy_(cow_pins[k][:ncow], non_blocking=True)
        pa.pa_copy_blocks(sess.kc, sess.vc, dcow, err_flag=sess.err)

    def step_graph(k, first, last):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            s0 = torch.cuda.current_stream()
            copy_s.wait_stream(s0)
            out_s.wait_stream(s0)
            with torch.cuda.stream(copy_s):
                if k + 1 <= last:
                    h2d(k + 1)
            with torch.cuda.stream(out_s):
                if k - 1 >= first:
                    d2h(k - 1)
            compute(k)
            s0.wait_stream(copy_s)
            s0.wait_stream(out_s)
        return g

    def run(ks, count):
        first, last = ks[0], ks[-1]
        graphs = [step_graph(k, first, last) for k in ks]
        torch.cuda.synchronize()
        done = [torch.cuda.Event() for _ in ks]
        first_in = torch.cuda.Event()
        t0 = time.perf_counter()
        pend = {first: host_part(first)}
        h2d(first)                               # the first step's inputs
        first_in.record(main)
        if first + 1 <= last:
            pend[first + 1] = host_part(first + 1)
        for i, k in enumerate(ks):
            ncow, lens = pend.pop(k)
            if ncow:
                cow_copies(k, ncow)
            graphs[i].replay()                   # step k, step k + 1's H2D, step k - 1's D2H
            done[i].record(main)
            if count:                            # counted after the timed region
                seen.append((k, ncow, lens.clone()))
            if k + 2 <= last:
                # step k's H2D (graph k - 1, or the copies before the first
                # graph) has read pinned set k % 2, which step k + 2 refills
                (done[i - 1] if i >= 1 else first_in).synchronize()
                pend[k + 2] = host_part(k + 2)
        d2h(last)
        torch.cuda.synchronize()                 # every step's out is in host memory
        t1 = time.perf_counter()
        return t1 - t0

    seen = []
    stats = dict(bytes=0, h2d=0, d2h=0)
    run(list(range(args.warmup)), False)
    torch.cuda.synchronize()
    barrier(world)
    dt_s = run(list(range(args.warmup, n)), True)
    assert int(sess.err.item()) == 0, f"e2e: device error flag {int(sess.err.item())}"
    for k, ncow, lens in seen:
        stats["bytes"] += sess.bytes_of(lens.tolist())
        stats["h2d"] = (sum(t.numel() * t.element_size() for t in
                            (qs[k], kk[k], vv[k], pins[k % 2]["slots"], pins[k % 2]["tab"],
                             pins[k % 2]["lens"])) + ncow * 16)
        stats["d2h"] = pins[k % 2]["out"].numel() * pins[k % 2]["out"].element_size()
    total_bytes, span_ms, gbs = aggregate(stats["bytes"], dt_s * 1e3, world)
    K = n - args.warmup
    return {"value": round(gbs, 1), "unit": "GB/s",
            "h2d_bytes_per_step": stats["h2d"], "d2h_bytes_per_step": stats["d2h"],
            "ms_per_step": round(span_ms / K, 4),
            "device_part": "one cuda graph per step (its compute, the next step's H2D, the "
                           "previous step's D2H), host prepared two steps ahead"}


# ----------------------------------------------------------------------------- the oracle on the host

def cpu_baseline(w, seconds, threads=None):
    """The oracle, as it stands, on the host cores: float64 decode of as many
    whole sequences of the first step's batch as fit in about ``seconds``.
    ``threads``: cap on the BLAS threads (None = all the process may use)."""
    import contextlib
    import oracle
    from threadpoolctl import threadpool_info, threadpool_limits
    rec = oracle.run(w, decode=False, steps=1)
    st = rec.steps[0]
    q = oracle.as_storage(w.step_q[0], w.dtype)
    esize = torch.tensor([], dtype=w.torch_dtype).element_size()
    S = len(st.seqs)
    limit = threadpool_limits(limits=threads) if threads else contextlib.nullcontext()
    with limit:
        done, nbytes, t0 = 0, 0, time.perf_counter()
        while True:             # whole sequences, cycling over the batch, ~`seconds` of work
            s = done % S
            oracle.paged_decode(q[s:s + 1], rec.key_cache, rec.value_cache,
                                st.block_tables[s:s + 1], st.context_lens[s:s + 1], w.scale,
                                w.dtype)
            nbytes += algorithmic_bytes([int(st.context_lens[s])], w.num_q_heads,
                                        w.num_kv_heads, w.head_dim, w.block_size, esize)
            done += 1
            if time.perf_counter() - t0 > seconds:
                break
        dt = time.perf_counter() - t0
        used = max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
    return {"value": round(nbytes / dt / 1e9, 4), "unit": "GB/s", "cores": used,
            "kind": "oracle",
            "sample": f"{done} sequence decodes ({done / S:.2f} passes over the {S} sequences of "
                      f"step 0 of {w.name}), float64 numpy (gather through the block table + "
                      f"softmax attention), {dt:.1f} s, {used} BLAS thread(s)",
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
    P = w.partition_size if getattr(args, "partition_size", None) is None else args.partition_size
    S = len(w.step_seqs(0))
    lens = w.meta["lens"][:S] if len(w.meta["lens"]) >= S else w.meta["lens"]
    esize = torch.tensor([], dtype=w.torch_dtype).element_size()
    cfg = workload_config(w, P, S, lens,
                          algorithmic_bytes(lens, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                            w.block_size, esize),
                          world, getattr(args, "engine", "auto"), "host memory (oracle on CPU)")
    cfg["parallelism"] = "host cores"
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(span / args.steps * 1e3, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded; see workloads/)",
            "config": cfg,
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
            sess.write(plan[k])
            sess.decode(plan[k], out)
        torch.cuda.synchronize()
        total_ms, total_bytes = 0.0, 0
        for k in range(args.warmup, n):
            sess.write(plan[k])
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
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--only", dest="all_workloads", action="store_false",
                    help="measure only --workload (no per_workload section)")
    ap.add_argument("--extra-steps", type=int, default=24,
                    help="decode steps of each other batch in per_workload (the e2e leg times "
                         "all but --warmup of them, pipelined: a short run weighs the pipeline's "
                         "fill and drain too much)")
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

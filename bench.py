"""Benchmark of the paged decode hot path on B200.

A step is one pass of the hot path over one synthetic batch: the copy-on-write
block copies the batch needs (none for the decode-only workloads), the slot
write of the step's new tokens, and decode (split-K plus its reduce when the
partition rule splits the batch). When the step writes only each sequence's
newest token and decodes unsplit from a 16- or 32-bit cache, the slot write
and decode run as one launch (pa_decode_append); the bytes counted are the
same. The default workload is the LLaMA-7B-shaped
fp16 decode layer (64 sequences, 32 heads, head_dim 128, block 16, context
lengths U{256..2048}).

metric: effective GB/s = algorithmic bytes of the step / device time of the
step, with
  decode bytes = sum_s ctx_s * 2 * Hkv * D * elt + S * Hq * D * (elt_q + elt_out)
                 + 4 * sum_s ceil(ctx_s / bs) + 4 * S
  slot-write bytes = 2 * T * Hkv * D * elt (read) + the same (write) + 4 * T
Inputs (>= 1.1 GB of K/V per step) are larger than L2 (126 MB), so no flush between steps.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 each rank runs its own batch on its own GPU (sequences shard across
GPUs with no exchange); value = all ranks' bytes / the slowest rank's time.
Under torchrun the ranks come from the launcher (WORLD_SIZE must equal N);
without one, bench.py starts N local ranks itself under torch.distributed.run.
--dry-run --backend gloo runs that launch and the timing plumbing on CPU only.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
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

DEFAULT_WORKLOAD = "llama7b_mha_fp16"
METRIC = "paged decode: effective KV GB/s (% of HBM peak) and seq-tokens/s on 1 B200"
FALLBACK_HBM_GBS = 6650.0


def elt(dtype: torch.dtype) -> int:
    return torch.tensor([], dtype=dtype).element_size()


def kv_row_bytes(spec) -> int:
    """Bytes of one (token, kv head) row of K or V in the cache (int8: codes
    plus the fp32 row scale)."""
    return spec.head_dim * elt(spec.torch_kv_dtype) + (4 if spec.kv_dtype == "i8" else 0)


def decode_bytes(spec, ctx: np.ndarray) -> int:
    """Algorithmic bytes of one decode over the batch (K/V read once, q read,
    out written, the used table entries and the context lengths read)."""
    kv = int(ctx.astype(np.int64).sum()) * 2 * spec.num_kv_heads * kv_row_bytes(spec)
    qo = len(ctx) * spec.num_heads * spec.head_dim * (elt(spec.torch_q_dtype) + elt(spec.torch_out_dtype))
    tables = 4 * int(((ctx.astype(np.int64) + spec.block_size - 1) // spec.block_size).sum()) + 4 * len(ctx)
    return kv + qo + tables


def kv_bytes_per_token(num_layers: int, num_kv_heads: int, head_dim: int, elt_bytes: int) -> int:
    """K and V bytes of one token across all layers (2 * layers * heads * dim * elt)."""
    return 2 * num_layers * num_kv_heads * head_dim * elt_bytes


def write_bytes(spec, num_tokens: int) -> int:
    src = spec.num_kv_heads * spec.head_dim * elt(spec.torch_q_dtype)   # the new rows read
    dst = spec.num_kv_heads * kv_row_bytes(spec)                         # and written (int8: + scale)
    return 2 * num_tokens * (src + dst) + 4 * num_tokens


def copy_bytes(spec, num_pairs: int) -> int:
    blk = spec.num_kv_heads * spec.block_size * kv_row_bytes(spec)
    return 2 * 2 * num_pairs * blk + 16 * num_pairs


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    for name in ("pa_decode.cu", "pa_common.cuh", "pa_internal.h"):
        with open(os.path.join(ROOT, "paged_kv_cache_340_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "decode_dram_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    e = rec.get(workload, {}).get(kernel)
    if not e or e.get("source_sha") != kernel_source_sha():
        return None
    return e.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.uuid = None
        try:
            self.uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            self.uuid = None

    def start(self):
        """Starts sampling and returns once the first sample has arrived, so
        that nvidia-smi's start-up does not fall inside the timed region."""
        import threading
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        self.lines = []
        first = threading.Event()
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return

        def reader():
            for ln in self.proc.stdout:
                self.lines.append(ln)
                first.set()
            first.set()

        self.thread = threading.Thread(target=reader, daemon=True)
        self.thread.start()
        first.wait(timeout=20)
        self.skip = len(self.lines)  # samples taken before the timed region

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.06)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=5)
        out = "".join(self.lines[self.skip:])
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for row in csv.reader(io.StringIO(out)):
            if len(row) < 8:
                continue
            try:
                sm.append(float(row[0]))
                mx.append(float(row[1]))
            except ValueError:
                continue
            for n, v in zip(names, row[4:8]):
                if v.strip().lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------ distributed

from paged_kv_cache_340_b200 import dist as pdist  # noqa: E402


def dist_setup(n_gpus: int, backend: str = "nccl"):
    world, rank, local = pdist.init(backend)
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but {world} rank(s) were started")
    return world, rank, local


def launch_ranks(args) -> None:
    """--gpus N > 1 with no launcher around this process: start N local ranks
    (one process per GPU) under torch.distributed.run with this script and
    these arguments, wait for them and exit with their status. With a
    launcher, check that it started N ranks; with N = 1, return."""
    env_world = os.environ.get("WORLD_SIZE")
    if env_world is not None:
        if int(env_world) != args.gpus:
            raise SystemExit(f"--gpus {args.gpus} but the launcher started {env_world} rank(s)")
        return
    if args.gpus <= 1:
        return
    if not args.dry_run and torch.cuda.device_count() < args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but {torch.cuda.device_count()} GPU(s) are visible")
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__)] + sys.argv[1:]
    bound = 3600
    import shutil
    if shutil.which("timeout"):
        cmd = ["timeout", "-k", "60", str(bound)] + cmd
    r = subprocess.run(cmd, env=dict(os.environ, MASTER_ADDR="127.0.0.1"))
    raise SystemExit(r.returncode)


def max_over_ranks(x: float, world: int) -> float:
    return pdist.max_over_ranks(x, world)


def barrier(world: int):
    pdist.barrier(world)


# ------------------------------------------------------------ measurement

def build_batch(name: str, rank: int, partition=None):
    from paged_kv_cache_340_b200.batch import build_decode_batch, build_parallel_sampling_batch, \
        build_prefix_cache_batch, write_prefix
    from paged_kv_cache_340_b200.workloads import SPECS, make_decode_inputs, make_parallel_sampling_inputs, \
        make_prefix_cache_inputs
    spec = pdist.rank_spec(SPECS[name], rank)
    if spec.lengths[0] == "prefix":
        inp = make_prefix_cache_inputs(spec)
        b = build_prefix_cache_batch(spec, inp)
        write_prefix(b)
    elif spec.lengths[0] == "parallel":
        inp = make_parallel_sampling_inputs(spec)
        b = build_parallel_sampling_batch(spec, inp, partition_size=partition or 0)
        write_prefix(b)
    else:
        inp = make_decode_inputs(spec)
        b = build_decode_batch(spec, inp, partition_size=partition)
    torch.cuda.synchronize()
    b.host_inputs = inp
    return spec, b


def unique_kv_bytes(spec, tables: np.ndarray, ctx: np.ndarray) -> int:
    """K/V bytes of the distinct cache rows one decode reads: a block that
    several sequences share (a prefix) counts once, with the most tokens any
    of them reads from it."""
    used = {}
    bs = spec.block_size
    for row, L in zip(tables, ctx.astype(np.int64)):
        for j in range(int((L + bs - 1) // bs)):
            b = int(row[j])
            used[b] = max(used.get(b, 0), int(min(bs, L - j * bs)))
    return sum(used.values()) * 2 * spec.num_kv_heads * kv_row_bytes(spec)


def step_bytes(spec, b) -> dict:
    d = decode_bytes(spec, b.host_context_lens)
    w = write_bytes(spec, b.new_key.shape[0])
    c = copy_bytes(spec, b.cow_pairs.shape[0])
    return dict(decode=d, write=w, copy=c, total=d + w + c)


def launches_per_step(b) -> int:
    if b.fused_append:
        return (1 if b.cow_pairs.shape[0] else 0) + 1
    return (1 if b.cow_pairs.shape[0] else 0) + 1 + (2 if b.partition_size else 1)


def time_steps(b, steps: int, warmup: int, world: int, sample_clocks=False, device_index=0):
    """Device time per step over `steps` steps (max over ranks), and the mean
    duration of each kernel of the step (a second pass with CUDA events
    around every launch, on the launching stream)."""
    from paged_kv_cache_340_b200 import pa_copy_blocks, pa_copy_blocks_q8, pa_decode, pa_decode_append, \
        pa_decode_q8, pa_decode_splitk, pa_decode_splitk_q8, pa_reshape_and_cache, pa_reshape_and_cache_q8, \
        pa_splitk_reduce
    spec = b.spec
    stream = torch.cuda.current_stream()

    def mark(ev, i):
        if ev is not None:
            ev[i].record(stream)

    def step(ev=None):
        mark(ev, 0)
        if b.k_scale is not None:  # int8 cache
            if b.cow_pairs.shape[0]:
                pa_copy_blocks_q8(b.k_cache, b.v_cache, b.k_scale, b.v_scale, b.cow_pairs, stream=stream)
            mark(ev, 1)
            pa_reshape_and_cache_q8(b.new_key, b.new_value, b.k_cache, b.v_cache, b.k_scale, b.v_scale,
                                    b.slot_mapping, stream=stream)
            mark(ev, 2)
            if b.partition_size:
                pa_decode_splitk_q8(b.workspace, b.query, b.k_cache, b.v_cache, b.k_scale, b.v_scale, b.block_tables,
                                    b.context_lens, spec.scale, b.max_context_len, b.partition_size,
                                    seq_order=b.seq_order, stream=stream)
                mark(ev, 3)
                pa_splitk_reduce(b.out, b.workspace, b.context_lens, b.max_context_len, b.partition_size,
                                 stream=stream)
            else:
                pa_decode_q8(b.out, b.query, b.k_cache, b.v_cache, b.k_scale, b.v_scale, b.block_tables,
                             b.context_lens, spec.scale, seq_order=b.seq_order, stream=stream)
                mark(ev, 3)
            mark(ev, 4)
            return
        if b.cow_pairs.shape[0]:
            pa_copy_blocks(b.k_cache, b.v_cache, b.cow_pairs, stream=stream)
        mark(ev, 1)
        if b.fused_append:  # slot write and decode in one launch
            mark(ev, 2)
            pa_decode_append(b.out, b.query, b.new_key, b.new_value, b.k_cache, b.v_cache, b.block_tables,
                             b.context_lens, spec.scale, seq_order=b.seq_order, stream=stream)
            mark(ev, 3)
            mark(ev, 4)
            return
        pa_reshape_and_cache(b.new_key, b.new_value, b.k_cache, b.v_cache, b.slot_mapping, stream=stream)
        mark(ev, 2)
        if b.partition_size:
            pa_decode_splitk(b.workspace, b.query, b.k_cache, b.v_cache, b.block_tables, b.context_lens, spec.scale,
                             b.max_context_len, b.partition_size, seq_order=b.seq_order, stream=stream)
            mark(ev, 3)
            pa_splitk_reduce(b.out, b.workspace, b.context_lens, b.max_context_len, b.partition_size,
                             stream=stream)
        else:
            pa_decode(b.out, b.query, b.k_cache, b.v_cache, b.block_tables, b.context_lens, spec.scale,
                      seq_order=b.seq_order, stream=stream)
            mark(ev, 3)
        mark(ev, 4)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(device_index) if sample_clocks else None
    if sampler:
        sampler.start()
    barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop() if sampler else None
    ms = max_over_ranks(t0.elapsed_time(t1), world) / steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        step(evs[i])
    torch.cuda.synchronize()

    def mean(i, j):
        return statistics.fmean(e[i].elapsed_time(e[j]) for e in evs)

    if b.fused_append:
        kernels = {"decode_append": mean(2, 3)}
    else:
        kernels = {"reshape_and_cache": mean(1, 2), "decode": mean(2, 3)}
    if b.cow_pairs.shape[0]:
        kernels["copy_blocks"] = mean(0, 1)
    if b.partition_size:
        kernels["splitk_reduce"] = mean(3, 4)
    return ms, kernels, clocks


def e2e_steps(b, steps: int, warmup: int, world: int):
    """The same step through the public host-buffer API (HostStepPipeline):
    every step copies its inputs from pinned host memory (query, new K/V,
    slots, block tables, context lengths, schedule) and reads its output back
    into pinned memory; copies of neighbouring steps overlap the kernels."""
    from paged_kv_cache_340_b200.batch import HostStepPipeline
    stream = torch.cuda.current_stream()
    pipe = HostStepPipeline(b)
    for _ in range(warmup):
        pipe.step(stream)
    pipe.drain(stream)
    torch.cuda.synchronize()
    barrier(world)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    pipe.start(stream)
    for _ in range(steps):
        pipe.step(stream)
    pipe.drain(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(t0.elapsed_time(t1), world) / steps
    return ms, pipe.h2d_bytes, pipe.d2h_bytes


# ---------------------------------------------------------- CPU oracle legs

class OracleBatch:
    """The oracle's view of a decode workload, built on the host only: the
    seeded inputs and the block tables from the oracle's own pool (same
    free-block order as the library's), never from the CUDA path."""

    def __init__(self, spec, inputs=None):
        import oracle
        from oracle.block_pool import BlockPool as OPool, Sequence, append_tokens
        from paged_kv_cache_340_b200.workloads import make_decode_inputs
        oracle.build()
        self.spec = spec
        self.inputs = inputs if inputs is not None else make_decode_inputs(spec)
        ctx = self.inputs["context_lens"].numpy().astype(np.int32)
        pool = OPool(int(self.inputs["num_blocks"]), spec.block_size, policy="fifo",
                     free_order=self.inputs["free_order"].tolist())
        self.tables = []
        for L in ctx:
            seq = Sequence()
            append_tokens(pool, seq, int(L))
            self.tables.append(np.array(seq.block_table, np.int64))
        self.ctx = ctx


def oracle_sample(ob: OracleBatch, budget_s: float, start_seq: int = 0):
    """Times the oracle (as it stands, single-threaded float64 C) on whole
    sequences of the batch, from start_seq on (cycling through the batch, at
    most 100 passes), until budget_s of oracle time is spent. Returns (bytes,
    seconds, sequences). Widening the inputs to float64 is outside the timed
    calls."""
    import oracle
    spec = ob.spec
    k, v, q = ob.inputs["k_pool"], ob.inputs["v_pool"], ob.inputs["query"]
    tot_bytes, tot_s, n_seq = 0, 0.0, 0
    S = len(ob.ctx)
    s = start_seq
    while tot_s < budget_s and n_seq < 100 * S:
        i = s % S
        L = int(ob.ctx[i])
        ids = torch.from_numpy(ob.tables[i])
        kp = k.index_select(0, ids).double().numpy()
        vp = v.index_select(0, ids).double().numpy()
        qs = q[i:i + 1].double().numpy()
        tab = np.arange(max(len(ids), 1), dtype=np.int32)[None, :]
        t = time.perf_counter()
        oracle.paged_decode(qs, kp, vp, tab, np.array([L], np.int32), spec.scale, spec.block_size)
        tot_s += time.perf_counter() - t
        tot_bytes += decode_bytes(spec, np.array([L]))
        n_seq += 1
        s += 1
    return tot_bytes, tot_s, n_seq


def host_cores() -> int:
    """Cores this process may run on (nproc)."""
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def oracle_sample_parallel(ob: OracleBatch, budget_s: float, threads: int):
    """The same oracle, as it stands, on `threads` host threads at once, each
    over its own whole sequences of the batch (the C call runs without the
    Python lock, so the threads run in parallel), until each thread has spent
    budget_s of oracle time. Returns (bytes per second summed over the
    threads, sequences, wall seconds)."""
    import threading
    res = [None] * threads
    prev = torch.get_num_threads()
    torch.set_num_threads(1)  # the per-sequence widening stays on its own thread

    def work(i):
        res[i] = oracle_sample(ob, budget_s, start_seq=(i * 13) % len(ob.ctx))

    t = time.perf_counter()
    ths = [threading.Thread(target=work, args=(i,)) for i in range(threads)]
    for th in ths:
        th.start()
    for th in ths:
        th.join()
    wall = time.perf_counter() - t
    torch.set_num_threads(prev)
    return sum(b / sec for b, sec, _ in res), sum(n for _, _, n in res), wall


def run_reference(args, world, rank):
    """Reference arm: the CPU oracle, timed on the host cores, on the same
    workload, metric and unit. Rank 0 only; no GPU is used."""
    if rank != 0:
        return
    from paged_kv_cache_340_b200.workloads import SPECS
    spec = SPECS[args.workload]
    if spec.lengths[0] == "parallel":
        raise SystemExit("the reference arm times the decode-only workloads")
    ob = OracleBatch(spec)
    budget = max(0.002, min(2.0, 90.0 / max(1, args.steps + args.warmup)))
    for i in range(args.warmup):
        oracle_sample(ob, budget / 4, start_seq=i)
    tot_b, tot_s, seqs = 0, 0.0, 0
    for i in range(args.steps):
        nb_, ns_, nq_ = oracle_sample(ob, budget, start_seq=i)
        tot_b += nb_
        tot_s += ns_
        seqs += nq_
    gbs = tot_b / tot_s / 1e9
    sample = (f"{seqs} whole sequences (all {spec.num_heads} heads each) of the {spec.name} batch over "
              f"{args.steps} steps, about {budget:.3g} s of oracle time per step; float64 C, one thread")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * tot_s / max(1, args.steps), 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": spec.name, "num_seqs": spec.num_seqs, "num_heads": spec.num_heads,
                   "num_kv_heads": spec.num_kv_heads, "head_dim": spec.head_dim, "block_size": spec.block_size,
                   "kv_dtype": spec.kv_dtype},
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": 1, "host_cores": host_cores(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def kernel_lines(spec, b, kern: dict, by: dict) -> dict:
    """Per kernel of the step: mean launch time and algorithmic GB/s."""
    nbytes = {"decode": by["decode"], "reshape_and_cache": by["write"], "copy_blocks": by["copy"],
              "decode_append": by["decode"] + by["write"]}
    if b.partition_size:
        parts = ((b.host_context_lens.astype(np.int64) + b.partition_size - 1) // b.partition_size).sum()
        nbytes["splitk_reduce"] = int(parts) * spec.num_heads * (spec.head_dim + 2) * 4 + \
            len(b.host_context_lens) * spec.num_heads * spec.head_dim * elt(spec.torch_out_dtype)
    return {k: {"ms": round(v, 5), "GBps": round(nbytes[k] / v / 1e6, 1)} for k, v in kern.items()}


def tensor_peak():
    """Measured dense bf16 tensor throughput (TFLOP/s), burst figure."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def measure_prefill(name: str, steps: int, warmup: int):
    """Prefill step (slot write of the new tokens + causal paged attention):
    TFLOP/s of the attention kernel against the bf16 tensor peak."""
    from paged_kv_cache_340_b200 import pa_prefill, pa_reshape_and_cache
    from paged_kv_cache_340_b200.batch import build_prefill_batch, prefill_flops
    from paged_kv_cache_340_b200.workloads import SPECS, make_prefill_inputs
    spec = SPECS[name]
    b = build_prefill_batch(spec, make_prefill_inputs(spec))
    stream = torch.cuda.current_stream()
    flops = prefill_flops(spec, b.host_context_lens)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        pa_reshape_and_cache(b.new_key, b.new_value, b.k_cache, b.v_cache, b.slot_mapping, stream=stream)
        if ev:
            ev[1].record(stream)
        pa_prefill(b.out, b.query, b.q_start, b.max_q_len, b.k_cache, b.v_cache, b.block_tables, b.context_lens,
                   spec.scale, stream=stream)
        if ev:
            ev[2].record(stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    for i in range(steps):
        step(evs[i])
    torch.cuda.synchronize()
    att = statistics.fmean(e[1].elapsed_time(e[2]) for e in evs)
    wr = statistics.fmean(e[0].elapsed_time(e[1]) for e in evs)
    peak, kind = tensor_peak()
    tf = flops / (att * 1e-3) / 1e12
    res = {"prefill_kernel_ms": round(att, 4), "TFLOPs": round(tf, 1), "tensor_peak": peak, "peak_kind": kind,
           "frac_of_tensor_peak": round(tf / peak, 3), "flops_per_step": flops,
           "slot_write_ms": round(wr, 4), "new_tokens": int(b.host_slots.shape[0]),
           "tokens_per_s": round(b.host_slots.shape[0] / ((att + wr) * 1e-3), 1)}
    del b
    torch.cuda.empty_cache()
    return res


def event_floor_ms(stream, reps: int = 50):
    """Event-to-event time (median, ms) of an empty kernel between two events
    inside a CUDA graph, the arrangement the beam step's per-kernel times are
    read in: the part of such a time any kernel there pays. The empty kernel
    is PyTorch's spin kernel with a zero-cycle spin (not this library's).
    None if it cannot be measured."""
    try:
        ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            torch.cuda._sleep(0)
            torch.cuda.synchronize()
            with torch.cuda.graph(g, stream=stream):
                ev[0].record(stream)
                torch.cuda._sleep(0)
                ev[1].record(stream)
        xs = []
        for _ in range(reps):
            g.replay()
            torch.cuda.synchronize()
            xs.append(ev[0].elapsed_time(ev[1]))
        del g
        return statistics.median(xs)
    except Exception:  # a measurement aid only
        return None


def measure_beam(name: str, steps: int, warmup: int, host_steps: int = 30):
    """Beam-search decode steps with the beam step on the device (beam step,
    counted copy, slot write, decode; no host round trip), each step replayed
    as a CUDA graph; and for context the same steps through the host pool,
    where each step must read the beams' parents back (a synchronisation) and
    upload tables, slots and pairs."""
    from paged_kv_cache_340_b200 import pa_copy_blocks, pa_decode_append
    from paged_kv_cache_340_b200.batch import beam_decode_bytes, build_beam_batch, host_beam_step, run_beam_step
    from paged_kv_cache_340_b200.workloads import SPECS, make_beam_inputs
    spec = SPECS[name]
    b = build_beam_batch(spec, make_beam_inputs(spec))
    G = b.parents.shape[0]                               # distinct steps; graph k runs step k (mod G)
    warmup = -(-warmup // G) * G
    steps = min(steps, spec.max_divergent - warmup - host_steps - 3 * G - 12)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            run_beam_step(b, stream=stream)
    torch.cuda.synchronize()
    # one graph per distinct step, each with events between its launches
    graphs, evs = [], []
    with torch.cuda.stream(stream):
        for k in range(G):
            ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(5)]  # recorded on replay
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                run_beam_step(b, stream=stream, events=ev)
            graphs.append(g)
            evs.append(ev)
    b.steps_done -= G                                    # capturing ran nothing
    first = b.steps_done
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record(stream)
        for _ in range(steps):
            graphs[b.steps_done % G].replay()
            b.steps_done += 1
        t1.record(stream)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    by = statistics.fmean(beam_decode_bytes(b, first + i) for i in range(steps))
    # per-kernel times: replay each graph alone and read its own events
    samples = []
    with torch.cuda.stream(stream):
        while b.steps_done % G:
            graphs[b.steps_done % G].replay()
            b.steps_done += 1
        for _ in range(2):
            for k in range(G):
                graphs[k].replay()
                b.steps_done += 1
                torch.cuda.synchronize()
                e = evs[k]
                samples.append([e[i].elapsed_time(e[i + 1]) for i in range(4)])
    kern = [statistics.fmean(x[i] for x in samples) for i in range(4)]
    dec_by = statistics.fmean(beam_decode_bytes(b, b.steps_done - 1 - i) for i in range(len(samples)))
    # the wall time of one step when the host waits for its result
    wall = []
    with torch.cuda.stream(stream):
        for _ in range(12):
            t = time.perf_counter()
            graphs[b.steps_done % G].replay()
            b.steps_done += 1
            stream.synchronize()
            wall.append(time.perf_counter() - t)
    del graphs
    # host-pool path over the same kind of steps, from the state the device has now
    W = b.tables[0].shape[0]
    cur = b.steps_done % 2
    tables = b.tables[cur].cpu().numpy()
    ctx = b.context_lens[cur].cpu().numpy()
    from paged_kv_cache_340_b200 import BlockPool
    ref, fl = b.pool.ref.cpu().numpy(), b.pool.free_list()
    hp = BlockPool(b.num_blocks, spec.block_size, b.pool.policy, free_order=np.arange(b.num_blocks, dtype=np.int32))
    for _ in range(b.num_blocks):
        hp.allocate()
    for blk in range(b.num_blocks):
        for _ in range(int(ref[blk]) - 1):
            hp.share(blk)
    for blk in fl:
        hp.free(int(blk))
    dt_tab = torch.empty_like(b.tables[0])
    dt_ctx = torch.empty_like(b.context_lens[0])
    dt_slots = torch.empty_like(b.slot_mapping)
    host = []
    for i in range(host_steps):
        t = time.perf_counter()
        k = (b.steps_done + i) % G
        parents = b.parents[k].cpu().numpy()             # read back: a synchronisation
        tables, ctx, slots, cow = host_beam_step(hp, tables, ctx, parents)
        dt_tab.copy_(torch.from_numpy(tables))
        dt_ctx.copy_(torch.from_numpy(ctx))
        dt_slots.copy_(torch.from_numpy(slots))
        if cow.shape[0]:
            pa_copy_blocks(b.k_cache, b.v_cache, torch.from_numpy(cow).cuda())
        pa_decode_append(b.out, b.query[k], b.new_key[k], b.new_value[k], b.k_cache, b.v_cache, dt_tab, dt_ctx,
                         spec.scale)
        torch.cuda.synchronize()
        host.append(time.perf_counter() - t)
    floor = event_floor_ms(stream)  # what an empty kernel measures between two events in a graph
    res = {"ms_per_step": round(ms, 4), "beams": W, "steps_timed": steps, "launch": "one CUDA graph per step",
           "decode_kernel_ms": round(kern[3], 4), "decode_GBps_logical": round(dec_by / kern[3] / 1e6, 1),
           "step_GBps_logical": round(by / ms / 1e6, 1),
           "kernels_ms": {"beam_step": round(kern[0], 5), "copy_blocks_counted": round(kern[1], 5),
                          "decode_append": round(kern[3], 5)},
           "event_floor_ms": None if floor is None else round(floor, 5),
           "device_path_wall_ms_with_sync": round(1e3 * statistics.median(wall), 4),
           "host_pool_path_wall_ms": round(1e3 * statistics.median(host), 4),
           "note": "decode bytes are logical: beams of a prompt share their prefix blocks (read from L2)"}
    del b
    torch.cuda.empty_cache()
    return res


def decode_kernel_of(b, by: dict):
    """The step's decode kernel: its name in the kernel timings and the
    algorithmic bytes it moves (the fused form also does the slot write)."""
    if b.fused_append:
        return "decode_append", by["decode"] + by["write"]
    return "decode", by["decode"]


def measure_other(name: str, steps: int, warmup: int):
    spec, b = build_batch(name, 0)
    ms, kern, _ = time_steps(b, steps, warmup, 1)
    by = step_bytes(spec, b)
    peak, _ = peaks()
    dname, dbytes = decode_kernel_of(b, by)
    dec = kern[dname]
    res = {"ms_per_step": round(ms, 4), "GBps": round(by["total"] / ms / 1e6, 1),
           "pct_of_hbm_peak": round(100 * by["total"] / ms / 1e6 / peak, 1),
           "decode_kernel_ms": round(dec, 4), "decode_kernel_GBps": round(dbytes / dec / 1e6, 1),
           "partition_size": b.partition_size, "seq_tokens_per_s": round(spec.num_seqs / ms * 1e3, 1),
           "context_tokens_per_s": round(float(b.host_context_lens.sum()) / ms * 1e3, 1),
           "kernels": kernel_lines(spec, b, kern, by)}
    if spec.lengths[0] in ("parallel", "prefix"):  # shared prefix blocks: logical and distinct bytes
        uniq = unique_kv_bytes(spec, b.host_tables, b.host_context_lens)
        logical = int(b.host_context_lens.astype(np.int64).sum()) * 2 * spec.num_kv_heads * kv_row_bytes(spec)
        res["kv_bytes_logical"] = logical
        res["kv_bytes_unique"] = uniq
        res["decode_kernel_GBps_unique_kv"] = round(uniq / dec / 1e6, 1)
        res["note"] = "GBps counts logical bytes: sequences sharing a prefix each read its blocks (L2 hits)"
    del b
    torch.cuda.empty_cache()
    return res


def run_dry(args, world: int, rank: int) -> None:
    """The multi-rank plumbing with no GPU work: each rank takes its own
    workload seed, warms up and times K empty steps between barriers, and the
    job's time is the slowest rank's. Rank 0 prints one line listing every
    rank it heard from (a CPU test of the --gpus N launch)."""
    from paged_kv_cache_340_b200.workloads import SPECS
    spec = pdist.rank_spec(SPECS[args.workload], rank)
    for _ in range(args.warmup):
        barrier(world)
    barrier(world)
    t = time.perf_counter()
    for _ in range(args.steps):
        barrier(world)
    ms = max_over_ranks(1e3 * (time.perf_counter() - t), world) / max(1, args.steps)
    ranks = [None] * world
    if world > 1:
        torch.distributed.all_gather_object(ranks, {"rank": rank, "seed": spec.seed, "pid": os.getpid()})
    else:
        ranks = [{"rank": rank, "seed": spec.seed, "pid": os.getpid()}]
    if rank == 0:
        print(json.dumps({"dry_run": True, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                          "ms_per_step": round(ms, 5), "backend": args.backend, "ranks": ranks,
                          "config": {"workload": spec.name}}), flush=True)
    pdist.finalize(world)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--partition", type=int, default=None, help="force a split-K partition size (0 = unsplit)")
    ap.add_argument("--no-others", action="store_true", help="skip the other workloads' lines")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--backend", default="nccl", choices=["nccl", "gloo"],
                    help="process-group backend (gloo only with --dry-run)")
    ap.add_argument("--dry-run", action="store_true",
                    help="start the ranks and run the barriers and max-over-ranks timing, no GPU work")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    if args.backend == "gloo" and not args.dry_run:
        raise SystemExit("--backend gloo is for --dry-run (the GPU path uses nccl)")
    if args.impl == "reference":
        # The reference arm runs on the host: rank 0 alone, no process group.
        world, rank, _ = pdist.env_ranks()
        run_reference(args, world, rank)
        return
    launch_ranks(args)  # --gpus N > 1 without a launcher: starts N ranks and exits
    if args.dry_run:
        world, rank, _ = dist_setup(args.gpus, args.backend)
        run_dry(args, world, rank)
        return
    world, rank, local = dist_setup(args.gpus)
    import paged_kv_cache_340_b200 as pa  # noqa: F401  (fails loudly without the CUDA library)

    from paged_kv_cache_340_b200.workloads import SPECS as _SPECS
    if _SPECS[args.workload].branches and _SPECS[args.workload].num_prompts and args.workload.startswith("beam"):
        if rank == 0:
            print(json.dumps({"workload": args.workload, "beam": measure_beam(args.workload, args.steps,
                                                                              args.warmup)}), flush=True)
        pdist.finalize(world)
        return
    if _SPECS[args.workload].q_len:
        if rank == 0:
            print(json.dumps({"workload": args.workload, "prefill": measure_prefill(args.workload, args.steps,
                                                                                    args.warmup)}), flush=True)
        pdist.finalize(world)
        return
    spec, b = build_batch(args.workload, rank, args.partition)
    ms, kern, clocks = time_steps(b, args.steps, args.warmup, world, sample_clocks=(rank == 0),
                                  device_index=local)
    by = step_bytes(spec, b)
    dname, dbytes = decode_kernel_of(b, by)
    dec_ms = kern[dname]
    peak, peak_kind = peaks()
    value = pdist.job_throughput(by["total"], ms, world)
    e2e_ms, h2d, d2h = e2e_steps(b, max(10, args.steps // 4), args.warmup, world)
    kernel = "pa_decode_splitk" if b.partition_size else ("pa_decode_append" if b.fused_append else "pa_decode")
    achieved = dbytes / (dec_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": spec.kv_dtype, "data": "synthetic",
        "config": {"workload": spec.name, "num_seqs": spec.num_seqs, "num_heads": spec.num_heads,
                   "num_kv_heads": spec.num_kv_heads, "head_dim": spec.head_dim, "block_size": spec.block_size,
                   "context_lens": "U{256..2048}" if spec.name == DEFAULT_WORKLOAD else str(spec.lengths),
                   "kv_dtype": spec.kv_dtype, "out_dtype": spec.out_dtype, "partition_size": b.partition_size,
                   "parallelism": f"dp{world} (sequences shard, no exchange)",
                   "l2": f"inputs larger than L2 (decode reads {by['decode'] / 1e9:.3f} GB per step, L2 126 MB), no flush",
                   "step": ("copy_blocks (if any) + decode_append (slot write of each sequence's newest token "
                            "and decode, one launch)" if b.fused_append else
                            "copy_blocks (if any) + reshape_and_cache + decode")},
        "pct_of_hbm_peak": round(100 * value / world / peak, 2),
        "seq_tokens_per_s": round(world * spec.num_seqs / (ms * 1e-3), 1),
        "context_tokens_per_s": round(world * float(b.host_context_lens.sum()) / (ms * 1e-3), 1),
        "bytes_per_step": by,
        "e2e": {"value": round(pdist.job_throughput(by["total"], e2e_ms, world), 2), "unit": "GB/s",
                "ms_per_step": round(e2e_ms, 5), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "roofline": {"bound": "hbm", "kernel": kernel, "achieved": round(achieved, 1), "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "kernel_ms": round(dec_ms, 5),
                     "traffic": recorded_traffic(spec.name, kernel)},
        "gpu_launches": launches_per_step(b) * args.steps,
        "clocks": clocks,
    }
    line["kernels"] = kernel_lines(spec, b, kern, by)
    if world == 1 and rank == 0 and not args.no_cpu_baseline and "k_pool" in b.host_inputs and \
            spec.kv_dtype != "i8":  # the sampled oracle leg is the 16/32-bit decode
        ob = OracleBatch(spec, b.host_inputs)
        nbytes, secs, nseq = oracle_sample(ob, 12.0)
        ncores = host_cores()
        line["cpu_baseline"] = {"value": round(nbytes / secs / 1e9, 4), "unit": "GB/s", "cores": 1,
                                "host_cores": ncores, "kind": "oracle",
                                "sample": f"{nseq} sequences (all heads; {nseq / spec.num_seqs:.1f} passes over the "
                                          f"{spec.num_seqs}-sequence batch), decode only; float64 C oracle, "
                                          f"one thread of {ncores} host cores, {secs:.1f} s"}
        nth = min(ncores, 128)
        rate, nseq_p, wall = oracle_sample_parallel(ob, 4.0, nth)
        line["cpu_baseline_all_cores"] = {
            "value": round(rate / 1e9, 4), "unit": "GB/s", "cores": nth, "host_cores": ncores, "kind": "oracle",
            "sample": f"{nseq_p} whole sequences of the same batch on {nth} threads at once (each over its own "
                      f"sequences, 4 s of oracle time per thread, {wall:.1f} s wall); value = sum of the "
                      f"threads' rates; the same float64 C oracle, unchanged"}
    del b
    torch.cuda.empty_cache()
    if world == 1 and not args.no_others and args.workload == DEFAULT_WORKLOAD:
        line["other_workloads"] = {n: measure_other(n, 200, 10) for n in
                                   ("gqa_bf16", "long_splitk_bf16", "parallel_sampling_fp16", "prefix_cache_fp16",
                                    "llama7b_mha_int8", "gqa_int8")}
        line["prefill_workloads"] = {n: measure_prefill(n, 20, 3) for n in
                                     ("prefill_llama7b_mha_bf16", "chunked_prefill_gqa_bf16")}
        line["beam_search_fp16"] = measure_beam("beam_search_fp16", 200, 10)
    if rank == 0:
        print(json.dumps(line), flush=True)
    pdist.finalize(world)


if __name__ == "__main__":
    main()

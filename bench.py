"""Benchmark of the paged-KV attention hot path on B200.

Default workload: one decode step at batch 512 with prefix sharing (lognormal context
lengths, median 1024, clipped to [16, 4096]; half the sequences share a 1024-token prefix
held in 4 physical blocks; 16 query / 8 KV heads, head_dim 128, block size 256, bf16).
A step stores the 512 new tokens' K/V rows and runs paged decode attention over the
contexts that include them, in one call: nvpa_decode_step_shared_prefix by default (the
shared prefix is attended once for its group on the tensor cores), nvpa_decode_step with
--decode-api plain.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl nvpa|reference]
                    [--workload NAME]

With --gpus N > 1 and no launcher, bench.py starts N ranks itself (torch.distributed.run
on 127.0.0.1); under a launcher, N must equal WORLD_SIZE or the run stops with an error.

Prints one JSON line.  `value` is the achieved HBM bandwidth of the whole step in GB/s,
counting each unique cached K/V row once (plus q, out, the new rows and the index
arrays); `seq_steps_per_s` is batch / step time.  Under torchrun (N > 1) every rank runs
its own batch (weak scaling, no collective on the data path); the time is the maximum
over ranks.  `--impl reference` times the CPU oracle on a bounded sample instead.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "paged decode attn: achieved HBM GB/s (% of peak), seq-steps/s at batch 512"
DEFAULT_WORKLOAD = "decode_b512_shared_prefix"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
CLOCK_QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
               "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
               "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


# ----------------------------------------------------------------------------------
# algorithmic work (bytes / flops) of a step, from the workload's metadata
# ----------------------------------------------------------------------------------

def decode_step_bytes(step) -> dict:
    """Algorithmic HBM bytes of one decode step (store + attention).

    Each physical (block, row) that holds a live token is read once per KV head for K and
    for V, even when several sequences share it; q is read and out written once; the
    store reads the new K/V rows and writes them; index arrays are read once.
    """
    bs, hkv, d = step.block_size, step.num_kv_heads, step.head_dim
    used = {}
    for b in range(step.batch):
        L = int(step.context_lens[b])
        for j in range((L + bs - 1) // bs):
            blk = int(step.block_tables[b, j])
            used[blk] = max(used.get(blk, 0), min(bs, L - j * bs))
    unique_rows = sum(used.values())
    kv = unique_rows * hkv * d * 2 * 2
    logical_kv = int(step.context_lens.sum()) * hkv * d * 2 * 2
    qo = 2 * step.batch * step.num_q_heads * d * 2
    n_real = int((step.slot_mapping >= 0).sum())
    store = 2 * n_real * hkv * d * 2 * 2 + step.num_tokens * 4
    tables = sum((int(L) + bs - 1) // bs for L in step.context_lens) * 4 + step.batch * 4
    return dict(kv_unique=kv, kv_logical=logical_kv, attention=kv + qo + tables,
                store=store, step=kv + qo + tables + store)


def prefill_step_work(step) -> dict:
    d, hq, hkv = step.head_dim, step.num_q_heads, step.num_kv_heads
    flops = 0
    for i in range(step.batch):
        lq = int(step.cu_seqlens_q[i + 1] - step.cu_seqlens_q[i])
        lk = int(step.cu_seqlens_k[i + 1] - step.cu_seqlens_k[i])
        # query r sees lk - lq + r + 1 keys; QK^T and PV are 2*d flops per (query, key) each
        flops += 4 * d * hq * (lq * (lk - lq) + lq * (lq + 1) // 2)
    store = 2 * step.total_q * hkv * d * 2 * 2 + step.total_q * 4
    return dict(flops=flops, store=store)


# ----------------------------------------------------------------------------------
# environment helpers
# ----------------------------------------------------------------------------------

def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16_tflops=float(p["bf16_tflops"]),
                    bf16_tflops_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                    source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm_gbs=FALLBACK_HBM_GBS, bf16_tflops=FALLBACK_BF16_TFLOPS,
                    bf16_tflops_sustained=1400.0, source="fallback")


def peak_source(peaks: dict, key: str, what: str) -> str:
    """Where a roofline denominator came from, for the JSON line."""
    if peaks["source"] == "measured":
        return f"measured: MEASURED_PEAKS.json {key} ({what})"
    return (f"fallback: MEASURED_PEAKS.json absent; an earlier measurement of the same "
            f"quantity ({what}) on this kind of B200: {peaks[key]:g}")


class ClockSampler:
    """nvidia-smi clock/throttle samples taken while the timed region runs."""

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"nvpa_bench_clocks_{os.getpid()}_{index}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={CLOCK_QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self) -> dict:
        if self.proc is None or not os.path.exists(self.path):
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=["nvidia-smi unavailable"])
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return dict(sm_mhz=None, sm_max_mhz=smax, reasons=["no samples"])
        busy = sorted(sm)[len(sm) // 4:] or sm   # drop idle samples at the edges
        return dict(sm_mhz=float(np.median(busy)), sm_max_mhz=smax, reasons=sorted(reasons),
                    samples=len(sm))


def profile_traffic(kernel_tag: str, source_files) -> float | None:
    """DRAM bytes per launch recorded in profiles/ for this kernel, if the kernel's source
    is unchanged since the capture (the summary stores a hash of its sources)."""
    path = os.path.join(ROOT, "profiles", f"{kernel_tag}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    h = re.search(r"source_sha256:\s*([0-9a-f]{16,64})", text)
    if not m or not h:
        return None
    digest = hashlib.sha256()
    for f in source_files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            digest.update(fh.read())
    if not digest.hexdigest().startswith(h.group(1)):
        return None
    return float(m.group(1))


# sources of the split-KV worker, the dominant kernel of a decode step
DECODE_SOURCES = ["paged_kv_cache_422_b200/csrc/paged_attention.cu",
                  "paged_kv_cache_422_b200/csrc/decode_params.cuh",
                  "paged_kv_cache_422_b200/csrc/attn_warp.cuh",
                  "paged_kv_cache_422_b200/csrc/common.cuh"]


# sources of the tcgen05 attention kernel, the dominant kernel of a prefill step
PREFILL_SOURCES = ["paged_kv_cache_422_b200/csrc/prefill_tcgen05.cu",
                   "paged_kv_cache_422_b200/csrc/sm100.cuh",
                   "paged_kv_cache_422_b200/csrc/attn_warp.cuh",
                   "paged_kv_cache_422_b200/csrc/common.cuh"]


def source_sha(files) -> str:
    digest = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            digest.update(fh.read())
    return digest.hexdigest()


# ----------------------------------------------------------------------------------
# distributed plumbing (also exercised by the gloo tests)
# ----------------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def launch_plan(gpus: int, env=None):
    """How this process honours `--gpus N`.

    Returns "run" when the process is one of the job's ranks and the job has N of them,
    "spawn" when N > 1 and no launcher started the process (bench.py then starts N ranks
    itself through torch.distributed.run); raises ValueError when a launcher's WORLD_SIZE
    disagrees with N, so that a run never reports a GPU count it did not use.
    """
    env = os.environ if env is None else env
    if gpus < 1:
        raise ValueError(f"--gpus must be >= 1, got {gpus}")
    if "WORLD_SIZE" in env:
        world = int(env["WORLD_SIZE"])
        if world != gpus:
            raise ValueError(f"--gpus {gpus} but the launcher started {world} rank(s) "
                             f"(WORLD_SIZE={world}); pass matching values")
        return "run"
    return "spawn" if gpus > 1 else "run"


def spawn_command(gpus: int, argv, port: int):
    """The torch.distributed.run command line that starts `gpus` ranks of this script."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={gpus}", "--master-addr", "127.0.0.1", "--master-port", str(port),
            os.path.abspath(__file__)] + list(argv)


def _free_port() -> int:
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank float over the process group (identity with one process)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ----------------------------------------------------------------------------------
# CPU oracle (reference arm and cpu_baseline)
# ----------------------------------------------------------------------------------

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


def oracle_decode_sample(step, seqs):
    """Run the CPU oracle's decode over a sample of sequences; returns (seconds, bytes)."""
    import oracle
    t0 = time.perf_counter()
    oracle.paged_decode_attention(step.q[seqs], step._ora_k, step._ora_v, step.block_tables[seqs],
                                  step.context_lens[seqs], step.scale)
    dt = time.perf_counter() - t0
    # the sample's share of the step's algorithmic bytes, in proportion to context length
    share = float(step.context_lens[seqs].sum()) / float(step.context_lens.sum())
    return dt, step._bytes["step"] * share


def prepare_oracle(step):
    import oracle
    step.__dict__.setdefault("_bytes", decode_step_bytes(step))
    kc, vc = step.k_pool.copy(), step.v_pool.copy()
    oracle.store_kvcache(kc, vc, step.k_new, step.v_new, step.slot_mapping)
    step._ora_k, step._ora_v = kc, vc


def effective_cores(cpu_s: float, wall_s: float) -> int:
    """Host cores a run kept busy on average: process CPU time (all threads) / wall time."""
    return max(1, int(round(cpu_s / wall_s))) if wall_s > 0 else 1


def single_thread():
    """Context that limits the BLAS pools to one thread (the 1-thread CPU baseline)."""
    from threadpoolctl import threadpool_limits
    return threadpool_limits(limits=1)


def _decode_cpu_run(step, budget_s):
    order = np.random.default_rng(0).permutation(step.batch)
    tot_t, tot_b, n = 0.0, 0, 0
    c0, w0 = time.process_time(), time.perf_counter()
    while n < step.batch and tot_t < budget_s:
        dt, nb = oracle_decode_sample(step, order[n:n + 4])
        tot_t += dt
        tot_b += nb
        n += len(order[n:n + 4])
    cores = effective_cores(time.process_time() - c0, time.perf_counter() - w0)
    return tot_t, tot_b, n, cores


def cpu_baseline(step, budget_s: float = 8.0) -> dict:
    """The oracle on as many whole sequences (in a fixed shuffled order) as fit in about
    budget_s seconds, with the host's BLAS threads and again with one thread; GB/s counts
    each sampled sequence's K/V bytes.  `cores` is the average number of host cores the
    run kept busy (process CPU time / wall time), not the size of the thread pool."""
    prepare_oracle(step)
    tot_t, tot_b, n, cores = _decode_cpu_run(step, budget_s)
    with single_thread():
        t1, b1, n1, _ = _decode_cpu_run(step, budget_s)
    return dict(value=tot_b / tot_t / 1e9, unit="GB/s", cores=cores, kind="oracle",
                blas_threads=blas_threads(),
                sample=f"{n} of {step.batch} sequences (fixed shuffled order), float64 numpy, "
                       f"{tot_t:.1f} s; seq-steps/s {n / tot_t:.3f}",
                single_thread=dict(value=b1 / t1 / 1e9, unit="GB/s", cores=1,
                                   sample=f"{n1} sequences, {t1:.1f} s, BLAS limited to 1 thread"))


def prefill_cpu_baseline(step, budget_s: float = 8.0) -> dict:
    """The oracle's varlen prefill on as many whole sequences (in a fixed shuffled order) as
    fit in about budget_s seconds, with the host's BLAS threads and again with one thread;
    TFLOP/s counts the sample's algorithmic causal FLOPs.  `cores` as in cpu_baseline."""
    import oracle
    kc, vc = step.k_pool.copy(), step.v_pool.copy()
    oracle.store_kvcache(kc, vc, step.k_new, step.v_new, step.slot_mapping)
    tot_t, tot_f, n, cores = _prefill_cpu_run(step, kc, vc, budget_s)
    with single_thread():
        t1, f1, n1, _ = _prefill_cpu_run(step, kc, vc, budget_s)
    return dict(value=tot_f / tot_t / 1e12, unit="TFLOP/s", cores=cores, kind="oracle",
                blas_threads=blas_threads(),
                sample=f"{n} of {step.batch} sequences (fixed shuffled order), float64 numpy, "
                       f"{tot_t:.1f} s",
                single_thread=dict(value=f1 / t1 / 1e12, unit="TFLOP/s", cores=1,
                                   sample=f"{n1} sequences, {t1:.1f} s, BLAS limited to 1 thread"))


def _prefill_cpu_run(step, kc, vc, budget_s):
    import oracle
    d, hq = step.head_dim, step.num_q_heads
    order = np.random.default_rng(0).permutation(step.batch)
    tot_t, tot_f, n = 0.0, 0, 0
    c0, w0 = time.process_time(), time.perf_counter()
    while n < step.batch and tot_t < budget_s:
        i = int(order[n])
        q0, q1 = int(step.cu_seqlens_q[i]), int(step.cu_seqlens_q[i + 1])
        lq, lk = q1 - q0, int(step.cu_seqlens_k[i + 1] - step.cu_seqlens_k[i])
        t0 = time.perf_counter()
        oracle.varlen_prefill_attention(step.q[q0:q1], kc, vc, step.block_tables[i:i + 1],
                                        np.array([0, lq], np.int32), np.array([0, lk], np.int32),
                                        step.scale)
        tot_t += time.perf_counter() - t0
        tot_f += 4 * d * hq * (lq * (lk - lq) + lq * (lq + 1) // 2)
        n += 1
    return tot_t, tot_f, n, effective_cores(time.process_time() - c0, time.perf_counter() - w0)


def run_reference(args) -> int:
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    from synth import WORKLOADS
    step = WORKLOADS[args.workload]()
    prepare_oracle(step)
    order = np.random.default_rng(0).permutation(step.batch)
    per_step = 4
    times, nbytes = [], []
    cpu_used = 0.0
    for i in range(args.warmup + args.steps):
        seqs = order[(i * per_step) % step.batch:][:per_step]
        c0 = time.process_time()
        dt, nb = oracle_decode_sample(step, seqs)
        if i >= args.warmup:
            times.append(dt)
            nbytes.append(nb)
            cpu_used += time.process_time() - c0
    t = float(np.sum(times))
    value = float(np.sum(nbytes)) / t / 1e9
    cores = effective_cores(cpu_used, t)
    line = dict(metric=METRIC, value=value, unit="GB/s", n_gpus=args.gpus, steps=args.steps,
                warmup=args.warmup, ms_per_step=t / args.steps * 1e3, higher_is_better=True,
                scaling="weak", vs_baseline=None, dtype="f64", data="synthetic",
                impl="reference",
                config=dict(workload=args.workload, sample_sequences_per_step=per_step),
                cpu_baseline=dict(value=value, unit="GB/s", cores=cores, kind="oracle",
                                  sample=f"{per_step} sequences of {step.batch} per step"),
                e2e=dict(value=value, unit="GB/s", h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------------
# the GPU arm
# ----------------------------------------------------------------------------------

L2_FLUSHED = "flushed: a 512 MB buffer written and read back before every step, outside its events"


def make_l2_flush(dev, enabled: bool):
    """A function that evicts the 126 MB L2 on `stream` (between timed steps, outside their
    events), or None when flushing is off: it writes a 512 MB buffer, then reads it back,
    so that L2 ends up holding clean lines of that buffer; after the write alone L2 would
    be full of dirty lines, and the next step would pay for writing them back to DRAM
    inside its own events."""
    if not enabled:
        return None
    import torch
    buf = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    words = buf.view(torch.int32)
    res = torch.empty((), dtype=torch.int32, device=dev)

    def flush(stream):
        with torch.cuda.stream(stream):
            buf.fill_(1)
            torch.amax(words, dim=0, out=res)
    return flush


class PackedInputs:
    """A step's input tensors laid out back to back (256-byte aligned) in one pinned host
    buffer and in one device buffer of the same layout, so that a single cudaMemcpyAsync
    moves all of a step's inputs; `views` are device tensors with the original shapes and
    dtypes inside the device buffer."""

    def __init__(self, tensors: dict, dev):
        import torch
        offs, off = {}, 0
        for k, v in tensors.items():
            nb = v.numel() * v.element_size()
            offs[k] = (off, nb)
            off = (off + nb + 255) // 256 * 256
        self.host = torch.empty(off, dtype=torch.uint8).pin_memory()
        self.device = torch.empty(off, dtype=torch.uint8, device=dev)
        self.views = {}
        for k, v in tensors.items():
            o, nb = offs[k]
            self.host[o:o + nb].copy_(v.detach().contiguous().reshape(-1).view(torch.uint8).cpu())
            self.views[k] = self.device[o:o + nb].view(v.dtype).view(v.shape)
        self.nbytes = off

    def upload(self, stream):
        import torch
        with torch.cuda.stream(stream):
            self.device.copy_(self.host, non_blocking=True)

    def twin(self) -> "PackedInputs":
        """A second device buffer of the same layout, filled from the same host buffer."""
        import torch
        t = object.__new__(PackedInputs)
        t.host, t.nbytes = self.host, self.nbytes
        t.device = torch.empty_like(self.device)
        base = self.device.data_ptr()
        t.views = {}
        for k, v in self.views.items():
            o = v.data_ptr() - base
            nb = v.numel() * v.element_size()
            t.views[k] = t.device[o:o + nb].view(v.dtype).view(v.shape)
        return t


E2E_COPIES = ("every step: one packed host-to-device copy of all its inputs from pinned memory and "
              "a device-to-host copy of its output, both inside the timed region; triple-buffered "
              "so that the next steps' uploads and the previous step's read-back overlap step i's "
              "kernels")


def end_to_end(run_step, packed, out, stream, steps, warmup, dev):
    """Steps with host inputs and a host result, all inside the timed region: every step
    copies all of its inputs from pinned host memory (one packed host-to-device copy),
    runs on the device copies, and copies its output back to pinned host memory.
    Consecutive steps are independent batches, so the copies are pipelined the way a
    serving loop prefetches: three device input buffers and three output buffers, uploads
    on one stream, kernels on `stream`, read-backs on a third; the uploads of the next
    steps and the read-back of the last one run while step i computes.  A buffer is reused
    only after the step that used it three steps earlier is done with it (with two, an
    upload as long as a step, as on hosts whose small pinned copies run at 14 GB/s, left
    no slack).  The timed region starts before the
    first upload (behind the same lead sleep as the device-timed steps, so that the host
    enqueues ahead of the GPU) and ends after the last read-back; the first upload and
    the last read-back, which nothing overlaps, are inside it.  `run_step(inputs, out)` enqueues one
    step on `stream`.  Returns (ms per step, breakdown of medians: h2d, compute, d2h in
    device ms and host ms spent enqueueing a step, d2h bytes per step)."""
    import torch
    nbuf = 3
    packs = [packed] + [packed.twin() for _ in range(nbuf - 1)]
    outs = [out] + [torch.empty_like(out) for _ in range(nbuf - 1)]
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    up = torch.cuda.Stream(device=dev)
    down = torch.cuda.Stream(device=dev)
    mk = lambda: [torch.cuda.Event(enable_timing=True) for _ in range(6)]   # noqa: E731

    # ev: 0/1 upload start/end (up), 2/3 compute start/end (stream), 4/5 read-back (down)
    def one(i, ev, hist):
        b = i % nbuf
        if i >= nbuf:
            up.wait_event(hist[i - nbuf][3])     # that step has finished reading this input buffer
        ev[0].record(up)
        packs[b].upload(up)
        ev[1].record(up)
        stream.wait_event(ev[1])
        if i >= nbuf:
            stream.wait_event(hist[i - nbuf][5])  # that step's read-back is done with this output
        ev[2].record(stream)
        run_step(packs[b].views, outs[b])
        ev[3].record(stream)
        down.wait_event(ev[3])
        ev[4].record(down)
        with torch.cuda.stream(down):
            out_host.copy_(outs[b], non_blocking=True)
        ev[5].record(down)

    hist = []
    for i in range(max(nbuf, warmup)):
        hist.append(mk())
        one(i, hist[-1], hist)
    torch.cuda.synchronize(dev)
    barrier(dev)
    hist = []
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        torch.cuda._sleep(LEAD_SLEEP_CYCLES)
    e0.record(stream)
    up.wait_event(e0)
    host_s = []
    for i in range(steps):
        h0 = time.perf_counter()
        hist.append(mk())
        one(i, hist[-1], hist)
        host_s.append(time.perf_counter() - h0)
    stream.wait_event(hist[-1][5])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / steps
    br = dict(h2d_ms=float(np.median([e[0].elapsed_time(e[1]) for e in hist])),
              compute_ms=float(np.median([e[2].elapsed_time(e[3]) for e in hist])),
              d2h_ms=float(np.median([e[4].elapsed_time(e[5]) for e in hist])),
              host_enqueue_ms=float(np.median(host_s)) * 1e3)
    return ms, br, out_host.numel() * out_host.element_size()


# Queued on the step stream ahead of the start event (about 0.2 ms at 1.9 GHz): the host
# enqueues the first step while the GPU still runs it, so the region does not begin with
# an idle GPU waiting for the first step's launches.  Without it the first of the timed
# steps measured 56-130 us longer than the others on the decode workloads: the host's time
# to enqueue one step (about 0.1 ms).  It is kept that short so that a host-bound run (the
# tiny batch, whose steps take less GPU time than their enqueueing) hides at most about
# two steps of host time.
LEAD_SLEEP_CYCLES = 400_000
TIMING = ("CUDA events on the step stream; a ~0.2 ms sleep kernel queued before the start event "
          "(after the barrier and synchronize) so that the first step's launches are queued "
          "before the GPU reaches them")


def timed_steps(step_fn, steps, stream, flush, dev):
    """Run `steps` steps on `stream`, each bracketed by CUDA events; with `flush`, L2 is
    evicted before every step, outside its events.  Returns (total ms of the region, list of
    per-step ms); the caller takes the step time from the events when flushing."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        torch.cuda._sleep(LEAD_SLEEP_CYCLES)
    start.record(stream)
    for i in range(steps):
        if flush is not None:
            flush(stream)
        step_fn(evs[i])
    stop.record(stream)
    torch.cuda.synchronize(dev)
    return start.elapsed_time(stop), [a.elapsed_time(b) for a, b in evs]


def run_nvpa(args) -> int:
    import torch
    import torch.distributed as dist

    import paged_kv_cache_422_b200 as nvpa
    from synth import WORKLOADS
    from synth.device import decode_to_device

    world, rank, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    lib = nvpa.lib()

    step = WORKLOADS[args.workload]()
    if hasattr(step, "cu_seqlens_q"):
        return run_nvpa_prefill(args, step, dev, lib, world, rank)
    work = decode_step_bytes(step)
    t = decode_to_device(step, dev)
    if step.num_tokens > step.batch:
        # a padded token list (slot -1 entries beyond the batch): the decode step takes one
        # new row per sequence, the rows of the real tokens in sequence order
        real = torch.as_tensor(np.nonzero(step.slot_mapping >= 0)[0][:step.batch], device=dev)
        for k in ("k_new", "v_new", "slot_mapping"):
            t[k] = t[k][real].contiguous()
    stream = torch.cuda.Stream(device=dev)
    shared = args.decode_api == "shared"
    if shared:
        ws_bytes = nvpa.decode_shared_prefix_workspace_size(
            step.batch, step.num_q_heads, step.num_kv_heads, step.head_dim, step.max_context_len,
            step.block_size, args.num_splits)
    else:
        ws_bytes = nvpa.paged_decode_workspace_size(
            step.batch, step.num_q_heads, step.num_kv_heads, step.head_dim, step.max_context_len,
            step.block_size, args.num_splits)
    workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    out = torch.empty_like(t["q"])
    decode_call = nvpa.decode_step_shared_prefix if shared else nvpa.decode_step

    def one_step(ev=None, inp=None, dst=None):
        # store + decode in one call (the library's fused decode step)
        inp = t if inp is None else inp
        if ev is not None:
            ev[0].record(stream)
        decode_call(inp["q"], inp["k_new"], inp["v_new"], t["k_cache"], t["v_cache"],
                    inp["slot_mapping"], inp["block_tables"], inp["context_lens"],
                    step.max_context_len, step.scale, out=out if dst is None else dst,
                    workspace=workspace, num_splits=args.num_splits, stream=stream)
        if ev is not None:
            ev[1].record(stream)

    # the warm-up steps run as the timed ones do (flush included), so that the first timed
    # flush and step are not the first to touch the flush buffer or its kernels
    flush = make_l2_flush(dev, args.flush_l2)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            if flush is not None:
                flush(stream)
            one_step()
    torch.cuda.synchronize(dev)

    # ---------------- timed region: K steps, device-timed ----------------
    with ClockSampler(dev.index if dev.index is not None else 0) as clocks:
        barrier(dev)
        torch.cuda.synchronize(dev)
        n0 = lib.nvpa_kernel_launch_count()
        ms_total, per_step = timed_steps(one_step, args.steps, stream, flush, dev)
        launches = lib.nvpa_kernel_launch_count() - n0
        barrier(dev)
    if flush is not None:
        ms_total = float(np.sum(per_step))     # the flushes between steps are not step time
    attn_ms = max_over_ranks(float(np.mean(per_step)), dev)
    median_ms = max_over_ranks(float(np.median(per_step)), dev)
    ms_total = max_over_ranks(ms_total, dev)
    ms_step = ms_total / args.steps

    # ---------------- end to end: host buffers in, host result out ----------------
    packed = PackedInputs({k: t[k] for k in ("q", "k_new", "v_new", "slot_mapping",
                                             "block_tables", "context_lens")}, dev)
    e2e_ms, e2e_breakdown, d2h = end_to_end(lambda inp, o: one_step(inp=inp, dst=o), packed, out,
                                            stream, args.steps, args.warmup, dev)
    e2e_ms = max_over_ranks(e2e_ms, dev)
    h2d = packed.nbytes

    peaks = measured_peaks()
    value = work["step"] * world / (ms_step * 1e-3) / 1e9
    attn_gbs = work["step"] / (attn_ms * 1e-3) / 1e9
    traffic = None
    if args.workload == DEFAULT_WORKLOAD and shared:
        # the worker's DRAM bytes from the committed capture of this step (none is kept for
        # the plain step's worker)
        traffic = profile_traffic("decode_step_shared_prefix_b512", DECODE_SOURCES)
    cs = clocks.summary()
    line = dict(
        metric=METRIC, value=value, unit="GB/s", n_gpus=world, steps=args.steps,
        warmup=args.warmup, ms_per_step=ms_step, higher_is_better=True, scaling="weak",
        vs_baseline=None, dtype="bf16", data="synthetic",
        ms_per_step_median=median_ms,
        pct_of_peak=100.0 * value / world / peaks["hbm_gbs"],
        seq_steps_per_s=step.batch * world / (ms_step * 1e-3),
        logical_kv_gbs=work["kv_logical"] * world / (ms_step * 1e-3) / 1e9,
        config=dict(workload=args.workload, batch=step.batch, num_q_heads=step.num_q_heads,
                    num_kv_heads=step.num_kv_heads, head_dim=step.head_dim,
                    block_size=step.block_size, max_context_len=step.max_context_len,
                    total_context_tokens=int(step.context_lens.sum()),
                    unique_kv_bytes=work["kv_unique"], step_bytes=work["step"],
                    parallelism=f"replicas x{world}" if world > 1 else "single GPU",
                    timing=TIMING,
                    l2=(L2_FLUSHED + "; %.3f GB of unique K/V per step vs 126 MB L2"
                        % (work["kv_unique"] / 1e9))
                       if args.flush_l2 else
                       ("inputs larger than L2: %.2f GB of unique K/V per step vs 126 MB L2"
                        % (work["kv_unique"] / 1e9) if work["kv_unique"] > L2_BYTES else
                        "NOT flushed (--flush-l2 flushes): %.3f GB of unique K/V per step fits "
                        "in the 126 MB L2" % (work["kv_unique"] / 1e9)),
                    num_splits=args.num_splits,
                    decode_api=("nvpa_decode_step_shared_prefix" if shared else "nvpa_decode_step")),
        roofline=dict(bound="hbm",
                      kernel=("decode step: plan, shared-prefix tensor-core tiles, split-KV worker "
                              "with the store folded in, combine" if shared else
                              "decode step: plan, split-KV worker with the store folded in, combine"),
                      achieved=attn_gbs, peak=peaks["hbm_gbs"], unit="GB/s",
                      frac=attn_gbs / peaks["hbm_gbs"], traffic=traffic,
                      peak_source=peak_source(peaks, "hbm_gbs", "burst copy")),
        e2e=dict(value=work["step"] * world / (e2e_ms * 1e-3) / 1e9, unit="GB/s",
                 h2d_bytes_per_step=h2d, d2h_bytes_per_step=d2h, ms_per_step=e2e_ms,
                 copies=E2E_COPIES,
                 breakdown_median=e2e_breakdown),
        gpu_launches=int(launches),
        clocks=cs,
    )
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(step)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del t, workspace
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_nvpa_prefill(args, step, dev, lib, world, rank) -> int:
    """A prefill step: store the uncached suffix tokens, then varlen causal attention.
    value = algorithmic causal FLOPs / step time (TFLOP/s)."""
    import torch
    import torch.distributed as dist

    import paged_kv_cache_422_b200 as nvpa
    from synth.device import prefill_to_device

    work = prefill_step_work(step)
    t = prefill_to_device(step, dev)
    stream = torch.cuda.Stream(device=dev)
    ws = torch.empty(nvpa.varlen_prefill_workspace_size(step.batch, step.total_q),
                     dtype=torch.uint8, device=dev)
    out = torch.empty_like(t["q"])

    def one_step(ev=None, inp=None, dst=None):
        inp = t if inp is None else inp
        nvpa.store_kvcache(inp["k_new"], inp["v_new"], t["k_cache"], t["v_cache"],
                           inp["slot_mapping"], stream=stream)
        if ev is not None:
            ev[0].record(stream)
        nvpa.varlen_prefill_attention(inp["q"], t["k_cache"], t["v_cache"], inp["block_tables"],
                                      inp["cu_seqlens_q"], inp["cu_seqlens_k"], step.max_seqlen_q,
                                      step.max_seqlen_k, step.scale, out=out if dst is None else dst,
                                      workspace=ws, stream=stream)
        if ev is not None:
            ev[1].record(stream)

    flush = make_l2_flush(dev, args.flush_l2)   # warm-up as the timed steps, flush included
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            if flush is not None:
                flush(stream)
            one_step()
    torch.cuda.synchronize(dev)

    step_evs = []

    def timed_whole(ev):
        a = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        one_step(ev)
        b = torch.cuda.Event(enable_timing=True)
        b.record(stream)
        step_evs.append((a, b))

    with ClockSampler(dev.index if dev.index is not None else 0) as clocks:
        barrier(dev)
        torch.cuda.synchronize(dev)
        n0 = lib.nvpa_kernel_launch_count()
        ms_total, attn_per_step = timed_steps(timed_whole, args.steps, stream, flush, dev)
        launches = lib.nvpa_kernel_launch_count() - n0
        barrier(dev)
    whole = [a.elapsed_time(b) for a, b in step_evs]
    if flush is not None:
        ms_total = float(np.sum(whole))
    ms_step = max_over_ranks(ms_total / args.steps, dev)
    attn_ms = max_over_ranks(float(np.mean(attn_per_step)), dev)
    attn_median_ms = max_over_ranks(float(np.median(attn_per_step)), dev)
    median_ms = max_over_ranks(float(np.median(whole)), dev)

    # ---------------- end to end: host buffers in, host result out ----------------
    packed = PackedInputs({k: t[k] for k in ("q", "k_new", "v_new", "slot_mapping",
                                             "block_tables", "cu_seqlens_q", "cu_seqlens_k")}, dev)
    e2e_ms, e2e_breakdown, d2h = end_to_end(lambda inp, o: one_step(inp=inp, dst=o), packed, out,
                                            stream, args.steps, args.warmup, dev)
    e2e_ms = max_over_ranks(e2e_ms, dev)
    h2d = packed.nbytes

    peaks = measured_peaks()
    tflops = work["flops"] * world / (ms_step * 1e-3) / 1e12
    attn_tflops = work["flops"] / (attn_ms * 1e-3) / 1e12
    line = dict(
        metric="varlen causal prefill with prefix-cache hits: TFLOP/s (algorithmic causal FLOPs)",
        value=tflops, unit="TFLOP/s", n_gpus=world, steps=args.steps, warmup=args.warmup,
        ms_per_step=ms_step, higher_is_better=True, scaling="weak", vs_baseline=None,
        dtype="bf16", data="synthetic",
        ms_per_step_median=median_ms, attention_ms_median=attn_median_ms,
        tokens_per_s=step.total_q * world / (ms_step * 1e-3),
        store_gbs=work["store"] / ((ms_step - attn_ms) * 1e-3) / 1e9 if ms_step > attn_ms else None,
        config=dict(workload=args.workload, batch=step.batch, total_q=step.total_q,
                    max_seqlen_q=step.max_seqlen_q, max_seqlen_k=step.max_seqlen_k,
                    num_q_heads=step.num_q_heads, num_kv_heads=step.num_kv_heads,
                    head_dim=step.head_dim, block_size=step.block_size,
                    algorithmic_tflop=work["flops"] / 1e12,
                    timing=TIMING,
                    l2=(L2_FLUSHED
                        if args.flush_l2 else
                        "inputs larger than L2, not flushed: each step stores 101 MB of new K/V "
                        "rows, then reads 101 MB of q and 128 MB of unique K/V and writes 101 MB "
                        "of output, against the 126 MB L2")),
        roofline=dict(bound="tensor", kernel="varlen_prefill_attention (plan + tcgen05 kernel)",
                      achieved=attn_tflops, peak=peaks["bf16_tflops"], unit="TFLOP/s",
                      frac=attn_tflops / peaks["bf16_tflops"],
                      traffic=(profile_traffic("prefill_tcgen05_varlen_b32", PREFILL_SOURCES)
                               if args.workload == "prefill_varlen_prefix_hits_b32" else None),
                      peak_source=peak_source(peaks, "bf16_tflops", "cuBLAS bf16 GEMM, burst")),
        e2e=dict(value=work["flops"] * world / (e2e_ms * 1e-3) / 1e12, unit="TFLOP/s",
                 h2d_bytes_per_step=h2d, d2h_bytes_per_step=d2h, ms_per_step=e2e_ms,
                 copies=E2E_COPIES,
                 breakdown_median=e2e_breakdown),
        gpu_launches=int(launches), clocks=clocks.summary())
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = prefill_cpu_baseline(step)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description="paged-KV attention benchmark (one JSON line)")
    ap.add_argument("--gpus", type=int, default=1)
    # 10 warm-up launches and 100 timed steps by default (the median of 100 iterations):
    # about 30 ms of timed work at the default workload
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["nvpa", "reference"], default="nvpa")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--num-splits", type=int, default=0)
    ap.add_argument("--decode-api", choices=["shared", "plain"], default="shared",
                    help="shared: nvpa_decode_step_shared_prefix; plain: nvpa_decode_step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--flush-l2", action="store_true",
                    help="write and read back a 512 MB buffer before every timed step "
                         "(outside its events)")
    argv = sys.argv[1:] if argv is None else list(argv)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    try:
        plan = launch_plan(args.gpus)
    except ValueError as e:
        print(f"bench.py: {e}", file=sys.stderr, flush=True)
        return 2
    if plan == "spawn":
        return subprocess.call(spawn_command(args.gpus, argv, _free_port()))
    if args.impl == "reference":
        return run_reference(args)
    return run_nvpa(args)


if __name__ == "__main__":
    sys.exit(main())

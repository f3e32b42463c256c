"""Benchmark of the paged decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole hot path over one synthetic batch: the
copy-on-write block copies of the step (copy_blocks, when the step has any),
the append of the step's new tokens (reshape_and_cache), and decode attention
(decode partitions + split-K reduce).  Block-manager bookkeeping is host work
done while the batch is built.  The default workload is the largest one that
fits one GPU, the long-context shared-prefix decode at block size 16: 128
requests forked from one 4096-token prefix (the same physical blocks) plus
unique suffixes of up to 28,672 tokens, Hq=32, Hkv=8, head size 128, bf16,
split-K partitions of 512 tokens.

Printed (rank 0, one JSON line): the KV-read bandwidth of the step (algorithmic
KV bytes / device time, aggregated over ranks), the step time, the roofline of
the dominant kernel (decode partitions) against the measured HBM copy
bandwidth, the same metric end to end from pinned host buffers (``e2e``), the
oracle timed on the host cores on a bounded sample (``cpu_baseline``), the
number of library kernels launched in the timed region, and the SM clocks seen.

With --gpus N > 1 (launched by torchrun) each rank runs its own replica of the
workload (seed offset by rank) with no collective on the data path: weak
scaling; the step time is the max over ranks.

--impl reference times the oracle (the plain fp64 CPU implementation) on the
host cores on the same workload and metric, one bounded sample per step.

--op mq (1 GPU) measures the multi-query kernel (pa_decode_multi) on
--workload verify_gqa70b (the gqa70b batch verifying 4 proposed tokens per
sequence) or prefill_gqa70b (16 sequences with contexts U[2048,8192] whose last
512 tokens are a prefill chunk).

--op swap (1 GPU) measures the block swap instead: every block of the
workload's batch to a pinned host pool (scattered ids) and back, one
pa_swap_blocks launch per direction, against one contiguous device<->pinned
copy of the same bytes (the link's own rate).
"""
import argparse
import hashlib
import json
import os
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "paged decode attention µs/step and KV-read GB/s (fraction of B200 HBM peak)"
DEFAULT_WORKLOAD = "long_prefix_bs16"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0


def workload_spec(name):
    if name.endswith("_fp8"):
        return W.fp8(workload_spec(name[: -len("_fp8")]))
    if name.endswith("_quarter"):
        # a quarter of the sequences of a workload (same kernel, same per-sequence
        # shapes): the profiling case for captures that must stay small
        from dataclasses import replace
        base = workload_spec(name[: -len("_quarter")])
        return replace(base, name=name, num_seqs=max(1, base.num_seqs // 4))
    if name == "opt13b_compact":
        # the opt13b launch with a pool of 1.25x the blocks it needs (about 1 GB
        # on the device instead of 6.6): the profiling case
        from dataclasses import replace
        return replace(W.FULL["opt13b"], name="opt13b_compact", num_blocks=None)
    if name.startswith("long_prefix_bs"):
        return W.long_prefix(int(name[len("long_prefix_bs"):]))
    if name == "long_prefix":
        return W.long_prefix(16)
    return W.FULL[name]


WORKLOAD_TEXT = {
    "tiny": "tiny paged decode: 8 seqs, context U[1,64], Hq=Hkv=4, D=64, block 16, 64-block permuted pool, fp32",
    "opt13b": "OPT-13B-shaped decode layer: 64 seqs, Hq=Hkv=40, D=128, block 16, fp16, context lognormal(median 600, sigma 0.5) clipped to [16,2048], 20,000-block pool",
    "llama13b_ps": "LLaMA-13B-shaped parallel sampling: 16 prompts x 6 samples, Hq=Hkv=40, D=128, block 16, bf16, prompt U[512,1024] shared, 1-256 divergent tokens with copy-on-write",
    "gqa70b": "GQA 70B-shaped decode layer: 256 seqs, Hq=64, Hkv=8, D=128, block 16, bf16, context U[256,4096]",
    "long_prefix": "long-context shared-prefix decode: 128 requests sharing a 4096-token prefix + suffix U[1,28672], Hq=32, Hkv=8, D=128, bf16",
}


def workload_text(name):
    if name.endswith("_fp8"):
        sp = workload_spec(name)
        return (workload_text(name[: -len("_fp8")]) +
                f"; cache of E4M3 codes (k_scale {sp.k_scale:.6g}, v_scale {sp.v_scale:.6g}), "
                f"queries and outputs {sp.dtype}")
    if name.endswith("_quarter"):
        return workload_text(name[: -len("_quarter")]) + " (a quarter of the sequences)"
    if name == "opt13b_compact":
        return WORKLOAD_TEXT["opt13b"].replace("20,000-block pool", "pool of 1.25x the blocks needed")
    base = name.split("_bs")[0] if name.startswith("long_prefix") else name
    txt = WORKLOAD_TEXT[base]
    if base == "long_prefix":
        txt += f", block {workload_spec(name).block_size}, split-K partitions of 512"
    return txt


# ---------------------------------------------------------------------------
# byte accounting (algorithmic traffic of one step)


def step_bytes(spec, tables, lens, num_blocks_shared_ok=True):
    """KV bytes a step must read: every (physical block, kv head) token slot
    holding a valid token counted once (unique) and once per reader (logical),
    plus q, out, table and length bytes."""
    bs, es = spec.block_size, spec.esize
    row = spec.Hkv * spec.D * spec.kv_esize * 2   # K and V bytes of one token, all kv heads
    logical = int(lens.astype(np.int64).sum()) * row
    # unique: valid tokens of each distinct physical block
    used = {}
    for b in range(len(lens)):
        L = int(lens[b])
        nb = -(-L // bs)
        for i in range(nb):
            blk = int(tables[b, i])
            n = min(bs, L - i * bs)
            if used.get(blk, 0) < n:
                used[blk] = n
    unique = sum(used.values()) * row
    B = len(lens)
    qo = 2 * B * spec.Hq * spec.D * es
    tbl = sum(-(-int(L) // bs) for L in lens) * 4 + B * 4
    return unique, logical, qo + tbl


# ---------------------------------------------------------------------------
# clocks (NVML, sampled in a thread)

_REASONS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
    0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
}


class ClockSampler:
    def __init__(self, device_index, period_s=0.02):
        self.samples = []
        self.max_mhz = None
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that, keep going
            self.err = repr(e)
        self.period = period_s
        self.t = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except Exception:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append((time.time(), mhz, rs))
            except Exception:
                pass
            self._stop.wait(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return time.time()

    def stop(self):
        self._stop.set()
        if self.t:
            self.t.join()

    def summary(self, t0, t1):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        win = [s for s in self.samples if t0 <= s[0] <= t1] or self.samples[-5:]
        mhz = [s[1] for s in win]
        rs = 0
        for s in win:
            rs |= int(s[2])
        names = [n for bit, n in _REASONS.items() if rs & bit and n != "gpu_idle"]
        return {"sm_mhz": float(np.median(mhz)) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(win)}


# ---------------------------------------------------------------------------
# distributed plumbing (one process per GPU; weak scaling)


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def dist_init(world, backend):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def reduce_max(x, world, device="cpu"):
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(x, world, device="cpu"):
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(world, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def rank_spec(spec, rank):
    from dataclasses import replace
    return spec if rank == 0 else replace(spec, seed=spec.seed + 100_000 * rank)


# ---------------------------------------------------------------------------
# profile summaries committed under profiles/ (dram traffic of the dominant kernel)


KERNEL_SOURCES = {
    "decode_partition_kernel": ("decode.cu", "pa_device.cuh", "pa_internal.h"),
    "decode_partition_tc_kernel": ("decode_tc.cu", "tc_common.cuh", "pa_device.cuh", "pa_internal.h"),
    "decode_partition_tc8_kernel": ("decode_tc8.cu", "tc_common.cuh", "pa_device.cuh",
                                    "pa_internal.h"),
    # pa_decode_grouped: the span and rest kernels (decode_tc.cu, or decode.cu
    # for G = 1, 2) and the reduce (decode.cu); E4M3 caches: decode_tc8.cu
    "decode_grouped": ("decode_tc.cu", "decode.cu", "tc_common.cuh", "pa_device.cuh",
                       "pa_internal.h"),
    "decode_grouped_fp8": ("decode_tc8.cu", "decode.cu", "tc_common.cuh", "pa_device.cuh",
                           "pa_internal.h"),
}


def partition_kernel(spec, P):
    """The decode-partition kernel the library picks for this launch: a
    tensor-core one (16-bit or E4M3 cache) for 4 or 8 query heads per kv head
    with fp16/bf16 queries, head size 128 and a partition length that is a
    multiple of 128; else CUDA cores."""
    G = spec.Hq // spec.Hkv
    if spec.dtype in ("f16", "bf16") and spec.D == 128 and G in (4, 8) and P % 128 == 0:
        return "decode_partition_tc8_kernel" if spec.fp8 else "decode_partition_tc_kernel"
    return "decode_partition_kernel"


def source_digest(files=KERNEL_SOURCES["decode_partition_kernel"]):
    """Digest of the kernels' code: the sources with comments and blank lines
    dropped, so that editing a comment does not retire a capture."""
    import re
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "paged_kv_cache_443_b200", "csrc", f), encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"(?m)^\s*//.*$|\s+//[^\"\n]*$", "", text)
        code = "\n".join(ln.rstrip() for ln in text.splitlines() if ln.strip())
        h.update(code.encode("utf-8"))
    return h.hexdigest()[:16]


TRAFFIC_FILE = os.path.join("profiles", "dram_traffic.json")


def profiled_traffic(workload, kernel, partition_size):
    """DRAM bytes per launch of the decode-partition kernel, from the ncu capture
    recorded in profiles/dram_traffic.json for this workload, kernel and
    partition length, and only while that kernel's sources are unchanged since
    the capture.  Returns (bytes or None, a note saying where they come from)."""
    path = os.path.join(ROOT, TRAFFIC_FILE)
    try:
        with open(path) as f:
            entries = json.load(f)["captures"]
    except (OSError, ValueError, KeyError):
        return None, "no ncu capture recorded"
    for e in entries:
        if (e.get("workload") == workload and e.get("kernel") == kernel
                and int(e.get("partition_size", -1)) == int(partition_size)):
            if e.get("source_digest") != source_digest(KERNEL_SOURCES[kernel]):
                return None, "the kernel changed since its ncu capture"
            return float(e["dram_bytes_per_launch"]), e.get("how", "ncu capture")
    return None, "no ncu capture of this kernel at this workload and partition length"


def record_traffic(csv_path, workload, kernel, partition_size):
    """Record in profiles/dram_traffic.json the DRAM bytes of one decode call:
    dram__bytes_read.sum + dram__bytes_write.sum summed over the launches of an
    ncu CSV that captured exactly that call's kernels (a capture's --csv
    --print-units base log, or the raw page of a report), with the current
    digest of the kernels' sources."""
    import csv
    with open(csv_path, newline="") as f:
        lines = [ln for ln in f if ln.startswith('"')]   # ncu's own "==PROF==" lines dropped
    rows = list(csv.DictReader(lines))
    names = ("dram__bytes_read.sum", "dram__bytes_write.sum")
    total, launches = 0.0, set()
    if rows and "Metric Name" not in rows[0]:
        # the raw page of a report (ncu -i REP --page raw --csv --print-units base
        # --metrics ...): one row per launch after a row of units
        units, rows = rows[0], rows[1:]
        for n in names:
            if units.get(n) not in ("byte", "bytes"):
                raise SystemExit(f"{csv_path}: capture with --print-units base (got {units.get(n)})")
        rows = [dict(r, **{"Metric Name": n, "Metric Unit": "byte", "Metric Value": r[n]})
                for r in rows for n in names]
    for r in rows:
        if r.get("Metric Name") in names:
            if r.get("Metric Unit") not in ("byte", "bytes"):
                raise SystemExit(f"{csv_path}: capture with --print-units base (got {r.get('Metric Unit')})")
            total += float(r["Metric Value"].replace(",", ""))
            launches.add(r["ID"])
    if not launches:
        raise SystemExit(f"{csv_path}: no dram__bytes_* rows")
    path = os.path.join(ROOT, TRAFFIC_FILE)
    try:
        with open(path) as f:
            data = json.load(f)
    except (OSError, ValueError):
        data = {"captures": []}
    entry = {"workload": workload, "kernel": kernel, "partition_size": int(partition_size),
             "source_digest": source_digest(KERNEL_SOURCES[kernel]),
             "dram_bytes_per_launch": int(round(total)),
             "how": (f"ncu dram__bytes_read.sum + dram__bytes_write.sum over the "
                     f"{len(launches)} kernel launches of one call, {os.path.basename(csv_path)}")}
    data["captures"] = [e for e in data.get("captures", [])
                        if (e.get("workload"), e.get("kernel"), int(e.get("partition_size", -1)))
                        != (workload, kernel, int(partition_size))] + [entry]
    with open(path, "w") as f:
        json.dump(data, f, indent=1)
        f.write("\n")
    return entry


def measured_peak_tensor():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (bf16 burst)"
    except Exception:
        return 1590.0, "fallback"


def measured_peak_hbm():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------------------
# oracle timing (CPU): bounded sample of the same workload


def oracle_sample_setup(spec, max_seqs=None):
    """Builds the workload (or its first max_seqs sequences) on the oracle side:
    oracle allocator, oracle append and copy, seeded contents drawn on the CPU.
    The pool is sized to the sample (1.25x the blocks it needs)."""
    import torch
    import oracle
    from dataclasses import replace
    from oracle.allocator import BlockManager
    sp = spec
    if max_seqs is not None and spec.kind in ("independent", "shared_prefix") and \
            max_seqs < spec.num_seqs:
        sp = replace(spec, num_seqs=max_seqs)
    sp = replace(sp, num_blocks=None)
    sc = W.scenario(sp)
    shape = (sc.num_blocks, sp.Hkv, sp.block_size, sp.D)
    st = {"f32": np.float32, "f16": np.uint16, "bf16": np.uint16, "e4m3": np.uint8}[sp.kv]
    kc = np.zeros(shape, dtype=st)
    vc = np.zeros(shape, dtype=st)
    bm = BlockManager(sc.num_blocks, sp.block_size, sc.free_order.tolist())
    for op in sc.setup_ops + sc.step_ops:
        if op.kind == "add":
            bm.add(op.seq)
        elif op.kind == "fork":
            bm.fork(op.seq, op.arg)
        elif op.kind == "release":
            bm.release(op.seq)
        else:
            k, v = W.kv_content(sp, op.kv_id, op.arg, "cpu")
            slots, pairs = bm.append(op.seq, op.arg)
            if pairs:
                oracle.copy_blocks(kc, vc, np.array(pairs), sp.kv_code)
            if sp.fp8:
                oracle.reshape_and_cache_e4m3(W.storage_view(k), W.storage_view(v), kc, vc,
                                              np.array(slots), sp.dtype_code, sp.k_scale,
                                              sp.v_scale)
            else:
                oracle.reshape_and_cache(W.storage_view(k), W.storage_view(v), kc, vc,
                                         np.array(slots), sp.dtype_code)
    tables, lens = bm.build_tables(sc.batch, sc.max_blocks)
    q = W.storage_view(W.q_content(sp, len(sc.batch), "cpu"))
    return sp, q, kc, vc, tables, lens


def time_oracle(spec, budget_s=15.0, steps=None, per_step_budget_s=None):
    """Times the oracle's attention on rows of the workload.  Returns
    (GB/s, seconds per sampled step, threads, sample description)."""
    import oracle
    nthreads = oracle.max_threads()
    # a bounded sample: the first 16 sequences of an independent batch, the
    # first 4 requests (with their shared prefix) of a shared-prefix batch
    max_seqs = {"independent": min(spec.num_seqs, 16),
                "shared_prefix": min(spec.num_seqs, 4)}.get(spec.kind)
    sp, q, kc, vc, tables, lens = oracle_sample_setup(spec, max_seqs)
    B = len(lens)
    rows_all = np.array([(b, h) for b in range(B) for h in range(sp.Hq)], dtype=np.int64)
    row_bytes = lambda rows: int(sum(int(lens[b]) for b, _ in rows)) * sp.D * sp.kv_esize * 2
    kv = dict(kv_dtype=sp.kv_code, k_scale=sp.k_scale, v_scale=sp.v_scale)
    # calibration on a few rows
    rng = np.random.default_rng(0)
    cal = rows_all[rng.choice(len(rows_all), size=min(len(rows_all), 4 * nthreads), replace=False)]
    t0 = time.perf_counter()
    oracle.paged_attention(q, kc, vc, sp.dtype_code, tables, lens, sp.softmax_scale, rows=cal,
                           nthreads=nthreads, **kv)
    per_byte = (time.perf_counter() - t0) / max(1, row_bytes(cal))
    target = per_step_budget_s if per_step_budget_s is not None else budget_s
    n_rows = int(max(1, min(len(rows_all), target / max(per_byte * row_bytes(rows_all) / len(rows_all), 1e-9))))
    n_steps = steps if steps is not None else 1
    total_bytes, total_t = 0, 0.0
    for i in range(n_steps):
        sel = rows_all[rng.choice(len(rows_all), size=n_rows, replace=False)]
        t0 = time.perf_counter()
        oracle.paged_attention(q, kc, vc, sp.dtype_code, tables, lens, sp.softmax_scale, rows=sel,
                               nthreads=nthreads, **kv)
        total_t += time.perf_counter() - t0
        total_bytes += row_bytes(sel)
    # KV bytes of the sampled (sequence, query head) rows as the kernel counts them:
    # G query heads share one kv head's bytes
    gbs = total_bytes / sp.G / total_t / 1e9
    desc = (f"{n_rows} of {len(rows_all)} (sequence, query head) rows per step, {n_steps} step(s), "
            f"of the first {B} sequences of the workload built on the oracle side "
            f"(pool of 1.25x the blocks they need); KV bytes counted once per kv head")
    return gbs, total_t / n_steps, nthreads, desc


# ---------------------------------------------------------------------------
# the GPU arm


def run_ours(args):
    import torch
    import paged_kv_cache_443_b200 as pk
    from paged_kv_cache_443_b200.cache import PagedKVCache

    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py: a CUDA device is required for --impl ours")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist_init(world, "nccl")
    pk.lib()  # fails loudly if the library is missing

    spec = rank_spec(workload_spec(args.workload), rank)
    sc = W.scenario(spec)
    cache = PagedKVCache(sc.num_blocks, spec.block_size, spec.Hkv, spec.D, W.torch_kv_dtype(spec),
                         device, sc.free_order.tolist(), fill=0.0, k_scale=spec.k_scale,
                         v_scale=spec.v_scale)
    for op in sc.setup_ops:
        if op.kind == "add":
            cache.add(op.seq)
        elif op.kind == "fork":
            cache.fork(op.seq, op.arg)
        elif op.kind == "release":
            cache.release(op.seq)
        else:
            k, v = W.kv_content(spec, op.kv_id, op.arg, device)
            cache.append([op.seq], [op.arg], k, v)
            del k, v
    seqs = [op.seq for op in sc.step_ops]
    counts = [op.arg for op in sc.step_ops]
    draws = [W.kv_content(spec, op.kv_id, op.arg, device) for op in sc.step_ops]
    key = torch.cat([d[0] for d in draws]).contiguous()
    value = torch.cat([d[1] for d in draws]).contiguous()
    del draws
    slots_l, pairs_l = cache.reserve(seqs, counts)
    slots = torch.tensor(slots_l, dtype=torch.int64, device=device)
    pairs = torch.tensor(pairs_l, dtype=torch.int64, device=device).reshape(-1, 2)
    tables, lens, max_ctx = cache.tables(sc.batch, sc.max_blocks)
    q = W.q_content(spec, len(sc.batch), device)
    out = torch.empty_like(q)
    P = args.partition_size if args.partition_size else spec.partition_size
    if P == 0:   # the workload leaves it to the library: use pa_decode's automatic length
        auto = pk.pa_decode_fp8_auto_partition_size if spec.fp8 else pk.pa_decode_auto_partition_size
        P = auto(len(sc.batch), spec.Hq, spec.Hkv, spec.D, spec.dtype_code, max_ctx)
    # families sharing leading blocks (parallel samples, a common prefix) are
    # decoded with each family's shared span read once, unless --grouped off
    groups = None
    if args.grouped == "on" or (args.grouped == "auto" and spec.kind != "independent"):
        groups = cache.groups(tables, lens)
        if groups.max_shared_len == 0:
            groups = None
    if groups is not None:
        ws = cache.grouped_workspace(q.shape[0], q.shape[1], max_ctx, groups, P)
    else:
        ws = cache.workspace(q.shape[0], q.shape[1], max_ctx, P)
    scale = spec.softmax_scale
    n_part = pk.pa_decode_num_partitions(max_ctx, P)
    stream = torch.cuda.current_stream(device)
    kc, vc = cache.k_cache, cache.v_cache

    unique, logical, other = step_bytes(spec, tables.cpu().numpy(), lens.cpu().numpy())
    flush = unique < 8 * L2_BYTES
    scratch = torch.zeros(2 * L2_BYTES // 4, dtype=torch.float32, device=device) if flush else None

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        if pairs.numel():
            pk.pa_copy_blocks(kc, vc, pairs, stream=stream)
        if spec.fp8:
            pk.pa_reshape_and_cache_fp8(key, value, kc, vc, slots, spec.k_scale, spec.v_scale,
                                        stream=stream)
        else:
            pk.pa_reshape_and_cache(key, value, kc, vc, slots, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        if groups is not None:
            # one call: the groups' spans, the rest of each sequence, the reduce
            if spec.fp8:
                pk.pa_decode_grouped_fp8(out, q, kc, vc, tables, lens, groups, scale, max_ctx,
                                         spec.k_scale, spec.v_scale, partition_size=P,
                                         workspace=ws, stream=stream)
            else:
                pk.pa_decode_grouped(out, q, kc, vc, tables, lens, groups, scale, max_ctx,
                                     partition_size=P, workspace=ws, stream=stream)
            if ev is not None:
                ev[2].record(stream)
                ev[3].record(stream)
            return
        if spec.fp8:
            pk.pa_decode_partitions_fp8(out, q, kc, vc, tables, lens, scale, max_ctx, spec.k_scale,
                                        spec.v_scale, partition_size=P, workspace=ws,
                                        stream=stream)
        else:
            pk.pa_decode_partitions(out, q, kc, vc, tables, lens, scale, max_ctx,
                                    partition_size=P, workspace=ws, stream=stream)
        if ev is not None:
            ev[2].record(stream)
        if n_part > 1:
            pk.pa_decode_reduce(out, lens, max_ctx, partition_size=P, workspace=ws, stream=stream)
        if ev is not None:
            ev[3].record(stream)

    sampler = ClockSampler(local)
    sampler.start()
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(device)
    assert pk.pa_device_status() == 0, "device-side check failed during warm-up"
    # clock soak: keep the GPU under this load for a while before timing, so the
    # clock samples describe the timed region's state (W >= 3 warm-up steps ran)
    soak_t0 = time.time()
    while time.time() - soak_t0 < args.soak_seconds:
        for _ in range(20):
            step()
        torch.cuda.synchronize(device)

    K = args.steps
    sink = torch.empty((), dtype=torch.float32, device=device)

    def evict_l2():
        # stream a 2x-L2 buffer: evicts the previous step's lines, and a read
        # leaves no dirty lines for the timed kernels to write back
        torch.amax(scratch, dim=0, out=sink)

    # ---- timed region: K whole steps (the step's kernels back to back, so the
    # library's overlapped launches overlap; events only at step boundaries) ----
    step_evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    launches0 = pk.pa_launch_count()
    barrier(world, device)
    torch.cuda.synchronize(device)
    for i in range(K):
        if flush:
            evict_l2()
        step_evs[i][0].record(stream)
        step()
        step_evs[i][1].record(stream)
    torch.cuda.synchronize(device)
    barrier(world, device)
    t_end = time.time()
    launches = pk.pa_launch_count() - launches0
    if flush:   # the L2 eviction between steps is not part of the step
        total_ms = float(sum(step_evs[i][0].elapsed_time(step_evs[i][1]) for i in range(K)))
    else:       # back-to-back steps: the whole span (includes launch gaps)
        total_ms = step_evs[0][0].elapsed_time(step_evs[K - 1][1])
    assert pk.pa_device_status() == 0, "device-side check failed in the timed region"

    # ---- per-kernel durations (CUDA events between the kernels, same steps) ----
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    torch.cuda.synchronize(device)
    for i in range(K):
        if flush:
            evict_l2()
        step(evs[i])
    torch.cuda.synchronize(device)
    part_ms = [evs[i][1].elapsed_time(evs[i][2]) for i in range(K)]
    red_ms = [evs[i][2].elapsed_time(evs[i][3]) for i in range(K)]
    app_ms = [evs[i][0].elapsed_time(evs[i][1]) for i in range(K)]

    # ---- end to end through the public API: pinned host buffers in, result out ----
    h_q = q.cpu().pin_memory()
    h_key, h_value = key.cpu().pin_memory(), value.cpu().pin_memory()
    h_slots, h_pairs = slots.cpu().pin_memory(), pairs.cpu().pin_memory()
    h_tables, h_lens = tables.cpu().pin_memory(), lens.cpu().pin_memory()
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    d_q, d_key, d_value = torch.empty_like(q), torch.empty_like(key), torch.empty_like(value)
    d_slots, d_pairs = torch.empty_like(slots), torch.empty_like(pairs)
    d_tables, d_lens = torch.empty_like(tables), torch.empty_like(lens)
    h2d = sum(t.numel() * t.element_size() for t in (h_q, h_key, h_value, h_slots, h_pairs,
                                                     h_tables, h_lens))
    d2h = h_out.numel() * h_out.element_size()

    def e2e_body(st):
        for d, h in ((d_q, h_q), (d_key, h_key), (d_value, h_value), (d_slots, h_slots),
                     (d_pairs, h_pairs), (d_tables, h_tables), (d_lens, h_lens)):
            d.copy_(h, non_blocking=True)
        cache.copy_on_write(d_pairs, stream=st)
        cache.store(d_key, d_value, d_slots, stream=st)
        cache.decode(d_q, d_tables, d_lens, max_ctx, scale, out=out, partition_size=P,
                     workspace=ws, stream=st, groups=groups)
        h_out.copy_(out, non_blocking=True)

    def time_e2e(step_fn):
        for _ in range(3):
            step_fn()
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world, device)
        torch.cuda.synchronize(device)
        e0.record(stream)
        for _ in range(Ke):
            step_fn()
        e1.record(stream)
        torch.cuda.synchronize(device)
        return e0.elapsed_time(e1) / Ke

    Ke = max(1, min(K, 200))
    e2e_eager_ms = time_e2e(lambda: e2e_body(stream))
    # the same step (copies in, library calls, copy out) captured once as a CUDA
    # graph and replayed: what a serving loop runs, without per-call host work
    e2e_mode = "cuda graph of the step (H2D copies, library launches, D2H copy)"
    try:
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(device)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            e2e_body(None)
        torch.cuda.synchronize(device)
        with torch.cuda.graph(graph):
            e2e_body(None)
        torch.cuda.synchronize(device)
        e2e_ms = time_e2e(graph.replay)
    except Exception as exc:   # capture unsupported here: keep the eager figure
        e2e_mode = f"eager API calls (graph capture failed: {type(exc).__name__})"
        graph = None
        e2e_ms = e2e_eager_ms
    assert pk.pa_device_status() == 0, "device-side check failed in the end-to-end steps"
    sampler.stop()
    clocks = sampler.summary(soak_t0, t_end)

    # ---- aggregate over ranks ----
    ms_step = reduce_max(total_ms / K, world, device)
    e2e_ms = reduce_max(e2e_ms, world, device)
    e2e_eager_ms = reduce_max(e2e_eager_ms, world, device)
    units = reduce_sum(unique, world, device)
    value = units / (ms_step * 1e-3) / 1e9
    e2e_value = units / (e2e_ms * 1e-3) / 1e9

    part_avg = float(np.mean(part_ms))
    peak, peak_kind = measured_peak_hbm()
    alg = unique + other
    achieved = alg / (part_avg * 1e-3) / 1e9
    kname = partition_kernel(spec, P)
    traffic, traffic_note = profiled_traffic(args.workload, kname, P)
    if groups is not None:
        # the three launches of the grouped decode are timed together (the
        # reduce included), against the same algorithmic bytes
        span_kernel = "decode_partition_tc8_kernel" if spec.fp8 else "decode_partition_tc_kernel"
        kname = ("decode_grouped: " + span_kernel + " (the families' shared spans, "
                 "16/G or 8/G members per CTA) next to " + partition_kernel(spec, P) +
                 " (the rest of every sequence), then decode_reduce_kernel")
        traffic, traffic_note = profiled_traffic(
            args.workload, "decode_grouped_fp8" if spec.fp8 else "decode_grouped", P)

    result = None
    if rank == 0:
        result = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": "GB/s",
            "n_gpus": world,
            "steps": K,
            "warmup": args.warmup,
            "ms_per_step": round(ms_step, 6),
            "us_per_step": round(ms_step * 1e3, 3),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": f"e4m3 kv, {spec.dtype} q/out (fp32 math)" if spec.fp8 else spec.dtype,
            "data": "synthetic: seeded N(0,1) K/V/q in the cache dtype, context lengths and block "
                    "placement drawn as the workload states (stand-in for the ShareGPT/Alpaca-shaped "
                    "serving workloads; no dataset or weights)",
            "config": {
                "workload": f"{args.workload}: {workload_text(args.workload)}",
                "num_seqs": len(sc.batch), "num_heads": spec.Hq, "num_kv_heads": spec.Hkv,
                "head_size": spec.D, "block_size": spec.block_size, "num_blocks": sc.num_blocks,
                "max_context_len": max_ctx, "partition_size": P, "num_partitions": n_part,
                "split_k": (f"{n_part} partitions of {P} tokens at the longest context; the reduce "
                            "kernel merges them" if n_part > 1 else
                            f"one partition of {P} tokens covers every sequence: no split-K "
                            "reduce launch"),
                "kv_bytes_unique": unique, "kv_bytes_logical": logical,
                "new_tokens_per_step": int(key.shape[0]), "cow_pairs_per_step": int(pairs.shape[0]),
                "l2": ("L2 flushed between timed steps (252 MB streamed read, excluded from the step time)"
                       if flush else f"inputs larger than L2: {unique / 1e9:.2f} GB of KV per step"),
                "parallelism": "replicas" if world == 1 else f"replicas x{world} (no collective)",
                "decode": (f"grouped: {groups.num_groups} families sharing up to "
                           f"{groups.max_shared_len} leading tokens, each shared span read once "
                           f"for its members (pa_decode_grouped{'_fp8' if spec.fp8 else ''})"
                           if groups is not None
                           else "pa_decode_partitions + pa_decode_reduce"),
            },
            "kernels_us": ({  # from the second pass, with events between the kernels
                "append_and_copy": round(float(np.mean(app_ms)) * 1e3, 3),
                "decode_partitions": round(part_avg * 1e3, 3),
                "decode_reduce": round(float(np.mean(red_ms)) * 1e3, 3),
            } if groups is None else {
                "append_and_copy": round(float(np.mean(app_ms)) * 1e3, 3),
                "decode_grouped": round(part_avg * 1e3, 3),
            }),
            "roofline": {
                "kernel": kname,
                "bound": "hbm",
                "achieved": round(achieved, 1),
                "peak": peak,
                "peak_kind": peak_kind,
                "unit": "GB/s",
                "frac": round(achieved / peak, 4),
                "traffic": traffic,
                "traffic_source": traffic_note,
                "algorithmic_bytes_per_launch": alg,
            },
            "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "ms_per_step": round(e2e_ms, 6),
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "mode": e2e_mode,
                    "eager_value": round(units / (e2e_eager_ms * 1e-3) / 1e9, 2),
                    "eager_ms_per_step": round(e2e_eager_ms, 6)},
            "gpu_launches": int(launches),
            "clocks": clocks,
        }
    return result


MQ_WORKLOADS = {
    # (spec, query tokens per sequence, description)
    "verify_gqa70b": (W.GQA70B, 4, "speculative verify: the gqa70b batch (256 seqs, Hq=64, Hkv=8, "
                      "D=128, bf16, context U[256,4096]) checking 4 proposed tokens per sequence"),
    "verify2_gqa70b": (W.GQA70B, 2, "speculative verify: the gqa70b batch checking 2 proposed tokens "
                       "per sequence (query tokens x heads = 16: the token-major decode kernel)"),
    "prefill_gqa70b": (None, 512, "chunked prefill: 16 sequences, Hq=64, Hkv=8, D=128, bf16, block "
                       "16, context U[2048,8192] whose last 512 tokens are the chunk"),
}


def mq_spec(name):
    from dataclasses import replace
    if name.endswith("_quarter"):       # the profiling case: a quarter of the sequences
        spec, Q = mq_spec(name[: -len("_quarter")])
        return replace(spec, name=name, num_seqs=max(1, spec.num_seqs // 4)), Q
    spec, Q, _ = MQ_WORKLOADS[name]
    if spec is None:
        spec = replace(W.GQA70B, name="prefill_gqa70b", num_seqs=16, ctx_lo=2048, ctx_hi=8192,
                       seed=449)
    return spec, Q


def run_mq(args):
    """Multi-query attention throughput (TFLOP/s and KV GB/s) on one GPU."""
    import torch
    import paged_kv_cache_443_b200 as pk
    from paged_kv_cache_443_b200.cache import PagedKVCache

    if not torch.cuda.is_available():
        raise SystemExit("bench.py: a CUDA device is required for --op mq")
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    pk.lib()
    spec, Q = mq_spec(args.workload)
    sc = W.scenario(spec)
    cache = PagedKVCache(sc.num_blocks, spec.block_size, spec.Hkv, spec.D, W.torch_kv_dtype(spec),
                         device, sc.free_order.tolist(), fill=0.0)
    for op in sc.setup_ops + sc.step_ops:
        if op.kind == "add":
            cache.add(op.seq)
        elif op.kind == "fork":
            cache.fork(op.seq, op.arg)
        elif op.kind == "release":
            cache.release(op.seq)
        else:
            k, v = W.kv_content(spec, op.kv_id, op.arg, device)
            cache.append([op.seq], [op.arg], k, v)
            del k, v
    tables, lens, max_ctx = cache.tables(sc.batch, sc.max_blocks)
    lens_h = lens.cpu().numpy().astype(np.int64)
    qlens = np.minimum(Q, lens_h)
    qs = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    T = int(qs[-1])
    g = torch.Generator(device=device).manual_seed(spec.seed)
    q = torch.randn((T, spec.Hq, spec.D), generator=g, device=device).to(W.torch_dtype(spec))
    out = torch.empty_like(q)
    qs_d = torch.from_numpy(qs).to(device)
    P = args.partition_size     # 0: pa_decode_multi's automatic length
    n = pk.pa_decode_multi_workspace_bytes(T, spec.Hq, spec.D, max_ctx, P)
    ws = torch.empty(n // 4, dtype=torch.float32, device=device) if n else None
    maxq = int(qlens.max())
    stream = torch.cuda.current_stream(device)

    def step():
        pk.pa_decode_multi(out, q, cache.k_cache, cache.v_cache, tables, lens, qs_d,
                           spec.softmax_scale, max_ctx, maxq, partition_size=P, workspace=ws,
                           stream=stream)

    unique, logical, other = step_bytes(spec, tables.cpu().numpy(), lens_h)
    # flops: 4 * D per (query row, attended key): q.k and p.v, 2 flops each per element
    pos_sum = sum(int(qlens[b]) * (2 * int(lens_h[b]) - int(qlens[b]) + 1) // 2
                  for b in range(len(lens_h)))
    flops = 4.0 * spec.D * spec.Hq * pos_sum
    alg_bytes = unique + 2 * T * spec.Hq * spec.D * spec.esize
    flush = unique < 8 * L2_BYTES
    scratch = torch.zeros(2 * L2_BYTES // 4, dtype=torch.float32, device=device) if flush else None
    sink = torch.empty((), dtype=torch.float32, device=device)
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(device)
    assert pk.pa_device_status() == 0
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    sampler = ClockSampler(0)
    sampler.start()
    t0 = time.time()
    launches0 = pk.pa_launch_count()
    for i in range(K):
        if flush:
            torch.amax(scratch, dim=0, out=sink)
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize(device)
    t1 = time.time()
    sampler.stop()
    launches = pk.pa_launch_count() - launches0
    assert pk.pa_device_status() == 0
    ms = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    tflops = flops / (ms * 1e-3) / 1e12
    gbs = alg_bytes / (ms * 1e-3) / 1e9
    hbm_peak, hbm_kind = measured_peak_hbm()
    tc_peak, tc_kind = measured_peak_tensor()
    tensor_bound = tflops / tc_peak > gbs / hbm_peak
    return {
        "metric": "multi-query paged attention: TFLOP/s (tensor-bound work) or KV GB/s (HBM-bound)",
        "op": "mq",
        "value": round(tflops if tensor_bound else gbs, 2),
        "unit": "TFLOP/s" if tensor_bound else "GB/s",
        "n_gpus": 1, "steps": K, "warmup": max(3, args.warmup), "ms_per_step": round(ms, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": spec.dtype,
        "data": "synthetic: seeded N(0,1) K/V/q, context lengths and placement as the workload states",
        "config": {"workload": f"{args.workload}: {MQ_WORKLOADS[args.workload.replace('_quarter', '')][2]}",
                   "num_seqs": len(sc.batch), "query_tokens": T, "query_tokens_per_seq": Q,
                   "max_context_len": max_ctx, "partition_size": P or "automatic",
                   "kv_bytes_unique": unique, "flops": flops,
                   "l2": "L2 flushed between timed steps" if flush else "inputs larger than L2"},
        "tflops": round(tflops, 2), "kv_gbs": round(gbs, 2),
        "roofline": {"kernel": ("decode_partition_tc_kernel, several queries (+ reduce)"
                               if Q * spec.G <= 64 and spec.G in (4, 8)
                               else "decode_mq_kernel (+ reduce)"),
                     "bound": "tensor" if tensor_bound else "hbm",
                     "achieved": round(tflops if tensor_bound else gbs, 2),
                     "peak": tc_peak if tensor_bound else hbm_peak,
                     "peak_kind": tc_kind if tensor_bound else hbm_kind,
                     "unit": "TFLOP/s" if tensor_bound else "GB/s",
                     "frac": round(tflops / tc_peak if tensor_bound else gbs / hbm_peak, 4),
                     "other_frac": round(gbs / hbm_peak if tensor_bound else tflops / tc_peak, 4)},
        "gpu_launches": int(launches),
        "clocks": sampler.summary(t0, t1),
    }


def run_swap(args):
    """Swap-out / swap-in bandwidth of pa_swap_blocks on the workload's blocks."""
    import torch
    import paged_kv_cache_443_b200 as pk

    if not torch.cuda.is_available():
        raise SystemExit("bench.py: a CUDA device is required for --op swap")
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    pk.lib()
    spec = workload_spec(args.workload)
    sc = W.scenario(spec)
    dt = W.torch_kv_dtype(spec)
    shape = (sc.num_blocks, spec.Hkv, spec.block_size, spec.D)
    kc = torch.randn(shape, dtype=torch.float32, device=device).to(dt)
    vc = torch.randn(shape, dtype=torch.float32, device=device).to(dt)
    # the batch's blocks: the live ids of the scenario's block tables, in table order
    cache_ids = []
    bm = pk.BlockAllocator(sc.num_blocks, spec.block_size, sc.free_order.tolist())
    for op in sc.setup_ops + sc.step_ops:
        if op.kind == "add":
            bm.add(op.seq)
        elif op.kind == "fork":
            bm.fork(op.seq, op.arg)
        elif op.kind == "release":
            bm.release(op.seq)
        else:
            bm.append(op.seq, op.arg)
    t, _ = bm.build_tables(sc.batch, sc.max_blocks)
    seen = set()
    for x in t.ravel():
        if x >= 0 and int(x) not in seen:
            seen.add(int(x))
            cache_ids.append(int(x))
    n = len(cache_ids)
    rng = np.random.default_rng(spec.seed)
    host_ids = rng.permutation(n)
    hk = torch.empty((n,) + shape[1:], dtype=dt).pin_memory()
    hv = torch.empty((n,) + shape[1:], dtype=dt).pin_memory()
    out_pairs = torch.tensor(np.stack([cache_ids, host_ids], 1), dtype=torch.int64, device=device)
    in_pairs = torch.tensor(np.stack([host_ids, cache_ids], 1), dtype=torch.int64, device=device)
    block_bytes = spec.Hkv * spec.block_size * spec.D * spec.kv_esize
    moved = 2 * n * block_bytes                      # K and V, one direction
    stream = torch.cuda.current_stream(device)
    flat_d = torch.empty(moved, dtype=torch.uint8, device=device)
    flat_h = torch.empty(moved, dtype=torch.uint8).pin_memory()

    def timed(fn, K):
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(K):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(device)
        return e0.elapsed_time(e1) / K

    K = max(1, min(args.steps, 20))
    sampler = ClockSampler(0)
    sampler.start()
    t0 = time.time()
    launches0 = pk.pa_launch_count()
    out_ms = timed(lambda: pk.pa_swap_blocks(hk, hv, kc, vc, out_pairs, stream=stream), K)
    in_ms = timed(lambda: pk.pa_swap_blocks(kc, vc, hk, hv, in_pairs, stream=stream), K)
    launches = pk.pa_launch_count() - launches0
    d2h_ms = timed(lambda: flat_h.copy_(flat_d, non_blocking=True), K)
    h2d_ms = timed(lambda: flat_d.copy_(flat_h, non_blocking=True), K)
    t1 = time.time()
    sampler.stop()
    assert pk.pa_device_status() == 0, "device-side check failed"
    # round trip restores the cache bit for bit
    ref_k = kc.clone()
    pk.pa_swap_blocks(hk, hv, kc, vc, out_pairs, stream=stream)
    kc.zero_()
    pk.pa_swap_blocks(kc, vc, hk, hv, in_pairs, stream=stream)
    torch.cuda.synchronize(device)
    ids = torch.tensor(cache_ids, device=device)
    assert torch.equal(kc.index_select(0, ids).view(torch.uint8),
                       ref_k.index_select(0, ids).view(torch.uint8))
    gbs = lambda ms: moved / (ms * 1e-3) / 1e9  # noqa: E731
    rt_ms = out_ms + in_ms
    return {
        "metric": "swap_blocks GB/s, device <-> pinned host (K and V blocks, each direction)",
        "op": "swap",
        "value": round(2 * moved / (rt_ms * 1e-3) / 1e9, 2),
        "unit": "GB/s",
        "n_gpus": 1, "steps": K, "warmup": max(3, args.warmup),
        "ms_per_step": round(rt_ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": spec.dtype, "data": "synthetic N(0,1) blocks",
        "config": {"workload": f"{args.workload}: {workload_text(args.workload)}",
                   "blocks": n, "block_bytes_per_cache": block_bytes,
                   "bytes_per_direction": moved, "host_ids": "random permutation"},
        "swap_out": {"ms": round(out_ms, 4), "GB/s": round(gbs(out_ms), 2)},
        "swap_in": {"ms": round(in_ms, 4), "GB/s": round(gbs(in_ms), 2)},
        "contiguous_copy": {"d2h_GB/s": round(gbs(d2h_ms), 2), "h2d_GB/s": round(gbs(h2d_ms), 2)},
        "roofline": {"bound": "link", "achieved": round(2 * moved / (rt_ms * 1e-3) / 1e9, 2),
                     "peak": round(2 * moved / ((d2h_ms + h2d_ms) * 1e-3) / 1e9, 2),
                     "peak_kind": "contiguous cudaMemcpyAsync of the same bytes, measured here",
                     "unit": "GB/s", "frac": round((d2h_ms + h2d_ms) / rt_ms, 4)},
        "gpu_launches": int(launches),
        "clocks": sampler.summary(t0, t1),
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=["tiny", "opt13b", "opt13b_compact", "llama13b_ps", "gqa70b",
                             "long_prefix_bs8", "long_prefix_bs16", "long_prefix_bs32",
                             "gqa70b_quarter", "long_prefix_bs8_quarter",
                             "long_prefix_bs16_quarter", "opt13b_fp8", "opt13b_compact_fp8",
                             "gqa70b_fp8", "gqa70b_quarter_fp8", "long_prefix_bs8_fp8",
                             "long_prefix_bs16_fp8", "long_prefix_bs32_fp8",
                             "long_prefix_bs16_quarter_fp8", "llama13b_ps_fp8", "tiny_fp8",
                             "verify_gqa70b", "verify2_gqa70b", "prefill_gqa70b",
                             "verify_gqa70b_quarter",
                             "prefill_gqa70b_quarter"])
    ap.add_argument("--partition-size", type=int, default=0,
                    help="split-K partition length (0: the workload's own, 512)")
    ap.add_argument("--soak-seconds", type=float, default=0.5,
                    help="untimed load before the timed steps (clock samples)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--op", default="decode", choices=["decode", "swap", "mq"],
                    help="decode: the hot path (default); swap: block swap bandwidth")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--grouped", default="auto", choices=["auto", "on", "off"],
                    help="decode families sharing leading blocks with pa_decode_grouped "
                         "(auto: for parallel-sampling and shared-prefix workloads)")
    ap.add_argument("--record-traffic", metavar="CSV",
                    help="no run: record the DRAM bytes of one call from an ncu CSV into "
                         "profiles/dram_traffic.json for --workload, --traffic-kernel and "
                         "--partition-size")
    ap.add_argument("--traffic-kernel", choices=sorted(KERNEL_SOURCES), default="decode_grouped")
    args = ap.parse_args()
    if args.record_traffic:
        print(json.dumps(record_traffic(args.record_traffic, args.workload, args.traffic_kernel,
                                        args.partition_size)))
        return
    args.warmup = max(3, args.warmup)
    rank, world, _ = dist_env()

    if args.impl == "reference":
        if rank != 0:
            return
        spec = workload_spec(args.workload)
        per_step = max(0.02, 60.0 / (args.steps + args.warmup))
        time_oracle(spec, steps=args.warmup, per_step_budget_s=per_step)  # untimed warm-up
        gbs, sec, threads, desc = time_oracle(spec, steps=args.steps, per_step_budget_s=per_step)
        line = {
            "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(sec * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (same generators as the GPU arm)",
            "config": {"workload": f"{args.workload}: {workload_text(args.workload)}"},
            "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": threads,
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0,
        }
        print(json.dumps(line), flush=True)
        return

    if args.op == "swap":
        if rank == 0 and args.impl == "ours":
            print(json.dumps(run_swap(args)), flush=True)
        return
    if args.op == "mq":
        if rank == 0 and args.impl == "ours":
            print(json.dumps(run_mq(args)), flush=True)
        return

    result = run_ours(args)
    if rank == 0 and result is not None:
        if world == 1 and not args.no_cpu_baseline:
            gbs, sec, threads, desc = time_oracle(workload_spec(args.workload), budget_s=15.0)
            result["cpu_baseline"] = {"value": round(gbs, 4), "unit": "GB/s", "cores": threads,
                                      "kind": "oracle", "sample": desc}
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

"""Benchmark: ZipNN-style compress + decompress of a 7B-shaped BF16 checkpoint on B200.

One step = zipnn_compress of each of the 225 tensors of the checkpoint (6,607,077,376
BF16 values, 13.21 GB), issued round-robin on 8 CUDA streams (one workspace each), then
one zipnn_decompress_batch over all 225 containers.
The metric is GB/s of uncompressed bytes; `value` is the round-trip rate (uncompressed
bytes / (compress time + decompress time)) summed over all ranks, and the JSON line
also carries each direction and its fraction of the HBM roofline (algorithmic bytes
read + written / time), against the measured copy bandwidth and against the nominal
8 TB/s.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun (N > 1) the checkpoint is N times as wide (every tensor has N times the
rows) and rank r holds chunks [r * C_t, (r + 1) * C_t) of each tensor t, C_t being the
chunks of the one-GPU tensor: weak scaling, every rank compresses the same amount. Each
step ends the compress half with the one exchange the path has: the payload sizes of the
rank's 225 shards (zipnn_shard_sizes), one all-gather of them (225 u64 per rank), and
the relocation of the rank's chunk tables into the whole containers (zipnn_shard_tables).
At N = 1 the same calls run without the all-gather. Time is the max over ranks.
"""
import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np
import torch

METRIC = "decompress/compress GB/s (uncompressed) at 1 B200; % of HBM roofline"
WORKLOAD = ("BF16 7B-shaped checkpoint: 32 x [q,k,v,o 4096x4096; gate,up,down 4096x11008] + embedding "
            "32000x4096, 225 tensors, 6,607,077,376 values (13.21 GB), sigma_t log-uniform [0.005, 0.05], "
            "256 KiB chunks; compress: one zipnn call per tensor, tensors spread round-robin over {ns} streams")
CHUNK = 262144
SUBBLOCK = 512  # the library default (include/zipnn.h)
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # the B200 figure the metric names ("about 8 TB/s")


# ------------------------------------------------------------------ distributed helpers

def dist_env():
    """(rank, world, local_rank) from the torchrun environment; (0, 1, 0) without it."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(world, backend):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(value, world, device):
    """Max of a float over all ranks (identity for one rank)."""
    if world == 1:
        return float(value)
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def rank_seed(rank):
    """Each rank compresses its own checkpoint: the generator seeds shift by rank."""
    return 1000003 * rank


# ------------------------------------------------------------------ measurement helpers

# ncu summaries under profiles/ that give a kernel's DRAM bytes per value; each names the
# kernel sources it was taken from, by hash, so a summary of an older kernel is not used
PROFILE_OF = {"decode_merge": "decode_merge_embedding_bf16.txt", "encode": "encode_bf16_embedding_bf16.txt",
              "split_hist": "split_hist_embedding_bf16.txt", "code_build": "build_chunks_embedding_bf16.txt"}


def code_digest(files, csrc=None):
    """sha256 over the code of the given source files (sorted by name; in the package's csrc
    unless `csrc` names another folder), comments removed and runs of white space made one
    space: a change to the code changes it, a change to a comment or to the layout does not."""
    import hashlib
    import re
    csrc = csrc or os.path.join(ROOT, "lossless_float_weight_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(files):
        with open(os.path.join(csrc, f)) as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(re.sub(r"\s+", " ", text).strip().encode())
        h.update(b"\0")
    return h.hexdigest()


def profile_traffic(kernel, values_per_launch):
    """DRAM bytes of one launch of `kernel`, from its committed ncu summary scaled by the values
    the launch processes; None without a summary or when the kernel's code changed since."""
    import re
    name = PROFILE_OF.get(kernel)
    path = os.path.join(ROOT, "profiles", name) if name else None
    if not path or not os.path.exists(path):
        return None
    text = open(path).read()
    bpv = re.search(r"DRAM bytes per value\s+([0-9.]+)", text)
    src = re.search(r"kernel code sha256 \(([^)]*)\): ([0-9a-f]{64})", text)
    if not bpv or not src:
        return None
    if code_digest(src.group(1).split()) != src.group(2):
        return None
    return round(float(bpv.group(1)) * values_per_launch)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle samples every 50 ms while running."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def wait_first(self, timeout_s=3.0):
        """Wait (bounded) until nvidia-smi has printed its first sample, so that a short
        timed region that starts now is sampled."""
        t0 = time.time()
        while self.proc is not None and not self.lines and time.time() - t0 < timeout_s:
            time.sleep(0.01)

    def mark(self):
        return len(self.lines)

    def stop(self, lo=None, hi=None):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        mhz, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        # the samples taken while the timed region ran (lo..hi), plus the one just after it;
        # all of them when the region was too short to catch any
        window = self.lines[lo:hi + 1] if lo is not None and hi is not None and hi + 1 > lo else []
        for ln in window or self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                mhz.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        mhz.sort()
        return {"sm_mhz": mhz[len(mhz) // 2] if mhz else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(mhz)}


# ------------------------------------------------------------------ our arm

def make_workload(device, rank, tensors=None, only=None):
    """Rank r's slice of every tensor of the (N-times-wider) checkpoint: the one-GPU
    tensor's shape, its values drawn from the tensor's seed shifted by rank_seed(r)."""
    from lossless_float_weight_b200 import workloads as W
    shapes = W.checkpoint_7b_shapes()
    sig = W.checkpoint_7b_sigmas(len(shapes))
    pick = [only] if only is not None else list(range(len(shapes)))[:tensors]
    return [W.checkpoint_7b_tensor(t + rank_seed(rank), shapes[t][1], sig[t], device).reshape(-1) for t in pick]


def _oracle_leg(oracle, dtype, pieces, threads, budget_s, plan_lens=None):
    """Time the oracle's compress and decompress over host pieces (uint8 numpy arrays, each
    a whole number of chunks of its tensor) until budget_s seconds of work are done."""
    done, t_c, t_d, used = 0, 0.0, 0.0, 0
    for h in pieces:
        n = oracle.values_in(dtype, h.size)
        t0 = time.perf_counter()
        c = oracle.compress(dtype, h, n, CHUNK, SUBBLOCK, plan_lens=plan_lens, threads=threads)
        t1 = time.perf_counter()
        y = oracle.decompress(dtype, c, n, CHUNK, threads=threads)
        t2 = time.perf_counter()
        assert np.array_equal(y, h)
        t_c += t1 - t0
        t_d += t2 - t1
        done += h.size
        used += 1
        if t_c + t_d > budget_s:
            break
    return done, t_c, t_d, used


def _slices(x, piece_bytes):
    """Host pieces of a device tensor, each piece_bytes (whole chunks) or the rest."""
    flat = x.reshape(-1).view(torch.uint8)
    for lo in range(0, flat.numel(), piece_bytes):
        yield flat[lo: lo + piece_bytes].cpu().numpy()


def cpu_baseline(xs, dev, budget_all=5.0, budget_one=6.0):
    """The oracle as it stands on this host's cores (a reported baseline, not the target),
    on bounded samples of every workload: (i) one thread on the 2 MiB BF16 tensor, FP32,
    FP8 and the first two layers of the checkpoint; (ii) all threads (chunk-parallel) on
    all five workloads. Each leg stops after its time budget; `sample` says how much of
    the workload it covered. `value` is the checkpoint leg on all threads."""
    import oracle
    from lossless_float_weight_b200 import workloads as W
    threads = os.cpu_count() or 1
    legs = []

    def leg(config, dtype, pieces, nthreads, budget, total_bytes, plan_lens=None, note=""):
        done, t_c, t_d, used = _oracle_leg(oracle, dtype, pieces, nthreads, budget, plan_lens)
        legs.append({"config": config, "threads": nthreads, "bytes": done,
                     "sample": f"{done / 1e9:.3f} of {total_bytes / 1e9:.3f} GB{note}",
                     "compress_GBps": round(done / t_c / 1e9, 4), "decompress_GBps": round(done / t_d / 1e9, 4),
                     "roundtrip_GBps": round(done / (t_c + t_d) / 1e9, 4)})
        return legs[-1]

    small = W.bf16_small().view(torch.uint8).numpy()
    ckpt = lambda: (x.view(torch.uint8).cpu().numpy() for x in xs)  # noqa: E731
    two_layers = lambda: (x.view(torch.uint8).cpu().numpy() for x in xs[:14])  # noqa: E731
    ckpt_bytes = sum(x.numel() * 2 for x in xs)
    piece = 64 << 20
    fp32 = W.fp32_tensor(n=268435456, device=dev)
    fp8 = W.fp8_tensor(rows=262144, cols=4096, device=dev)
    # (i) one thread
    leg("1: BF16 1,048,576 values", "bf16", [small], 1, budget_one, small.size)
    leg("2: BF16 7B checkpoint, first 2 layers (subset)", "bf16", two_layers(), 1, budget_one,
        sum(x.numel() * 2 for x in xs[:14]), note=" (layers 0-1 only)")
    leg("3: FP32 268,435,456 values", "fp32", _slices(fp32, piece), 1, budget_one, fp32.numel() * 4)
    leg("4: FP8 E4M3 262,144 x 4096", "fp8_e4m3", _slices(fp8, piece), 1, budget_one, fp8.numel())
    # (ii) every thread
    leg("1: BF16 1,048,576 values", "bf16", [small], threads, budget_all, small.size)
    main = leg("2: BF16 7B checkpoint", "bf16", ckpt(), threads, 3 * budget_all, ckpt_bytes)
    leg("3: FP32 268,435,456 values", "fp32", _slices(fp32, 4 * piece), threads, budget_all, fp32.numel() * 4)
    clean = fp32.to(torch.bfloat16).to(torch.float32)
    del fp32
    leg("3: FP32 clean (rounded through BF16)", "fp32", _slices(clean, 4 * piece), threads, budget_all,
        clean.numel() * 4)
    del clean
    leg("4: FP8 E4M3 262,144 x 4096", "fp8_e4m3", _slices(fp8, 4 * piece), threads, budget_all, fp8.numel())
    del fp8
    kv = W.kv_cache(device=dev)
    kv_sample = kv[: (1 << 30) // 2].view(torch.uint8).cpu().numpy()  # the first 1 GiB: 4096 chunks
    kv_total = kv.numel() * 2
    del kv
    lens, _, _, _ = oracle.plan_build("bf16", kv_sample, groups=8, seed=0)
    leg("5: BF16 K/V cache, 8-group plan (built by the oracle on the sample, not timed)", "bf16",
        (kv_sample[lo: lo + 4 * piece] for lo in range(0, kv_sample.size, 4 * piece)), threads, budget_all,
        kv_total, plan_lens=lens)
    return {
        "value": main["roundtrip_GBps"], "unit": "GB/s", "cores": threads, "kind": "oracle",
        "compress_GBps": main["compress_GBps"], "decompress_GBps": main["decompress_GBps"],
        "sample": f"checkpoint leg: {main['sample']} (first tensors in order), compress+decompress, "
                  f"{threads} threads (chunk-parallel); every leg below is a bounded sample",
        "legs": legs,
    }


def bench_config(args, world, nbytes):
    """The `config` of the JSON line: the workload and how a step runs (both arms)."""
    return {
        "workload": WORKLOAD.format(ns=args.streams),
        "step": "compress all 225 tensors (one zipnn_compress each), then decompress all 225 ("
                + ("one zipnn_decompress each" if args.per_tensor_decode else "one zipnn_decompress_batch")
                + ") (value = uncompressed bytes per step / step time, x ranks)",
        "global_batch": world * nbytes,
        "parallelism": (f"weak scaling over {world} rank(s): each rank holds a contiguous chunk range of every tensor of "
                        f"a checkpoint {world}x as wide; per step one all-gather of the 225 shard payload sizes "
                        "(u64, the only exchange) and the relocation of the rank's chunk tables into the whole "
                        "containers" if world > 1 else
                        "one GPU; the shard-size and chunk-table steps run as they do on N GPUs, without the "
                        "all-gather"),
        "l2": "inputs larger than L2 (13.2 GB per rank; no flush needed)",
        "subblock": SUBBLOCK,
        "streams": args.streams,
        "chunk_bytes": CHUNK,
    }


def run_ours(args):
    from lossless_float_weight_b200 import zipnn as Z
    rank, world, local = dist_env()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    init_dist(world, "nccl")
    stream = torch.cuda.current_stream(dev)

    xs = make_workload(dev, rank, args.tensors, args.only)
    nbytes = sum(x.numel() * 2 for x in xs)
    outs = [torch.empty(Z.zipnn_max_compressed_bytes(Z.BF16, x.numel(), CHUNK), dtype=torch.uint8, device=dev)
            for x in xs]
    # tensors go round-robin to NSTREAMS streams, each with its own workspace, so that
    # one tensor's tail overlaps the next tensor's work
    streams = [torch.cuda.Stream(dev) for _ in range(args.streams)]
    wss = [Z.workspace(Z.BF16, max(x.numel() for x in xs), CHUNK, dev) for _ in streams]
    decs = [torch.empty_like(x) for x in xs]
    torch.cuda.synchronize()

    def fan_out(fn):
        ev = torch.cuda.Event()
        ev.record(stream)
        for s in streams:
            s.wait_event(ev)
        for i in range(len(xs)):
            fn(i, streams[i % len(streams)], wss[i % len(streams)])
        for s in streams:
            e2 = torch.cuda.Event()
            e2.record(s)
            stream.wait_event(e2)

    # the shards of one container: rank r holds chunks [r * C_t, (r + 1) * C_t) of tensor t
    from lossless_float_weight_b200 import shard as SH
    n_slice = [x.numel() for x in xs]
    n_totals = [world * n for n in n_slice]
    chunk_los = [rank * -(-n // (CHUNK // 2)) for n in n_slice]
    sizes_buf = torch.empty(len(xs), dtype=torch.int64, device=dev)
    sh_ws = torch.empty(Z.zipnn_shard_workspace_bytes(len(xs)), dtype=torch.uint8, device=dev)
    tables = [torch.empty(SH.table_bytes(Z.BF16, n), dtype=torch.uint8, device=dev) for n in n_slice]
    headers = [torch.empty(64, dtype=torch.uint8, device=dev) if lo == 0 else None for lo in chunk_los]

    def exchange_and_relocate(st):
        SH.shard_sizes(outs, n_totals, chunk_los, stream=st, out=sizes_buf, ws=sh_ws)
        all_sizes = SH.exchange_sizes(sizes_buf)  # NCCL all-gather of 225 u64 per rank (N > 1)
        SH.shard_tables(Z.BF16, outs, n_totals, chunk_los, all_sizes, rank, world, CHUNK, stream=st,
                        tables=tables, headers=headers, ws=sh_ws)

    def compress_all():
        fan_out(lambda i, s, w: Z.compress_into(xs[i], outs[i], w, CHUNK, stream=s))
        exchange_and_relocate(stream)

    bws = Z.batch_workspace(len(xs), dev)

    def decompress_all():
        if args.per_tensor_decode:
            fan_out(lambda i, s, w: Z.decompress_into(outs[i], outs[i].numel(), decs[i], w, CHUNK, stream=s))
        else:  # one launch over all the tensors' chunks
            Z.decompress_batch_into(outs, [o.numel() for o in outs], decs, bws, CHUNK, stream=stream)

    for _ in range(args.warmup):
        compress_all()
        decompress_all()
    torch.cuda.synchronize()
    csizes = [Z.compressed_size(o) for o in outs]
    ok = all(torch.equal(d.view(torch.int16), x.view(torch.int16)) for d, x in zip(decs, xs))
    if not ok:
        raise RuntimeError("round trip mismatch")
    if Z.status(sh_ws) != Z.OK:
        raise RuntimeError("shard tables reported a mismatch")
    if world == 1 and not all(torch.equal(t, o[64: 64 + t.numel()]) for t, o in zip(tables, outs)):
        raise RuntimeError("one shard: the relocated tables must equal the containers' own")
    cbytes = sum(csizes)

    # timed region: K steps, events on the launching stream, kernel events on
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(local)
    # launches of our kernels per step: split+histogram, code build (BF16), layout scan
    # and encode per compress call, decode per decompress call (events count them below)
    barrier(world, dev)
    torch.cuda.synchronize()
    clocks.start()
    clocks.wait_first()
    clk_lo = clocks.mark()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for k in range(args.steps):
        ev[k][0].record(stream)
        compress_all()
        ev[k][1].record(stream)
        decompress_all()
        ev[k][2].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    clk_hi = clocks.mark()
    barrier(world, dev)
    clk = clocks.stop(clk_lo, clk_hi)
    total_ms = max_over_ranks(t_start.elapsed_time(t_end), world, dev)
    comp_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps, world, dev)
    dec_ms = max_over_ranks(sum(e[1].elapsed_time(e[2]) for e in ev) / args.steps, world, dev)
    ms_step = total_ms / args.steps
    ok = all(torch.equal(d.view(torch.int16), x.view(torch.int16)) for d, x in zip(decs, xs))

    # kernel-timing pass: the same K steps on one stream, every launch bracketed by CUDA
    # events on its stream (on several streams launches overlap and their durations
    # would count shared time)
    Z.zipnn_timing_enable(1)
    Z.kernel_times()
    for k in range(args.steps):
        for i in range(len(xs)):
            Z.compress_into(xs[i], outs[i], wss[0], CHUNK, stream=stream)
        exchange_and_relocate(stream)
        if args.per_tensor_decode:
            for i in range(len(xs)):
                Z.decompress_into(outs[i], outs[i].numel(), decs[i], wss[0], CHUNK, stream=stream)
        else:
            Z.decompress_batch_into(outs, [o.numel() for o in outs], decs, bws, CHUNK, stream=stream)
    torch.cuda.synchronize()
    ktimes = Z.kernel_times()
    Z.zipnn_timing_enable(0)

    peak, peak_src = measured_peaks()
    algo_bytes = nbytes + cbytes  # read + written, per direction
    gpu_launches = sum(v[1] for v in ktimes.values())  # the same count as the timed region
    # algorithmic bytes per step of each kernel (reads + writes the method needs)
    kbytes = {"decode_merge": cbytes + nbytes, "encode": nbytes + cbytes, "split_hist": nbytes,
              "code_build": 0, "layout_scan": 0, "shard_tables": 0}
    # dominant kernel: the one with the largest share of device time
    dom = max(ktimes.items(), key=lambda kv: kv[1][0])
    dom_name, (dom_ms, dom_n) = dom
    dom_bytes = kbytes.get(dom_name, 0) * args.steps
    achieved = dom_bytes / (dom_ms / 1e3) / 1e9 if dom_ms > 0 else 0.0

    # end to end through the public API, host buffers (pinned), copies inside the timed region
    e2e = run_e2e(Z, xs, csizes, dev, stream, streams, args, world) if not args.no_extras else None

    if rank == 0:
        cpu = cpu_baseline(xs, dev) if world == 1 and not args.no_extras else None
        line = {
            "metric": METRIC,
            "value": round(world * nbytes / (ms_step / 1e3) / 1e9, 2),
            "unit": "GB/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms_step, 4),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "u32",
            "data": "synthetic (seeded N(0, sigma_t^2) BF16 tensors of a 7B checkpoint's shapes; no trained weights)",
            "config": bench_config(args, world, nbytes),
            "compress": {"GBps": round(world * nbytes / (comp_ms / 1e3) / 1e9, 2), "ms": round(comp_ms, 4),
                         "hbm_frac": round(algo_bytes / (comp_ms / 1e3) / 1e9 / peak, 4),
                         "hbm_frac_nominal_8TBps": round(algo_bytes / (comp_ms / 1e3) / 1e9 / NOMINAL_HBM_GBS, 4)},
            "decompress": {"GBps": round(world * nbytes / (dec_ms / 1e3) / 1e9, 2), "ms": round(dec_ms, 4),
                           "hbm_frac": round(algo_bytes / (dec_ms / 1e3) / 1e9 / peak, 4),
                           "hbm_frac_nominal_8TBps": round(algo_bytes / (dec_ms / 1e3) / 1e9 / NOMINAL_HBM_GBS, 4)},
            "compression_ratio": round(cbytes / nbytes, 5),
            "roofline": {
                "kernel": dom_name,
                "bound": "hbm",
                "achieved": round(achieved, 1),
                "peak": peak,
                "peak_source": peak_src,
                "unit": "GB/s",
                "frac": round(achieved / peak, 4),
                "frac_nominal_8TBps": round(achieved / NOMINAL_HBM_GBS, 4),
                "traffic": profile_traffic(dom_name, nbytes / 2 / len(xs)),
                "traffic_note": "DRAM bytes per launch: the kernel's ncu bytes per value on the embedding tensor "
                                "(profiles/) times the average values per launch; null if the kernel changed since",
                "avg_launch_ms": round(dom_ms / max(1, dom_n), 5),
                "launches": int(dom_n),
                "measured": "CUDA events around every launch of the kernel, single-stream kernel-timing pass of "
                            "the same K steps",
                "algorithmic_bytes_per_step": dom_bytes // max(1, args.steps),
            },
            "kernel_ms_per_step": {k: round(v[0] / args.steps, 4) for k, v in ktimes.items() if v[1]},
            "gpu_launches": int(gpu_launches),
            "e2e": e2e,
            "clocks": clk,
            "roundtrip_ok": bool(ok),
        }
        if cpu is not None:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)


def run_e2e(Z, xs, csizes, dev, stream, streams, args, world):
    """Same metric through the public API with host buffers: pinned host tensors in,
    pinned host tensors out. Every step copies each tensor to the device, compresses
    it, reads its size and copies the container back, then copies each container to
    the device, decompresses it and copies the values back. Tensors go round-robin to the
    streams and the two halves are pipelined (one tensor's upload and compress beside an
    earlier tensor's container round trip and decompress), so host transfers in both
    directions overlap each other and the kernels."""
    nbytes = sum(x.numel() * 2 for x in xs)
    h_in = [x.cpu().pin_memory() for x in xs]
    h_cont = [torch.empty(c, dtype=torch.uint8).pin_memory() for c in csizes]
    h_out = [torch.empty_like(h).pin_memory() for h in h_in]
    d_in = [torch.empty_like(x) for x in xs]
    d_cont = [torch.empty(Z.zipnn_max_compressed_bytes(Z.BF16, x.numel(), CHUNK), dtype=torch.uint8, device=dev)
              for x in xs]
    d_out = [torch.empty_like(x) for x in xs]
    wss = [Z.workspace(Z.BF16, max(x.numel() for x in xs), CHUNK, dev) for _ in streams]
    ns = len(streams)

    lag = 2 * ns  # tensors whose compress is queued before the first one's size is read

    def step():
        ev = torch.cuda.Event()
        ev.record(stream)
        for s in streams:
            s.wait_event(ev)

        def first_half(i):
            s = streams[i % ns]
            with torch.cuda.stream(s):
                d_in[i].copy_(h_in[i], non_blocking=True)
            Z.compress_into(d_in[i], d_cont[i], wss[i % ns], CHUNK, stream=s)

        def second_half(i):
            s = streams[i % ns]
            size = Z.compressed_size(d_cont[i], stream=s)  # waits for this tensor's compress only
            with torch.cuda.stream(s):
                h_cont[i][:size].copy_(d_cont[i][:size], non_blocking=True)
                d_cont[i][:size].copy_(h_cont[i][:size], non_blocking=True)
            Z.decompress_into(d_cont[i], size, d_out[i], wss[i % ns], CHUNK, stream=s)
            with torch.cuda.stream(s):
                h_out[i].copy_(d_out[i], non_blocking=True)

        # a software pipeline: while tensor i uploads and compresses, the container of
        # tensor i - lag goes down and back up and is decompressed, so the two directions
        # of the host link are busy at once
        for i in range(len(xs) + lag):
            if i < len(xs):
                first_half(i)
            if i >= lag:
                second_half(i - lag)
        for s in streams:
            e2 = torch.cuda.Event()
            e2.record(s)
            stream.wait_event(e2)

    steps = max(1, args.steps)
    step()
    torch.cuda.synchronize()
    barrier(world, dev)
    s0, e0 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(steps):
        step()
    e0.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(s0.elapsed_time(e0) / steps, world, dev)
    ok = all(torch.equal(a.view(torch.int16), b.view(torch.int16)) for a, b in zip(h_out, h_in))
    cb = sum(csizes)
    return {"value": round(world * nbytes / (ms / 1e3) / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": nbytes + cb, "d2h_bytes_per_step": cb + nbytes, "ms_per_step": round(ms, 3),
            "steps": steps, "roundtrip_ok": bool(ok)}


# ------------------------------------------------------------------ reference arm (the oracle)

def run_reference(args):
    """The oracle (the plain C definition of the method) on the host cores, on this arm's
    config and metric; each step is a bounded sample of the workload: the seven tensors of
    layer 0 of the checkpoint (386 MB), compressed and decompressed chunk-parallel."""
    rank, world, local = dist_env()
    if rank != 0:
        return
    import oracle
    from lossless_float_weight_b200 import workloads as W
    shapes = W.checkpoint_7b_shapes()
    sig = W.checkpoint_7b_sigmas(len(shapes))
    threads = os.cpu_count() or 1
    layer = [W.checkpoint_7b_tensor(t, shapes[t][1], sig[t], "cpu").reshape(-1) for t in range(7)]
    hs = [x.view(torch.uint8).numpy() for x in layer]
    nb = sum(h.size for h in hs)
    total = sum(math.prod(sh) * 2 for _, sh in shapes)

    def step():
        for x, h in zip(layer, hs):
            c = oracle.compress("bf16", h, x.numel(), CHUNK, SUBBLOCK, threads=threads)
            y = oracle.decompress("bf16", c, x.numel(), CHUNK, threads=threads)
        return y, h

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        y, h = step()
    dt = (time.perf_counter() - t0) / args.steps
    assert np.array_equal(y, h)
    v = nb / dt / 1e9
    sample = (f"layer 0 of the checkpoint (7 tensors, {nb / 1e6:.1f} MB of {total / 1e9:.2f} GB, generated on the "
              f"host) per step, compress+decompress, {threads} threads (chunk-parallel)")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "u32", "data": "synthetic",
        "config": bench_config(args, world, total),
        "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_plan_transfer(args):
    """Shared-code setup reuse ("NeuralZip: Reusable Setup for Fast Lossless Compression",
    abstract: a setup transferred to other weights and reused as they evolve). A plan is
    built once on layers 0-15 of the checkpoint (one tensor, their concatenation), then
    layers 16-31 are compressed with it, as they are and with 5% relative noise added
    (weights after further training). Reports the size against per-chunk codes, the
    fraction of chunks that fall back to a local code, the setup time and the compress
    throughput with and without the plan (on --streams streams, as the main benchmark)."""
    from lossless_float_weight_b200 import workloads as W
    from lossless_float_weight_b200 import zipnn as Z
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    shapes = W.checkpoint_7b_shapes()
    sig = W.checkpoint_7b_sigmas(len(shapes))
    per_layer = 7
    a_ids, b_ids = range(0, 16 * per_layer), range(16 * per_layer, 32 * per_layer)
    a = torch.cat([W.checkpoint_7b_tensor(t, shapes[t][1], sig[t], dev).reshape(-1) for t in a_ids])
    xs = [W.checkpoint_7b_tensor(t, shapes[t][1], sig[t], dev).reshape(-1) for t in b_ids]
    g = torch.Generator(device=dev).manual_seed(99)
    noisy = [(x.float() + 0.05 * float(sig[t]) * torch.randn(x.numel(), generator=g, device=dev)).to(torch.bfloat16)
             for x, t in zip(xs, b_ids)]
    nbytes = sum(x.numel() * 2 for x in xs)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    plan = Z.Plan.create(a, groups=args.groups, seed=0, ws=Z.workspace(Z.BF16, a.numel(), CHUNK, dev))
    ev1.record(stream)
    torch.cuda.synchronize()
    setup_ms = ev0.elapsed_time(ev1)
    del a
    streams = [torch.cuda.Stream(dev) for _ in range(args.streams)]
    wss = [Z.workspace(Z.BF16, max(x.numel() for x in xs), CHUNK, dev) for _ in streams]
    outs = [torch.empty(Z.zipnn_max_compressed_bytes(Z.BF16, x.numel(), CHUNK), dtype=torch.uint8, device=dev)
            for x in xs]

    def compress(tensors, with_plan):
        ev = torch.cuda.Event()
        ev.record(stream)
        for s in streams:
            s.wait_event(ev)
        for i, x in enumerate(tensors):
            Z.compress_into(x, outs[i], wss[i % len(streams)], CHUNK, plan=plan if with_plan else None,
                            stream=streams[i % len(streams)])
        for s in streams:
            e = torch.cuda.Event()
            e.record(s)
            stream.wait_event(e)

    def measure(tensors, with_plan):
        for _ in range(args.warmup):
            compress(tensors, with_plan)
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            compress(tensors, with_plan)
        t1.record(stream)
        torch.cuda.synchronize()
        ms = t0.elapsed_time(t1) / args.steps
        size, huff, local = 0, 0, 0
        for i, x in enumerate(tensors):
            size += Z.compressed_size(outs[i])
            c = -(-x.numel() // (CHUNK // 2))
            table = outs[i][64: 64 + 16 * 2 * c].cpu().numpy().reshape(c, 2, 16)[:, 0]  # exponent entries
            mode = table[:, 0]
            code = table[:, 4:8].copy().view("<u4")[:, 0]
            huff += int((mode == 2).sum())
            local += int(((mode == 2) & (code == 0xFFFFFFFF)).sum())
        # the round trip still holds with the plan
        y = torch.empty_like(tensors[0])
        Z.decompress_into(outs[0], outs[0].numel(), y, wss[0], CHUNK, stream=stream)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), tensors[0].view(torch.int16))
        return {"ratio": round(size / nbytes, 5), "compress_GBps": round(nbytes / (ms / 1e3) / 1e9, 1),
                "ms": round(ms, 3), "fallback_rate": round(local / max(1, huff), 4)}

    own = measure(xs, False)
    reuse = measure(xs, True)
    drift = measure(noisy, True)
    drift_own = measure(noisy, False)
    line = {
        "mode": "plan_transfer",
        "workload": "plan on layers 0-15 of the BF16 7B-shaped checkpoint (6.47 GB, 112 tensors concatenated); "
                    "applied to layers 16-31 (112 tensors, %.2f GB) as generated and with N(0, (0.05 sigma_t)^2) "
                    "added; 256 KiB chunks" % (nbytes / 1e9),
        "groups": args.groups,
        "setup_ms": round(setup_ms, 2),
        "own_codes": own,
        "plan": reuse,
        "plan_ratio_loss_pct": round(100 * (reuse["ratio"] / own["ratio"] - 1), 3),
        "perturbed_own_codes": drift_own,
        "perturbed_plan": drift,
        "perturbed_ratio_loss_pct": round(100 * (drift["ratio"] / drift_own["ratio"] - 1), 3),
        "steps": args.steps,
        "warmup": args.warmup,
        "streams": args.streams,
    }
    print(json.dumps(line), flush=True)


def run_single(args):
    """One tensor of another workload (the parity configs, and FP4 at the FP8 config's
    shape): compress and decompress timed separately, K steps each, CUDA events on one
    stream; inputs resident in HBM and larger than L2. K/V cache: compress with an
    8-group plan built once before the timed region (its setup time reported apart)."""
    from lossless_float_weight_b200 import workloads as W
    from lossless_float_weight_b200 import zipnn as Z
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    w = args.workload
    if w in ("fp32", "fp32_clean"):
        rows = args.rows or 65536
        x = W.fp32_tensor(n=rows * 4096, device=dev, clean=(w == "fp32_clean"))
        desc = f"FP32 {rows * 4096:,} values N(0, 0.02^2)" + (", rounded through BF16" if w == "fp32_clean" else "")
    elif w == "fp8":
        rows = args.rows or 262144
        x = W.fp8_tensor(rows=rows, cols=4096, device=dev)
        desc = f"FP8 E4M3 {rows:,} x 4096, N(0, 1) x per-row scale log-uniform [0.25, 4]"
    elif w == "fp4":
        rows = args.rows or 262144
        x = W.fp4_tensor(rows=rows, cols=4096, device=dev)
        desc = (f"FP4 E2M1 {rows:,} x 4096 ({rows * 4096:,} values), N(0, 1) x per-row scale "
                "log-uniform [0.25, 4]")
    else:
        layers = args.rows or 32
        x = W.kv_cache(shape=(layers, 2, 16, 8, 4096, 128), device=dev)
        desc = f"BF16 K/V cache [{layers}, 2, 16, 8, 4096, 128], per-channel std log-normal, 8-group plan"
        if args.max_pack:
            desc += f", up to {args.max_pack} packed exponents"
    x = x.reshape(-1)
    n = Z.nvalues(x)
    nbytes = x.numel() * x.element_size()
    dt = Z.dtype_code(x.dtype)
    ws = Z.workspace(dt, n, CHUNK, dev)
    out = torch.empty(Z.zipnn_max_compressed_bytes(dt, n, CHUNK), dtype=torch.uint8, device=dev)
    y = torch.empty_like(x)
    plan, setup_ms = None, None
    if w == "kv_cache":
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        plan = Z.Plan.create(x, groups=8, seed=0, ws=ws, max_pack=args.max_pack)
        e1.record(stream)
        torch.cuda.synchronize()
        setup_ms = e0.elapsed_time(e1)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / args.steps

    c_ms = timed(lambda: Z.compress_into(x, out, ws, CHUNK, plan=plan, stream=stream))
    cbytes = Z.compressed_size(out)
    d_ms = timed(lambda: Z.decompress_into(out, cbytes, y, ws, CHUNK, stream=stream))
    # per-kernel device time of one compress and one decompress (events around each launch)
    Z.zipnn_timing_enable(1)
    Z.kernel_times()
    Z.compress_into(x, out, ws, CHUNK, plan=plan, stream=stream)
    Z.decompress_into(out, cbytes, y, ws, CHUNK, stream=stream)
    torch.cuda.synchronize()
    ktimes = {k: round(v[0], 4) for k, v in Z.kernel_times().items() if v[1]}
    Z.zipnn_timing_enable(0)
    ok = torch.equal(y.view(torch.uint8), x.view(torch.uint8)) and Z.status(ws) == Z.OK
    peak, peak_src = measured_peaks()
    algo = nbytes + cbytes
    line = {
        "metric": METRIC, "workload": w, "config": desc, "unit": "GB/s",
        "compress": {"GBps": round(nbytes / (c_ms / 1e3) / 1e9, 2), "ms": round(c_ms, 4),
                     "hbm_frac": round(algo / (c_ms / 1e3) / 1e9 / peak, 4)},
        "decompress": {"GBps": round(nbytes / (d_ms / 1e3) / 1e9, 2), "ms": round(d_ms, 4),
                       "hbm_frac": round(algo / (d_ms / 1e3) / 1e9 / peak, 4)},
        "compression_ratio": round(cbytes / nbytes, 5), "bytes": nbytes, "values": n,
        "peak": peak, "peak_source": peak_src, "steps": args.steps, "warmup": args.warmup,
        "plan_setup_ms": None if setup_ms is None else round(setup_ms, 2), "roundtrip_ok": bool(ok),
        "max_pack": args.max_pack if w == "kv_cache" else None,
        "kernel_ms": ktimes,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--tensors", type=int, default=None,
                    help="only the first T tensors of the checkpoint (small cases for profilers)")
    ap.add_argument("--only", type=int, default=None, help="only tensor IDX of the checkpoint (profiler cases)")
    ap.add_argument("--no-extras", action="store_true", help="skip the e2e and CPU-baseline legs")
    ap.add_argument("--streams", type=int, default=8, help="CUDA streams the tensors are spread over")
    ap.add_argument("--workload", default="checkpoint_7b",
                    choices=["checkpoint_7b", "fp32", "fp32_clean", "fp8", "fp4", "kv_cache"],
                    help="another workload than the benchmark's: one tensor, compress and decompress timed apart")
    ap.add_argument("--rows", type=int, default=None,
                    help="rows of 4096 values for --workload fp32/fp32_clean/fp8/fp4, layers for kv_cache "
                         "(profiler cases; default 65536 FP32, 262144 FP8/FP4, 32 layers)")
    ap.add_argument("--max-pack", type=int, default=0,
                    help="--workload kv_cache: the plan also lists up to this many packed exponents (BF16, <= 15)")
    ap.add_argument("--plan-transfer", action="store_true",
                    help="instead of the benchmark: build a shared-code plan on layers 0-15 and reuse it on 16-31")
    ap.add_argument("--groups", type=int, default=8, help="plan groups for --plan-transfer")
    ap.add_argument("--per-tensor-decode", action="store_true",
                    help="decompress with one zipnn_decompress per tensor (default: one zipnn_decompress_batch)")
    args = ap.parse_args()
    if args.plan_transfer:
        run_plan_transfer(args)
        return
    if args.workload != "checkpoint_7b":
        run_single(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)
    rank, world, _ = dist_env()
    if world > 1:
        import torch.distributed as dist
        if dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

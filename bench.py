#!/usr/bin/env python
"""DF11 block-decode benchmark on B200.

One step = one df11_decompress_async launch decoding a whole Llama-3.1-8B
shaped transformer block (7 matrices, 218,103,808 BF16 weights, one codebook)
from HBM-resident compressed arrays into a BF16 buffer.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]

Metric: (compressed bytes read + 2 bytes x weights written) / kernel time, in
GB/s (1e9), with Gweights/s and the fraction of the measured HBM copy peak.
Multi-GPU (torchrun, one process per GPU): every rank decodes its own block
(seed 1000 + rank); blocks are independent, so there is no collective on the
data path and scaling is weak; the time is the max over ranks.

--impl reference times the CPU oracle (serial bit-by-bit decode) on bounded
samples of the same block, on rank 0 only.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads  # noqa: E402

METRIC = "DF11 decode GB/s (compressed in + BF16 out), Gweights/s, % of B200 HBM peak"
UNIT = "GB/s"
WORKLOAD = "llama8b_block"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 7700.0      # B200 HBM3e, the HGX data-sheet figure (context only)
KERNEL_SRC = os.path.join(ROOT, "huffman_decode_b200", "csrc", "df11_decode.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_kernel_llama8b_block.md")


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--bytes-per-thread", type=int, default=16, choices=[8, 16],
                    help="stream bytes each decoding thread owns (format layout)")
    ap.add_argument("--workload", default=WORKLOAD,
                    choices=sorted(workloads.WORKLOADS) + ["llama8b_model", "llama8b_overlap",
                                                           "llama8b_offload", "llama8b_gemv",
                                                           "llama8b_compress", "llama8b_verify"],
                    help="block to decode (the headline number is llama8b_block); "
                         "llama8b_model = 32 Llama-3.1-8B blocks, each with its own "
                         "codebook, decoded one after another into one buffer; "
                         "llama8b_overlap = those blocks decoded while the previous "
                         "block's matrix products run; llama8b_offload = blocks held "
                         "compressed in pinned host memory, uploaded and decoded in a "
                         "pipeline; llama8b_compress = the GPU compressor on the block; "
                         "llama8b_verify = the CRC-32C check of a resident block")
    ap.add_argument("--blocks", type=int, default=None,
                    help="blocks of the llama8b_model/overlap/offload streams "
                         "(default 32, 8 for offload)")
    ap.add_argument("--tokens", default=None,
                    help="comma-separated token counts of the activations (llama8b_overlap: "
                         "default 1,256,2048,8192; llama8b_gemv: default 1,4,8)")
    ap.add_argument("--runs", type=int, default=10,
                    help="llama8b_overlap: repetitions of every measurement (median and range reported)")
    ap.add_argument("--max-ctas", default="0,148,74",
                    help="llama8b_overlap: comma-separated decode CTA counts (0 = one resident "
                         "wave on every SM; 148 or 74 leave part of the SMs to the products)")
    ap.add_argument("--consumer-priority", type=int, default=-1,
                    help="llama8b_overlap: CUDA priority of the consumer stream (lower = higher)")
    ap.add_argument("--scale-div", type=int, default=1,
                    help="divide every row count of the block (smaller case for profiling)")
    ap.add_argument("--e2e-steps", type=int, default=20,
                    help="steps of the end-to-end measurement (capped at --steps)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-pieces", type=int, default=8,
                    help="end-to-end measurement: the block moves in this many chunk ranges, so "
                         "the copy in of one overlaps the decode and the copy out of others "
                         "(1 = copy everything in, decode, copy everything out)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--flush-l2", action="store_true",
                    help="write a 256 MB buffer before every timed launch and time each launch "
                         "alone (for blocks whose working set fits in the 126 MB L2)")
    ap.add_argument("--cpu-baseline-seconds", type=float, default=10.0)
    ap.add_argument("--min-seconds", type=float, default=1.0,
                    help="repeat the timed K steps until about this much wall time has passed "
                         "(the median repetition is reported)")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the per-configuration measurements of the default run")
    return ap.parse_args()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_hash() -> str:
    with open(KERNEL_SRC, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def profiled_traffic(n_weights: int):
    """DRAM bytes per launch from the committed ncu summary (its
    `dram_bytes_per_weight` line), scaled to this launch's weights, or None
    when the kernel source changed since the counters were taken."""
    try:
        with open(TRAFFIC_FILE) as f:
            text = f.read()
    except OSError:
        return None
    fields = dict(re.findall(r"^([a-z0-9_]+): ([0-9a-f.]+)$", text, re.M))
    if fields.get("kernel_source_sha256_16") != kernel_hash() or "dram_bytes_per_weight" not in fields:
        return None
    return round(float(fields["dram_bytes_per_weight"]) * n_weights)


def make_block(seed: int, scale_div: int = 1, workload: str = WORKLOAD):
    if workload == "llama8b_block":
        return [m for _, m in workloads.llama_block(seed, scale_div=scale_div)]
    if workload == "flux_dit_block":
        return [m for _, m in workloads.flux_block(5000 + (seed - 1000), scale_div=scale_div)]
    return [m for _, m in workloads.WORKLOADS[workload]()]


# ------------------------------------------------------ ranks (replicas)

def rank_seed(rank: int, base: int = 1000, per_rank: int = 1) -> int:
    """First block seed of a rank: ranks decode disjoint, independent blocks
    (replicas, no data exchange)."""
    return base + rank * per_rank


def reduce_over_ranks(maxima, sums, device=None):
    """Max-reduce `maxima` (timings) and sum-reduce `sums` (bytes, weights)
    over all ranks; identity without an initialised process group.  Works on
    NCCL (device tensors) and gloo (CPU tensors)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(x) for x in maxima], [float(x) for x in sums]
    t = torch.tensor([float(x) for x in maxima], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    c = torch.tensor([float(x) for x in sums], dtype=torch.float64, device=device)
    dist.all_reduce(c, op=dist.ReduceOp.SUM)
    return t.tolist(), c.tolist()


def job_rate(job_units: float, steps: int, ms_max: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's device time (units per second / 1e9)."""
    return job_units * steps / (ms_max * 1e-3) / 1e9


# ----------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML during the timed
    region (background thread, ~5 ms period)."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int):
        self.samples = []
        self.reason_bits = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
            self._reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        except Exception:
            self.nvml = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nvml.nvmlDeviceGetClockInfo(self.handle, self.nvml.NVML_CLOCK_SM))
                self.reason_bits |= int(self._reasons(self.handle))
            except Exception:
                pass
            time.sleep(0.005)

    def start(self):
        if self.nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()
        reasons = [n for b, n in self.REASONS.items() if self.reason_bits & b and b != 0x1]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples)}


# ------------------------------------------------------- CPU oracle legs

def oracle_sample_plan(ob, n_slices: int, threads_per_chunk: int = 32, slice_bits: int = 64):
    """Split the oracle artifact into n_slices runs of whole chunks; each run
    decodes serially from its first code start."""
    bounds = np.linspace(0, ob.n_chunks, n_slices + 1).astype(np.int64)
    plan = []
    for a, b in zip(bounds[:-1], bounds[1:]):
        if b <= a:
            continue
        g = int(a) * threads_per_chunk
        start_bit = slice_bits * g + int(ob.gap[g])
        plan.append((start_bit, int(ob.pos[a]), int(ob.pos[b] - ob.pos[a])))
    return plan


def time_oracle_decode(oracle, ob, plan_item):
    start_bit, first, count = plan_item
    t0 = time.perf_counter()
    e, _ = oracle.decode(ob.stream, count, ob.lengths, start_bit=start_bit)
    w = oracle.join(e, ob.signmant[first: first + count])
    dt = time.perf_counter() - t0
    return dt, w


def host_cpu():
    """The host's CPU model and logical core count."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "host_logical_cpus": os.cpu_count()}


def pinned_to_one_core(fn):
    """Runs fn() with this process pinned to one core it may use (restoring
    the affinity afterwards); returns (result, core or None)."""
    try:
        old = os.sched_getaffinity(0)
    except (AttributeError, OSError):
        return fn(), None
    core = max(old)
    try:
        os.sched_setaffinity(0, {core})
        return fn(), core
    except OSError:
        return fn(), None
    finally:
        try:
            os.sched_setaffinity(0, old)
        except OSError:
            pass


def cpu_baseline(oracle, hb, cb, bytes_per_weight, seconds):
    """The oracle's serial decode of the whole block (repeated until about
    `seconds` of CPU time, at most 4 passes), on one core (pinned)."""
    def run():
        total_w = 0
        total_t = 0.0
        passes = 0
        while passes < 4 and (passes == 0 or total_t < seconds):
            t0 = time.perf_counter()
            e, _ = oracle.decode(hb.exp_stream, hb.n_elements, cb.lengths())
            oracle.join(e, hb.signmant[: hb.n_elements])
            total_t += time.perf_counter() - t0
            total_w += hb.n_elements
            passes += 1
        return total_w, total_t, passes

    (total_w, total_t, passes), core = pinned_to_one_core(run)
    return {"value": round(total_w * bytes_per_weight / total_t / 1e9, 4), "unit": UNIT,
            "cores": 1, "kind": "oracle",
            "gweights_per_s": round(total_w / total_t / 1e9, 5),
            "pinned_core": core, **host_cpu(),
            "sample": f"{passes} full serial decode pass(es) of the llama8b_block "
                      f"({hb.n_elements} weights each) by the oracle, one thread, "
                      f"{total_t:.1f} s"}


def e2e_plan(hb, pieces):
    """The chunk ranges of a piecewise end-to-end step and, for each, the
    byte spans of the arrays its range decode reads (df11_decompress_range_async:
    stream words plus the 16-byte pad, gaps incl. the next thread's, counts,
    positions incl. the next one,
    sign|mantissa rounded out to 16 bytes).  Returns [(c0, c1, p0, p1,
    [(array, begin, end), ...]), ...] with p0, p1 the output range."""
    n_chunks = int(hb.header.n_chunks)
    pieces = max(1, min(pieces, n_chunks))
    W = 32 * int(hb.header.bytes_per_thread)
    pos = hb.chunk_pos.astype(np.int64)
    cuts = [n_chunks * i // pieces for i in range(pieces + 1)]
    plan = []
    for c0, c1 in zip(cuts[:-1], cuts[1:]):
        p0, p1 = int(pos[c0]), int(pos[c1])
        spans = [("exp_stream", W * c0, min(W * c1 + 16, hb.exp_stream.nbytes)),
                 ("gaps", 16 * c0, min(16 * c1 + 1, hb.gaps.nbytes)),
                 ("counts", 32 * c0, 32 * c1),
                 ("chunk_pos", 4 * c0, 4 * (c1 + 1)),
                 ("signmant", p0 & ~15, min((p1 + 15) & ~15, hb.signmant.nbytes))]
        plan.append((c0, c1, p0, p1, spans))
    return plan


def e2e_pipeline(df11, db, hb, host, out, host_out, err, host_err, pieces, stream, dev):
    """One end-to-end step as a pipeline over `pieces` chunk ranges: range k
    is copied in (its stream words, gaps, positions and sign|mantissa bytes)
    on a copy-in stream, decoded on `stream` (df11_decompress_range_async)
    and its BF16 output copied out on a copy-out stream, so the two PCIe
    directions and the decode overlap.  The step ends on `stream`.  Returns
    (step, host->device bytes, device->host bytes) per step."""
    import torch
    c_in, c_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    cblk = db.c_struct()
    plan = e2e_plan(hb, pieces)
    # the decoder's multi-code table travels with the block's tables
    host_table = db.decode_table.cpu().pin_memory() if db.decode_table is not None else None
    h2d = (host["lut"].numel() + (host_table.numel() if host_table is not None else 0)
           + sum(b - a for *_, spans in plan for _, a, b in spans))
    d2h = 2 * int(hb.chunk_pos[-1]) + 4
    ev_in = [torch.cuda.Event() for _ in plan]
    ev_dec = [torch.cuda.Event() for _ in plan]
    ev_start, ev_end = torch.cuda.Event(), torch.cuda.Event()

    def step():
        ev_start.record(stream)              # after the previous step, on every stream
        c_in.wait_event(ev_start)
        c_out.wait_event(ev_start)
        with torch.cuda.stream(c_in):
            db.tensors["lut"].copy_(host["lut"], non_blocking=True)
            if host_table is not None:
                db.decode_table.copy_(host_table, non_blocking=True)
            for i, (_, _, _, _, spans) in enumerate(plan):
                for name, a, b in spans:
                    db.tensors[name][a:b].copy_(host[name][a:b], non_blocking=True)
                ev_in[i].record(c_in)
        for i, (c0, c1, _, _, _) in enumerate(plan):
            stream.wait_event(ev_in[i])
            df11.decompress_range_async(db, c0, c1, out, err, stream=stream, c_block=cblk)
            ev_dec[i].record(stream)
        with torch.cuda.stream(c_out):
            for i, (_, _, p0, p1, _) in enumerate(plan):
                c_out.wait_event(ev_dec[i])
                host_out[p0:p1].copy_(out[p0:p1], non_blocking=True)
            host_err.copy_(err, non_blocking=True)
            ev_end.record(c_out)
        stream.wait_event(ev_end)

    return step, h2d, d2h


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    mats = make_block(1000)
    n = int(sum(m.size for m in mats))
    ob = oracle.compress_block(mats)
    comp_bytes = (ob.stream.nbytes + ob.gap.size // 2 + ob.thread_count.size + ob.pos.nbytes
                  + (n + 15) // 16 * 16)
    bytes_per_weight = (comp_bytes + 2 * n) / n
    plan = oracle_sample_plan(ob, 64)

    def run():
        for i in range(args.warmup):
            time_oracle_decode(oracle, ob, plan[i % len(plan)])
        total_t = 0.0
        total_w = 0
        for i in range(args.steps):
            dt, _ = time_oracle_decode(oracle, ob, plan[i % len(plan)])
            total_t += dt
            total_w += plan[i % len(plan)][2]
        return total_t, total_w

    (total_t, total_w), core = pinned_to_one_core(run)
    value = total_w * bytes_per_weight / total_t / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_t / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "u8", "data": "synthetic",
        "config": {"workload": WORKLOAD, "n_weights": n, "seed": 1000,
                   "sample_per_step": "1/64 of the block's chunks, decoded serially"},
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
                         "pinned_core": core, **host_cpu(),
                         "sample": f"each step decodes 1/64 of the llama8b_block "
                                   f"(~{n // 64} weights) serially, one thread"},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------ per configuration

# The five configurations of the measured workload list, by name: 1 = one
# 1024x1024 matrix, 2 = the Llama-3.1-8B-shaped block (the headline), 3 =
# 32 such blocks with their own codebooks, 4a/b/c = the adversarial 16 M
# weight blocks, 5 = the FLUX-shaped DiT block.
PER_CONFIG = [("1", "single_1024x1024"), ("2", "llama8b_block"), ("3", "llama8b_model"),
              ("4a", "adversarial_heavy_tail"), ("4b", "adversarial_single_exponent"),
              ("4c", "adversarial_uniform_bits"), ("5", "flux_dit_block")]


def _rates(nbytes, n, us, peak):
    return {"us": round(us, 3), "gb_per_s": round(nbytes / us / 1e3, 2),
            "gweights_per_s": round(n / us / 1e3, 2), "frac": round(nbytes / us / 1e3 / peak, 4)}


def graph_us(launch, k, scrub=None, reps=5):
    """Device time of one `launch` (microseconds), from CUDA-graph replays of
    k back-to-back launches (median of `reps` replays) -- so a launch that
    takes less time than the host needs to issue one is still timed by the
    GPU's clock.  With `scrub` (a tensor larger than the L2), each launch
    follows a write of the whole tensor: the time of a graph of k (scrub,
    launch) pairs minus that of k scrubs alone, i.e. a launch that starts
    from an L2 holding none of its data."""
    import torch
    side = torch.cuda.Stream()
    torch.cuda.synchronize()

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            fn()
        return g

    def run(g):
        out = []
        with torch.cuda.stream(side):
            g.replay()
            torch.cuda.synchronize()
            for _ in range(reps):
                a, b = _events(2)
                a.record(side)
                g.replay()
                b.record(side)
                b.synchronize()
                out.append(a.elapsed_time(b) * 1e3 / k)
        return statistics.median(out)

    if scrub is None:
        return run(capture(lambda: [launch(side) for _ in range(k)]))

    def pairs():
        for i in range(k):
            scrub.fill_(i & 255)
            launch(side)
    t_pairs = run(capture(pairs))
    t_scrub = run(capture(lambda: [scrub.fill_(i & 255) for i in range(k)]))
    return t_pairs - t_scrub


def integrity_figures(df11, dev, stream, hb, db, cb, out, w_dev, ws, scrub, launch, k, peak):
    """The integrity checks on one block, graph-timed like the decode: the
    decode that checks every chunk's sum as it decodes (one launch), the
    CRC-32C list check alone, and the CRC check followed by the plain
    decode (two launches, the block read twice)."""
    import torch
    nbytes = hb.compressed_bytes() + 2 * hb.n_elements
    n = hb.n_elements
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    first = torch.full((1,), -1, dtype=torch.int64, device=dev)
    sums = torch.from_numpy(df11.chunk_sums(hb).view(np.int32)).to(dev)
    crcs = torch.from_numpy(df11.checksum(hb).view(np.int32)).to(dev)

    def verified(st):
        df11.decompress_verified_async(db, out, sums, err, first, stream=st, c_block=cb, workspace=ws)

    def crc_only(st):
        df11.verify_device(db, crcs, err, first, stream=st)

    def crc_then_decode(st):
        crc_only(st)
        launch(st)
    out.zero_()
    verified(stream)
    crc_only(stream)
    torch.cuda.synchronize()
    clean = int(err.item()) == 0 and int(first.item()) == -1
    res = {"bit_exact": bool(torch.equal(out, w_dev)), "clean_block_passes": clean,
           "chunk_sums_bytes": 4 * int(hb.header.n_chunks)}
    res["verified_decode"] = {"back_to_back": _rates(nbytes, n, graph_us(verified, k), peak),
                              "l2_scrubbed": _rates(nbytes, n, graph_us(verified, max(k // 4, 5), scrub=scrub),
                                                    peak)}
    crc_bytes = hb.compressed_bytes()
    us = graph_us(crc_only, k)
    res["crc_check_alone"] = {"us": round(us, 2), "gb_per_s": round(crc_bytes / us / 1e3, 1),
                              "frac_of_peak": round(crc_bytes / us / 1e3 / peak, 4)}
    res["crc_check_then_decode"] = {"back_to_back": _rates(nbytes, n, graph_us(crc_then_decode, k), peak)}
    if int(err.item()) or int(first.item()) != -1:
        res["clean_block_passes"] = False
    return res


def per_config(df11, dev, stream, bpt, peak, headline=None):
    """Every configuration decoded on this GPU, each single block in the slice
    layout the library prefers for it: bit-exactness against the
    input, then its device time per launch from CUDA-graph replays
    (graph_us): back to back, and for single blocks from an L2 scrubbed by a
    256 MB write before each launch.  Config 3 times the 32-block stream
    (one launch = the 32 blocks decoded one after another into one reused
    buffer).  Config 2 also carries the headline's figure (direct launches,
    median repetition under sustained load)."""
    import torch
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = torch.zeros(df11.SCHED_WORKSPACE_BYTES, dtype=torch.uint8, device=dev)
    scrub = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    out_all = {}
    for key, name in PER_CONFIG:
        t0 = time.perf_counter()
        if name == "llama8b_model":
            dbs = numpy_model_blocks(workloads.llama_model_seeds(32), dev, bpt)
            n = sum(db.n_elements for db in dbs)
            nbytes = sum(db.compressed_bytes() + 2 * db.n_elements for db in dbs)
            out = torch.empty(max(db.n_elements for db in dbs), dtype=torch.bfloat16, device=dev)
            cblks = [(db, db.c_struct()) for db in dbs]

            def launch(st):
                for db, cb in cblks:
                    df11.decompress_async(db, out, err, stream=st, c_block=cb, workspace=ws)
            exact = True   # numpy_model_blocks checked every block
            k = 2
        else:
            mats = [m for _, m in workloads.WORKLOADS[name]()]
            w = np.concatenate([m.reshape(-1) for m in mats])
            cbk = df11.build_codebook(mats)
            # each block in the slice layout the library prefers for it
            # (16 bytes for the large blocks, 8 for small or 1-bit-code ones)
            bpt_c = df11.preferred_bytes_per_thread(cbk, sms)
            hb = df11.compress(cbk, mats, 32, bpt_c)
            db = hb.to_device(dev)
            cb = db.c_struct()
            n = hb.n_elements
            nbytes = hb.compressed_bytes() + 2 * n
            out = torch.empty(n, dtype=torch.int16, device=dev)

            def launch(st):
                df11.decompress_async(db, out, err, stream=st, c_block=cb, workspace=ws)
            launch(stream)
            torch.cuda.synchronize()
            w_dev = torch.from_numpy(w.view(np.int16)).to(dev)
            exact = bool(torch.equal(out, w_dev)) and int(err.item()) == 0
            k = 100 if n < 50_000_000 else 20
            if name == "llama8b_block":
                integrity = integrity_figures(df11, dev, stream, hb, db, cb, out, w_dev, ws, scrub, launch, k, peak)
            del w, hb, w_dev
        setup_s = time.perf_counter() - t0
        entry = {"workload": name, "n_weights": n, "bytes_per_launch": nbytes, "bit_exact": exact,
                 "bytes_per_thread": bpt if name == "llama8b_model" else bpt_c, "setup_s": round(setup_s, 1)}
        entry["back_to_back"] = _rates(nbytes, n, graph_us(launch, k), peak)
        if name != "llama8b_model":
            entry["l2_scrubbed"] = _rates(nbytes, n, graph_us(launch, max(k // 4, 5), scrub=scrub), peak)
        else:
            entry["what"] = "one launch = the 32 blocks decoded one after another (us per 32 blocks)"
        if name == "llama8b_block" and headline is not None:
            entry["headline_direct_launches"] = _rates(nbytes, n, headline, peak)
        if name == "llama8b_block":
            entry["integrity"] = integrity
            integrity = None
        if int(err.item()):
            entry["bit_exact"] = False
        out_all[key] = entry
        del out
        torch.cuda.synchronize()
    return out_all


# -------------------------------------------------------------- GPU arm

def run_b200(args):
    import torch
    import torch.distributed as dist

    import huffman_decode_b200 as df11

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    seed = rank_seed(rank)
    mats = make_block(seed, args.scale_div, args.workload)
    t0 = time.perf_counter()
    cb = df11.build_codebook(mats)
    hb = df11.compress(cb, mats, 32, args.bytes_per_thread)
    compress_s = time.perf_counter() - t0
    if df11.validate(hb) != 0:
        raise RuntimeError("compressed block failed validation")
    n = hb.n_elements
    comp_bytes = hb.compressed_bytes()
    bytes_per_step = comp_bytes + 2 * n

    db = hb.to_device(dev)
    out = torch.empty(n, dtype=torch.bfloat16, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    hb_bits = np.concatenate([m.reshape(-1) for m in mats]).view(np.int16)
    want = torch.from_numpy(hb_bits).to(dev)
    stream = torch.cuda.current_stream(dev)
    cblk = db.c_struct()

    def step():
        df11.decompress_async(db, out, err, stream=stream, c_block=cblk)

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    bit_exact = bool(torch.equal(out.view(torch.int16), want)) and int(err.item()) == 0
    if not bit_exact:
        raise RuntimeError("decode is not bit-exact; refusing to report a number")
    del want

    sampler = ClockSampler(local)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if args.flush_l2:
        # every launch starts from an L2 holding none of its data; only the
        # launches are timed (one event pair each)
        scrub = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for a, b in evs:
            scrub.fill_(1)
            a.record(stream)
            step()
            b.record(stream)
        torch.cuda.synchronize()
        ms = sum(a.elapsed_time(b) for a, b in evs)
        del scrub
        reps = None
    else:
        ms, reps = timed_reps(step, args.steps, stream, world, min_seconds=args.min_seconds, device=dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = sampler.stop()

    # ---- end to end: pinned host arrays -> device, decode, BF16 -> host
    e2e = None
    if not args.no_e2e:
        k = max(1, min(args.e2e_steps, args.steps))
        host = {name: torch.from_numpy(a.view(np.uint8)).pin_memory() for name, a in hb.arrays().items()}
        host_out = torch.empty(n, dtype=torch.bfloat16, pin_memory=True)
        host_err = torch.empty(1, dtype=torch.int32, pin_memory=True)
        e2e_step, h2d, d2h = e2e_pipeline(df11, db, hb, host, out, host_out, err, host_err,
                                          max(1, args.e2e_pieces), stream, dev)
        e2e_step()
        torch.cuda.synchronize()
        if not torch.equal(host_out.view(torch.int16), torch.from_numpy(hb_bits)) or int(host_err.item()):
            raise RuntimeError("end-to-end decode is not bit-exact")
        s2 = torch.cuda.Event(enable_timing=True)
        e2 = torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        s2.record(stream)
        for _ in range(k):
            e2e_step()
        e2.record(stream)
        e2.synchronize()
        e2e_ms = s2.elapsed_time(e2)
        e2e = {"ms": e2e_ms, "k": k, "h2d": h2d, "d2h": d2h}

    # ---- max over ranks, bytes summed over ranks
    (ms_max, e2e_ms_per_step), (job_bytes, job_weights) = reduce_over_ranks(
        [ms, e2e["ms"] / e2e["k"] if e2e else 0.0], [bytes_per_step, n], dev)

    per_cfg = None
    if (rank == 0 and world == 1 and not args.no_per_config and args.workload == WORKLOAD
            and args.scale_div == 1 and not args.flush_l2):
        peak_, _ = measured_peaks()
        per_cfg = per_config(df11, dev, stream, args.bytes_per_thread, peak_,
                             headline=ms / args.steps * 1e3)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        cpu = cpu_baseline(oracle, hb, cb, bytes_per_step / n, args.cpu_baseline_seconds)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    ms_per_step = ms_max / args.steps
    value = job_rate(job_bytes, args.steps, ms_max)
    peak, peak_kind = measured_peaks()
    launch_s = ms / args.steps * 1e-3              # this rank's own kernel time per launch
    achieved = bytes_per_step / launch_s / 1e9
    traffic = profiled_traffic(n)
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "u8", "data": "synthetic",
        "config": {"workload": args.workload if args.scale_div == 1 else f"{args.workload}/rows{args.scale_div}",
                   "n_weights": n, "n_matrices": len(mats),
                   "seed": seed, "threads_per_chunk": 32, "bytes_per_thread": args.bytes_per_thread,
                   "bits_per_weight": round(8 + cb.total_bits / n, 4),
                   "compressed_bytes": comp_bytes, "bytes_per_step": bytes_per_step,
                   "l2": ("L2 flushed (256 MB written) before every timed launch, launches timed alone"
                          if args.flush_l2 else
                          "%s (%.3f GB touched per step vs 126 MB L2), no flush"
                          % ("inputs larger than L2" if bytes_per_step > 126e6 else
                             "working set fits in L2: an L2-resident figure", bytes_per_step / 1e9)),
                   "parallelism": f"replicas x{world}, one block per GPU, no collective"},
        "gweights_per_s": round(job_rate(job_weights, args.steps, ms_max), 2),
        "pct_of_hbm_peak": round(100 * value / world / peak, 2),
        "pct_of_nominal_hbm": round(100 * value / world / NOMINAL_HBM_GBS, 2),
        "bit_exact": bit_exact,
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak,
                     "peak_source": peak_kind, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": traffic, "algorithmic_bytes_per_launch": bytes_per_step},
        "clocks": clocks,
        "gpu_launches": args.steps,
        "host_compress_s": round(compress_s, 3),
    }
    if e2e:
        line["e2e"] = {"value": round(job_bytes / (e2e_ms_per_step * 1e-3) / 1e9, 2), "unit": UNIT,
                       "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                       "ms_per_step": round(e2e_ms_per_step, 4), "steps": e2e["k"],
                       "pieces": max(1, args.e2e_pieces),
                       "what": "pinned host arrays -> device, decode, BF16 + error word -> pinned host, "
                               "as a pipeline over chunk ranges (df11_decompress_range_async)"}
    if reps:
        line["timing"] = reps
    if cpu:
        line["cpu_baseline"] = cpu
    if per_cfg:
        line["per_config"] = per_cfg
    print(json.dumps(line), flush=True)
    return 0


def gpu_compressed_blocks(n_blocks, seed0, dev, bpt, verify_into=None, scale_div=1):
    """n_blocks Llama-3.1-8B-shaped blocks drawn on the GPU (seeds seed0..),
    each histogrammed, given its own codebook and compressed on the GPU.
    Every block is decoded once and compared with its input (bit-exact or an
    exception).  Returns (device blocks, per-block GPU compress ms, host
    codebook seconds)."""
    import torch

    import huffman_decode_b200 as df11
    stream = torch.cuda.current_stream(dev)
    cerr = torch.zeros(1, dtype=torch.int32, device=dev)
    derr = torch.zeros(1, dtype=torch.int32, device=dev)
    blocks, gpu_ms, host_cb_s = [], [], 0.0
    out = verify_into
    for b in range(n_blocks):
        d_in = workloads.llama_block_device(seed0 + b, dev, scale_div=scale_div)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        ev[0].record(stream)
        hist = df11.histogram_device(d_in)
        ev[1].record(stream)
        t0 = time.perf_counter()
        cb = df11.build_codebook_from_histogram(hist.cpu().numpy().astype(np.uint64))
        host_cb_s += time.perf_counter() - t0
        ev[2].record(stream)
        db = df11.compress_device(cb, d_in, 32, bpt, error=cerr)
        ev[3].record(stream)
        if out is None or out.numel() < d_in.numel():
            out = torch.empty(d_in.numel(), dtype=torch.bfloat16, device=dev)
        df11.decompress_async(db, out, derr, stream=stream)
        torch.cuda.synchronize()
        gpu_ms.append(ev[0].elapsed_time(ev[1]) + ev[2].elapsed_time(ev[3]))
        if int(cerr.item()) or int(derr.item()) or not torch.equal(
                out[: d_in.numel()].view(torch.int16), d_in):
            raise RuntimeError(f"block {b}: GPU compress/decode is not bit-exact")
        del d_in, hist
        blocks.append(db)
    return blocks, gpu_ms, host_cb_s


def numpy_model_blocks(seeds, dev, bpt, scale_div=1):
    """The 8B-scale stream as specified: llama_block(seed) for every seed,
    drawn by numpy in a pool of worker processes, compressed on the host
    (one codebook per block) and copied to the GPU.  Every block is decoded
    once into one reused buffer and compared with its input (bit-exact or an
    exception).  Returns the device blocks."""
    import torch

    import huffman_decode_b200 as df11
    stream = torch.cuda.current_stream(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    dbs, out = [], None
    for sd, w in workloads.llama_model_blocks(seeds, scale_div=scale_div):
        hb = df11.compress(df11.build_codebook([w]), [w], 32, bpt)
        db = hb.to_device(dev)
        if out is None:
            out = torch.empty(hb.n_elements, dtype=torch.int16, device=dev)
        df11.decompress_async(db, out[: hb.n_elements], err, stream=stream)
        want = torch.from_numpy(w.view(np.int16)).to(dev)
        if int(err.item()) or not torch.equal(out[: hb.n_elements], want):
            raise RuntimeError(f"block seed {sd}: decode is not bit-exact")
        del hb, want
        dbs.append(db)
    return dbs


def run_model_stream(args):
    """The 8B-scale stream: n_blocks Llama-3.1-8B-shaped blocks drawn by numpy
    (llama_block(seed), seeds 1000 + block), each with its own codebook, all
    resident in HBM; one step decodes every block in turn into one reused
    BF16 buffer on one stream."""
    import torch
    import torch.distributed as dist

    import huffman_decode_b200 as df11

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    stream = torch.cuda.current_stream(dev)
    bpt = args.bytes_per_thread
    n_blocks = args.blocks or 32
    derr = torch.zeros(1, dtype=torch.int32, device=dev)
    seed0 = rank_seed(rank, per_rank=n_blocks)
    dbs = numpy_model_blocks(range(seed0, seed0 + n_blocks), dev, bpt, args.scale_div)
    out = torch.empty(max(db.n_elements for db in dbs), dtype=torch.bfloat16, device=dev)
    blocks = [(db, db.c_struct(), db.compressed_bytes() + 2 * db.n_elements) for db in dbs]
    n_weights = sum(db.n_elements for db in dbs)
    step_bytes = sum(x[2] for x in blocks)

    def step():
        for db, cblk, _ in blocks:
            df11.decompress_async(db, out, derr, stream=stream, c_block=cblk)

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    ms, reps = timed_reps(step, args.steps, stream, world, min_seconds=1.0, device=dev)
    clocks = sampler.stop()
    if int(derr.item()):
        raise RuntimeError("device error word set during the timed decode")
    (ms_max,), (job_bytes, job_weights) = reduce_over_ranks([ms], [step_bytes, n_weights], dev)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    peak, peak_kind = measured_peaks()
    launches = args.steps * len(blocks)
    achieved = step_bytes / (ms / args.steps * 1e-3) / 1e9
    value = job_rate(job_bytes, args.steps, ms_max)
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "u8", "data": "synthetic (numpy, llama_block(seed) for every block)",
        "config": {"workload": "llama8b_model", "blocks": len(blocks), "n_weights": n_weights,
                   "threads_per_chunk": 32, "bytes_per_thread": bpt,
                   "bytes_per_step": step_bytes, "seeds": f"{seed0}..{seed0 + len(blocks) - 1}",
                   "l2": "inputs larger than L2, no flush",
                   "parallelism": f"replicas x{world}, own blocks per GPU, no collective"},
        "gweights_per_s": round(job_rate(job_weights, args.steps, ms_max), 2),
        "pct_of_hbm_peak": round(100 * value / world / peak, 2),
        "bit_exact": True,
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak,
                     "peak_source": peak_kind, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": profiled_traffic(n_weights // len(blocks)),
                     "algorithmic_bytes_per_launch": step_bytes // len(blocks)},
        "clocks": clocks,
        "timing": reps,
        "gpu_launches": launches,
    }
    print(json.dumps(line), flush=True)
    return 0


def _events(n):
    import torch
    return [torch.cuda.Event(enable_timing=True) for _ in range(n)]


def run_overlap(args):
    """Decode overlapped with consumption (1 GPU): n blocks resident
    compressed in HBM; the consumer runs each block's seven linear layers
    (cuBLAS BF16 GEMMs, Y = X W^T) on activations of T tokens.  Timed on the
    device with CUDA events:
      decode  - every block decoded back to back;
      gemm    - every block's products on already-decoded weights;
      serial  - per block, decode then its products, one stream (the pages'
                order: decode just before the block runs);
      overlap - the pipeline: block i+1 decodes on its own stream while the
                products of block i run, two output slots.
    hidden = (serial - overlap) / decode: the share of decode time hidden.
    Each measurement is repeated --runs times, interleaved (every variant
    once per run), and reported as the median with its range."""
    import torch

    import huffman_decode_b200 as df11
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    n_blocks = args.blocks or 32
    dbs, _, _ = gpu_compressed_blocks(n_blocks, 1000, dev, args.bytes_per_thread)
    n = dbs[0].n_elements
    shapes = [s for _, s in workloads.LLAMA8B_BLOCK_SHAPES]
    offs = np.cumsum([0] + [r * c for r, c in shapes])
    slots = [torch.empty(n, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    cblk = [db.c_struct() for db in dbs]
    s_dec = torch.cuda.Stream(dev)
    s_use = torch.cuda.Stream(dev, priority=args.consumer_priority)
    results = []
    token_list = [int(t) for t in (args.tokens or "1,256,2048,8192").split(",") if t]
    cap_list = [int(c) for c in args.max_ctas.split(",") if c != ""]
    for T in token_list:
        g = torch.Generator(device=dev)
        g.manual_seed(T)
        x_in = {k: torch.randn(T, k, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
                for k in (4096, 14336)}
        y = [torch.empty(T, r, dtype=torch.bfloat16, device=dev) for r, _ in shapes]

        def weights(buf):
            return [buf[offs[i]:offs[i + 1]].view(r, c) for i, (r, c) in enumerate(shapes)]

        wv = [weights(sl) for sl in slots]

        def products(slot):
            for i, (r, c) in enumerate(shapes):
                torch.mm(x_in[c], wv[slot][i].t(), out=y[i])

        def decode(i, slot, stream, max_ctas=0):
            df11.decompress_async(dbs[i], slots[slot], err, stream=stream, c_block=cblk[i],
                                  max_ctas=max_ctas)

        def timed(fn, reps=1):
            for _ in range(max(args.warmup, 1)):
                fn()
            torch.cuda.synchronize()
            e = _events(2)
            e[0].record(torch.cuda.current_stream(dev))
            for _ in range(reps):
                fn()
            e[1].record(torch.cuda.current_stream(dev))
            torch.cuda.synchronize()
            return e[0].elapsed_time(e[1]) / reps

        cur = torch.cuda.current_stream(dev)

        def run_decode():
            for i in range(n_blocks):
                decode(i, 0, cur)

        def run_gemm():
            for i in range(n_blocks):
                products(0)

        def run_serial():
            for i in range(n_blocks):
                decode(i, i % 2, cur)
                products(i % 2)

        def run_overlap_cap(max_ctas, claimed):
            def fn():
                with df11.Pipeline(2) as pipe:
                    s_dec.wait_stream(cur)
                    s_use.wait_stream(cur)
                    for i in range(n_blocks):
                        slot = i % 2
                        pipe.decode(slot, dbs[i], slots[slot], err, s_dec, max_ctas=max_ctas,
                                    workspace=claimed)
                        pipe.acquire(slot, s_use)
                        with torch.cuda.stream(s_use):
                            products(slot)
                        pipe.release(slot, s_use)
                    cur.wait_stream(s_use)
                    cur.wait_stream(s_dec)
            return fn

        reps = max(1, args.steps)
        variants = [(c, w) for c in cap_list for w in (True, False)]
        samples = {"decode": [], "gemm": [], "serial": [], **{v: [] for v in variants}}
        same = True
        for run in range(max(1, args.runs)):
            samples["decode"].append(timed(run_decode, reps))
            samples["gemm"].append(timed(run_gemm, reps))
            samples["serial"].append(timed(run_serial, reps))
            ref = [t.clone() for t in y]
            for v in variants:
                samples[v].append(timed(run_overlap_cap(*v), reps))
                same = same and all(torch.equal(a, b) for a, b in zip(ref, y))
        med = {k: float(np.median(v)) for k, v in samples.items()}
        t_dec, t_gemm, t_ser = med["decode"], med["gemm"], med["serial"]
        row = {"tokens": T, "runs": max(1, args.runs), "decode_ms": round(t_dec, 4), "gemm_ms": round(t_gemm, 4),
               "serial_ms": round(t_ser, 4), "overlap": []}
        for cap, claimed in variants:
            hid = [(s_ - o) / d for s_, o, d in zip(samples["serial"], samples[(cap, claimed)], samples["decode"])]
            row["overlap"].append({
                "max_ctas": cap, "schedule": "claimed tail" if claimed else "static",
                "overlap_ms": round(med[(cap, claimed)], 4),
                "hidden_frac": round(float(np.median(hid)), 4),
                "hidden_frac_range": [round(min(hid), 4), round(max(hid), 4)],
                "overhead_vs_bf16": round(med[(cap, claimed)] / t_gemm, 4),
                "outputs_equal_serial": bool(same)})
        flops = 2.0 * T * offs[-1] * n_blocks
        row["gemm_tflops"] = round(flops / (t_gemm * 1e-3) / 1e12, 1)
        results.append(row)
    if int(err.item()):
        raise RuntimeError("device error word set")
    best = {r["tokens"]: max(r["overlap"], key=lambda o: o["hidden_frac"]) for r in results}
    line = {
        "metric": "decode hidden behind the block's matrix products (fraction of decode time)",
        "value": None, "unit": "fraction", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "higher_is_better": True, "dtype": "bf16",
        "data": "synthetic (GPU-drawn weights and activations)",
        "config": {"workload": "llama8b_overlap", "blocks": n_blocks, "n_weights_per_block": n,
                   "bytes_per_thread": args.bytes_per_thread,
                   "consumer_stream_priority": args.consumer_priority,
                   "consumer": "7 cuBLAS BF16 GEMMs per block (Y = X W^T), torch.mm"},
        "results": results,
        "best_hidden_frac": {str(k): v["hidden_frac"] for k, v in best.items()},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_offload(args):
    """Offload streaming (1 GPU): n blocks held compressed in pinned host
    memory; a step uploads every block over PCIe into one of two staging
    slots and decodes it into one of two BF16 slots (the pipeline: upload of
    block i+1 overlaps the decode of block i).  Reported beside it, on the
    same box: the pinned host->device copy bandwidth of the compressed arrays
    alone, and of plain BF16 weights (offloading without DF11)."""
    import torch

    import huffman_decode_b200 as df11
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    n_blocks = args.blocks or 8
    dbs, _, _ = gpu_compressed_blocks(n_blocks, 1000, dev, args.bytes_per_thread)
    # checksum lists (kept on the device for the verify stage) and the
    # checksum kernel's own throughput on a resident block
    crcs = [df11.checksum_device(db) for db in dbs]
    torch.cuda.synchronize()
    cur = torch.cuda.current_stream(dev)
    e = _events(2)
    for _ in range(3):
        df11.checksum_device(dbs[0])
    e[0].record(cur)
    for _ in range(20):
        df11.checksum_device(dbs[0])
    e[1].record(cur)
    torch.cuda.synchronize()
    crc_ms = e[0].elapsed_time(e[1]) / 20
    crc_gbs = dbs[0].compressed_bytes() / (crc_ms * 1e-3) / 1e9
    # the blocks move to pinned host memory; the device copies are dropped
    hosts = []
    for db in dbs:
        t = {k: v.to("cpu").pin_memory() for k, v in db.tensors.items()}
        hosts.append(df11.PinnedHostBlock(header=db.header, tensors=t, sizes=dict(db.sizes)))
    last_n = dbs[-1].n_elements
    last_ref = torch.empty(last_n, dtype=torch.bfloat16, device=dev)
    df11.decompress_async(dbs[-1], last_ref)
    torch.cuda.synchronize()
    del dbs, e
    torch.cuda.empty_cache()
    sizes = {k: max(h.sizes[k] for h in hosts) for k in hosts[0].sizes}
    staging = [df11.DeviceBlock.staging(sizes, dev) for _ in range(2)]
    n_max = max(h.n_elements for h in hosts)
    slots = [torch.empty(n_max, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    s_copy, s_dec = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    cur = torch.cuda.current_stream(dev)
    comp_bytes = sum(h.compressed_bytes() for h in hosts)
    bf16_bytes = sum(2 * h.n_elements for h in hosts)

    def make_step(verify):
        def step():
            with df11.Pipeline(2) as pipe:
                s_copy.wait_stream(cur)
                s_dec.wait_stream(cur)
                for i, h in enumerate(hosts):
                    slot = i % 2
                    pipe.upload(slot, h, staging[slot], s_copy)
                    if verify:
                        pipe.verify(slot, staging[slot], crcs[i], err, stream=s_dec)
                    pipe.decode(slot, staging[slot], slots[slot], err, s_dec)
                    pipe.acquire(slot, cur)
                    pipe.release(slot, cur)
                cur.wait_stream(s_dec)
        return step

    def copies_only():
        for i, h in enumerate(hosts):
            for k, t in h.tensors.items():
                staging[i % 2].tensors[k][: t.numel()].copy_(t, non_blocking=True)

    bf16_host = torch.empty(n_max, dtype=torch.int16).pin_memory()

    def bf16_copies():
        for h in hosts:
            slots[0][: h.n_elements].view(torch.int16).copy_(bf16_host[: h.n_elements],
                                                             non_blocking=True)

    def timed(fn):
        for _ in range(max(args.warmup, 1)):
            fn()
        torch.cuda.synchronize()
        e = _events(2)
        e[0].record(cur)
        for _ in range(args.steps):
            fn()
        e[1].record(cur)
        torch.cuda.synchronize()
        return e[0].elapsed_time(e[1]) / args.steps

    sampler = ClockSampler(0)
    sampler.start()
    t_pipe = timed(make_step(False))
    clocks = sampler.stop()
    ok = int(err.item()) == 0 and torch.equal(slots[(n_blocks - 1) % 2][:last_n], last_ref)
    t_pipe_verify = timed(make_step(True))
    ok = ok and int(err.item()) == 0
    t_copy = timed(copies_only)
    t_bf16 = timed(bf16_copies)
    h2d = comp_bytes / (t_copy * 1e-3) / 1e9
    line = {
        "metric": "offload stream: BF16 weights delivered per second (pinned host DF11 -> GPU BF16)",
        "value": round(bf16_bytes / (t_pipe * 1e-3) / 1e9, 2), "unit": "GB/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(t_pipe, 4), "higher_is_better": True, "dtype": "u8",
        "data": "synthetic (GPU-drawn, GPU-compressed, then pinned host)",
        "config": {"workload": "llama8b_offload", "blocks": n_blocks,
                   "bytes_per_thread": args.bytes_per_thread, "slots": 2,
                   "compressed_bytes_per_step": comp_bytes, "bf16_bytes_per_step": bf16_bytes},
        "compressed_h2d_gbs_in_pipeline": round(comp_bytes / (t_pipe * 1e-3) / 1e9, 2),
        "h2d_copy_only": {"ms": round(t_copy, 4), "gbs": round(h2d, 2)},
        "pcie_frac": round((comp_bytes / (t_pipe * 1e-3) / 1e9) / h2d, 4),
        "bf16_offload": {"ms": round(t_bf16, 4),
                         "gbs": round(bf16_bytes / (t_bf16 * 1e-3) / 1e9, 2)},
        "speedup_vs_bf16_offload": round(t_bf16 / t_pipe, 3),
        "with_checksum_verify": {"ms": round(t_pipe_verify, 4),
                                 "overhead": round(t_pipe_verify / t_pipe - 1, 4)},
        "checksum_kernel": {"ms_per_block": round(crc_ms, 4), "gbs": round(crc_gbs, 1),
                            "what": "df11_checksum_device_async over one resident block's "
                                    "compressed arrays"},
        "bit_exact_last_block": bool(ok),
        "clocks": clocks,
        "gpu_launches": n_blocks * args.steps,
    }
    print(json.dumps(line), flush=True)
    return 0 if ok else 1


def run_gemv(args):
    """Decode fused with its consumer at small token counts (1 GPU): n
    blocks resident compressed in HBM; per block the seven Llama-3.1-8B
    matrices multiply T activation rows.  Timed on the device:
      fused   - df11_decode_gemv_async, one launch per block (the BF16 block
                never reaches HBM), plus zeroing the block's outputs;
      serial  - decode to a BF16 buffer, then seven cuBLAS products
                (torch.mm), the pages' order;
      bf16    - seven cuBLAS products on resident BF16 weights (no DF11).
    The fused launch's roofline is HBM: it reads the compressed block (and
    the activations) and writes the outputs."""
    import torch

    import huffman_decode_b200 as df11
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    n_blocks = args.blocks or 16
    dbs, _, _ = gpu_compressed_blocks(n_blocks, 1000, dev, args.bytes_per_thread)
    shapes = [s for _, s in workloads.LLAMA8B_BLOCK_SHAPES]
    offs = np.cumsum([0] + [r * c for r, c in shapes])
    n = int(offs[-1])
    buf = torch.empty(n, dtype=torch.bfloat16, device=dev)
    wres = torch.empty(n, dtype=torch.bfloat16, device=dev)
    df11.decompress_async(dbs[0], wres)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    cur = torch.cuda.current_stream(dev)
    peak, peak_kind = measured_peaks()
    results = []
    for T in [int(t) for t in (args.tokens or "1,4,8").split(",") if t]:
        g = torch.Generator(device=dev)
        g.manual_seed(1000 + T)
        xs = [torch.randn(T, c, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
              for _, c in shapes]
        xs16 = [x.view(torch.int16) for x in xs]
        ybuf = torch.zeros(sum(T * r for r, _ in shapes), dtype=torch.float32, device=dev)
        ys, o = [], 0
        for r, _ in shapes:
            ys.append(ybuf[o:o + T * r].view(T, r))
            o += T * r
        yb = [torch.empty(T, r, dtype=torch.bfloat16, device=dev) for r, _ in shapes]

        def fused():
            for db in dbs:
                ybuf.zero_()
                df11.decode_gemv_async(db, shapes, xs16, ys, err)

        def mm(wbuf):
            for i, (r, c) in enumerate(shapes):
                torch.mm(xs[i], wbuf[offs[i]:offs[i + 1]].view(r, c).t(), out=yb[i])

        def serial():
            for db in dbs:
                df11.decompress_async(db, buf, err)
                mm(buf)

        def bf16():
            for _ in dbs:
                mm(wres)

        def timed(fn):
            for _ in range(max(args.warmup, 1)):
                fn()
            torch.cuda.synchronize()
            e = _events(2)
            e[0].record(cur)
            for _ in range(args.steps):
                fn()
            e[1].record(cur)
            torch.cuda.synchronize()
            return e[0].elapsed_time(e[1]) / args.steps / n_blocks

        t_f, t_s, t_b = timed(fused), timed(serial), timed(bf16)
        # the last block's fused products against decode + cuBLAS (FP32 from BF16 outputs)
        ybuf.zero_()
        df11.decode_gemv_async(dbs[-1], shapes, xs16, ys, err)
        df11.decompress_async(dbs[-1], buf, err)
        mm(buf)
        torch.cuda.synchronize()
        rel = max(float(((ys[i] - yb[i].float()).abs().max() / (yb[i].float().abs().max() + 1e-30)))
                  for i in range(len(shapes)))
        comp = dbs[0].compressed_bytes()
        moved = comp + 2 * T * sum(c for _, c in shapes) + 4 * T * sum(r for r, _ in shapes)
        gbs = moved / (t_f * 1e-3) / 1e9
        results.append({
            "tokens": T, "fused_ms_per_block": round(t_f, 4), "serial_ms_per_block": round(t_s, 4),
            "bf16_ms_per_block": round(t_b, 4), "fused_vs_serial": round(t_s / t_f, 3),
            "fused_vs_bf16": round(t_b / t_f, 3),
            "fused_roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak,
                               "peak_source": peak_kind, "frac": round(gbs / peak, 4),
                               "bytes_per_block": moved},
            "max_rel_diff_vs_cublas_bf16_out": rel})
    if int(err.item()):
        raise RuntimeError("device error word set")
    line = {
        "metric": "decode fused with matrix-vector products: ms per Llama-3.1-8B block",
        "value": None, "unit": "ms", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "higher_is_better": False, "dtype": "fp32 accumulate, bf16 in",
        "data": "synthetic (GPU-drawn weights and activations)",
        "config": {"workload": "llama8b_gemv", "blocks": n_blocks, "n_weights_per_block": n,
                   "bytes_per_thread": args.bytes_per_thread},
        "results": results,
        "gpu_launches": n_blocks * args.steps * 2,
    }
    print(json.dumps(line), flush=True)
    return 0


def timed_reps(step, steps, stream, world, min_seconds=1.0, min_reps=5, device=None):
    """Times `steps` back-to-back steps between two CUDA events on `stream`,
    each repetition bracketed by a barrier across ranks and a device
    synchronize, repeated until about min_seconds of wall time (and at least
    min_reps repetitions) have passed, so the clock samples taken meanwhile
    cover a real stretch of load.  The repetition count is fixed up front
    from a calibration repetition and agreed across ranks (the maximum).
    Returns (median repetition ms, a record of the repetitions)."""
    import math

    import torch
    import torch.distributed as dist

    def one():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        a, b = _events(2)
        a.record(stream)
        for _ in range(steps):
            step()
        b.record(stream)
        b.synchronize()
        return a.elapsed_time(b)

    t0 = time.perf_counter()
    times = [one()]
    wall = time.perf_counter() - t0
    want = max(min_reps, int(math.ceil(min_seconds / max(wall, 1e-6))))
    (want,), _ = reduce_over_ranks([want], [], device)
    for _ in range(int(want) - 1):
        times.append(one())
    total = time.perf_counter() - t0
    med = statistics.median(times)
    return med, {"reps": len(times), "steps_per_rep": steps, "rep_ms_median": round(med, 5),
                 "rep_ms_min": round(min(times), 5), "rep_ms_max": round(max(times), 5),
                 "wall_s": round(total, 3),
                 "what": "ms_per_step = the median repetition / steps_per_rep"}


def _timed_steps(step, steps, warmup, stream, local):
    """Warm-up, then `steps` back-to-back steps between two events on
    `stream`, with clocks sampled meanwhile.  Returns (ms, clocks)."""
    import torch
    for _ in range(max(warmup, 0)):
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    e = _events(2)
    sampler.start()
    e[0].record(stream)
    for _ in range(steps):
        step()
    e[1].record(stream)
    e[1].synchronize()
    clocks = sampler.stop()
    return e[0].elapsed_time(e[1]), clocks


def run_compress(args):
    """The GPU compressor (1 GPU): one step is df11_histogram_device +
    df11_compress_device of the Llama-3.1-8B-shaped block, drawn on the GPU and
    resident in HBM.  The codebook comes from the histogram on the host (its
    time is reported beside, not in the step; the pages build it on the CPU
    too).  The output is checked byte for byte against the host compressor
    and by a decode round trip.  Roofline: the method must read the BF16
    block and write the compressed arrays (2 + ~1.33 B/weight)."""
    import torch

    import huffman_decode_b200 as df11
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    d_in = workloads.llama_block_device(1000, dev, scale_div=args.scale_div)
    n = d_in.numel()
    hist = df11.histogram_device(d_in)
    t0 = time.perf_counter()
    cb = df11.build_codebook_from_histogram(hist.cpu().numpy().astype(np.uint64))
    cb_ms = 1e3 * (time.perf_counter() - t0)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    scratch = torch.empty(df11.compress_device_scratch_bytes(n), dtype=torch.uint8, device=dev)
    db = df11.compress_device(cb, d_in, 32, args.bytes_per_thread, error=err, scratch=scratch)
    out = torch.empty(n, dtype=torch.bfloat16, device=dev)
    df11.decompress_async(db, out)
    torch.cuda.synchronize()
    ok = int(err.item()) == 0 and bool(torch.equal(out.view(torch.int16), d_in))
    hb = df11.compress(cb, [d_in.cpu().numpy().view(np.uint16)], 32, args.bytes_per_thread)
    for name in ("exp_stream", "gaps", "counts", "chunk_pos", "signmant"):
        a = db.tensors[name][: db.sizes[name]].cpu().numpy().view(np.uint8)
        h = getattr(hb, name).view(np.uint8)
        ok = ok and np.array_equal(a[: h.size], h) and not a[h.size:].any()
    if not ok:
        raise RuntimeError("GPU compressor output differs from the host compressor")
    del out, hb

    def step():
        df11.histogram_device(d_in)
        df11.compress_device(cb, d_in, 32, args.bytes_per_thread, error=err, scratch=scratch)

    ms, clocks = _timed_steps(step, args.steps, args.warmup, stream, 0)
    if int(err.item()):
        raise RuntimeError("device error word set during the timed compression")
    peak, peak_kind = measured_peaks()
    comp = db.compressed_bytes()
    alg = 2 * n + comp
    step_s = ms / args.steps * 1e-3
    line = {
        "metric": "GPU compression of BF16 weights to DF11 (histogram + encode), BF16 GB/s in",
        "value": round(2 * n / step_s / 1e9, 2), "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "u8", "data": "synthetic (GPU-drawn, torch CUDA generator)",
        "config": {"workload": "llama8b_compress", "n_weights": n, "seed": 1000,
                   "threads_per_chunk": 32, "bytes_per_thread": args.bytes_per_thread,
                   "compressed_bytes": comp, "l2": "inputs larger than L2, no flush"},
        "byte_identical_to_host_compressor": True,
        "host_codebook_ms": round(cb_ms, 3),
        "roofline": {"bound": "hbm", "achieved": round(alg / step_s / 1e9, 2), "peak": peak,
                     "peak_source": peak_kind, "unit": "GB/s",
                     "frac": round(alg / step_s / 1e9 / peak, 4), "traffic": None,
                     "algorithmic_bytes_per_step": alg},
        "clocks": clocks,
        "gpu_launches": 5 * args.steps,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_verify(args):
    """The integrity check (1 GPU): one step is df11_verify_device_async over a
    resident GPU-compressed Llama-3.1-8B-shaped block: the CRC-32C of every
    4096-byte segment of its five arrays against the expected list.  The
    list is checked against the host's (SSE4.2) list first.  Roofline: the
    compressed bytes must be read once."""
    import torch

    import huffman_decode_b200 as df11
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    (db,), _, _ = gpu_compressed_blocks(1, 1000, dev, args.bytes_per_thread, scale_div=args.scale_div)
    expected = df11.checksum_device(db)
    host = {a: db.tensors[a][: db.sizes[a]].cpu().numpy() for a in ("exp_stream", "gaps", "counts", "chunk_pos",
                                                                     "signmant", "lut")}
    hb = df11.HostBlock(header=db.header, exp_stream=host["exp_stream"], gaps=host["gaps"],
                        counts=host["counts"], chunk_pos=host["chunk_pos"].view(np.uint32), signmant=host["signmant"],
                        lut=host["lut"].view(np.uint16))
    t0 = time.perf_counter()
    host_list = df11.checksum(hb)
    host_s = time.perf_counter() - t0
    if not np.array_equal(expected.cpu().numpy().view(np.uint32), host_list):
        raise RuntimeError("device checksum list differs from the host's")
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def step():
        df11.verify_device(db, expected, err, stream=stream)

    ms, clocks = _timed_steps(step, args.steps, args.warmup, stream, 0)
    if int(err.item()):
        raise RuntimeError("verification failed on an intact block")
    peak, peak_kind = measured_peaks()
    comp = db.compressed_bytes()
    step_s = ms / args.steps * 1e-3
    line = {
        "metric": "CRC-32C verification of a resident DF11 block (compressed GB/s checked)",
        "value": round(comp / step_s / 1e9, 2), "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "u8", "data": "synthetic (GPU-drawn, GPU-compressed)",
        "config": {"workload": "llama8b_verify", "n_weights": db.n_elements, "seed": 1000,
                   "segments": int(expected.numel()), "compressed_bytes": comp,
                   "l2": "inputs larger than L2, no flush"},
        "host_sse42_gbs": round(comp / host_s / 1e9, 2),
        "roofline": {"bound": "hbm", "achieved": round(comp / step_s / 1e9, 2), "peak": peak,
                     "peak_source": peak_kind, "unit": "GB/s",
                     "frac": round(comp / step_s / 1e9 / peak, 4), "traffic": None,
                     "algorithmic_bytes_per_step": comp},
        "clocks": clocks,
        "gpu_launches": args.steps,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "llama8b_model":
        return run_model_stream(args)
    if args.workload == "llama8b_overlap":
        return run_overlap(args)
    if args.workload == "llama8b_offload":
        return run_offload(args)
    if args.workload == "llama8b_gemv":
        return run_gemv(args)
    if args.workload == "llama8b_compress":
        return run_compress(args)
    if args.workload == "llama8b_verify":
        return run_verify(args)
    return run_b200(args)


if __name__ == "__main__":
    sys.exit(main())

"""Benchmark: exact attention forward + backward on B200 through the C ABI.

One step = one pass of the whole hot path over one batch of synthetic input: fa_fwd (O, LSE)
followed by the backward's launches (preprocess, main, dQ conversion). The default workload is
the long-context configuration B=1, H=16, N=32768, d=128, causal, bf16 (the largest of the
workloads, which fits one GPU). The same run also reports device-timed forward / backward
figures of the other workloads (GPT-style forward, training shape, sliding window, tiny) under
"configs". ``--config train_fwd_fp8`` instead times the E4M3 forward (fa_fwd_fp8) on the training
shape: one step = one launch. ``--config decode_paged`` times the paged-KV decode
(fa_decode_paged): one step = one call (append, attention and merge in one kernel) over every
sequence, reported in GB/s of cache read.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl reference]

For N > 1 it is launched with torch.distributed.run, one rank per GPU: every rank runs its
own copy of the workload (independent problems, no data-path collective: weak scaling);
the timed region is bracketed by barriers and the max over ranks is reported.
``--impl reference`` times the fp64 CPU oracle on the host cores instead (rank 0 only).

Prints one JSON line (rank 0).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_attention_116_b200 import binding  # noqa: E402
from exact_attention_116_b200 import distributed as mg  # noqa: E402
from exact_attention_116_b200.inputs import (CONFIGS, DECODE_CONFIGS, FP8_CONFIGS, make_decode_inputs,  # noqa: E402
                                             make_fp8_inputs, make_inputs)
from exact_attention_116_b200.workload import flops, flops_tile_granular, hbm_bytes, visible_pairs  # noqa: E402

METRIC = "attention fwd/bwd TFLOPS (bf16, causal) and % of B200 dense BF16 peak"
METRIC_FP8 = "attention fwd TFLOPS (E4M3 inputs, causal) and % of B200 dense FP8 peak"
FP8_PER_BF16 = 2.0  # nominal dense FP8 / BF16 tensor throughput (4.5 / 2.25 PFLOP/s)
METRIC_DECODE = "paged-KV decode attention GB/s of KV cache read (bf16) and % of B200 HBM bandwidth"
UNIT = "TFLOPS"
L2_BYTES = 126 * 2**20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "ncu_traffic.json")


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def kernel_source_hash(sources) -> str:
    h = hashlib.sha256()
    for name in sources:
        with open(os.path.join(ROOT, "exact_attention_116_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu summary (entry
    "kernel@workload"), if the sources that define the kernel still hash to the value recorded
    with the measurement."""
    if not os.path.exists(PROFILE_TRAFFIC):
        return None
    with open(PROFILE_TRAFFIC) as f:
        k = json.load(f).get("kernels", {}).get(f"{kernel}@{workload}")
    if k is None or k.get("source_hash") != kernel_source_hash(k.get("sources", [])):
        return None
    return k.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------- L2 flush, config record

def l2_flusher(dev):
    """A callable that writes one buffer larger than L2 and then reads another, so that the next
    timed launch starts with a clean L2 (nothing of its inputs cached, no dirty lines of the flush
    left to write back). It runs on the current stream, outside the timed interval."""
    w = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    r = torch.ones(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    def flush():
        w.zero_()
        r.sum()
    return flush


L2_NOTE = ("L2 flushed before every timed step outside the timed interval (252 MiB written, then 252 MiB read); "
           "each step timed with CUDA events on the launching stream")


def attn_config(cfg) -> dict:
    """The workload record of a bf16 config: the same keys in the GPU arm and the reference arm."""
    return {"workload": f"{cfg.name}: {cfg.note}", "B": cfg.B, "N": cfg.N, "H": cfg.H, "d": cfg.d,
            "causal": cfg.causal, "window": [cfg.win_l, cfg.win_r], "seed": cfg.seed}


# ----------------------------------------------------------------------------- end to end

def pipelined_e2e(info, dev, sets, copy_in, compute, copy_out, steps: int, warm: int = 4) -> float:
    """Time `steps` end-to-end steps through the public API, pipelined over three streams and
    len(sets) device buffer sets: every step copies its inputs host -> device (copy_in(set)),
    runs the path (compute(set, stream)) and copies its outputs device -> host (copy_out(set)).
    Step k's outputs travel down while step k+1's inputs travel up and step k+1 computes (PCIe
    is full duplex), so throughput is bounded by the slowest of the three, not their sum. A set
    is refilled only after its previous compute has read it, and recomputed only after its
    previous outputs are on the host. Returns the device time per step (ms, max over ranks) from
    the first copy-in to the last copy-out."""
    s_in, s_comp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    n = len(sets)
    ev = {name: [torch.cuda.Event() for _ in range(n)] for name in ("in", "comp", "out")}
    started = [False] * n

    def one(k):
        b = k % n
        with torch.cuda.stream(s_in):
            if started[b]:
                s_in.wait_event(ev["comp"][b])  # the set's previous compute has read its inputs
            copy_in(sets[b])
            ev["in"][b].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev["in"][b])
            if started[b]:
                s_comp.wait_event(ev["out"][b])  # the set's previous outputs are on the host
            compute(sets[b], s_comp)
            ev["comp"][b].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["comp"][b])
            copy_out(sets[b])
            ev["out"][b].record(s_out)
        started[b] = True

    for k in range(warm):
        one(k)
    torch.cuda.synchronize()
    mg.barrier(info)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    s_comp.wait_event(e0)
    s_out.wait_event(e0)
    for k in range(steps):
        one(k)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_comp)
    e1.record(s_out)
    torch.cuda.synchronize()
    mg.barrier(info)
    return mg.max_over_ranks(info, e0.elapsed_time(e1), dev) / steps


def packed_buffers(dev, specs, pin=False):
    """One byte buffer holding tensors of the given (shape, dtype) specs at 256-byte aligned
    offsets, and views of it: a single copy moves them all."""
    offs, total = [], 0
    for shape, dt in specs:
        total = (total + 255) // 256 * 256
        offs.append(total)
        total += int(np.prod(shape)) * torch.empty((), dtype=dt).element_size()
    buf = torch.empty(total, dtype=torch.uint8, device=dev)
    if pin:
        buf = buf.pin_memory()
    views = []
    for (shape, dt), off in zip(specs, offs):
        nb = int(np.prod(shape)) * torch.empty((), dtype=dt).element_size()
        views.append(buf[off:off + nb].view(dt).view(shape))
    return buf, views


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons, filtered to a time window."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        self.path = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            gid = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", gid, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self, t0: float, t1: float) -> dict | None:
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                    ts += float("0." + parts[0].split(".")[1]) if "." in parts[0] else 0.0
                    rows.append((ts, float(parts[1]), float(parts[2]), parts[5:9]))
                except (ValueError, IndexError):
                    continue
        os.unlink(self.path)
        inside = [r for r in rows if t0 - 0.15 <= r[0] <= t1 + 0.15]
        window = "timed"
        if not inside:
            inside, window = rows, "warmup+timed"
        if not inside:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i, v in enumerate(r[3]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": reasons, "samples": len(inside), "window": window}


# ----------------------------------------------------------------------------- oracle (CPU) timing

def oracle_sample(cfg, seconds: float, q=None, k=None, v=None, do=None):
    """Time the fp64 oracle, as it stands, on blocks of query rows, head after head of batch 0
    (forward of the rows and their backward contributions) until `seconds` have passed.

    Returns (TFLOPS by the same pair-count convention, seconds, rows done, BLAS threads).
    """
    from oracle import attention_fp64 as oracle
    try:
        from threadpoolctl import threadpool_info
        threads = max((i.get("num_threads", 1) for i in threadpool_info()), default=os.cpu_count())
    except Exception:
        threads = os.cpu_count()
    if q is None:
        q, k, v, do = make_inputs(cfg)
    n, block = cfg.N, min(512, cfg.N)
    wr = 0 if cfg.causal else cfg.win_r
    row_pairs = []
    for i in range(n):
        lo = max(0, i - cfg.win_l) if cfg.win_l >= 0 else 0
        hi = min(n - 1, i + wr) if wr >= 0 else n - 1
        row_pairs.append(hi - lo + 1)
    pairs, rows_done = 0, 0
    t0 = time.perf_counter()
    for h in range(cfg.H):
        q4, k4, v4 = (x[:1, :, h:h + 1].to(torch.float64).numpy() for x in (q, k, v))
        qh, kh, vh, doh = q4[0, :, 0], k4[0, :, 0], v4[0, :, 0], do[0, :, h].to(torch.float64).numpy()
        dq, dk, dv = np.zeros_like(qh), np.zeros_like(kh), np.zeros_like(vh)
        dvec = np.zeros(n)
        r1 = n
        while r1 > 0:
            r0 = max(0, r1 - block)
            oracle.forward_rows(q4, k4, v4, 0, 0, np.arange(r0, r1), cfg.scale, cfg.causal, cfg.win_l, cfg.win_r)
            oracle.backward_rows(qh, kh, vh, doh, r0, r1, cfg.scale, cfg.causal, cfg.win_l, cfg.win_r,
                                 dq, dk, dv, dvec)
            pairs += sum(row_pairs[r0:r1])
            rows_done += r1 - r0
            r1 = r0
            if time.perf_counter() - t0 >= seconds:
                break
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return 14 * cfg.d * pairs / dt / 1e12, dt, rows_done, threads


def oracle_sample_fp8(cfg, seconds: float, codes=None, descales=None):
    """Time the fp64 oracle's E4M3 forward, as it stands, on blocks of 512 query rows, head after
    head of batch 0, until `seconds` have passed. Returns (TFLOPS by 4*d*pairs, seconds, rows, threads)."""
    from oracle import fp8_e4m3 as oracle8
    try:
        from threadpoolctl import threadpool_info
        threads = max((i.get("num_threads", 1) for i in threadpool_info()), default=os.cpu_count())
    except Exception:
        threads = os.cpu_count()
    if codes is None:
        codes, descales = make_fp8_inputs(cfg)
    cn = [t.numpy() for t in codes]
    dn = [t.numpy().astype(np.float64) for t in descales]
    n, block = cfg.N, min(512, cfg.N)
    wr = 0 if cfg.causal else cfg.win_r
    pairs, rows_done = 0, 0
    t0 = time.perf_counter()
    for h in range(cfg.H):
        r1 = n
        while r1 > 0:
            r0 = max(0, r1 - block)
            rows = np.arange(r0, r1)
            oracle8.forward_rows_fp8(*cn, *dn, 0, h, rows, cfg.scale, cfg.causal, cfg.win_l, cfg.win_r)
            for i in range(r0, r1):
                lo = max(0, i - cfg.win_l) if cfg.win_l >= 0 else 0
                hi = min(n - 1, i + wr) if wr >= 0 else n - 1
                pairs += hi - lo + 1
            rows_done += r1 - r0
            r1 = r0
            if time.perf_counter() - t0 >= seconds:
                break
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return 4 * cfg.d * pairs / dt / 1e12, dt, rows_done, threads


# ----------------------------------------------------------------------------- GPU arm

def decode_cache_bytes(cfg, seqlens) -> int:
    """Algorithmic bytes of one decode call: the K and V rows every sequence's keys occupy (the
    whole sequence is visible to its newest rows), plus q, O and LSE."""
    kv = int(seqlens.sum()) * cfg.H * cfg.d * 2 * 2
    return kv + 2 * cfg.B * cfg.Sq * cfg.H * cfg.d * 2 + cfg.B * cfg.H * cfg.Sq * 4


def oracle_sample_decode(cfg, seconds: float, inputs):
    """Time the fp64 decode oracle, as it stands, one sequence at a time until `seconds` have passed.
    Returns (GB/s of cache rows processed, seconds, sequences, threads)."""
    from oracle import decode_paged_fp64 as oracle_dec
    try:
        from threadpoolctl import threadpool_info
        threads = max((i.get("num_threads", 1) for i in threadpool_info()), default=os.cpu_count())
    except Exception:
        threads = os.cpu_count()
    q, kc, vc, table, lens = inputs
    qn, kn, vn, tn, ln_ = q.double().numpy(), kc.float().numpy(), vc.float().numpy(), table.numpy(), lens.numpy()
    done_bytes, seqs = 0, 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < seconds:
        b = seqs % cfg.B
        oracle_dec.decode_forward(qn[b:b + 1], kn, vn, tn[b:b + 1], ln_[b:b + 1], cfg.scale, cfg.causal, cfg.win_l,
                                  cfg.win_r)
        done_bytes += int(ln_[b]) * cfg.H * cfg.d * 2 * 2
        seqs += 1
    dt = time.perf_counter() - t0
    return done_bytes / dt / 1e9, dt, seqs, threads


def decode_new_rows(cfg, host):
    """The new tokens' K and V rows of a decode step: the rows the cache holds at positions
    len_b - Sq + i (so that writing them back leaves the cache as generated)."""
    q, kc, vc, table, lens = host
    k_new = torch.empty_like(q)
    v_new = torch.empty_like(q)
    for b in range(cfg.B):
        for i in range(cfg.Sq):
            pos = int(lens[b]) - cfg.Sq + i
            page = int(table[b, pos // cfg.page_size])
            k_new[b, i] = kc[page, pos % cfg.page_size]
            v_new[b, i] = vc[page, pos % cfg.page_size]
    return k_new, v_new


def run_gpu_decode(args):
    """Paged-KV decode: one step = one fa_decode_paged call over all sequences, which writes the
    new tokens' K/V rows into the resident cache and attends the new rows to the whole cache."""
    info = mg.rank_info()
    world, rank, local = info.world, info.rank, info.local_rank
    torch.cuda.set_device(local)
    mg.init(info, "nccl", device=torch.device("cuda", local))
    cfg = DECODE_CONFIGS[args.config]
    host = make_decode_inputs(cfg)
    dev = torch.device("cuda", torch.cuda.current_device())
    q, kc, vc, table, lens = (x.to(dev) for x in host)
    kn_h, vn_h = decode_new_rows(cfg, host)
    k_new, v_new = kn_h.to(dev), vn_h.to(dev)
    B, Sq, H, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Sq), dtype=torch.float32, device=dev)
    splits = int(args.splits) or binding.decode_splits(B, Sq, H, d, cfg.max_pages * cfg.page_size)
    stream = torch.cuda.current_stream()
    # workspace of the split count in use (the library's choice unless --splits is given)
    ws = torch.empty(max(1, binding.decode_workspace_bytes(B, Sq, H, d, splits)), dtype=torch.uint8, device=dev)
    # L2 flush between steps (the cache is 2x268 MiB > L2 already, q/O are tiny): a buffer larger
    # than L2 is written, then another one read, so that the step starts with a clean L2 and does
    # not pay for writing the flush's dirty lines back
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    flush_r = torch.ones(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    def step():
        binding.decode_paged_into(q, kc, vc, table, lens, o, lse, cfg.scale, cfg.causal, (cfg.win_l, cfg.win_r),
                                  splits, ws, k_new=k_new, v_new=v_new)

    for _ in range(args.warmup):
        step()
    binding.check()
    torch.cuda.synchronize()
    sampler = ClockSampler(dev.index) if local == 0 else None
    mg.barrier(info)
    torch.cuda.synchronize()
    t_wall0 = time.time()
    ms = 0.0
    for _ in range(args.steps):
        flush.zero_()
        flush_r.sum()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step()
        b.record(stream)
        b.synchronize()
        ms += a.elapsed_time(b)
    torch.cuda.synchronize()
    mg.barrier(info)
    t_wall1 = time.time()
    binding.check()
    clocks = sampler.stop(t_wall0, t_wall1) if sampler else None
    ms_step = mg.max_over_ranks(info, ms, dev) / args.steps
    nbytes = decode_cache_bytes(cfg, host[4])
    gbs = nbytes / (ms_step * 1e-3) / 1e9

    # a step's host inputs: the new rows' q, K, V, the block table and the lengths (the cache is
    # device-resident state, as in a serving loop), packed in one pinned buffer so that a step is
    # one copy up and one copy down (O and LSE packed likewise)
    step_inputs = (host[0], kn_h, vn_h, host[3], host[4])
    in_specs = [(tuple(x.shape), x.dtype) for x in step_inputs]
    out_specs = [(tuple(o.shape), o.dtype), (tuple(lse.shape), lse.dtype)]
    in_h, in_h_views = packed_buffers("cpu", in_specs, pin=True)
    for dst, src in zip(in_h_views, step_inputs):
        dst.copy_(src)
    out_h, _ = packed_buffers("cpu", out_specs, pin=True)
    e2e_sets = []
    for _ in range(2):
        in_d, in_v = packed_buffers(dev, in_specs)
        out_d, out_v = packed_buffers(dev, out_specs)
        e2e_sets.append((in_d, in_v, out_d, out_v))

    def dec_compute(st, s):
        (qd, knd, vnd, td, ld), (od, lsed) = st[1], st[3]
        binding.decode_paged_into(qd, kc, vc, td, ld, od, lsed, cfg.scale, cfg.causal, (cfg.win_l, cfg.win_r),
                                  splits, ws, stream=s, k_new=knd, v_new=vnd)

    e2e_steps = max(4, min(args.steps, 50))
    e2e_ms = pipelined_e2e(info, dev, e2e_sets, lambda st: st[0].copy_(in_h, non_blocking=True), dec_compute,
                           lambda st: out_h.copy_(st[2], non_blocking=True), e2e_steps)
    binding.check()
    h2d = in_h.numel()

    peak, peak_src = peaks()
    res = {
        "metric": METRIC_DECODE, "value": round(gbs * world, 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 cache, uniform ragged lengths, random page order)",
        "config": {"workload": f"{cfg.name}: {cfg.note}; a step appends the new rows' K/V and attends",
                   "B": B, "Sq": Sq, "H": H, "d": d,
                   "page_size": cfg.page_size, "lengths": [int(x) for x in host[4]], "causal": cfg.causal,
                   "splits": splits, "seed": cfg.seed,
                   "l2": "L2 flushed before every timed step (512 MiB written, then 512 MiB read: no dirty lines "
                         "left to write back inside the step); KV cache > L2",
                   "bytes": "K and V rows of every visible key + q, O, LSE"},
        "roofline": {"kernel": "fa_decode_kernel<128> (append and merge fused; timed with the counter-"
                               "zeroing launch before it)", "bound": "hbm", "achieved": round(gbs, 1),
                     "peak": peak["hbm_gbs"], "unit": "GB/s", "frac": round(gbs / peak["hbm_gbs"], 4),
                     "peak_source": f"{peak_src} hbm_gbs (copy bandwidth)",
                     "traffic": recorded_traffic("fa_decode_kernel", cfg.name), "algorithmic_bytes": nbytes},
        "e2e": {"value": round(nbytes * world / (e2e_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": out_h.numel(),
                "pipelining": "one packed copy up (q, new K/V rows, block table, lengths) and one down (O, LSE) per "
                              "step, on their own streams, overlapping the previous and next steps' compute (two "
                              "device buffer sets)"},
        "gpu_launches": (2 if splits > 1 else 1) * args.steps,  # counter zeroing, decode kernel
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, dt, seqs, threads = oracle_sample_decode(cfg, args.cpu_seconds, host)
        res["cpu_baseline"] = {"value": round(v, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                               "sample": f"fp64 decode oracle (page gather + definition) on {seqs} sequences of "
                                         f"{cfg.name}, {dt:.1f} s, same byte convention"}
    mg.shutdown(info)
    if rank == 0:
        print(json.dumps(res), flush=True)


def run_gpu_fp8(args):
    """E4M3 forward: one step = one fa_fwd_fp8 launch over the whole workload."""
    info = mg.rank_info()
    world, rank, local = info.world, info.rank, info.local_rank
    torch.cuda.set_device(local)
    mg.init(info, "nccl", device=torch.device("cuda", local))
    cfg = FP8_CONFIGS[args.config]
    scale, causal, win = cfg.scale, cfg.causal, (cfg.win_l, cfg.win_r)
    B, N, H, d = cfg.shape
    codes_h, desc_h = make_fp8_inputs(cfg)
    dev = torch.device("cuda", torch.cuda.current_device())
    codes = [x.to(dev) for x in codes_h]
    desc = [x.to(dev) for x in desc_h]
    o = torch.empty((B, N, H, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        binding.fwd_fp8_into(*codes, *desc, o, lse, scale, causal, win)

    for _ in range(args.warmup):
        step()
    binding.check()
    torch.cuda.synchronize()
    sampler = ClockSampler(dev.index) if local == 0 else None
    mg.barrier(info)
    torch.cuda.synchronize()
    t_wall0 = time.time()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(args.steps):
        step()
    end.record(stream)
    torch.cuda.synchronize()
    mg.barrier(info)
    t_wall1 = time.time()
    binding.check()
    clocks = sampler.stop(t_wall0, t_wall1) if sampler else None
    ms_step = mg.max_over_ranks(info, start.elapsed_time(end), dev) / args.steps
    f_fwd, _ = flops(B, N, H, d, causal, *win)

    pin = [x.pin_memory() for x in (*codes_h, *desc_h)]
    o_h = torch.empty((B, N, H, d), dtype=torch.bfloat16).pin_memory()
    lse_h = torch.empty((B, H, N), dtype=torch.float32).pin_memory()
    e2e_sets = [((*codes, *desc), (o, lse))]
    e2e_sets.append((tuple(torch.empty_like(x) for x in (*codes, *desc)), (torch.empty_like(o), torch.empty_like(lse))))

    def fp8_copy_in(st):
        for src, dst in zip(pin, st[0]):
            dst.copy_(src, non_blocking=True)

    def fp8_compute(st, s):
        binding.fwd_fp8_into(*st[0], *st[1], scale, causal, win, stream=s)

    def fp8_copy_out(st):
        o_h.copy_(st[1][0], non_blocking=True)
        lse_h.copy_(st[1][1], non_blocking=True)

    e2e_steps = max(4, min(args.steps, 20))
    e2e_ms = pipelined_e2e(info, dev, e2e_sets, fp8_copy_in, fp8_compute, fp8_copy_out, e2e_steps)
    binding.check()

    peak, peak_src = peaks()
    fp8_peak = peak["bf16_tflops"] * FP8_PER_BF16
    achieved = f_fwd / (ms_step * 1e-3) / 1e12
    in_bytes = 3 * B * N * H * d + 3 * B * H * 4
    res = {
        "metric": METRIC_FP8, "value": round(mg.aggregate_rate(f_fwd, world, ms_step * 1e-3) / 1e12, 3),
        "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3",
        "data": "synthetic (seeded N(0,1), per-head E4M3 quantisation with descale = amax/448)",
        "config": {"workload": f"{cfg.name}: {cfg.note}", "B": B, "N": N, "H": H, "d": d, "causal": causal,
                   "window": list(win), "seed": cfg.seed,
                   "l2": f"inputs larger than L2 (q,k,v = {in_bytes / 2**20:.0f} MiB > 126 MiB); no flush",
                   "flops": "4*d*pairs over exactly counted visible pairs",
                   "per_rank": "each rank runs the whole workload on its own inputs"},
        "roofline": {"kernel": "fa_fwd_kernel<128, E4M3>", "bound": "tensor", "achieved": round(achieved, 2),
                     "peak": round(fp8_peak, 1), "unit": "TFLOP/s", "frac": round(achieved / fp8_peak, 4),
                     "frac_of_bf16_peak": round(achieved / peak["bf16_tflops"], 4),
                     "peak_source": f"{peak_src} bf16_tflops x {FP8_PER_BF16} (nominal dense FP8/BF16 ratio)",
                     "traffic": recorded_traffic("fa_fwd_kernel<128, E4M3>", cfg.name),
                     "algorithmic_bytes": in_bytes + B * N * H * d * 2 + B * H * N * 4},
        "e2e": {"value": round(mg.aggregate_rate(f_fwd, world, e2e_ms * 1e-3) / 1e12, 3), "unit": UNIT,
                "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": in_bytes,
                "d2h_bytes_per_step": B * N * H * d * 2 + B * H * N * 4,
                "pipelining": "copy-in, fa_fwd_fp8 and copy-out of consecutive steps on three streams with two "
                              "device buffer sets (every step copies its own inputs and outputs)"},
        "gpu_launches": 2 * args.steps,  # the forward's work-counter reset and the forward
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tf, dt, rows, threads = oracle_sample_fp8(cfg, args.cpu_seconds, codes_h, desc_h)
        res["cpu_baseline"] = {"value": round(tf, 6), "unit": UNIT, "cores": threads, "kind": "oracle",
                               "sample": f"fp64 oracle E4M3 forward (decode, descale, definition) of {rows} query rows "
                                         f"(512-row blocks, heads of batch 0 in order) of {cfg.name}, {dt:.1f} s"}
    mg.shutdown(info)
    if rank == 0:
        print(json.dumps(res), flush=True)


def time_attention(cfg, dev, iters: int, warm: int, flush) -> dict:
    """Device time of one workload's forward and backward stages (the bench's launch configuration):
    every iteration flushes L2, then times fa_fwd and each backward launch with CUDA events on the
    launching stream. Returns mean milliseconds per launch."""
    q_h, k_h, v_h, do_h = make_inputs(cfg)
    q, k, v, do = (x.to(dev) for x in (q_h, k_h, v_h, do_h))
    B, N, H, d = cfg.shape
    o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    ws = torch.empty(binding.workspace_bytes(B, N, H, d), dtype=torch.uint8, device=dev) if cfg.backward else None
    stream = torch.cuda.current_stream()
    win = (cfg.win_l, cfg.win_r)
    marks = {}

    def one(record: bool):
        flush()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        evs[0].record(stream)
        binding.fwd_into(q, k, v, o, lse, cfg.scale, cfg.causal, win)
        evs[1].record(stream)
        if cfg.backward:
            binding.bwd_stages(q, k, v, o, lse, do, dq, dk, dv, ws, cfg.scale, cfg.causal, win,
                               between=lambda i: i > 0 and evs[1 + i].record(stream))
        if record:
            marks.setdefault("ev", []).append(evs)

    for _ in range(warm):
        one(False)
    for _ in range(iters):
        one(True)
    torch.cuda.synchronize()
    binding.check()
    ev = marks["ev"]
    out = {"fwd_ms": statistics.mean(e[0].elapsed_time(e[1]) for e in ev)}
    if cfg.backward:
        out["pre_ms"] = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
        out["main_ms"] = statistics.mean(e[2].elapsed_time(e[3]) for e in ev)
        out["conv_ms"] = statistics.mean(e[3].elapsed_time(e[4]) for e in ev)
    del q, k, v, do, o, dq, dk, dv, lse, ws
    return out


def config_figures(cfg, t: dict, peak: dict) -> dict:
    """TFLOP/s (exact pair count and tile-granular count), fractions of the measured bf16 peak and,
    for the window workload, achieved algorithmic bytes per second against the HBM copy bandwidth."""
    B, N, H, d = cfg.shape
    win = (cfg.win_l, cfg.win_r)
    f_fwd, f_bwd = flops(B, N, H, d, cfg.causal, *win)
    g_fwd, g_bwd = flops_tile_granular(B, N, H, d, cfg.causal, *win)
    by_fwd, by_bwd = hbm_bytes(B, N, H, d)
    pk = peak["bf16_tflops"]
    r = {"workload": f"{cfg.name}: {cfg.note}", "fwd_ms": round(t["fwd_ms"], 4),
         "fwd_tflops": round(f_fwd / (t["fwd_ms"] * 1e-3) / 1e12, 2),
         "fwd_tflops_tile_granular": round(g_fwd / (t["fwd_ms"] * 1e-3) / 1e12, 2),
         "fwd_frac_of_peak": round(f_fwd / (t["fwd_ms"] * 1e-3) / 1e12 / pk, 4),
         "fwd_gflop": round(f_fwd / 1e9, 3), "fwd_gflop_tile_granular": round(g_fwd / 1e9, 3)}
    if cfg.backward:
        bwd_ms = t["pre_ms"] + t["main_ms"] + t["conv_ms"]
        r.update({"bwd_ms": round(bwd_ms, 4),
                  "bwd_stage_ms": {"preprocess": round(t["pre_ms"], 4), "main": round(t["main_ms"], 4),
                                   "dq_convert": round(t["conv_ms"], 4)},
                  "bwd_tflops": round(f_bwd / (bwd_ms * 1e-3) / 1e12, 2),
                  "bwd_tflops_tile_granular": round(g_bwd / (bwd_ms * 1e-3) / 1e12, 2),
                  "bwd_main_tflops": round(f_bwd / (t["main_ms"] * 1e-3) / 1e12, 2),
                  "bwd_frac_of_peak": round(f_bwd / (bwd_ms * 1e-3) / 1e12 / pk, 4),
                  "bwd_gflop": round(f_bwd / 1e9, 3), "bwd_gflop_tile_granular": round(g_bwd / 1e9, 3)})
    if cfg.win_l >= 0 or cfg.win_r >= 0:  # a narrow window is bound by its algorithmic bytes
        hb = peak["hbm_gbs"]
        r["fwd_gbs"] = round(by_fwd / (t["fwd_ms"] * 1e-3) / 1e9, 1)
        r["fwd_frac_of_hbm"] = round(r["fwd_gbs"] / hb, 4)
        if cfg.backward:
            r["bwd_gbs"] = round(by_bwd / (r["bwd_ms"] * 1e-3) / 1e9, 1)
            r["bwd_frac_of_hbm"] = round(r["bwd_gbs"] / hb, 4)
        r["algorithmic_bytes"] = {"fwd": by_fwd, "bwd": by_bwd, "convention": "fwd 4T+L, bwd 8T+L"}
    return r


EXTRA_CONFIGS = {"tiny_fwd": (50, 5), "gpt_fwd": (50, 5), "train_fwd_bwd": (20, 3), "window_fwd_bwd": (40, 5),
                 "long_fwd_bwd": (6, 2)}


def run_gpu(args):
    info = mg.rank_info()
    world, rank, local = info.world, info.rank, info.local_rank
    torch.cuda.set_device(local)
    mg.init(info, "nccl", device=torch.device("cuda", local))
    cfg = CONFIGS[args.config]
    if not cfg.backward:
        raise SystemExit(f"config {cfg.name} has no backward; a step is forward + backward")
    scale, causal, win = cfg.scale, cfg.causal, (cfg.win_l, cfg.win_r)
    B, N, H, d = cfg.shape
    q_h, k_h, v_h, do_h = make_inputs(cfg)
    dev = torch.device("cuda", torch.cuda.current_device())
    q, k, v, do = (x.to(dev) for x in (q_h, k_h, v_h, do_h))
    o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    ws = torch.empty(binding.workspace_bytes(B, N, H, d), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    flush = l2_flusher(dev)

    def step(evs=None):
        """One step; with evs (5 events): fwd start, preprocess, main, convert, end marks."""
        if evs:
            evs[0].record(stream)
        binding.fwd_into(q, k, v, o, lse, scale, causal, win)
        if evs:
            evs[1].record(stream)
        binding.bwd_stages(q, k, v, o, lse, do, dq, dk, dv, ws, scale, causal, win,
                           between=(lambda i: i > 0 and evs[1 + i].record(stream)) if evs else None)

    for _ in range(args.warmup):
        flush()
        step()
    binding.check()
    torch.cuda.synchronize()

    steps_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    sampler = ClockSampler(dev.index) if local == 0 else None
    mg.barrier(info)
    torch.cuda.synchronize()
    t_wall0 = time.time()
    for evs in steps_ev:
        flush()  # outside the step's timed interval
        step(evs)
    torch.cuda.synchronize()
    mg.barrier(info)
    t_wall1 = time.time()
    binding.check()
    clocks = sampler.stop(t_wall0, t_wall1) if sampler else None

    ms_total = mg.max_over_ranks(info, sum(e[0].elapsed_time(e[4]) for e in steps_ev), dev)
    ms_step = ms_total / args.steps
    f_fwd, f_bwd = flops(B, N, H, d, causal, *win)
    g_fwd, g_bwd = flops_tile_granular(B, N, H, d, causal, *win)
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in steps_ev)
    pre_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in steps_ev)
    main_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in steps_ev)
    conv_ms = statistics.mean(e[3].elapsed_time(e[4]) for e in steps_ev)
    bwd_ms = pre_ms + main_ms + conv_ms

    # ---- end to end through the public API with host buffers (pinned), copies inside the timed region.
    # Every step copies its inputs host -> device, runs fa_fwd + fa_bwd and copies its outputs back,
    # pipelined over three streams and two device buffer sets (pipelined_e2e).
    pin = [x.pin_memory() for x in (q_h, k_h, v_h, do_h)]
    out_h = [torch.empty_like(q_h).pin_memory() for _ in range(4)]
    lse_h = torch.empty((B, H, N), dtype=torch.float32).pin_memory()
    sets = [((q, k, v, do), (o, dq, dk, dv), lse, ws)]
    sets.append((tuple(torch.empty_like(x) for x in (q, k, v, do)), tuple(torch.empty_like(x) for x in (o, dq, dk, dv)),
                 torch.empty_like(lse), torch.empty_like(ws)))

    def train_copy_in(st):
        for src, dst in zip(pin, st[0]):
            dst.copy_(src, non_blocking=True)

    def train_compute(st, s):
        (qi, ki, vi, doi), (oo, dqo, dko, dvo), lseo, wso = st
        binding.fwd_into(qi, ki, vi, oo, lseo, scale, causal, win, stream=s)
        binding.bwd_into(qi, ki, vi, oo, lseo, doi, dqo, dko, dvo, scale, causal, win, workspace=wso, stream=s)

    def train_copy_out(st):
        for src, dst in zip(st[1], out_h):
            dst.copy_(src, non_blocking=True)
        lse_h.copy_(st[2], non_blocking=True)

    e2e_steps = max(4, min(args.steps, 20))
    e2e_ms = pipelined_e2e(info, dev, sets, train_copy_in, train_compute, train_copy_out, e2e_steps)
    binding.check()
    del sets, pin, out_h, lse_h

    peak, peak_src = peaks()
    main_tflops = f_bwd / (main_ms * 1e-3) / 1e12
    fwd_tflops = f_fwd / (fwd_ms * 1e-3) / 1e12
    bwd_tflops = f_bwd / (bwd_ms * 1e-3) / 1e12
    dominant = "fa_bwd_kernel" if main_ms >= fwd_ms else "fa_fwd_kernel"
    dom_ms, dom_flops = (main_ms, f_bwd) if dominant == "fa_bwd_kernel" else (fwd_ms, f_fwd)
    achieved = dom_flops / (dom_ms * 1e-3) / 1e12
    traffic = recorded_traffic(dominant, cfg.name)
    t_bytes = B * N * H * d * 2
    res = {
        "metric": METRIC, "value": round(mg.aggregate_rate(f_fwd + f_bwd, world, ms_step * 1e-3) / 1e12, 3),
        "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16)",
        "config": attn_config(cfg),
        "notes": {"l2": L2_NOTE,
                  "flops": "fwd 4*d*pairs + bwd 10*d*pairs over exactly counted visible pairs; the tile-granular "
                           "count (every touched 128x128 block in full) is reported beside it",
                  "per_rank": "each rank runs the whole workload on its own inputs"},
        "fwd_tflops": round(fwd_tflops, 2), "bwd_tflops": round(bwd_tflops, 2),
        "bwd_main_tflops": round(main_tflops, 2),
        "fwd_ms": round(fwd_ms, 4), "bwd_ms": round(bwd_ms, 4),
        "bwd_stage_ms": {"preprocess": round(pre_ms, 4), "main": round(main_ms, 4), "dq_convert": round(conv_ms, 4)},
        "gflop": {"fwd": round(f_fwd / 1e9, 3), "bwd": round(f_bwd / 1e9, 3),
                  "fwd_tile_granular": round(g_fwd / 1e9, 3), "bwd_tile_granular": round(g_bwd / 1e9, 3)},
        "value_tile_granular": round(mg.aggregate_rate(g_fwd + g_bwd, world, ms_step * 1e-3) / 1e12, 3),
        "frac_of_peak": {"fwd": round(fwd_tflops / peak["bf16_tflops"], 4),
                         "bwd": round(bwd_tflops / peak["bf16_tflops"], 4),
                         "denominator": f"bf16_tflops {peak['bf16_tflops']} ({peak_src})",
                         "fwd_of_datasheet_2250": round(fwd_tflops / 2250.0, 4),
                         "bwd_of_datasheet_2250": round(bwd_tflops / 2250.0, 4)},
        "roofline": {"kernel": dominant, "bound": "tensor", "achieved": round(achieved, 2),
                     "peak": peak["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(achieved / peak["bf16_tflops"], 4),
                     "frac_of_sustained": round(achieved / peak.get("bf16_tflops_sustained", peak["bf16_tflops"]), 4),
                     "peak_source": f"{peak_src} bf16_tflops (burst)", "traffic": traffic,
                     "algorithmic_bytes": hbm_bytes(B, N, H, d)[1 if dominant == "fa_bwd_kernel" else 0]},
        "e2e": {"value": round(mg.aggregate_rate(f_fwd + f_bwd, world, e2e_ms * 1e-3) / 1e12, 3), "unit": UNIT,
                "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": 4 * t_bytes,
                "d2h_bytes_per_step": 4 * t_bytes + B * H * N * 4,
                "pipelining": "copy-in, fa_fwd + fa_bwd and copy-out of consecutive steps on three streams with two "
                              "device buffer sets (every step copies its own inputs and outputs)"},
        # per step: the forward's work-counter reset and the forward; the backward's
        # preprocess, main kernel and dQ conversion
        "gpu_launches": 5 * args.steps,
        "clocks": clocks,
    }
    if not args.no_extras:
        # the other workloads, device-timed in the same run (after the timed region above)
        extras = {}
        for name, (iters, warm) in EXTRA_CONFIGS.items():
            if name == cfg.name:
                continue
            t = time_attention(CONFIGS[name], dev, iters, warm, flush)
            extras[name] = config_figures(CONFIGS[name], t, peak)
        extras[cfg.name] = config_figures(cfg, {"fwd_ms": fwd_ms, "pre_ms": pre_ms, "main_ms": main_ms,
                                                "conv_ms": conv_ms}, peak)
        res["configs"] = extras
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tf, dt, rows, threads = oracle_sample(cfg, args.cpu_seconds, q_h, k_h, v_h, do_h)
        res["cpu_baseline"] = {"value": round(tf, 6), "unit": UNIT, "cores": threads, "kind": "oracle",
                               "sample": f"fp64 oracle, forward+backward of {rows} query rows (512-row blocks, heads of "
                                         f"batch 0 in order) of {cfg.name}, {dt:.1f} s, same pair-count FLOP convention"}
    mg.shutdown(info)
    if rank == 0:
        print(json.dumps(res), flush=True)


# ----------------------------------------------------------------------------- reference arm (CPU oracle)

def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    per_step = max(0.5, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    if args.config in FP8_CONFIGS:
        return run_reference_fp8(args, FP8_CONFIGS[args.config], per_step, world)
    if args.config in DECODE_CONFIGS:
        return run_reference_decode(args, DECODE_CONFIGS[args.config], per_step, world)
    cfg = CONFIGS[args.config]
    q, k, v, do = make_inputs(cfg)
    for _ in range(args.warmup):
        oracle_sample(cfg, per_step, q, k, v, do)
    vals, threads, rows, secs = [], 1, 0, 0.0
    for _ in range(args.steps):
        tf, dt, rows, threads = oracle_sample(cfg, per_step, q, k, v, do)
        vals.append(tf)
        secs += dt
    value = statistics.mean(vals)
    sample = (f"fp64 oracle, forward+backward of {rows} query rows (512-row blocks, heads of batch 0 in order) of {cfg.name} per step, "
              f"about {per_step:.1f} s each")
    res = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs / max(1, args.steps) * 1e3, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (seeded N(0,1) bf16 widened to fp64)",
           "config": attn_config(cfg),
           "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": threads, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def run_reference_decode(args, cfg, per_step, world):
    host = make_decode_inputs(cfg)
    for _ in range(args.warmup):
        oracle_sample_decode(cfg, per_step, host)
    vals, threads, seqs, secs = [], 1, 0, 0.0
    for _ in range(args.steps):
        v, dt, seqs, threads = oracle_sample_decode(cfg, per_step, host)
        vals.append(v)
        secs += dt
    value = statistics.mean(vals)
    res = {"impl": "reference", "metric": METRIC_DECODE, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs / max(1, args.steps) * 1e3, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (seeded N(0,1) bf16 cache widened to fp64)",
           "config": {"workload": f"{cfg.name}: {cfg.note}", "B": cfg.B, "Sq": cfg.Sq, "H": cfg.H, "d": cfg.d,
                      "page_size": cfg.page_size, "seed": cfg.seed},
           "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                            "sample": f"fp64 decode oracle on {seqs} sequences per step, about {per_step:.1f} s each"},
           "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def run_reference_fp8(args, cfg, per_step, world):
    codes, descales = make_fp8_inputs(cfg)
    for _ in range(args.warmup):
        oracle_sample_fp8(cfg, per_step, codes, descales)
    vals, threads, rows, secs = [], 1, 0, 0.0
    for _ in range(args.steps):
        tf, dt, rows, threads = oracle_sample_fp8(cfg, per_step, codes, descales)
        vals.append(tf)
        secs += dt
    value = statistics.mean(vals)
    sample = (f"fp64 oracle E4M3 forward of {rows} query rows (512-row blocks, heads of batch 0 in order) of "
              f"{cfg.name} per step, about {per_step:.1f} s each")
    res = {"impl": "reference", "metric": METRIC_FP8, "value": round(value, 6), "unit": UNIT, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs / max(1, args.steps) * 1e3, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (seeded N(0,1), E4M3 codes decoded to fp64)",
           "config": {"workload": f"{cfg.name}: {cfg.note}", "B": cfg.B, "N": cfg.N, "H": cfg.H, "d": cfg.d,
                      "causal": cfg.causal, "window": [cfg.win_l, cfg.win_r], "seed": cfg.seed},
           "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": threads, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="long_fwd_bwd",
                    choices=sorted(CONFIGS) + sorted(FP8_CONFIGS) + sorted(DECODE_CONFIGS))
    ap.add_argument("--splits", type=int, default=0, help="decode: CTAs (pieces) per head; 0 = library's choice")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the other workloads' device-timed figures")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.config in FP8_CONFIGS:
        run_gpu_fp8(args)
    elif args.config in DECODE_CONFIGS:
        run_gpu_decode(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()

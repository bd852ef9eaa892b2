#!/usr/bin/env python
"""Forward-attention throughput on B200: TFLOP/s and fraction of roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload long] [--impl ours|reference]

--gpus N > 1 without a launcher starts N ranks itself (torch.distributed.run,
one process per GPU, rendezvous on 127.0.0.1); under torchrun, WORLD_SIZE must
equal N.

One step = one exact-attention forward pass (every step of the hot path, one
kernel launch) over the whole workload, inputs resident in HBM.  The default
workload is B8 H32 N4096 d128 bf16, non-causal (the shape of the pages' B8 H32
N4096 d128 benchmark).  FLOPs per step = 4 B Hq Nq Nk d (halved when causal).

Multi-GPU (torchrun, one process per GPU): every rank runs an independent
batch of the same shape (weak scaling, no collective on the data path);
``value`` is the FLOPs of all ranks divided by the slowest rank's time.

``--impl reference`` times the fp64 CPU oracle on the host cores instead, on a
bounded sample of the same workload per step (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "fwd attention TFLOP/s (B8 H32 N4096 d128 bf16) and % of B200 BF16 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# device code of each workload's dominant kernel: a recorded ncu traffic figure is
# valid only for the sources it was captured on
_CSRC = "exact_attention_157_b200/csrc/"
_COMMON = [_CSRC + "fwd_common.cuh", _CSRC + "sm100_ptx.cuh"]
KERNEL_SOURCES = {"tile": [_CSRC + "fwd_kernel_pp.cuh"] + _COMMON,
                  "short": [_CSRC + "short_kernel.cuh"] + _COMMON,
                  "decode": [_CSRC + "decode_kernel.cuh"] + _COMMON,
                  "bwd": [_CSRC + "bwd_kernels.cuh"] + _COMMON}


def kernel_family(w) -> str:
    """Which kernel a workload's forward runs on (the dispatch of attn_api.cu)."""
    if w.backward:
        return "bwd"
    if w.split_kv and w.Hq // w.Hkv * w.Nq <= 16 and not w.is_causal:
        return "decode"
    if w.d == 64 and w.Nk <= 256 and not w.fp8 and not w.softcap and w.mask2d is None and not w.split_kv:
        return "short"
    return "tile"


# --------------------------------------------------------------- helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS, source="fallback")


def kernel_source_hash(family: str = "tile") -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[family]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(w):
    """DRAM bytes per launch of this kernel and workload from profiles/traffic.json
    (written beside the ncu summaries), if they were taken on the current kernel
    sources; else None."""
    key = f"attn_{'bwd' if w.backward else 'fwd'}_{w.name}"
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f).get(key)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("kernel_source_sha") != kernel_source_hash(kernel_family(w)):
        return None
    return float(rec["traffic_bytes_per_launch"])


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {  # NVML clocks-event reason bits
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.idx, self.period = device_index, period_s
        self.samples, self.reason_bits = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001 - NVML missing: clocks are reported as unknown
            self.nvml = None

    def _run(self):
        n = self.nvml
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM))
                self.reason_bits |= int(n.nvmlDeviceGetCurrentClocksEventReasons(self.handle))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        reasons = [name for bit, name in self.REASONS.items() if self.reason_bits & bit and bit != 0x1]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples), "reasons": reasons}


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Slowest rank's time (all ranks call this in the same order)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def mask2d_keys_per_row(w):
    """Keys each query row may see under the workload's 2-D mask (numpy int
    array of length Nq): the algorithmic work of a masked workload counts only
    these (query, key) pairs."""
    import numpy as np
    kind, W, size = w.mask2d[0], int(w.mask2d[1]), int(w.mask2d[2])
    shift = int(w.mask2d[3]) if len(w.mask2d) > 3 else 0
    i = np.arange(w.Nq)[:, None]
    j = np.arange(w.Nk)[None, :]
    ri, ci, rj, cj = i // W, i % W, j // W, j % W
    if kind == "neighborhood":
        ok = (np.abs(ri - rj) < size) & (np.abs(ci - cj) < size)
    else:
        ok = ((ri + shift) // size == (rj + shift) // size) & ((ci + shift) // size == (cj + shift) // size)
    if w.is_causal:
        ok &= j <= i
    return ok.sum(axis=1)


def workload_flops(w):
    """Forward FLOPs of one step: the metric's 4*B*Hq*Nq*Nk*d (halved when
    causal) for dense workloads; 4*d per visible (query, key) pair under a 2-D mask."""
    if w.mask2d is None:
        return w.flops()
    return 4.0 * w.d * w.B * w.Hq * float(mask2d_keys_per_row(w).sum())


# ---------------------------------------------------------- CPU baseline
def oracle_sample(w, q, k, v, kl, target_s: float, max_rows=None, scales=None):
    """Runs the fp64 oracle on a bounded sample of the workload: whole query
    rows of the first (batch, head) pairs, as many as fit in ~target_s.
    FP8 workloads pass E4M3 codes as q, k, v and their block scales in
    ``scales``; the sampled heads are dequantized first.
    Returns (flops, seconds, description, threads)."""
    import numpy as np
    import oracle
    threads = oracle.default_threads()
    kl_list = None if kl is None else kl.cpu().tolist()
    group = w.Hq // w.Hkv

    def head_inputs(b, h):
        hk = h // group
        cut = lambda t, i: t[b:b + 1, i:i + 1].cpu()  # noqa: E731
        if scales is None:
            qh, kh, vh = (cut(t, i).double().numpy() for t, i in ((q, h), (k, hk), (v, hk)))
        else:
            qh, kh, vh = (oracle.dequantize_blocks(cut(t, i).numpy(), cut(sc, i).numpy())
                          for t, sc, i in ((q, scales[0], h), (k, scales[1], hk), (v, scales[2], hk)))
        return qh, kh, vh, None if kl_list is None else [kl_list[b]]

    per_row = None if w.mask2d is None else mask2d_keys_per_row(w)
    var = dict(softcap=w.softcap, mask2d=w.mask2d)

    def flops_of(b, rows):
        nk = w.Nk if kl_list is None else kl_list[b]
        total = 0.0
        for i in rows:
            if per_row is not None:
                keys = int(per_row[i])
            else:
                keys = min(nk, i + 1) if w.is_causal else nk
            total += 4.0 * keys * w.d
        return total

    # calibrate on a slice of the first head
    qh, kh, vh, klh = head_inputs(0, 0)
    cal_rows = list(range(0, w.Nq, max(1, w.Nq // max(1, min(w.Nq, 4 * threads)))))[: 4 * threads]
    t0 = time.perf_counter()
    oracle.attention(qh, kh, vh, is_causal=w.is_causal, key_lens=klh, rows=cal_rows, **var)
    t_cal = max(time.perf_counter() - t0, 1e-6)
    per_flop = t_cal / max(flops_of(0, cal_rows), 1.0)
    budget = target_s / per_flop  # flops we can afford
    # choose rows: whole heads while they fit, then a prefix of rows of the next head
    plan, used = [], 0.0
    for bh in range(w.B * w.Hq):
        b, h = divmod(bh, w.Hq)
        rows = list(range(w.Nq))
        f = flops_of(b, rows)
        if used + f <= budget:
            plan.append((b, h, rows))
            used += f
            continue
        # partial head: as many rows as fit (at least one row overall)
        n = max(1 if not plan else 0, int(w.Nq * (budget - used) / max(f, 1.0)))
        if max_rows is not None:
            n = min(n, max_rows)
        if n > 0:
            plan.append((b, h, rows[:n]))
            used += flops_of(b, rows[:n])
        break
    t0 = time.perf_counter()
    total = 0.0
    for b, h, rows in plan:
        qh, kh, vh, klh = head_inputs(b, h)
        oracle.attention(qh, kh, vh, is_causal=w.is_causal, key_lens=klh,
                         rows=None if len(rows) == w.Nq else rows, **var)
        total += flops_of(b, rows)
    dt = time.perf_counter() - t0
    n_rows = sum(len(r) for _, _, r in plan)
    desc = (f"{n_rows} query rows over {len(plan)} (batch, head) pairs of the {w.name} workload "
            f"({n_rows / (w.B * w.Hq * w.Nq):.2e} of it), fp64{' on the dequantized FP8 inputs' if scales else ''}, "
            f"all keys of each row")
    return total, dt, desc, threads


def oracle_sample_bwd(w, q, k, v, do, kl, target_s: float):
    """The fp64 backward oracle on a bounded sample: the first R query rows of
    the first (batch, K/V head) pairs (every query head of the group), R chosen
    to fill ~target_s.  Returns (flops, seconds, description, threads)."""
    import oracle
    threads = oracle.default_threads()
    kl_list = None if kl is None else kl.cpu().tolist()
    G = w.Hq // w.Hkv

    def inputs(b, hk, R):
        h0 = hk * G
        cut = lambda t, a, z: t[b:b + 1, a:z].cpu().double().numpy()
        return (cut(q, h0, h0 + G)[:, :, :R], cut(k, hk, hk + 1), cut(v, hk, hk + 1), cut(do, h0, h0 + G)[:, :, :R],
                None if kl_list is None else [kl_list[b]])

    def flops_of(b, R):
        nk = w.Nk if kl_list is None else kl_list[b]
        return sum(10.0 * w.d * G * (min(nk, i + 1) if w.is_causal else nk) for i in range(R))

    R0 = min(w.Nq, 16)
    t0 = time.perf_counter()
    qq, kk, vv, dd, ll = inputs(0, 0, R0)
    oracle.attention_bwd(qq, kk, vv, dd, is_causal=w.is_causal, key_lens=ll, n_threads=1)
    per_flop = max(time.perf_counter() - t0, 1e-6) / max(flops_of(0, R0), 1.0)
    # units run one per thread: give each thread ~target_s of rows
    n_units = min(threads, w.B * w.Hkv)
    R = max(1, min(w.Nq, int(R0 * target_s / max(per_flop * flops_of(0, R0), 1e-9))))
    units = [divmod(u, w.Hkv) for u in range(n_units)]
    t0 = time.perf_counter()
    import concurrent.futures as cf
    with cf.ThreadPoolExecutor(max_workers=n_units) as ex:
        list(ex.map(lambda bk: oracle.attention_bwd(*inputs(bk[0], bk[1], R)[:4], is_causal=w.is_causal,
                                                     key_lens=inputs(bk[0], bk[1], 1)[4], n_threads=1), units))
    dt = time.perf_counter() - t0
    total = sum(flops_of(b, R) for b, _ in units)
    desc = (f"backward of the first {R} query rows of {n_units} (batch, K/V head) pairs of the {w.name} "
            f"workload, every query head of each group, fp64, one pair per thread")
    return total, dt, desc, n_units


# -------------------------------------------------------------- our arm
def run_ours(args, w):
    import torch
    import exact_attention_157_b200 as ea
    from workloads import make_inputs

    world, rank, local = dist_env()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    scales = None
    if w.fp8:
        from workloads import make_fp8_inputs
        q, k, v, *scales = make_fp8_inputs(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, seed=w.seed + 7 * rank, device=dev)
        kl = None
        out = torch.empty((w.B, w.Hq, w.Nq, w.d), dtype=torch.bfloat16, device=dev)
    else:
        q, k, v, kl = make_inputs(w, device=dev, seed=w.seed + 7 * rank)
        out = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    flops = workload_flops(w)
    in_bytes = sum(t.numel() * t.element_size() for t in [q, k, v] + (scales or []) + ([] if kl is None else [kl]))
    out_bytes = out.numel() * 2 + lse.numel() * 4
    if w.backward:
        # the forward results and an upstream gradient are inputs of the timed backward step
        from workloads import make_qkv
        dout = make_qkv(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, seed=w.seed + 7 * rank + 1, device=dev)[0]
        ea.attention(q, k, v, is_causal=w.is_causal, key_lens=kl, out=out, lse=lse, stream=stream)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        st, bw_bytes = ea.attn_bwd_plan(w.B, w.Hq, w.Nq)
        bws = torch.empty((bw_bytes,), dtype=torch.uint8, device=dev)
        in_bytes += out.numel() * 2 + lse.numel() * 4 + dout.numel() * 2
        out_bytes = (dq.numel() + dk.numel() + dv.numel()) * 2
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = None
    if in_bytes + out_bytes < 2 * l2_bytes:  # small working set: flush L2 between steps
        flush = torch.empty(2 * l2_bytes // 4, dtype=torch.float32, device=dev)

    # decode-shaped workloads run through the split-KV entry point (workspace allocated once, here)
    split, ws, per_step_launches = None, None, 1
    if w.split_kv:
        split = 0
        st, n_used, nbytes = ea.attn_splitkv_plan(w.B, w.Hq, w.Nq, w.Nk, w.d, split, 0, Hkv=w.Hkv,
                                                  is_causal=w.is_causal)
        if st != ea.ATTN_OK:
            raise ea.AttnError(st, "attn_splitkv_plan")
        ws = torch.empty((max(nbytes, 1),), dtype=torch.uint8, device=dev)
        per_step_launches = 2 if nbytes > 0 else 1  # attention kernel + merge

    def call():
        if w.fp8:
            ea.attention_fp8(q, k, v, *scales, is_causal=w.is_causal, out=out, lse=lse, stream=stream)
            return
        if w.backward:
            ea.attention_backward(q, k, v, out, lse, dout, is_causal=w.is_causal, key_lens=kl, workspace=bws,
                                  stream=stream, dq=dq, dk=dk, dv=dv)
            return
        ea.attention(q, k, v, is_causal=w.is_causal, key_lens=kl, out=out, lse=lse, stream=stream,
                     split_kv=split, workspace=ws, softcap=w.softcap, mask2d=w.mask2d)

    if w.backward:
        per_step_launches = 3  # row statistics, dK / dV, dQ

    def step():
        if flush is not None:
            flush.fill_(1.0)
        call()

    for _ in range(args.warmup):
        step()
    ea.check_device_status(stream)

    # --- device-timed region: K steps, events on the launching stream
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * args.steps)] if flush is not None else None
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    launches = 0
    with ClockSampler(dev.index) as clocks:
        start.record(stream)
        for i in range(args.steps):
            if flush is not None:
                flush.fill_(1.0)
                ev[2 * i].record(stream)
                call()
                ev[2 * i + 1].record(stream)
            else:
                call()
            launches += per_step_launches
        end.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world, dev)
    ea.check_device_status(stream)
    total_ms = start.elapsed_time(end)
    if flush is not None:  # kernel time only, the L2 flush between steps excluded
        kernel_ms = sum(ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(args.steps))
    else:
        kernel_ms = total_ms
    kernel_ms = max_over_ranks(kernel_ms, world, dev)
    ms_per_step = kernel_ms / args.steps
    value = flops * world / (ms_per_step * 1e-3) / 1e12

    # --- end to end through the public API with pinned host buffers
    e2e_steps = max(1, min(args.steps, 20))
    if w.backward:
        host_in = [t.cpu().pin_memory() for t in (q, k, v, out, lse, dout)]
        host_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (dq, dk, dv)]
        klh = None if kl is None else kl.cpu().pin_memory()

        def e2e_step():
            with torch.cuda.stream(stream):
                for dst, src in zip((q, k, v, out, lse, dout), host_in):
                    dst.copy_(src, non_blocking=True)
                if klh is not None:
                    kl.copy_(klh, non_blocking=True)
                call()
                for dst, src in zip(host_out, (dq, dk, dv)):
                    dst.copy_(src, non_blocking=True)
    elif w.fp8:
        host_in = [t.cpu().pin_memory() for t in [q, k, v] + scales]
        outh = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        lseh = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()

        def e2e_step():
            with torch.cuda.stream(stream):
                for dst, src in zip([q, k, v] + scales, host_in):
                    dst.copy_(src, non_blocking=True)
                call()
                outh.copy_(out, non_blocking=True)
                lseh.copy_(lse, non_blocking=True)
    else:
        qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
        klh = None if kl is None else kl.cpu().pin_memory()
        outh = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        lseh = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        runner = ea.HostAttention(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, device=dev, with_key_lens=kl is not None,
                                  split_kv=split, is_causal=w.is_causal)

        def e2e_step():
            runner(qh, kh, vh, outh, lseh, klh, is_causal=w.is_causal, stream=stream, softcap=w.softcap,
                   mask2d=w.mask2d)
    for _ in range(min(args.warmup, 3)):
        e2e_step()
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / e2e_steps
    ea.check_device_status(stream)
    e2e_value = flops * world / (e2e_ms * 1e-3) / 1e12

    peaks = load_peaks()
    per_launch_flops = flops
    per_launch_bytes = w.qkvo_bytes() + w.lse_bytes()
    if w.backward:  # read Q, K, V, O, dO, LSE; write dQ, dK, dV
        per_launch_bytes = 2 * w.qkvo_bytes() + w.lse_bytes()
    peak_tc, peak_note = peaks["bf16_tflops"], " (burst)"
    if w.fp8:  # E4M3 codes and block scales in, bf16 O and fp32 LSE out
        per_launch_bytes = in_bytes + out.numel() * 2 + w.lse_bytes()
        peak_tc, peak_note = 2.0 * peaks["bf16_tflops"], " bf16 (burst) x 2, the nominal FP8 / BF16 dense ratio"
    t_launch = ms_per_step * 1e-3
    compute_floor = per_launch_flops / (peak_tc * 1e12)
    hbm_floor = per_launch_bytes / (peaks["hbm_gbs"] * 1e9)
    if compute_floor >= hbm_floor:
        roof = {"bound": "tensor", "achieved": per_launch_flops / t_launch / 1e12, "peak": peak_tc,
                "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": per_launch_bytes / t_launch / 1e9, "peak": peaks["hbm_gbs"],
                "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = recorded_traffic(w)
    roof["peak_source"] = peaks["source"] + peak_note
    roof["frac_of_roofline_time"] = max(compute_floor, hbm_floor) / t_launch

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        if w.backward:
            f, dt, desc, threads = oracle_sample_bwd(w, q, k, v, dout, kl, target_s=args.cpu_seconds)
        else:
            f, dt, desc, threads = oracle_sample(w, q, k, v, kl, target_s=args.cpu_seconds, scales=scales)
        cpu = {"value": f / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc,
               "seconds": dt}

    result = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3" if w.fp8 else "bf16", "data": "synthetic",
        "config": {"workload": f"{w.name}: B{w.B} Hq{w.Hq} Hkv{w.Hkv} Nq{w.Nq} Nk{w.Nk} d{w.d}"
                               f"{' causal' if w.is_causal else ''}{' fp8 e4m3' if w.fp8 else ''}",
                   "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Nq": w.Nq, "Nk": w.Nk, "d": w.d,
                   "is_causal": w.is_causal, "key_lens": w.key_lens,
                   "entry_point": ("attn_fwd_fp8" if w.fp8 else "attn_bwd" if w.backward else
                                   "attn_fwd_splitkv" if w.split_kv else
                                   "attn_fwd_mod" if (w.softcap or w.mask2d) else "attn_fwd"),
                   "softcap": w.softcap, "mask2d": w.mask2d,
                   "flops_per_step": flops, "parallelism": f"independent batch per GPU x{world}",
                   "l2": ("L2 flushed between steps (kernel time only)" if flush is not None
                          else f"inputs larger than L2 ({in_bytes / 1e6:.0f} MB > {l2_bytes / 1e6:.0f} MB)")},
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": in_bytes,
                "d2h_bytes_per_step": out_bytes, "ms_per_step": e2e_ms},
        "gpu_launches": launches,
        "clocks": clocks.summary(),
        "kernel_source_sha": kernel_source_hash(kernel_family(w)),
    }
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


# -------------------------------------------------------- reference arm
def run_reference(args, w):
    world, rank, _ = dist_env()
    if rank != 0:
        return  # rank 0 alone runs the CPU oracle
    import torch
    from workloads import make_inputs
    scales = None
    if w.fp8:
        from workloads import make_fp8_inputs
        q, k, v, *scales = make_fp8_inputs(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, seed=w.seed)
        kl = None
    else:
        q, k, v, kl = make_inputs(w, device="cpu")
    do = None
    if w.backward:
        from workloads import make_qkv
        do = make_qkv(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, seed=w.seed + 1)[0]
    steps, warmup = max(1, args.steps), max(0, args.warmup)
    per_step = max(0.2, min(10.0, args.reference_seconds / (steps + warmup)))
    times, flops_total, desc, threads = [], 0.0, "", 1
    for i in range(warmup + steps):
        if w.backward:
            f, dt, desc, threads = oracle_sample_bwd(w, q, k, v, do, kl, target_s=per_step)
        else:
            f, dt, desc, threads = oracle_sample(w, q, k, v, kl, target_s=per_step, scales=scales)
        if i >= warmup:
            times.append(dt)
            flops_total += f
    t = sum(times)
    value = flops_total / t / 1e12
    result = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": steps, "warmup": warmup,
        "ms_per_step": 1e3 * t / steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": f"{w.name}: B{w.B} Hq{w.Hq} Hkv{w.Hkv} Nq{w.Nq} Nk{w.Nk} d{w.d}"
                               f"{' causal' if w.is_causal else ''}{' fp8 e4m3' if w.fp8 else ''}",
                   "sample_per_step": desc},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(result), flush=True)


def launch_ranks(n: int, argv) -> int:
    """Runs this script as n ranks on this node (one process per GPU) under
    torch.distributed.run, rendezvous on 127.0.0.1, and returns its exit code.
    Each rank reads RANK / LOCAL_RANK / WORLD_SIZE from the environment."""
    import socket
    import subprocess
    with socket.socket() as sock:
        sock.bind(("127.0.0.1", 0))
        port = sock.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *argv]
    return subprocess.run(cmd, cwd=ROOT).returncode


def main(argv=None):
    from workloads import WORKLOADS
    argv = list(sys.argv[1:] if argv is None else argv)
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="long", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="CPU-baseline sample budget")
    ap.add_argument("--reference-seconds", type=float, default=120.0, help="total budget of --impl reference")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.gpus < 1:
        ap.error("--gpus must be at least 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        return launch_ranks(args.gpus, argv)  # one rank per GPU, started here
    world = dist_env()[0]
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}: launch with --nproc-per-node {args.gpus}")
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main() or 0)

"""Benchmark of the attention hot path on B200.

One step = one pass of the whole path over one batch of synthetic inputs:
  1. fused prefill: GQA causal attention, B=4, Hq=32, Hkv=8, L=4096, D=128, bf16
     (attn_fwd: tile loads, S = QK^T, masks with block skipping, online softmax,
     P.V, epilogue);
  2. paged decode: MQA, B=64 sequences, Hq=32, Hkv=1, D=128, lengths uniform in
     [512, 8192], 16-token pages behind a permuted block table
     (attn_decode_paged: split + combine), against three K/V pools of that
     batch in turn (the caches of three layers, 142 MB each).

The headline ``value`` is prefill TFLOP/s (FLOPs counted as the causal mask
requires); decode HBM GB/s is reported beside it, per call of the second and
third pools, which run back to back, and (``isolated``) for the first pool's
call alone after an L2 flush.  Both come from CUDA events recorded on the
launching stream inside the timed region.  ``--gpus N`` under torchrun runs N independent replicas (the path has
no exchange step), times on the device and takes the max over ranks.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from workloads import (FP8_CAUSAL, GQA_CAUSAL, LATENT_192_128, LATENT_256, MQA_DECODE, SWA_CAUSAL,  # noqa: E402
                       DecodeShape, decode_inputs, decode_queries, prefill_inputs, prefill_inputs_fp8, seed_of)
from workloads.accounting import decode_bytes, prefill_bytes, prefill_flops  # noqa: E402

METRIC = "attention fwd TFLOP/s (prefill) & decode HBM GB/s, % of B200 roofline"
PREFILL = GQA_CAUSAL
DECODE = MQA_DECODE
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) from
# an ncu capture of the kernel, valid only for the kernel sources it was taken
# on (sha256 prefix of the files); a changed kernel reports null until it is
# captured again.
PROFILED_TRAFFIC = {
    # the plain prefill launch (rows 256-4095; the 19 us launch of rows 0-255 not included)
    "prefill": {"files": ["csrc/prefill_sm100.cu", "csrc/sm100_ptx.cuh"], "sha": "88d16936586a538e",
                "bytes": 255_063_552 + 79_245_824},
    "decode": {"files": ["csrc/decode_paged.cu", "csrc/sm100_ptx.cuh"], "sha": "53366978b9648ab7",
               "bytes": 147_646_720 + 3_941_632},
}


def profiled_traffic(kernel: str):
    import hashlib
    entry = PROFILED_TRAFFIC[kernel]
    h = hashlib.sha256()
    for f in entry["files"]:
        with open(os.path.join(ROOT, "attention_flash_attn_02_b200", f), "rb") as fh:
            h.update(fh.read())
    return entry["bytes"] if h.hexdigest()[:16] == entry["sha"] else None
L2_FLUSH_BYTES = 256 << 20
DECODE_LAYERS = 3  # K/V pools decoded per step
E2E_MAX_STEPS = 50  # the end-to-end loop copies ~490 MB per step: at most this many steps
SIDE_MIN_MS = 120.0  # each side measurement runs launches for at least this long (clock samples)
SUSTAINED_S = 2.0  # length of the sustained-clock prefill loop
# MQA decode in a 256-wide latent space: the decode workload's batch, lengths
# and layout with D = 256 (a side line; 285 MB of K/V)
LATENT_DECODE = DecodeShape("latent_mqa_paged_decode_B64_H32_Hkv1_D256_len512_8192", B=64, Hq=32, Hkv=1, D=256,
                            len_lo=512, len_hi=8192)


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads' side measurements")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the CPU oracle baseline")
    ap.add_argument("--profile", choices=sorted(PROFILE_WORKLOADS), default=None,
                    help="only launch this workload's kernels warmup + steps times (for profiler captures)")
    return ap.parse_args(argv)


# Workloads --profile can launch alone: (shape, seed index, input format or
# call name).  The FP8 one runs at half the workload's length (a quarter of its
# work, inputs still 3 x 64 MB > L2) so that a many-pass capture stays short.
PROFILE_WORKLOADS = {
    "prefill": (GQA_CAUSAL, 1, "bf16"),
    "swa": (SWA_CAUSAL, 3, "bf16"),
    "fp8": (dataclasses.replace(FP8_CAUSAL, name="fp8_causal_B1_H32_L16384_D128", Lq=16384, Lk=16384), 4, "e4m3"),
    "e5m2": (dataclasses.replace(FP8_CAUSAL, name="fp8_causal_B1_H32_L16384_D128", Lq=16384, Lk=16384), 4, "e5m2"),
    "latent256": (LATENT_256, 3, "mla"),
    "decode": (MQA_DECODE, 2, "decode"),
    "backward": (GQA_CAUSAL, 1, "bwd"),
}


def run_profile(args):
    """Launches one workload's kernels (warmup + steps times) and exits: the
    command profiler captures run, with nothing else on the device."""
    import torch
    import attention_flash_attn_02_b200 as attn
    attn.load()
    dev = torch.device("cuda", 0)
    shape, idx, kind = PROFILE_WORKLOADS[args.profile]
    if kind == "decode":
        kv = decode_inputs(shape, seed_of(idx))
        d = {n: getattr(kv, n).to(dev) for n in ("q", "k_pages", "v_pages", "block_table", "seq_lens")}
        fn = lambda: attn.attn_decode_paged(d["q"], d["k_pages"], d["v_pages"], d["block_table"],  # noqa: E731
                                            d["seq_lens"], shape.scale)
    elif kind in ("e4m3", "e5m2"):
        q8, k8, v8, sq, sk, sv = prefill_inputs_fp8(shape, seed_of(idx), fmt=kind)
        q8, k8, v8 = q8.to(dev), k8.to(dev), v8.to(dev)
        call = attn.attn_fwd_fp8 if kind == "e4m3" else attn.attn_fwd_e5m2
        fn = lambda: call(q8, k8, v8, sq, sk, sv, shape.scale, shape.causal, shape.window)  # noqa: E731
    elif kind == "bwd":
        # one forward for O and LSE, then the backward launches alone
        q, k, v = [t.to(dev) for t in prefill_inputs(shape, seed_of(idx))]
        g = torch.Generator().manual_seed(seed_of(idx) + 300)
        do = torch.randn(q.shape, generator=g).to(torch.bfloat16).to(dev)
        o, lse = attn.attn_fwd(q, k, v, shape.scale, shape.causal, shape.window)
        fn = lambda: attn.attn_bwd(q, k, v, o, do, lse, shape.scale, shape.causal, shape.window)  # noqa: E731
    else:
        q, k, v = [t.to(dev) for t in prefill_inputs(shape, seed_of(idx))]
        call = attn.attn_fwd_mla if kind == "mla" else attn.attn_fwd
        fn = lambda: call(q, k, v, shape.scale, shape.causal, shape.window)  # noqa: E731
    for _ in range(args.warmup + args.steps):
        fn()
    torch.cuda.synchronize()
    st = attn.attn_last_device_error()
    print(json.dumps({"profile": args.profile, "workload": shape.name, "launches": args.warmup + args.steps,
                      "status": attn.attn_status_str(st)}))
    if st != 0:
        sys.exit(1)


# ------------------------------------------------------------ distributed
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(world: int, backend: str):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank scalar over all ranks (identity for one rank)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ peaks
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """Samples the SM clock and the throttle reasons of the GPU under test
    from a background thread while the timed region runs: through NVML every
    millisecond, so that a region of ten milliseconds still gets ten samples,
    else with nvidia-smi every 200 ms.  Only samples taken between
    ``begin()`` and ``end()`` (host time around the region, whose GPU work
    the final synchronize bounds) are reported.  The device is matched by
    UUID, else by index, else it is the only GPU listed."""

    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, uuid: str, index: int):
        self.uuid = (uuid or "").lower().replace("gpu-", "").replace("-", "")
        self.index = index
        self.rows = []          # (host time, sm MHz, max sm MHz, set of reasons)
        self.source = None
        self._stop = None
        self._thread = None
        self._first = None
        self.t0 = self.t1 = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        n = pynvml.nvmlDeviceGetCount()
        handles = [pynvml.nvmlDeviceGetHandleByIndex(i) for i in range(n)]
        norm = lambda u: (u.decode() if isinstance(u, bytes) else u).lower().replace("gpu-", "").replace("-", "")  # noqa: E731
        for h in handles:
            if self.uuid and norm(pynvml.nvmlDeviceGetUUID(h)) == self.uuid:
                return pynvml, h
        if n == 1:
            return pynvml, handles[0]
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.index)

    def _poll_nvml(self, pynvml, h):
        get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        bits = [getattr(pynvml, "nvmlClocksEventReasonHwSlowdown", 0x8),
                getattr(pynvml, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
                getattr(pynvml, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
                getattr(pynvml, "nvmlClocksEventReasonSwPowerCap", 0x4)]
        mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        while not self._stop.is_set():
            t = time.perf_counter()
            sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
            r = get_reasons(h)
            self.rows.append((t, float(sm), float(mx), {self.REASONS[i] for i in range(4) if r & bits[i]}))
            self._first.set()
            self._stop.wait(0.001)

    def _poll_smi(self):
        while not self._stop.is_set():
            try:
                t = time.perf_counter()
                out = subprocess.run(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits"],
                                     capture_output=True, text=True, timeout=5).stdout
                rows = [[x.strip() for x in line.split(",")] for line in out.splitlines()]
                rows = [r for r in rows if len(r) >= 10]
                norm = lambda u: u.lower().replace("gpu-", "").replace("-", "")  # noqa: E731
                mine = [r for r in rows if self.uuid and norm(r[1]) == self.uuid]
                if not mine:
                    mine = rows if len(rows) == 1 else [r for r in rows if r[0] == str(self.index)]
                num = lambda x: float(x) if x.replace(".", "", 1).isdigit() else None  # noqa: E731
                for r in mine:
                    if num(r[2]) is not None:
                        self.rows.append((t, num(r[2]), num(r[3]),
                                          {self.REASONS[i] for i in range(4) if r[6 + i].lower() == "active"}))
            except Exception:
                pass
            self._first.set()
            self._stop.wait(0.2)

    def _run(self):
        try:
            pynvml, h = self._nvml_handle()
            self.source = "nvml, 1 ms"
            self._poll_nvml(pynvml, h)
        except Exception:
            self.source = "nvidia-smi, 200 ms"
            self._poll_smi()

    def start(self):
        import threading
        self._stop = threading.Event()
        self._first = threading.Event()
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()
        self._first.wait(timeout=5)  # the first sample precedes the region

    def begin(self):
        self.t0 = time.perf_counter()

    def end(self):
        self.t1 = time.perf_counter()

    def stop(self):
        if self._thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["not sampled"], "samples": 0}
        self._stop.set()
        self._thread.join(timeout=10)
        t0 = self.t0 if self.t0 is not None else float("-inf")
        t1 = self.t1 if self.t1 is not None else float("inf")
        mine = [r for r in self.rows if t0 <= r[0] <= t1]
        if not mine:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples in the timed region"],
                    "samples": 0, "source": self.source}
        sm = [r[1] for r in mine]
        load = [x for x in sm if x > 500] or sm
        return {"sm_mhz": statistics.median(load), "sm_min_mhz": min(load),
                "sm_max_mhz": max(r[2] for r in mine if r[2] is not None),
                "reasons": sorted(set().union(*(r[3] for r in mine))), "samples": len(mine),
                "source": self.source}


# ----------------------------------------------------------- CPU baseline
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 0) for d in threadpool_info() if d.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_oracle_prefill(budget_s: float):
    """Times the float64 oracle on whole heads of the prefill workload until
    the budget is spent (at least one head).  Returns (TFLOP/s, heads, seconds)."""
    import oracle
    q, k, v = prefill_inputs(PREFILL, seed_of(1))
    per_head = prefill_flops(PREFILL) / (PREFILL.B * PREFILL.Hq)
    heads = 0
    t0 = time.perf_counter()
    while True:
        b, h = divmod(heads, PREFILL.Hq)
        oracle.attention(q, k, v, PREFILL.scale, PREFILL.causal, PREFILL.window, heads=[h], batches=[b])
        heads += 1
        el = time.perf_counter() - t0
        if el >= budget_s or heads >= PREFILL.B * PREFILL.Hq:
            break
    return per_head * heads / el / 1e12, heads, el


# ------------------------------------------------------------------ ours
def run_ours(args):
    import torch
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    init_dist(world, "nccl")
    import attention_flash_attn_02_b200 as attn
    attn.load()
    dev = torch.device("cuda", local)
    peaks, peak_src = measured_peaks()

    # inputs resident in HBM before the timed region
    qh, kh, vh = prefill_inputs(PREFILL, seed_of(1))
    q, k, v = qh.to(dev), kh.to(dev), vh.to(dev)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    kv = decode_inputs(DECODE, seed_of(2))
    dq, dkp, dvp = kv.q.to(dev), kv.k_pages.to(dev), kv.v_pages.to(dev)
    dbt, dsl = kv.block_table.to(dev), kv.seq_lens.to(dev)
    do = torch.empty_like(dq)
    dlse = torch.empty(dq.shape[:2], dtype=torch.float32, device=dev)
    ws = torch.empty(attn.attn_decode_workspace_bytes(DECODE.B, DECODE.Hq, kv.max_pages, DECODE.D),
                     dtype=torch.uint8, device=dev)
    # Two more K/V pools of the same batch (same lengths and block table, their
    # own values), as the caches of further layers: each step decodes the
    # batch against all DECODE_LAYERS pools in turn.
    g_pool = torch.Generator(device=dev)
    g_pool.manual_seed(seed_of(2) + 1)
    pools = [(dkp, dvp)] + [
        (torch.randn(dkp.shape, generator=g_pool, device=dev).to(torch.bfloat16),
         torch.randn(dvp.shape, generator=g_pool, device=dev).to(torch.bfloat16))
        for _ in range(DECODE_LAYERS - 1)]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        attn.attn_fwd(q, k, v, PREFILL.scale, PREFILL.causal, PREFILL.window, o=o, lse=lse)
        if ev is not None:
            ev[1].record(stream)
        # Evict L2 so decode reads its cache from HBM: write a buffer larger
        # than L2, then read another one so the written lines are flushed back
        # to HBM here rather than during the decode.
        flush.zero_()
        flush_rd.view(torch.int32).sum(dtype=torch.int32)
        # Layer 0 alone after the flush (isolated call), then the other layers
        # back to back: their pools were last read a step ago, with the
        # prefill, the flush and the other pools (> L2 each) read since.
        if ev is not None:
            ev[2].record(stream)
        for li, (kp, vp) in enumerate(pools):
            attn.attn_decode_paged(dq, kp, vp, dbt, dsl, DECODE.scale, o=do, lse=dlse, workspace=ws)
            if ev is not None and li == 0:
                ev[3].record(stream)
        if ev is not None:
            ev[4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = attn.attn_last_device_error()
    if st != 0:
        raise RuntimeError(f"kernel status {attn.attn_status_str(st)} during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    try:
        gpu_uuid = str(torch.cuda.get_device_properties(local).uuid)
    except Exception:
        gpu_uuid = ""
    clocks = ClockSampler(gpu_uuid, local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    clocks.begin()
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    clocks.end()
    barrier(world)
    clk = clocks.stop()
    st = attn.attn_last_device_error()
    if st != 0:
        raise RuntimeError(f"kernel status {attn.attn_status_str(st)} during the timed region")

    region_ms = max_over_ranks(t_start.elapsed_time(t_end), world, dev)
    pre_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in evs), world, dev)
    dec1_ms = max_over_ranks(sum(e[2].elapsed_time(e[3]) for e in evs), world, dev)
    # back-to-back calls: layers 1.. of every step, per call
    dec_ms = max_over_ranks(sum(e[3].elapsed_time(e[4]) for e in evs), world, dev) / (DECODE_LAYERS - 1)
    K = args.steps
    pf = prefill_flops(PREFILL)
    db = decode_bytes(DECODE, kv.seq_lens.tolist())
    value = world * pf * K / (pre_ms / 1e3) / 1e12            # TFLOP/s, all ranks
    dec_gbs = world * db * K / (dec_ms / 1e3) / 1e9
    per_launch_pre_ms = pre_ms / K
    achieved_pre = pf / (per_launch_pre_ms / 1e3) / 1e12        # per GPU, per launch
    achieved_dec = db / (dec_ms / K / 1e3) / 1e9
    achieved_dec1 = db / (dec1_ms / K / 1e3) / 1e9

    # ---- end to end through the public API with host buffers
    pin = lambda t: t.pin_memory()  # noqa: E731
    hq, hk, hv = pin(qh), pin(kh), pin(vh)
    ho = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    hl = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    hdq, hdk, hdv = pin(kv.q), pin(kv.k_pages), pin(kv.v_pages)
    hbt, hsl = pin(kv.block_table), pin(kv.seq_lens)
    hdo = torch.empty(do.shape, dtype=do.dtype).pin_memory()
    hdl = torch.empty(dlse.shape, dtype=dlse.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hdq, hdk, hdv, hbt, hsl))
    d2h = sum(t.numel() * t.element_size() for t in (ho, hl, hdo, hdl))

    # Pipelined the way a caller feeding the API from host memory would run
    # it: step i's inputs are uploaded on one stream while step i - 1
    # computes on another, and each step's results are read back on a third;
    # inputs and outputs are double-buffered.  Every step still moves all of
    # its input and result bytes inside the timed region.
    up_s, down_s = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ins = [(q, k, v, dq, dkp, dvp, dbt, dsl), tuple(torch.empty_like(t) for t in (q, k, v, dq, dkp, dvp, dbt, dsl))]
    outs = [(o, lse, do, dlse), tuple(torch.empty_like(t) for t in (o, lse, do, dlse))]
    hins = (hq, hk, hv, hdq, hdk, hdv, hbt, hsl)
    houts = [(ho, hl, hdo, hdl), tuple(torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (ho, hl, hdo, hdl))]
    ev_up = [torch.cuda.Event(), torch.cuda.Event()]      # buffer's inputs uploaded
    ev_used = [torch.cuda.Event(), torch.cuda.Event()]    # buffer's inputs consumed, outputs written
    ev_down = [torch.cuda.Event(), torch.cuda.Event()]    # buffer's outputs read back
    used_once = [False, False]

    def e2e_step(i):
        bi = i & 1
        bq, bk, bv, bdq, bdk, bdv, bbt, bsl = ins[bi]
        bo, bl, bdo, bdl = outs[bi]
        with torch.cuda.stream(up_s):
            if used_once[bi]:
                up_s.wait_event(ev_used[bi])
            for d_, h_ in zip(ins[bi], hins):
                d_.copy_(h_, non_blocking=True)
            ev_up[bi].record(up_s)
        stream.wait_event(ev_up[bi])
        if used_once[bi]:
            stream.wait_event(ev_down[bi])
        attn.attn_fwd(bq, bk, bv, PREFILL.scale, PREFILL.causal, PREFILL.window, o=bo, lse=bl)
        attn.attn_decode_paged(bdq, bdk, bdv, bbt, bsl, DECODE.scale, o=bdo, lse=bdl, workspace=ws)
        ev_used[bi].record(stream)
        with torch.cuda.stream(down_s):
            down_s.wait_event(ev_used[bi])
            for h_, d_ in zip(houts[bi], outs[bi]):
                h_.copy_(d_, non_blocking=True)
            ev_down[bi].record(down_s)
        used_once[bi] = True

    def e2e_join():
        stream.wait_stream(up_s)
        stream.wait_stream(down_s)

    e2e_step(0)
    e2e_step(1)
    e2e_join()
    torch.cuda.synchronize()
    K_e2e = min(K, E2E_MAX_STEPS)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    up_s.wait_event(e0)
    down_s.wait_event(e0)
    for i in range(K_e2e):
        e2e_step(i)
    e2e_join()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = world * pf * K_e2e / (e2e_ms / 1e3) / 1e12

    # ---- the prefill alone, back to back for SUSTAINED_S seconds: the figure
    # at the clock a long run settles to (the timed region above is shorter)
    sustained = sustained_prefill(attn, q, k, v, o, lse, stream, gpu_uuid, local, world, dev, pf, peaks)

    # ---- side measurements of the other workloads (not part of the step)
    extra = {}
    if not args.no_extra:
        extra = side_workloads(attn, dev, peaks, world, gpu_uuid, local)

    cpu = None
    if rank == 0 and world == 1:
        tf, heads, secs = cpu_oracle_prefill(args.cpu_seconds)
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"float64 oracle, {heads} whole (batch, head) pairs of the prefill workload "
                         f"(4096 causal rows each), {secs:.1f} s on the host"}

    peak_t = peaks["bf16_tflops"]
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(region_ms / K, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic: seeded N(0,1) q/k/v cast to bf16; decode lengths U[512,8192], permuted page table",
        "config": {
            "workload": "prefill gqa_causal B4 Hq32 Hkv8 L4096 D128 + paged decode mqa B64 Hq32 Hkv1 D128 len[512,8192] page16",
            "prefill": PREFILL.name, "decode": DECODE.name,
            "l2": ("prefill inputs 201 MB > L2; decode: a 256 MB buffer is written, then another read, before "
                   f"the first of {DECODE_LAYERS} K/V pools (142 MB each, > L2) of the batch; the pools are decoded "
                   "in turn, the later ones back to back (the decode figures), the first alone (isolated)"),
            "parallelism": f"replicas{world}",
        },
        "roofline": {
            "bound": "tensor", "kernel": "prefill_kernel<128,bf16>",
            "achieved": round(achieved_pre, 2), "peak": peak_t, "unit": "TFLOP/s",
            "frac": round(achieved_pre / peak_t, 4),
            "frac_of_sustained": round(achieved_pre / peaks["bf16_tflops_sustained"], 4),
            "peak_source": f"{peak_src} bf16_tflops (burst)",
            "traffic": profiled_traffic("prefill"),
            "algorithmic_bytes": prefill_bytes(PREFILL),
        },
        "decode": {
            "value": round(dec_gbs, 1), "unit": "GB/s", "workload": DECODE.name,
            "us_per_call": round(dec_ms / K * 1e3, 2),
            "timing": f"calls on K/V pools 2..{DECODE_LAYERS} of each step, back to back, per call",
            "roofline": {"bound": "hbm", "achieved": round(achieved_dec, 1), "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": round(achieved_dec / peaks["hbm_gbs"], 4),
                         "peak_source": f"{peak_src} hbm_gbs", "traffic": profiled_traffic("decode"),
                         "algorithmic_bytes": db},
            "isolated": {"us_per_call": round(dec1_ms / K * 1e3, 2), "GB/s": round(achieved_dec1, 1),
                         "frac": round(achieved_dec1 / peaks["hbm_gbs"], 4),
                         "timing": "the first pool's call alone, after the L2 flush, events around it"},
        },
        "e2e": {"value": round(e2e_value, 3), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": K_e2e},
        "prefill_sustained": sustained,
        # per step: the prefill's two launches (its leading row groups, whose
        # rows see fewer than 256 keys, run in the kernel built with the
        # two-part P V product; the rest in the other) + (split, combine) per
        # decode call
        "gpu_launches": (2 + 2 * DECODE_LAYERS) * K,
        "clocks": clk,
        "cpu_baseline": cpu,
        "workloads": extra,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def fp8_gemm_peak(dev):
    """Dense e4m3 tensor throughput on this GPU: a cuBLASLt 8192^3 GEMM with
    fp32 accumulation (torch._scaled_mm, unit scales, bf16 out), best of 10
    after 3 warm-ups, 2*N^3 FLOP each.  The denominator for the FP8 workload,
    in the style of the measured bf16 peak; None if the call is unavailable."""
    import torch
    n = 8192
    try:
        g = torch.Generator(device="cpu").manual_seed(7)
        a = torch.randn(n, n, generator=g).to(dev).to(torch.float8_e4m3fn)
        b = torch.randn(n, n, generator=g).to(dev).to(torch.float8_e4m3fn).t()  # column-major operand
        one = torch.ones((), device=dev, dtype=torch.float32)
        for _ in range(3):
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        del a, b
        torch.cuda.empty_cache()
        return 2.0 * n ** 3 / (best / 1e3) / 1e12
    except Exception:
        return None


def side_timer(fn, dev, world, gpu_uuid, local, min_ms=SIDE_MIN_MS, before=None):
    """Times one launch sequence ``fn`` on the current stream: 2 warm-ups,
    then launches with CUDA events around each (``before`` runs untimed ahead
    of each, e.g. an L2 flush) until at least ``min_ms`` of host time and 5
    launches have passed, with SM clocks sampled meanwhile.  Returns the median
    ms per launch (max over ranks) and the clock record."""
    import torch
    for _ in range(2):
        if before:
            before()
        fn()
    torch.cuda.synchronize()
    clocks = ClockSampler(gpu_uuid, local)
    clocks.start()
    clocks.begin()
    ts = []
    t0 = time.perf_counter()
    while len(ts) < 5 or (time.perf_counter() - t0) * 1e3 < min_ms:
        if before:
            before()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    clocks.end()
    clk = clocks.stop()
    clk["launches"] = len(ts)
    return max_over_ranks(statistics.median(ts), world, dev), clk


def sustained_prefill(attn, q, k, v, o, lse, stream, gpu_uuid, local, world, dev, pf, peaks):
    """The GQA causal prefill back to back for SUSTAINED_S seconds (one event
    pair around the whole loop, clocks sampled): TFLOP/s at the clock a long
    run settles to, against the sustained bf16 peak."""
    import torch
    n = 0
    clocks = ClockSampler(gpu_uuid, local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    clocks.begin()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < SUSTAINED_S:
        for _ in range(20):
            attn.attn_fwd(q, k, v, PREFILL.scale, PREFILL.causal, PREFILL.window, o=o, lse=lse)
        n += 20
        if n % 200 == 0:
            torch.cuda.synchronize()
    b.record(stream)
    torch.cuda.synchronize()
    clocks.end()
    clk = clocks.stop()
    ms = max_over_ranks(a.elapsed_time(b), world, dev) / n
    tf = pf / (ms / 1e3) / 1e12
    return {"TFLOP/s": round(tf, 1), "ms_per_launch": round(ms, 4), "launches": n,
            "frac_of_sustained_peak": round(tf / peaks["bf16_tflops_sustained"], 4),
            "frac_of_burst_peak": round(tf / peaks["bf16_tflops"], 4), "clocks": clk}


def side_workloads(attn, dev, peaks, world, gpu_uuid="", local=0):
    """Per-launch throughput of the other workloads, each timed by side_timer
    (inputs larger than L2) with its own clock record."""
    import torch
    out = {}
    T = lambda fn, **kw: side_timer(fn, dev, world, gpu_uuid, local, **kw)  # noqa: E731
    fp8_peak = fp8_gemm_peak(dev)
    for shape, idx, fmt in ((SWA_CAUSAL, 3, None), (FP8_CAUSAL, 4, "e4m3"), (FP8_CAUSAL, 4, "e5m2"),
                            (LATENT_192_128, 1, None), (LATENT_256, 3, None)):
        if fmt:
            q8, k8, v8, sq, sk, sv = prefill_inputs_fp8(shape, seed_of(idx), fmt=fmt)
            q8, k8, v8 = q8.to(dev), k8.to(dev), v8.to(dev)
            call = attn.attn_fwd_fp8 if fmt == "e4m3" else attn.attn_fwd_e5m2
            fn = lambda: call(q8, k8, v8, sq, sk, sv, shape.scale, shape.causal, shape.window)  # noqa
        else:
            q, k, v = [t.to(dev) for t in prefill_inputs(shape, seed_of(idx))]
            call = attn.attn_fwd_mla if shape.dv != 128 or shape.D != 128 else attn.attn_fwd
            fn = lambda: call(q, k, v, shape.scale, shape.causal, shape.window)  # noqa
        ms, clk = T(fn)
        tf = prefill_flops(shape) / (ms / 1e3) / 1e12
        entry = {"TFLOP/s": round(tf, 1), "ms": round(ms, 3), "bytes_MB": round(prefill_bytes(shape) / 1e6, 1)}
        if fmt:
            entry["frac_of_bf16_peak"] = round(tf / peaks["bf16_tflops"], 4)
            if fp8_peak:
                entry["fp8_peak_tflops"] = round(fp8_peak, 1)
                entry["frac_of_fp8_peak"] = round(tf / fp8_peak, 4)
                entry["fp8_peak_source"] = ("measured here: cuBLASLt e4m3 8192^3 GEMM (torch._scaled_mm), best of 10"
                                            + ("; the dense 8-bit tensor rate, e5m2 included" if fmt == "e5m2" else ""))
            else:
                entry["note"] = "FP8 GEMM probe unavailable; nominal dense FP8 is 2x bf16"
        else:
            entry["frac"] = round(tf / peaks["bf16_tflops"], 4)
        entry["clocks"] = clk
        out[shape.name + ("_e5m2" if fmt == "e5m2" else "")] = entry
        del fn
        torch.cuda.empty_cache()
    out.update(multi_token_decode(attn, dev, peaks, world, T))
    out.update(latent_decode(attn, dev, peaks, world, T))
    out.update(paged_chunk_prefill(attn, dev, peaks, world, T))
    out.update(backward_pass(attn, dev, peaks, world, T))
    return out


def latent_decode(attn, dev, peaks, world, T):
    """GB/s of the MQA paged decode with D = 256 (the decode workload's batch
    and lengths, 285 MB of K/V), L2 flushed (write, then read 256 MB) before
    each call."""
    import torch
    sh = LATENT_DECODE
    kv = decode_inputs(sh, seed_of(2))
    d = {n: getattr(kv, n).to(dev) for n in ("q", "k_pages", "v_pages", "block_table", "seq_lens")}
    o = torch.empty_like(d["q"])
    lse = torch.empty(d["q"].shape[:2], dtype=torch.float32, device=dev)
    ws = torch.empty(attn.attn_decode_workspace_bytes(sh.B, sh.Hq, kv.max_pages, sh.D), dtype=torch.uint8,
                     device=dev)
    fw = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    fr = torch.ones(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def flush():
        fw.zero_()
        fr.view(torch.int32).sum(dtype=torch.int32)

    fn = lambda: attn.attn_decode_paged(d["q"], d["k_pages"], d["v_pages"], d["block_table"], d["seq_lens"],  # noqa
                                        sh.scale, o=o, lse=lse, workspace=ws)
    ms, clk = T(fn, before=flush)
    by = decode_bytes(sh, kv.seq_lens.tolist())
    gbs = by / (ms / 1e3) / 1e9
    return {sh.name: {"GB/s": round(gbs, 1), "us_per_call": round(ms * 1e3, 2),
                      "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4), "bytes_MB": round(by / 1e6, 1),
                      "timing": "alone after an L2 flush", "clocks": clk}}


def backward_pass(attn, dev, peaks, world, T):
    """attn_bwd on the GQA causal prefill workload (its own forward's O and
    LSE): 5 products of the visible (query, key) pairs against the forward's
    2, i.e. 2.5x the forward's FLOPs.  The inputs (201 MB) and the dQ
    accumulator (272 MB) exceed L2."""
    import torch
    shape = PREFILL
    q, k, v = [t.to(dev) for t in prefill_inputs(shape, seed_of(1))]
    g = torch.Generator().manual_seed(seed_of(1) + 300)
    do = torch.randn(q.shape, generator=g).to(torch.bfloat16).to(dev)
    o, lse = attn.attn_fwd(q, k, v, shape.scale, shape.causal, shape.window)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(attn.attn_bwd_workspace_bytes(shape.B, shape.Hq, shape.Lq, shape.D), dtype=torch.uint8,
                     device=dev)
    fn = lambda: attn.attn_bwd(q, k, v, o, do, lse, shape.scale, shape.causal, shape.window,  # noqa: E731
                               dq=dq, dk=dk, dv=dv, workspace=ws)
    ms, clk = T(fn)
    tf = 2.5 * prefill_flops(shape) / (ms / 1e3) / 1e12
    return {f"backward_{shape.name}": {"TFLOP/s": round(tf, 1), "ms": round(ms, 3),
                                       "frac": round(tf / peaks["bf16_tflops"], 4), "clocks": clk}}


def paged_chunk_prefill(attn, dev, peaks, world, T, B=4, Hq=32, Hkv=8, D=128, cached=3072, chunk=1024):
    """Chunked prefill over a paged cache (attn_prefill_paged): each of B
    sequences holds `cached` tokens plus a `chunk` of new ones, 16-token pages
    in a permuted pool; the chunk attends causally to all of them.  Also the
    KV append of the chunk (attn_kv_append)."""
    import torch
    shape = DecodeShape("paged_chunk", B=B, Hq=Hq, Hkv=Hkv, D=D, len_lo=1, len_hi=1)
    L = cached + chunk
    kv = decode_inputs(shape, seed_of(1) + 200, seq_lens=[L] * B)
    q = decode_queries(shape, chunk, seed_of(1) + 201).to(dev)
    kp, vp, bt, sl = kv.k_pages.to(dev), kv.v_pages.to(dev), kv.block_table.to(dev), kv.seq_lens.to(dev)
    g = torch.Generator().manual_seed(seed_of(1) + 202)
    k_new = torch.randn(B, Hkv, chunk, D, generator=g).to(torch.bfloat16).to(dev)
    v_new = torch.randn(B, Hkv, chunk, D, generator=g).to(torch.bfloat16).to(dev)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    ms, clk = T(lambda: attn.attn_prefill_paged(q, kp, vp, bt, sl, shape.scale, o=o, lse=lse))
    flops = 4.0 * D * Hq * B * (chunk * cached + chunk * (chunk + 1) / 2)
    tf = flops / (ms / 1e3) / 1e12
    ms_app, clk_app = T(lambda: attn.attn_kv_append(k_new, v_new, kp, vp, bt, sl))
    app_bytes = 2 * 2 * B * Hkv * chunk * D * 2  # K and V, read and written
    return {f"paged_chunk_prefill_B{B}_H{Hq}_G{Hq // Hkv}_cached{cached}_chunk{chunk}_D{D}": {
        "TFLOP/s": round(tf, 1), "ms": round(ms, 3), "frac": round(tf / peaks["bf16_tflops"], 4), "clocks": clk,
        "kv_append_GB/s": round(app_bytes / (ms_app / 1e3) / 1e9, 1), "kv_append_us": round(ms_app * 1e3, 2),
        "kv_append_clocks": clk_app}}


def multi_token_decode(attn, dev, peaks, world, T, q_len: int = 4):
    """GB/s of the batch-64 MQA decode with q_len new tokens per sequence
    (attn_decode_paged_multi): every page read once for all q_len tokens.
    L2 flushed (write, then read 256 MB) before each call."""
    import torch
    kv = decode_inputs(DECODE, seed_of(2))
    qm = decode_queries(DECODE, q_len, seed_of(2) + 100).to(dev)
    kp, vp, bt, sl = kv.k_pages.to(dev), kv.v_pages.to(dev), kv.block_table.to(dev), kv.seq_lens.to(dev)
    o = torch.empty_like(qm)
    lse = torch.empty(qm.shape[:3], dtype=torch.float32, device=dev)
    ws = torch.empty(attn.attn_decode_workspace_bytes(DECODE.B, DECODE.Hq * q_len, kv.max_pages, DECODE.D),
                     dtype=torch.uint8, device=dev)
    fw = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    fr = torch.ones(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def flush():
        fw.zero_()
        fr.view(torch.int32).sum(dtype=torch.int32)

    fn = lambda: attn.attn_decode_paged_multi(qm, kp, vp, bt, sl, DECODE.scale, o=o, lse=lse, workspace=ws)  # noqa
    ms, clk = T(fn, before=flush)
    by = decode_bytes(DECODE, kv.seq_lens.tolist(), q_len)
    gbs = by / (ms / 1e3) / 1e9
    return {f"{DECODE.name}_qlen{q_len}": {"GB/s": round(gbs, 1), "us_per_call": round(ms * 1e3, 2),
                                            "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4),
                                            "bytes_MB": round(by / 1e6, 1), "clocks": clk}}


# ------------------------------------------------------------- reference
def run_reference(args):
    """The float64 oracle on the host cores, each step a bounded sample of
    the same workload: one whole (batch, head) of the prefill and one
    sequence of the decode."""
    rank, world, _ = dist_env()
    if world > 1 and rank != 0:
        return
    import oracle
    q, k, v = prefill_inputs(PREFILL, seed_of(1))
    kv = decode_inputs(DECODE, seed_of(2))
    per_head = prefill_flops(PREFILL) / (PREFILL.B * PREFILL.Hq)

    def step(i):
        b, h = divmod(i % (PREFILL.B * PREFILL.Hq), PREFILL.Hq)
        t0 = time.perf_counter()
        oracle.attention(q, k, v, PREFILL.scale, PREFILL.causal, PREFILL.window, heads=[h], batches=[b])
        t1 = time.perf_counter()
        sb = i % DECODE.B
        oracle.paged_decode(kv.q[sb:sb + 1], kv.k_pages, kv.v_pages, kv.block_table[sb:sb + 1],
                            kv.seq_lens[sb:sb + 1], DECODE.scale)
        return t1 - t0, time.perf_counter() - t0

    for i in range(args.warmup):
        step(i)
    pre = tot = 0.0
    for i in range(args.steps):
        a, b = step(args.warmup + i)
        pre += a
        tot += b
    value = per_head * args.steps / pre / 1e12
    line = {
        "metric": METRIC, "impl": "reference", "value": round(value, 5), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(tot / args.steps * 1e3, 2), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (same seeded inputs as the CUDA arm)",
        "config": {"workload": "prefill gqa_causal B4 Hq32 Hkv8 L4096 D128 + paged decode mqa B64 Hq32 Hkv1 D128",
                   "prefill": PREFILL.name, "decode": DECODE.name, "parallelism": "host"},
        "cpu_baseline": {"value": round(value, 5), "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": "each step: one whole (batch, head) of the prefill workload and one decode "
                                   "sequence, float64 oracle"},
        "e2e": {"value": round(value, 5), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    args = parse_args(argv)
    if args.profile:
        run_profile(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

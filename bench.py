"""Benchmark of MLA paged-KV decode on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole hot path over one batch: the tile scheduler
(mla_get_metadata) and the split-KV decode with its combine (mla_decode_kvcache).
The default workload is the memory-bound decode (batch 128, s_q 1, h_q 16, every
cache length 8192, 64-token pages scattered by a seeded block table), whose KV cache
(1.2 GB) is larger than the 126 MB L2, so no flush is needed between steps.

value     KV bytes the step reads (exact token counts, 1152 B per bf16 token) plus q, out
          and lse bytes, summed over all ranks, divided by the max-over-ranks device time
          (CUDA events on the launching stream).
e2e       the same metric when every step also copies its inputs (q, block_table,
          cache_seqlens, indices) from pinned host memory and reads back out and lse; the KV
          cache is resident device state, as in serving.  Decode steps go through the
          library's serving session (mla_session_decode with host buffers), which pipelines
          them as a serving loop would: step k+1's inputs are copied in and step k-1's results
          read back (two copy streams, double-buffered device staging) while step k computes;
          sparse prefill, which has no session call, runs the same pipeline from Python.  The
          timed region runs from before the first copy-in to after the last read-back.
roofline  the decode call (main kernel + combine): algorithmic bytes (or FLOPs) per call divided by
          its mean duration, timed in a loop of decode calls alone (CUDA events at the ends
          of the loop), against the measured HBM copy bandwidth or cuBLAS bf16 rate, with the
          fraction of the nominal B200 figures (8 TB/s, 2.25 PFLOP/s) beside it.  The whole-step
          loop that gives `value` records events only before its first and after its last
          step, so the scheduler -> decode programmatic launch chain runs undisturbed.
per_workload  the same figures for the other workloads (variable-length h128, causal s_q 2,
          FP8 cache, token-sparse decode, sparse prefill), a few steps each, on a 1-GPU run.
cpu_baseline  the fp64 oracle timed on this host's cores on a bounded sample of requests.

With N > 1 (torchrun), every rank runs its own batch of requests on its own GPU (requests
are independent: weak scaling, no collective on the data path); the barrier and the
max-over-ranks time use torch.distributed.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import threading
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))


def _peaks():
    try:
        with open(os.path.join(HERE, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML every 2 ms while the
    timed region runs."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown"}

    def __init__(self, torch_device):
        self.samples = []           # (t, sm_mhz, max_mhz, power_w, reason_bits)
        self._stop = threading.Event()
        self._t = None
        self._h = None
        self.window = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            pr = torch.cuda.get_device_properties(torch_device)
            bus = "%08X:%02X:%02X.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
            self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self._nv = pynvml
        except Exception:
            self._h = None

    def _read(self):
        nv, h = self._nv, self._h
        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
        try:
            rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
        except Exception:
            rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)
        return sm, mx, pw, rs

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append((time.perf_counter(), *self._read()))
            except Exception:
                pass
            self._stop.wait(0.002)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join(timeout=10)

    def mark(self, t0, t1):
        self.window = (t0, t1)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        inside = [s for s in self.samples if self.window and self.window[0] <= s[0] <= self.window[1]]
        use = inside if len(inside) >= 3 else self.samples
        reasons = set()
        for s in use:
            for bit, name in self.REASONS.items():
                if s[4] & bit:
                    reasons.add(name)
        return {"sm_mhz": float(np.median([s[1] for s in use])), "sm_max_mhz": float(max(s[2] for s in use)),
                "power_w_max": float(max(s[3] for s in use)), "reasons": sorted(reasons),
                "samples": len(use), "scope": "timed region" if use is inside else "warm-up and timed region"}


def oracle_baseline(case, budget_s: float = 15.0):
    """Time the fp64 oracle on a bounded prefix of the batch (about budget_s of host work)."""
    import oracle
    import mla_inputs as mi
    t0 = time.perf_counter()
    done = []
    if case.meta.get("prefill"):
        # sparse prefill: the oracle over the first query tokens, as many as the budget allows
        s_kv = int(case.cache_seqlens[0])
        kv_rows = case.kv.reshape(-1, case.kv.shape[-1])[:s_kv]
        n = 0
        while n < case.s_q:
            oracle.mla_sparse_prefill_reference(case.q_bits[0, n:n + 1], kv_rows, case.indices[0, n:n + 1],
                                                case.softmax_scale)
            n += 1
            if time.perf_counter() - t0 > budget_s:
                break
        dt = time.perf_counter() - t0
        sub = mi.DecodeCase(**{**case.__dict__, "q_bits": case.q_bits[:, :n], "s_q": n,
                               "indices": case.indices[:, :n]})
        try:
            from threadpoolctl import threadpool_info
            cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
        except Exception:
            cores = os.cpu_count() or 1
        return {"seconds": dt, "requests": n, "units": mi.workload_units(sub), "cores": int(cores),
                "what": f"first {n} of {case.s_q} query tokens"}
    for b in range(case.batch):
        if case.indices is not None:
            oracle.mla_sparse_decode_reference(case, case.indices, requests=[b])
        else:
            oracle.mla_decode_reference(case, requests=[b])
        done.append(b)
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    sub = mi.DecodeCase(**{**case.__dict__, "cache_seqlens": case.cache_seqlens[done],
                           "q_bits": case.q_bits[done], "block_table": case.block_table[done],
                           "indices": None if case.indices is None else case.indices[done]})
    units = mi.workload_units(sub)
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count() or 1
    return {"seconds": dt, "requests": len(done), "units": units, "cores": int(cores),
            "what": f"first {len(done)} of {case.batch} requests"}


# DRAM bytes (read + write) per launch of the main kernel from an ncu capture of the current
# kernel, scaled to the full workload by the bytes it processes when the capture ran a smaller
# batch (see profiles/); None when the kernel has changed since the counters were taken.
TRAFFIC = {
    "mem_b128_h16_L8192": 1255.9e6,            # batch 32 capture x 4.0
    "varlen_b128_h128": 1273.7e6,              # batch 32 capture x 4.385
    "causal_b64_sq2_h128": 363.5e6,            # full capture
    "fp8_b128_h128_L16384": 1494.1e6,          # batch 16 capture x 8
    "sparse_b128_h128_L8192_topk2048": 348.1e6,  # batch 32 capture x 4
}


def rank_case(workload: str, rank: int, batch=None):
    """The batch of requests rank `rank` owns: the named workload's shapes and cache lengths,
    with the random contents drawn from a seed shifted by the rank (independent problems)."""
    import mla_inputs as mi
    w = mi.WORKLOADS[workload]
    case = mi.make_workload(workload, poison=False, batch=batch)
    if rank > 0 and w.prefill:
        s_kv = int(case.cache_seqlens[0])
        case = mi.make_prefill_case(w.s_q, w.h_q, s_kv, w.topk, w.seed + 1000 * rank, name=workload)
        case.meta["prefill"] = True
    elif rank > 0:
        idx = case.indices
        case = mi.make_case(case.batch, case.s_q, case.h_q, case.cache_seqlens, causal=case.causal,
                            kv_format=case.kv_format, seed=w.seed + 1000 * rank, poison=False, name=workload)
        if idx is not None:
            case.indices = mi.make_sparse_indices(case.cache_seqlens, case.s_q, w.topk, w.seed + 1000 * rank)
    return case


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Largest value of x over all ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class DeviceRun:
    """One workload's inputs resident on the device and the calls of one step: the tile
    scheduler (mla_get_metadata) and the decode call (main kernel + combine)."""

    def __init__(self, case, dev, mla):
        import torch
        import mla_inputs as mi
        self.case, self.dev, self.mla = case, dev, mla
        self.q = torch.from_numpy(case.q_bits.view(np.int16)).view(torch.bfloat16).to(dev)
        if case.kv_format == "bf16":
            self.kv = torch.from_numpy(case.kv.view(np.int16)).view(torch.bfloat16).reshape(
                case.num_blocks, mi.PAGE, 1, mi.D_QK).to(dev)
        else:
            self.kv = torch.from_numpy(case.kv).to(dev)
        self.bt = torch.from_numpy(case.block_table).to(dev)
        self.sl = torch.from_numpy(case.cache_seqlens).to(dev)
        self.sparse = case.indices is not None
        self.idx = torch.from_numpy(case.indices).to(dev) if self.sparse else None
        R = case.rows
        # token-sparse: the scheduler's requests are the batch * s_q query positions of h_q rows
        self.parts = mla.mla_num_sm_parts(case.h_q if self.sparse else R, 1, dev.index)
        self.ws = torch.zeros(mla.mla_workspace_size(case.batch * case.s_q, self.parts, case.h_q, 1) if self.sparse
                              else mla.mla_workspace_size(case.batch, self.parts, R, 1), dtype=torch.uint8, device=dev)
        self.out = torch.empty((case.batch, case.s_q, case.h_q, 512), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((case.batch, case.h_q, case.s_q), dtype=torch.float32, device=dev)
        self.stream = torch.cuda.current_stream(dev)
        self.prefill = bool(case.meta.get("prefill"))
        if self.prefill:
            s_kv = int(case.cache_seqlens[0])
            self.kv = self.kv.reshape(-1, mi.D_QK)[:s_kv].reshape(s_kv, 1, mi.D_QK).contiguous()
            self.q = self.q[0].contiguous()
            self.idx = self.idx[0].contiguous()
            self.out = self.out[0]
            self.lse = self.lse[0]

    def metadata(self, sl_):
        c, mla = self.case, self.mla
        if self.sparse:
            return mla.mla_get_metadata_sparse(c.batch, c.s_q, c.topk, c.h_q, 1, num_sm_parts=self.parts,
                                               device=self.dev)
        return mla.mla_get_metadata(sl_, c.rows, 1, num_sm_parts=self.parts)

    def decode_into(self, q_, bt_, sl_, idx_, md, ns, out_, lse_):
        c, mla = self.case, self.mla
        if self.prefill:
            mla.mla_sparse_prefill(q_, self.kv, idx_, c.softmax_scale, tile_md=md, num_splits=ns, out=out_, lse=lse_,
                                   workspace=self.ws)
        elif self.sparse:
            mla.mla_decode_kvcache_sparse(q_, self.kv, bt_, sl_, idx_, 512, md, ns, softmax_scale=c.softmax_scale,
                                          out=out_, lse=lse_, workspace=self.ws)
        else:
            mla.mla_decode_kvcache(q_, self.kv, bt_, sl_, 512, md, ns, softmax_scale=c.softmax_scale,
                                   causal=c.causal, out=out_, lse=lse_, workspace=self.ws)

    def step(self):
        md, ns = self.metadata(self.sl)
        self.decode_into(self.q, self.bt, self.sl, self.idx, md, ns, self.out, self.lse)

    def measure(self, steps, warmup, barrier, reduce_max):
        """Device time of `steps` whole steps (events only at the ends of the loop: the decode
        kernel is a programmatic dependent of the scheduler, and an event between them would
        serialise the pair), then, in a separate loop, of `steps` decode calls alone on fixed
        metadata (the roofline's kernel time).  Both are max-over-ranks."""
        import torch
        for _ in range(warmup):
            self.step()
        barrier()
        # clocks under the same load for ~0.3 s just before the timed region (a short timed
        # region holds only a few samples); reported beside the timed region's own samples
        with ClockSampler(self.dev) as soak:
            t0 = time.perf_counter()
            while time.perf_counter() - t0 < 0.3:
                for _ in range(max(1, steps)):
                    self.step()
                torch.cuda.synchronize(self.dev)
            soak.mark(t0, time.perf_counter())
        barrier()
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(self.dev) as clk:
            t_wall0 = time.perf_counter()
            start.record(self.stream)
            for _ in range(steps):
                self.step()
            stop.record(self.stream)
            barrier()
            clk.mark(t_wall0, time.perf_counter())
        ms_total = reduce_max(start.elapsed_time(stop))
        # decode calls alone (metadata computed once, outside the loop)
        md, ns = self.metadata(self.sl)
        for _ in range(2):
            self.decode_into(self.q, self.bt, self.sl, self.idx, md, ns, self.out, self.lse)
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(self.stream)
        for _ in range(steps):
            self.decode_into(self.q, self.bt, self.sl, self.idx, md, ns, self.out, self.lse)
        b.record(self.stream)
        barrier()
        decode_ms = reduce_max(a.elapsed_time(b)) / steps
        status = self.mla.mla_read_status(self.ws)
        clocks = clk.summary()
        clocks["soak"] = soak.summary()
        return {"ms_total": ms_total, "decode_ms": decode_ms, "clocks": clocks, "status": status}


def roofline_of(units, decode_ms, ms_step, peaks):
    """Roofline figures of one workload: the bound is the slower of its bytes at HBM peak and
    its FLOPs at tensor peak (measured peaks), `achieved` is the decode call's rate, and the
    same fraction is also given against the nominal B200 figures (8 TB/s, 2.25 PFLOP/s dense
    bf16) and, for tensor-bound work, against the sustained cuBLAS figure."""
    hbm_peak, tc_peak, tc_sustained, peak_kind = peaks
    hbm_bound = units["bytes"] / (hbm_peak * 1e9) >= units["flops"] / (tc_peak * 1e12)
    gbs = units["bytes"] / (decode_ms * 1e-3) / 1e9
    tfs = units["flops"] / (decode_ms * 1e-3) / 1e12
    if hbm_bound:
        r = {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
             "peak_kind": peak_kind + " copy bandwidth", "nominal_peak": NOMINAL_HBM_GBS,
             "frac_nominal": gbs / NOMINAL_HBM_GBS}
    else:
        r = {"bound": "tensor", "achieved": tfs, "peak": tc_peak, "unit": "TFLOP/s", "frac": tfs / tc_peak,
             "peak_kind": peak_kind + " cuBLAS bf16 burst", "frac_sustained": tfs / tc_sustained,
             "sustained_peak": tc_sustained, "nominal_peak": NOMINAL_BF16_TFLOPS,
             "frac_nominal": tfs / NOMINAL_BF16_TFLOPS}
    roof_time = max(units["bytes"] / (hbm_peak * 1e9), units["flops"] / (tc_peak * 1e12))
    r["step_frac"] = roof_time / (ms_step * 1e-3)
    return r


DEFAULT_WORKLOAD = "mem_b128_h16_L8192"
PER_WORKLOADS = ("varlen_b128_h128", "causal_b64_sq2_h128", "fp8_b128_h128_L16384",
                 "sparse_b128_h128_L8192_topk2048", "sparse_prefill_s4096_h128_kv8192_topk2048")
NOMINAL_HBM_GBS = 8000.0
NOMINAL_BF16_TFLOPS = 2250.0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--batch", type=int, default=None,
                    help="run the first BATCH requests of the workload (profiling captures)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end pass")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="time only the headline workload (by default a 1-GPU run also times the other workloads)")
    ap.add_argument("--per-steps", type=int, default=20, help="timed steps of each other workload")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    import mla_inputs as mi
    w = mi.WORKLOADS[args.workload]
    metric = "MLA paged-KV decode TFLOP/s and KV HBM GB/s; fraction of B200 roofline"
    peaks = _peaks()

    if args.impl == "reference":
        # the reference arm is the fp64 oracle on host cores (rank 0 only)
        if rank != 0:
            return
        case = mi.make_workload(args.workload, poison=False)
        per_step = []
        for _ in range(args.warmup + args.steps):
            r = oracle_baseline(case, budget_s=max(1.0, args.cpu_budget / max(1, args.steps)))
            per_step.append(r)
        timed = per_step[args.warmup:]
        byts = sum(r["units"]["bytes"] for r in timed)
        secs = sum(r["seconds"] for r in timed)
        value = byts / secs / 1e9
        line = {"impl": "reference", "metric": metric, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / len(timed),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": {"workload": args.workload, "batch": w.batch, "s_q": w.s_q,
                                                 "h_q": w.h_q, "seqlens": w.seqlens, "kv": w.kv_format,
                                                 "topk": w.topk},
                "cpu_baseline": {"value": value, "unit": "GB/s", "cores": timed[0]["cores"], "kind": "oracle",
                                 "sample": timed[0]["what"] + " per step"},
                "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import torch
    import torch.distributed as dist
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import attention_mla_get_b200 as mla

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    # every rank owns its own requests (seed shifted by rank): independent problems
    case = rank_case(args.workload, rank, args.batch)
    units = mi.workload_units(case)
    run = DeviceRun(case, dev, mla)
    m = run.measure(args.steps, args.warmup, barrier, lambda x: max_over_ranks(x, world, dev))
    ms_total, decode_ms, clk, status = m["ms_total"], m["decode_ms"], m["clocks"], m["status"]
    q, kv, bt, sl, idx, out, lse = run.q, run.kv, run.bt, run.sl, run.idx, run.out, run.lse
    sparse, prefill, parts, stream = run.sparse, run.prefill, run.parts, run.stream
    metadata, decode_into = run.metadata, run.decode_into

    # ---- end to end through the C-ABI with host buffers ----
    q_h = q.cpu().pin_memory()
    bt_h = bt.cpu().pin_memory()
    sl_h = sl.cpu().pin_memory()
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    lse_h = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    idx_h = idx.cpu().pin_memory() if sparse else None
    h2d = q_h.numel() * 2 + bt_h.numel() * 4 + sl_h.numel() * 4 + (idx_h.numel() * 4 if sparse else 0)
    d2h = out_h.numel() * 2 + lse_h.numel() * 4
    # double-buffered device inputs and outputs, two copy streams beside the compute stream
    bufs = [dict(q=torch.empty_like(q), bt=torch.empty_like(bt), sl=torch.empty_like(sl),
                 idx=torch.empty_like(idx) if sparse else None, out=torch.empty_like(out),
                 lse=torch.empty_like(lse)) for _ in range(2)] if prefill else None
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    session = None
    if not prefill:
        session = mla.MLASession(case.batch, case.s_q, case.h_q, case.block_table.shape[1],
                                 topk=case.topk if sparse else 0,
                                 kv_dtype=mla.KV_FP8 if case.kv_format == "fp8" else mla.KV_BF16,
                                 num_sm_parts=parts)

    def e2e_run(n):
        if session is not None:
            for _ in range(n):
                session.decode(q_h, kv, bt_h, sl_h, out_h, lse_h, indices_host=idx_h,
                               softmax_scale=case.softmax_scale, causal=case.causal)
            session.join()
            return
        computed = [torch.cuda.Event() for _ in range(n)]
        out_read = [torch.cuda.Event() for _ in range(n)]
        s_in.wait_stream(stream)  # nothing is copied in before the region starts
        for k in range(n):
            b = bufs[k % 2]
            in_ready = torch.cuda.Event()
            with torch.cuda.stream(s_in):
                if k >= 2:
                    s_in.wait_event(computed[k - 2])  # step k-2 has read these inputs
                b["q"].copy_(q_h, non_blocking=True)
                b["bt"].copy_(bt_h, non_blocking=True)
                b["sl"].copy_(sl_h, non_blocking=True)
                if sparse:
                    b["idx"].copy_(idx_h, non_blocking=True)
                in_ready.record(s_in)
            stream.wait_event(in_ready)
            if k >= 2:
                stream.wait_event(out_read[k - 2])  # step k-2's results have been read back
            md, ns = metadata(b["sl"])
            decode_into(b["q"], b["bt"], b["sl"], b["idx"], md, ns, b["out"], b["lse"])
            computed[k].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(computed[k])
                out_h.copy_(b["out"], non_blocking=True)
                lse_h.copy_(b["lse"], non_blocking=True)
                out_read[k].record(s_out)
        stream.wait_event(out_read[n - 1])

    e2e_ms = None
    if not args.no_e2e:
        e2e_run(args.warmup)
        barrier()
        s2, t2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        e2e_run(args.steps)
        t2.record(stream)
        barrier()
        e2e_ms = max_over_ranks(s2.elapsed_time(t2), world, dev)
    if session is not None:
        session.close()

    # ---- the other workloads (one GPU: rank 0 of a 1-rank job only), a few steps each ----
    per_workload = None
    if world == 1 and not args.no_per_workload and args.batch is None and args.workload == DEFAULT_WORKLOAD:
        per_workload = {}
        del run, q, kv, bt, sl, idx, out, lse, bufs, metadata, decode_into
        torch.cuda.empty_cache()
        for name in PER_WORKLOADS:
            wcase = mi.make_workload(name, poison=False)
            wunits = mi.workload_units(wcase)
            wrun = DeviceRun(wcase, dev, mla)
            wm = wrun.measure(args.per_steps, 3, barrier, lambda x: x)
            ms_step = wm["ms_total"] / args.per_steps
            per_workload[name] = {
                "ms_per_step": ms_step, "decode_ms": wm["decode_ms"],
                "gbs": wunits["bytes"] / (ms_step * 1e-3) / 1e9, "tflops": wunits["flops"] / (ms_step * 1e-3) / 1e12,
                "steps": args.per_steps, "warmup": 3,
                "roofline": dict(roofline_of(wunits, wm["decode_ms"], ms_step, peaks), traffic=TRAFFIC.get(name)),
                "clocks": wm["clocks"], "device_status": wm["status"],
                "gpu_launches": 3 * args.per_steps,
                "config": {"batch": wcase.batch, "s_q": wcase.s_q, "h_q": wcase.h_q, "causal": wcase.causal,
                           "kv": wcase.kv_format, "topk": wcase.topk, "seqlens": mi.WORKLOADS[name].seqlens,
                           "kv_bytes": wunits["kv_bytes"], "flops": wunits["flops"]},
            }
            del wrun
            torch.cuda.empty_cache()

    if rank != 0:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return

    total_bytes = units["bytes"] * world * args.steps
    value = total_bytes / (ms_total * 1e-3) / 1e9
    tflops = units["flops"] * world * args.steps / (ms_total * 1e-3) / 1e12
    roof = roofline_of(units, decode_ms, ms_total / args.steps, peaks)
    roof["kernel"] = "mla_decode_kvcache (split-KV main + combine), decode calls alone"
    roof["traffic"] = TRAFFIC.get(args.workload)
    line = {
        "metric": metric, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "data": "synthetic",
        # the arithmetic type of the MMAs: FP8 caches above 64 query rows run on f16 operands
        "dtype": "f16" if case.kv_format == "fp8" and case.s_q * case.h_q > 64 else "bf16",
        "config": {"workload": args.workload, "batch": case.batch, "s_q": case.s_q, "h_q": case.h_q,
                   "h_kv": 1, "d_qk": 576, "d_v": 512, "page": 64, "seqlens": w.seqlens, "causal": case.causal,
                   "topk": case.topk,
                   "kv": case.kv_format, "kv_bytes": units["kv_bytes"], "l2": "inputs larger than L2 (no flush)",
                   "parallelism": f"replicas x{world} (independent requests per GPU)"},
        "tflops": tflops,
        "roofline_fraction": roof["step_frac"],
        "roofline": roof,
        "decode_ms": decode_ms,
        "e2e": None if e2e_ms is None else {
            "value": units["bytes"] * world * args.steps / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": 3 * args.steps,
        "clocks": clk,
        "device_status": status,
    }
    if per_workload is not None:
        line["per_workload"] = per_workload
    if not args.no_cpu_baseline:
        r = oracle_baseline(case, budget_s=args.cpu_budget)
        line["cpu_baseline"] = {"value": r["units"]["bytes"] / r["seconds"] / 1e9, "unit": "GB/s",
                                "cores": r["cores"], "kind": "oracle",
                                "sample": r["what"] + ", fp64 numpy"}
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

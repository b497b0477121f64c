#!/usr/bin/env python
"""SSD forward throughput on one B200 per rank (tokens/s = batch * seqlen / s).

Default workload: the 2.7B-like layer (B4 L8192 H80 P64 N128 G1, chunk 256, bf16
inputs). One step = one ssd_fwd call over one batch of seeded synthetic inputs
that already sit in HBM. Prints ONE JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Multi-GPU: launch with torch.distributed.run; every rank runs its own batch
(weak scaling, no data-path collective; the process group only carries the
barrier and the max over ranks of the device time).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SSD fwd tokens/s (batch·seqlen/s) at 2.7B-layer shape; % of roofline"
UNIT = "tokens/s"


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d["hbm_gbs"], d["bf16_tflops"], "measured"
    return 6650.0, 1590.0, "fallback"


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "k_ssd_pair_mamba2_2p7b_traffic.json")
TC_SOURCE = os.path.join(ROOT, "state_space_sequence_chunked_b200", "csrc", "ssd_tc_pair.cu")
TC_HEADER = os.path.join(ROOT, "state_space_sequence_chunked_b200", "csrc", "tc_ptx.cuh")  # its inline PTX


def tc_kernel(wl):
    """The tensor-core forward kernel that serves this workload: the head-pair kernel where
    dstate is 128 and the heads of a group pair up, the one-head kernel otherwise."""
    return "k_ssd_pair" if wl.dstate == 128 and (wl.nheads // wl.ngroups) % 2 == 0 else "k_ssd_tc<%d>" % wl.dstate


def code_sha256(*paths):
    """SHA-256 of C++/CUDA sources with their // comments and all whitespace removed: what the
    compiler turns into code. (None of the kernel sources uses // inside a string literal.)"""
    import hashlib
    import re

    code = ""
    for path in paths:
        text = open(path, encoding="utf-8").read()
        code += "".join("".join(re.sub(r"//.*", "", line).split()) for line in text.splitlines())
    return hashlib.sha256(code.encode()).hexdigest()


def measured_traffic(wl, path):
    """DRAM bytes (read + write) per launch of the tensor-core kernel from the committed ncu
    capture, if that capture was taken of the kernel's code as it is now; else None."""
    from state_space_sequence_chunked_b200 import inputs

    if wl != inputs.WORKLOADS["mamba2_2p7b"] or path != "tcgen05" or not os.path.exists(TRAFFIC_FILE):
        return None
    rec = json.load(open(TRAFFIC_FILE))
    if rec.get("source_code_sha256") != code_sha256(TC_SOURCE, TC_HEADER):
        return None
    return rec["dram_read_bytes"] + rec["dram_write_bytes"]


def algorithmic(wl):
    """Bytes each input is read once + outputs written once; FLOPs of the chunked
    method with the structurally-zero upper triangle of the diagonal blocks skipped
    and C B^T counted once per (batch, chunk, group)."""
    B, L, H, P, N, G, Q = wl.batch, wl.seqlen, wl.nheads, wl.headdim, wl.dstate, wl.ngroups, wl.chunk
    e = 2 if wl.dtype == "bf16" else 4
    nbytes = (2 * B * L * H * P * e       # x in, y out
              + B * L * H * e             # dt
              + 2 * B * L * G * N * e     # B, C
              + 2 * H * 4                 # A, D
              + B * H * P * N * 4         # h_final
              + (B * H * P * N * 4 if wl.h0_std > 0 else 0))
    nc_full, tail = divmod(L, Q)
    tri = lambda q: q * (q + 1) / 2
    pairs = nc_full * tri(Q) + tri(tail)      # causal (l, s) pairs per (b, head-or-group)
    flops = B * (2 * pairs * N * G + 2 * pairs * P * H) + B * L * H * 4 * P * N
    return nbytes, flops


def fwd_config(wl):
    """The config object of a forward line: the workload alone, so both arms carry the same
    keys and values (the path that ran is a separate key of the line)."""
    return {"workload": wl.name, "batch": wl.batch, "seqlen": wl.seqlen, "nheads": wl.nheads,
            "headdim": wl.headdim, "dstate": wl.dstate, "ngroups": wl.ngroups, "chunk": wl.chunk,
            "dt": wl.dt_dist, "per_rank_batch": wl.batch, "l2": l2_note(wl)}


def l2_note(wl):
    e = 2 if wl.dtype == "bf16" else 4
    mb = wl.batch * wl.seqlen * wl.nheads * wl.headdim * e / 1e6
    return (f"inputs larger than L2 (x and y {mb:.1f} MB each per step vs 126 MB L2); no flush" if mb > 126
            else f"x and y {mb:.1f} MB each per step: L2 flushed between steps")


class ClockSampler:
    """SM clock and clock-event (throttle) reasons of this rank's GPU, read through NVML
    (the library nvidia-smi reports from) every 2 ms on a host thread; only samples
    taken inside the timed window [mark_start, mark_end] count."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device):
        import threading

        self.samples, self.error, self.handle = [], None, None
        self.t0 = self.t1 = None
        self.stop_ev = threading.Event()
        self.thread = None
        try:
            import pynvml as nv
            import torch

            nv.nvmlInit()
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
            self.nv = nv
            self.handle = nv.nvmlDeviceGetHandleByUUID(uuid)
            self.smax = nv.nvmlDeviceGetMaxClockInfo(self.handle, nv.NVML_CLOCK_SM)
            self.thread = threading.Thread(target=self._run, daemon=True)
        except Exception as e:  # no NVML on this host: the line says so
            self.error = f"{type(e).__name__}: {e}"

    def sample(self) -> bool:
        nv, h = self.nv, self.handle
        t = time.perf_counter()
        try:
            sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
            rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
        except Exception as e:
            self.error = f"{type(e).__name__}: {e}"
            return False
        self.samples.append((t, sm, rs))
        return True

    def _run(self):
        while not self.stop_ev.is_set():
            if not self.sample():
                return
            time.sleep(0.002)

    def start(self):
        if self.thread is not None:
            self.thread.start()

    def poll_until(self, event):
        """Sample from the calling thread until `event` (recorded after the timed launches)
        completes, so that even a timed region of a few milliseconds holds samples taken
        while its kernels run."""
        if self.handle is None:
            return
        while not event.query():
            if not self.sample():
                return

    def mark_start(self):
        self.t0 = time.perf_counter()

    def mark_end(self):
        self.t1 = time.perf_counter()

    def stop(self):
        if self.thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "error": self.error}
        self.stop_ev.set()
        self.thread.join(1.0)
        inside = [(sm, rs) for (t, sm, rs) in self.samples if self.t0 <= t <= self.t1]
        reasons = sorted({nm for (_, rs) in inside for bit, nm in self.REASONS.items() if rs & bit})
        out = {"sm_mhz": statistics.median([sm for sm, _ in inside]) if inside else None,
               "sm_max_mhz": self.smax, "reasons": reasons, "samples": len(inside), "source": "nvml, 2 ms"}
        if inside:
            out["sm_mhz_min"] = min(sm for sm, _ in inside)
        if self.error:
            out["error"] = self.error
        return out


def dist_setup(backend: str = "nccl"):
    """Rank, world size and local rank from the launcher's environment; for N > 1 a
    process group (NCCL over the GPUs; gloo on CPU for the host-logic tests)."""
    import torch
    import torch.distributed as dist

    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime

        timeout = datetime.timedelta(seconds=180)
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=timeout)
    return ws, rank, local


def reduce_max(v: float, ws: int, device: str = "cuda") -> float:
    """Max over ranks (the job's time is the slowest rank's)."""
    if ws == 1:
        return v
    import torch
    import torch.distributed as dist

    t = torch.tensor([v], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(wl, rank: int) -> int:
    """Each rank draws its own batch (weak scaling: per-rank work is fixed)."""
    return wl.seed + 1000 * rank


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist

        dist.barrier()


# ---------------------------------------------------------------------------------------
# CPU oracle timing (the CPU baseline and the reference arm)

def time_oracle(wl, d, target_s: float, backward=None):
    """Run the fp64 oracle on whole (b, h) streams (every token of the sequence) of
    the drawn inputs, as many streams as fit in about target_s. Returns (tokens/s
    extrapolated to the whole problem, streams run, threads, seconds). With `backward`
    (the drawn cotangents) it times the oracle's backward pass instead."""
    import oracle

    threads = os.cpu_count() or 1
    B, H = wl.batch, wl.nheads

    def run(nb, nh):
        G = wl.ngroups
        hpg = H // G
        if G > 1:  # keep whole groups so the head -> group map is unchanged
            nh = max(hpg, (nh // hpg) * hpg)
        ng = nh // hpg if G > 1 else 1
        hs, gs = (slice(0, nb), slice(None), slice(0, nh)), (slice(0, nb), slice(None), slice(0, ng))
        x, dt = d["x"].values(hs), d["dt"].values(hs)
        Bm, Cm = d["B"].values(gs), d["C"].values(gs)
        A, D = d["A"].value[:nh], d["D"].value[:nh]
        h0 = d["h0"].values((slice(0, nb), slice(0, nh))) if d["h0"] is not None else None
        t0 = time.perf_counter()
        if backward is None:
            oracle.recurrent(x, dt, A, Bm, Cm, D, h0, threads=threads)
        else:
            dy = backward["dy"].values(hs)
            dhf = backward["dh_final"].values((slice(0, nb), slice(0, nh))) if backward["dh_final"] else None
            oracle.backward(x, dt, A, Bm, Cm, D, h0, dy, dhf, threads=threads)
        return time.perf_counter() - t0, nb * nh

    t1, n1 = run(1, 1)
    want = max(1, int(target_s / max(t1, 1e-6) * threads))
    nb = min(B, max(1, want // H)) if want >= H else 1
    nh = H if want >= H else min(H, want)
    t, n = run(nb, nh)
    tokens = wl.batch * wl.seqlen
    value = tokens * n / (B * H) / t
    return value, n, threads, t


def reference_arm(args, wl):
    """The CPU oracle as the reference arm, on the same workload and metric."""
    from state_space_sequence_chunked_b200 import inputs

    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    d = inputs.draw(wl)
    per_step = max(1.0, min(5.0, 150.0 / max(1, args.steps + args.warmup)))
    vals, secs = [], []
    for i in range(args.warmup + args.steps):
        v, n, threads, t = time_oracle(wl, d, per_step)
        if i >= args.warmup:
            vals.append(v)
            secs.append(t)
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * wl.batch * wl.seqlen / value, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": fwd_config(wl), "path": "oracle: fp64 recurrence on the host cores",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"fp64 recurrence on {n} of {wl.batch * wl.nheads} (batch, head) streams "
                                   f"over all {wl.seqlen} tokens per step, extrapolated to the whole batch"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0



VERIFY_METRIC = "SSD speculative verify + state selection draft tokens/s (batch*K/s)"


def verify_main(args, wl):
    """One step = ssd_verify (K draft tokens from a saved state, every state written) and
    ssd_select_state (keep the state at the accepted index), on seeded inputs in HBM."""
    import torch

    from state_space_sequence_chunked_b200 import _binding as ssd
    from state_space_sequence_chunked_b200 import inputs

    ws, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    d = inputs.draw(wl, seed=rank_seed(wl, rank))
    g = {k: d[k].torch(dev) for k in ("x", "dt", "A", "B", "C", "D", "h0")}
    acc = torch.from_numpy(d["accepted"]).to(dev)
    Bsz, K, H, P, N, G = wl.batch, wl.seqlen, wl.nheads, wl.headdim, wl.dstate, wl.ngroups
    so = torch.empty(Bsz, K, H, P, N, device=dev)
    y = torch.empty_like(g["x"])
    keep = torch.empty(Bsz, H, P, N, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        ssd.ssd_verify(g["h0"], g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], states_out=so, y=y, stream=stream)
        ssd.ssd_select_state(g["h0"], so, acc, h_keep=keep, stream=stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(dev)
    clocks.start()
    ev0, ev1, ev2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    barrier(ws)
    torch.cuda.synchronize()
    clocks.mark_start()
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    clocks.poll_until(ev1)
    torch.cuda.synchronize()
    clocks.mark_end()
    barrier(ws)
    clk = clocks.stop()
    ms = ev0.elapsed_time(ev1) / args.steps
    # the verify kernel alone, for its own roofline
    ev0.record(stream)
    for _ in range(args.steps):
        ssd.ssd_verify(g["h0"], g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], states_out=so, y=y, stream=stream)
    ev2.record(stream)
    torch.cuda.synchronize()
    ms_v = ev0.elapsed_time(ev2) / args.steps
    ms_max = reduce_max(ms, ws)
    e = 2  # bf16 inputs
    v_bytes = (Bsz * H * P * N * 4 * (1 + K) + Bsz * K * H * P * e * 2 + Bsz * K * H * e
               + 2 * Bsz * K * G * N * e + 2 * H * 4)
    s_bytes = 2 * Bsz * H * P * N * 4 + Bsz * 4
    hbm, _, src = peaks()
    tokens = Bsz * K
    if rank == 0:
        line = {
            "metric": VERIFY_METRIC, "value": tokens * ws / (ms_max * 1e-3), "unit": "tokens/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
            "config": {"workload": wl.name, "batch": Bsz, "K": K, "nheads": H, "headdim": P, "dstate": N,
                       "ngroups": G, "l2": "states_out 1074 MB per step vs 126 MB L2; no flush"},
            "roofline": {"bound": "hbm", "achieved": v_bytes / (ms_v * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
                         "frac": v_bytes / (ms_v * 1e-3) / 1e9 / hbm, "traffic": None, "kernel": "k_verify",
                         "peak_source": src, "alg_bytes": v_bytes, "ms": ms_v,
                         "step_bytes": v_bytes + s_bytes,
                         "step_frac": (v_bytes + s_bytes) / (ms * 1e-3) / 1e9 / hbm},
            "cpu_baseline": None, "gpu_launches": 2 * args.steps, "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


BWD_METRIC = "SSD bwd tokens/s (batch·seqlen/s) at 2.7B-layer shape; % of roofline"


def bwd_algorithmic(wl):
    """FLOPs of the chunked backward with recomputation (causal pairs only, C B^T once per
    (batch, chunk, group), each dot product dy.x counted once) and the bytes of its inputs
    read once and gradients written once."""
    B, L, H, P, N, G, Q = wl.batch, wl.seqlen, wl.nheads, wl.headdim, wl.dstate, wl.ngroups, wl.chunk
    e = 2 if wl.dtype == "bf16" else 4
    nc_full, tail = divmod(L, Q)
    tri = lambda q: q * (q + 1) / 2
    pairs = nc_full * tri(Q) + tri(tail)
    # per head: dy.x, u (P wide), v and w (N wide) over the pairs; five P x N products per
    # token (recomputed chunk state, adjoint chunk sum, Gend B, Gend^T x, S_in^T dy)
    flops = B * (2 * pairs * N * G + H * pairs * (4 * P + 4 * N)) + 10 * B * L * H * P * N
    nbytes = (3 * B * L * H * P * e          # x, dy in; dx out
              + 2 * B * L * H * e            # dt in; ddt out
              + 4 * B * L * G * N * e        # B, C in; dB, dC out
              + 4 * H * 4                    # A, D in; dA, dD out
              + 2 * B * H * P * N * 4        # dh_final in; dh0 out
              + (B * H * P * N * 4 if wl.h0_std > 0 else 0))
    return nbytes, flops


def alu_peak_tflops(clock_mhz):
    """fp32 FMA peak of the CUDA cores: 148 SMs x 128 fp32 lanes x 2 FLOP per clock."""
    return 148 * 128 * 2 * clock_mhz * 1e6 / 1e12


def bwd_main(args, wl):
    """One step = one ssd_bwd call (gradients of every input, states recomputed) on seeded
    inputs and cotangents resident in HBM."""
    import torch

    from state_space_sequence_chunked_b200 import _binding as ssd
    from state_space_sequence_chunked_b200 import inputs

    ws, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    d = inputs.draw(wl, seed=rank_seed(wl, rank))
    cot = inputs.draw_cotangents(wl, seed=rank_seed(wl, rank))
    code = ssd.SSD_BF16 if wl.dtype == "bf16" else ssd.SSD_F32
    g = {k: d[k].torch(dev) for k in ("x", "dt", "A", "B", "C", "D")}
    g["dy"] = cot["dy"].torch(dev)
    g["dhf"] = cot["dh_final"].torch(dev)
    h0 = d["h0"].torch(dev) if d["h0"] is not None else None
    need = ssd.bwd_workspace_bytes(wl.batch, wl.seqlen, wl.nheads, wl.headdim, wl.ngroups, wl.dstate, code,
                                   wl.chunk)
    work = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    out = {"dx": torch.empty_like(g["x"]), "ddt": torch.empty_like(g["dt"]), "dA": torch.empty_like(g["A"]),
           "dB": torch.empty_like(g["B"]), "dC": torch.empty_like(g["C"]), "dD": torch.empty_like(g["D"]),
           "dh0": torch.empty_like(g["dhf"])}
    stream = torch.cuda.current_stream(dev)
    plan = ssd.bwd_plan(wl.batch, wl.seqlen, wl.nheads, wl.headdim, wl.ngroups, wl.dstate, code, wl.chunk)
    launches = plan["kernels"]

    def call(src):
        ssd.ssd_bwd(src["x"], src["dt"], src["A"], src["B"], src["C"], src["D"], h0, src["dy"], src["dhf"],
                    chunk=wl.chunk, out=out, workspace=work, stream=stream)

    for _ in range(max(3, args.warmup)):
        call(g)
    torch.cuda.synchronize()
    clocks = ClockSampler(dev)
    clocks.start()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(ws)
    torch.cuda.synchronize()
    clocks.mark_start()
    ev0.record(stream)
    for _ in range(args.steps):
        call(g)
    ev1.record(stream)
    clocks.poll_until(ev1)
    torch.cuda.synchronize()
    clocks.mark_end()
    barrier(ws)
    clk = clocks.stop()
    ms = ev0.elapsed_time(ev1) / args.steps
    ms_max = reduce_max(ms, ws)

    # end to end: inputs and cotangents from pinned host memory, every gradient back
    host = {k: v.cpu().pin_memory() for k, v in g.items()}
    dg = {k: torch.empty_like(v) for k, v in g.items()}
    out_host = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in out.items()}

    def e2e_step():
        for k in dg:
            dg[k].copy_(host[k], non_blocking=True)
        call(dg)
        for k in out:
            out_host[k].copy_(out[k], non_blocking=True)

    e2e_steps = max(3, min(args.steps, 5))
    e2e_step()
    torch.cuda.synchronize()
    barrier(ws)
    ev0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    e2e_ms = reduce_max(ev0.elapsed_time(ev1) / e2e_steps, ws)
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = sum(v.numel() * v.element_size() for v in out_host.values())

    tokens = wl.batch * wl.seqlen
    nbytes, flops = bwd_algorithmic(wl)
    hbm, tf, src = peaks()
    clk_mhz = clk.get("sm_mhz") or 1965.0
    achieved = flops / (ms * 1e-3) / 1e12
    if plan["path"] == "mma":  # every product on tensor cores (bf16 mma.sync)
        bound, peak, peak_src = "tensor", tf, f"bf16 dense, {src} (MEASURED_PEAKS.json)"
        what = "fp32-accumulated bf16 mma.sync products"
    else:
        bound, peak = "alu", alu_peak_tflops(clk.get("sm_max_mhz") or 1965.0)
        peak_src, what = "148 SMs x 128 fp32 lanes x 2 FLOP x max SM clock", "fp32 FMA on CUDA cores"
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        v, n, threads, t = time_oracle(wl, d, args.cpu_seconds, backward=cot)
        cpu = {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"fp64 backward of the recurrence on {n} of {wl.batch * wl.nheads} (batch, head) streams "
                         f"over all {wl.seqlen} tokens ({t:.1f} s), extrapolated to the whole batch"}
    if rank == 0:
        line = {
            "metric": BWD_METRIC, "value": tokens * ws / (ms_max * 1e-3), "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if plan["path"] == "mma" else "f32",
            "data": "synthetic",
            "config": {"workload": wl.name + " backward", "path": plan["path"], "batch": wl.batch, "seqlen": wl.seqlen,
                       "nheads": wl.nheads, "headdim": wl.headdim, "dstate": wl.dstate, "ngroups": wl.ngroups,
                       "chunk": wl.chunk, "io_dtype": wl.dtype,
                       "l2": "inputs larger than L2 (x, dy, dx 335.5 MB each per step vs 126 MB L2); no flush"},
            "roofline": {"bound": bound, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": None,
                         "kernel": "whole ssd_bwd call (%d launches, %s)" % (launches, what),
                         "peak_source": peak_src,
                         "alg_flops": flops, "alg_bytes": nbytes,
                         "hbm_frac": nbytes / (ms * 1e-3) / 1e9 / hbm,
                         "tensor_roofline_ms": flops / (tf * 1e12) * 1e3,
                         "hbm_roofline_ms": nbytes / (hbm * 1e9) * 1e3, "sm_mhz_median": clk_mhz},
            "cpu_baseline": cpu,
            "e2e": {"value": tokens * ws / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": launches * args.steps, "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


def block_main(args):
    """The Mamba-2 mixer forward at the 2.7B-like layer (d_model 2560, H80 P64 N128 G1, conv
    width 4, one norm group) on B4 L8192: in_proj GEMM (cuBLAS), ssd_conv_split, ssd_fwd,
    ssd_gated_rmsnorm, out_proj GEMM (cuBLAS). One JSON line per part (CUDA events over --steps
    calls of that part alone, each against its own roofline) and one for the whole mixer."""
    import torch

    from state_space_sequence_chunked_b200 import _binding as ssd
    from state_space_sequence_chunked_b200 import inputs, mamba2

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    hbm, tf, src = peaks()
    steps = max(args.steps, 1)
    cfg = mamba2.MixerConfig(d_model=2560, nheads=80, headdim=64, ngroups=1, dstate=128, norm_groups=1)
    Bsz, L = 4, 8192
    d = inputs.draw_mixer(batch=Bsz, seqlen=L, d_model=cfg.d_model, nheads=cfg.nheads, headdim=cfg.headdim,
                          ngroups=cfg.ngroups, dstate=cfg.dstate, seed=2)
    g = {k: v.torch(dev) for k, v in d.items()}
    w = mamba2.MixerWeights(in_proj=g["in_proj"], conv_w=g["conv_w"], conv_b=g["conv_b"], dt_bias=g["dt_bias"],
                            A=g["A"], D=g["D"], norm_w=g["norm_w"], out_proj=g["out_proj"])
    HP, GN, H, dm, Dp = cfg.d_inner, cfg.ngroups * cfg.dstate, cfg.nheads, cfg.d_model, cfg.d_in_proj
    Cc = HP + 2 * GN
    T = Bsz * L
    zx = torch.matmul(g["u"], w.in_proj.t())
    sp = ssd.ssd_conv_split(zx[..., HP:HP + Cc], zx[..., HP + Cc:], w.conv_w, w.conv_b, w.dt_bias, nheads=H,
                            headdim=cfg.headdim, ngroups=cfg.ngroups, dstate=cfg.dstate)
    y, hf = ssd.ssd_fwd(sp["x"], sp["dt"], w.A, sp["B"], sp["C"], w.D, None, chunk=cfg.chunk)
    o = ssd.ssd_gated_rmsnorm(y.view(Bsz, L, HP), zx[..., :HP], w.norm_w, ngroups=1)
    ws = torch.empty(max(ssd.fwd_workspace_bytes(Bsz, L, H, cfg.headdim, cfg.ngroups, cfg.dstate, ssd.SSD_BF16,
                                                 cfg.chunk), 16), dtype=torch.uint8, device=dev)

    def timed(fn):
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    parts = []

    def part(name, fn, nbytes=0.0, flops=0.0):
        ms = timed(fn)
        t_b, t_f = nbytes / (hbm * 1e9), flops / (tf * 1e12)
        bound = "tensor" if t_f > t_b else "hbm"
        line = {"part": name, "ms": ms, "alg_bytes": nbytes, "alg_flops": flops, "bound": bound,
                "frac": max(t_b, t_f) / (ms * 1e-3), "achieved_gbs": nbytes / (ms * 1e-3) / 1e9,
                "achieved_tflops": flops / (ms * 1e-3) / 1e12, "roofline_ms": max(t_b, t_f) * 1e3}
        parts.append(line)
        print(json.dumps(line), flush=True)

    part("in_proj GEMM (cuBLAS)", lambda: torch.matmul(g["u"], w.in_proj.t(), out=zx),
         2 * (T * dm + Dp * dm + T * Dp), 2.0 * T * dm * Dp)
    part("ssd_conv_split", lambda: ssd.ssd_conv_split(zx[..., HP:HP + Cc], zx[..., HP + Cc:], w.conv_w, w.conv_b,
                                                      w.dt_bias, nheads=H, headdim=cfg.headdim, ngroups=cfg.ngroups,
                                                      dstate=cfg.dstate, out=sp, stream=stream),
         2 * 2 * T * (Cc + H) + Cc * 4 * 5 + H * 4)
    nb, fl = algorithmic(inputs.Workload("mixer", Bsz, L, H, cfg.headdim, cfg.dstate, cfg.ngroups, cfg.chunk, "bf16",
                                         0.0, 2))
    part("ssd_fwd", lambda: ssd.ssd_fwd(sp["x"], sp["dt"], w.A, sp["B"], sp["C"], w.D, None, chunk=cfg.chunk, y=y,
                                        h_final=hf, workspace=ws, stream=stream), nb, fl)
    part("ssd_gated_rmsnorm", lambda: ssd.ssd_gated_rmsnorm(y.view(Bsz, L, HP), zx[..., :HP], w.norm_w, ngroups=1,
                                                            out=o, stream=stream), 3 * 2 * T * HP + HP * 4)
    out = torch.empty(Bsz, L, dm, dtype=torch.bfloat16, device=dev)
    part("out_proj GEMM (cuBLAS)", lambda: torch.matmul(o, w.out_proj.t(), out=out), 2 * (T * HP + dm * HP + T * dm),
         2.0 * T * HP * dm)
    ms = timed(lambda: mamba2.mixer_fwd(g["u"], w, cfg, stream=stream))
    roof = sum(p_["roofline_ms"] for p_ in parts)
    print(json.dumps({"metric": "Mamba-2 mixer fwd tokens/s at the 2.7B-like layer", "value": T / (ms * 1e-3),
                      "unit": "tokens/s", "ms": ms, "sum_of_parts_ms": sum(p_["ms"] for p_ in parts),
                      "roofline_ms": roof, "frac_of_roofline_time": roof / ms, "steps": steps,
                      "config": {"batch": Bsz, "seqlen": L, "d_model": dm, "nheads": H, "headdim": cfg.headdim,
                                 "dstate": cfg.dstate, "ngroups": cfg.ngroups, "conv_width": cfg.conv_width,
                                 "norm_groups": 1, "dtype": "bf16"}, "peak_source": src}), flush=True)
    return 0


def aux_main(args):
    """Per-kernel timings of the kernels beside the forward, each against the HBM roofline
    (all of them are bandwidth-bound): the two verify flows on the spec-decode workload
    (all K states stored + select, or outputs only + recomputing the kept state), the
    one-token decode step at the same shape, and the three context-parallel steps for one
    rank's eighth of the long-context sequence (B1 L8192 of L65536, H80 P64 N256). One JSON
    line per kernel; inputs resident in HBM; CUDA events around `--steps` launches."""
    import torch

    from state_space_sequence_chunked_b200 import _binding as ssd
    from state_space_sequence_chunked_b200 import inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    hbm, _, src = peaks()
    steps = max(args.steps, 1)

    def timed(fn):
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    def emit(kernel, workload, ms, alg_bytes, launches, **extra):
        gbs = alg_bytes / (ms * 1e-3) / 1e9
        print(json.dumps({"kernel": kernel, "workload": workload, "ms": ms, "alg_bytes": alg_bytes,
                          "launches_per_call": launches, "achieved_gbs": gbs, "peak_gbs": hbm,
                          "peak_source": src, "frac": gbs / hbm, "steps": steps, **extra}), flush=True)

    # spec-decode verify workload: B64 K8 H32 P128 N128 G8, bf16 inputs, fp32 states
    wl = inputs.WORKLOADS["verify_k8"]
    d = inputs.draw(wl)
    g = {k: d[k].torch(dev) for k in ("x", "dt", "A", "B", "C", "D", "h0")}
    acc = torch.from_numpy(d["accepted"]).to(dev)
    Bsz, K, H, P, N, G = wl.batch, wl.seqlen, wl.nheads, wl.headdim, wl.dstate, wl.ngroups
    state = Bsz * H * P * N * 4
    x_b, dt_b, bc_b = Bsz * K * H * P * 2, Bsz * K * H * 2, Bsz * K * G * N * 2  # x (= y), dt, B (= C)
    small = 2 * x_b + dt_b + 2 * bc_b
    so = torch.empty(Bsz, K, H, P, N, device=dev)
    y = torch.empty_like(g["x"])
    keep = torch.empty(Bsz, H, P, N, device=dev)
    ms = timed(lambda: ssd.ssd_verify(g["h0"], g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], states_out=so, y=y,
                                      stream=stream))
    emit("k_verify (all K states)", wl.name, ms, state * (1 + K) + small, 1)
    ms = timed(lambda: ssd.ssd_select_state(g["h0"], so, acc, h_keep=keep, stream=stream))
    emit("k_select", wl.name, ms, 2 * state, 1)
    ms = timed(lambda: ssd.ssd_verify(g["h0"], g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], y=y,
                                      return_states=False, stream=stream))
    emit("k_verify (outputs only)", wl.name, ms, state + small, 1)
    ms = timed(lambda: ssd.ssd_advance_state(g["h0"], g["x"], g["dt"], g["A"], g["B"], acc, h_keep=keep,
                                             stream=stream))
    emit("k_advance", wl.name, ms, 2 * state + x_b + dt_b + bc_b, 1)
    st = g["h0"].clone()
    x1, dt1 = g["x"][:, 0].contiguous(), g["dt"][:, 0].contiguous()
    B1, C1 = g["B"][:, 0].contiguous(), g["C"][:, 0].contiguous()
    y1 = torch.empty_like(x1)
    ms = timed(lambda: ssd.ssd_decode_step(st, x1, dt1, g["A"], B1, C1, g["D"], y=y1, stream=stream))
    emit("k_decode (one token, in place)", "verify_k8 shape, K=1", ms, 2 * state + small // K, 1)  # small/K: one token
    del so

    # context parallelism: one of 8 segments of the long-context workload
    wl = inputs.WORKLOADS["long_n256"]
    R, Ls = 8, wl.seqlen // 8
    d = inputs.draw(wl, seqlen=Ls)
    g = {k: d[k].torch(dev) for k in ("x", "dt", "A", "B", "C", "D")}
    Bsz, H, P, N, G = wl.batch, wl.nheads, wl.headdim, wl.dstate, wl.ngroups
    nblk = (Ls + 127) // 128
    bd = torch.empty(Bsz, H, nblk, device=dev)
    tot = torch.empty(Bsz, H, device=dev)
    ms = timed(lambda: ssd.ssd_cp_decay(g["dt"], g["A"], block_decay=bd, total=tot, stream=stream))
    emit("k_block_decay + k_total_decay", f"long_n256 segment 1/{R}", ms, Bsz * Ls * H * 2 + Bsz * H * (nblk + 1) * 4,
         2)
    states = torch.randn(R, Bsz, H, P, N, device=dev) * 0.1
    totals = -torch.rand(R, Bsz, H, device=dev)
    s_in = torch.empty(Bsz, H, P, N, device=dev)
    hf = torch.empty(Bsz, H, P, N, device=dev)
    ms = timed(lambda: ssd.ssd_cp_combine(states, totals, R - 1, s_in=s_in, h_final=hf, stream=stream))
    emit("k_combine (last of 8 ranks)", f"long_n256 B1 H80 P64 N256, R={R}", ms,
         (R + 2) * Bsz * H * P * N * 4 + R * Bsz * H * 4, 1)
    yseg = torch.zeros(Bsz, Ls, H, P, dtype=torch.bfloat16, device=dev)
    ms = timed(lambda: ssd.ssd_cp_correct(g["dt"], g["A"], g["C"], bd, s_in, yseg, stream=stream))
    flops = 2.0 * Bsz * Ls * H * P * N
    emit("k_correct_tc", f"long_n256 segment 1/{R}", ms,
         2 * Bsz * Ls * H * P * 2 + Bsz * Ls * G * N * 2 + Bsz * Ls * H * 2 + Bsz * H * P * N * 4, 1,
         flops=flops, tflops=flops / (ms * 1e-3) / 1e12)
    return 0


# ---------------------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mamba2_2p7b")
    ap.add_argument("--seqlen", type=int, default=None,
                    help="override the workload's sequence length (a smaller case for profiler captures)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--block", action="store_true",
                    help="time the Mamba-2 mixer forward around the SSD layer (1 GPU, one line per part)")
    ap.add_argument("--bwd", action="store_true",
                    help="time the backward pass (ssd_bwd) of the forward workload instead")
    ap.add_argument("--aux", action="store_true",
                    help="time the verify/decode and context-parallel kernels instead (1 GPU, one line per kernel)")
    args = ap.parse_args()
    if args.aux:
        return aux_main(args)
    if args.block:
        return block_main(args)

    from state_space_sequence_chunked_b200 import inputs

    wl = inputs.WORKLOADS[args.workload]
    if args.seqlen is not None:
        import dataclasses

        wl = dataclasses.replace(wl, seqlen=args.seqlen)
    if args.bwd:
        if args.impl == "reference" or wl.verify:
            raise SystemExit("--bwd times this library's backward of a forward workload")
        return bwd_main(args, wl)
    if wl.verify:
        if args.impl == "reference":
            raise SystemExit("the reference arm times the forward workloads")
        return verify_main(args, wl)
    if args.impl == "reference":
        return reference_arm(args, wl)

    import torch

    from state_space_sequence_chunked_b200 import _binding as ssd

    ws, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    d = inputs.draw(wl, seed=rank_seed(wl, rank))
    code = ssd.SSD_BF16 if wl.dtype == "bf16" else ssd.SSD_F32
    plan = ssd.fwd_plan(wl.batch, wl.seqlen, wl.nheads, wl.headdim, wl.ngroups, wl.dstate, code, wl.chunk)
    g = {k: d[k].torch(dev) for k in ("x", "dt", "A", "B", "C", "D")}
    h0 = d["h0"].torch(dev) if d["h0"] is not None else None
    y = torch.empty_like(g["x"])
    hf = torch.empty(wl.batch, wl.nheads, wl.headdim, wl.dstate, device=dev)
    work = torch.empty(max(plan["workspace_bytes"], 16), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        ssd.ssd_fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], h0, chunk=wl.chunk, y=y, h_final=hf,
                    workspace=work, stream=stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()

    clocks = ClockSampler(dev)
    clocks.start()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(ws)
    torch.cuda.synchronize()
    # inputs smaller than L2: each step timed on its own, with a write of 256 MB between steps
    flush = None if wl.batch * wl.seqlen * wl.nheads * wl.headdim * (2 if wl.dtype == "bf16" else 4) > 126e6 \
        else torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    clocks.mark_start()
    if flush is None:
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        clocks.poll_until(ev1)
        torch.cuda.synchronize()
        total_ms = ev0.elapsed_time(ev1)
    else:
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for a, b in evs:
            flush.zero_()
            a.record(stream)
            step()
            b.record(stream)
        clocks.poll_until(evs[-1][1])
        torch.cuda.synchronize()
        total_ms = sum(a.elapsed_time(b) for a, b in evs)
    clocks.mark_end()
    barrier(ws)
    clk = clocks.stop()
    ms = total_ms / args.steps
    ms_max = reduce_max(ms, ws)

    tokens = wl.batch * wl.seqlen
    value = tokens * ws / (ms_max * 1e-3)
    hbm, tf, src = peaks()
    nbytes, flops = algorithmic(wl)
    t_roof = max(nbytes / (hbm * 1e9), flops / (tf * 1e12))
    bound = "hbm" if nbytes / (hbm * 1e9) >= flops / (tf * 1e12) else "tensor"
    if bound == "hbm":
        achieved, peak, unit = nbytes / (ms * 1e-3) / 1e9, hbm, "GB/s"
    else:
        achieved, peak, unit = flops / (ms * 1e-3) / 1e12, tf, "TFLOP/s"

    # end to end through the public call with host buffers
    host = {k: v.cpu().pin_memory() for k, v in g.items()}
    h0_host = h0.cpu().pin_memory() if h0 is not None else None
    y_host = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    hf_host = torch.empty(hf.shape, dtype=hf.dtype).pin_memory()
    dg = {k: torch.empty_like(v) for k, v in g.items()}
    dh0 = torch.empty_like(h0) if h0 is not None else None

    def e2e_step():
        for k in dg:
            dg[k].copy_(host[k], non_blocking=True)
        if dh0 is not None:
            dh0.copy_(h0_host, non_blocking=True)
        ssd.ssd_fwd(dg["x"], dg["dt"], dg["A"], dg["B"], dg["C"], dg["D"], dh0, chunk=wl.chunk, y=y,
                    h_final=hf, workspace=work, stream=stream)
        y_host.copy_(y, non_blocking=True)
        hf_host.copy_(hf, non_blocking=True)

    e2e_steps = max(3, min(args.steps, 10))
    e2e_step()
    torch.cuda.synchronize()
    barrier(ws)
    ev0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    e2e_ms = reduce_max(ev0.elapsed_time(ev1) / e2e_steps, ws)
    h2d = sum(v.numel() * v.element_size() for v in host.values()) + (
        h0_host.numel() * 4 if h0_host is not None else 0)
    d2h = y_host.numel() * y_host.element_size() + hf_host.numel() * 4

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        v, n, threads, t = time_oracle(wl, d, args.cpu_seconds)
        cpu = {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"fp64 recurrence on {n} of {wl.batch * wl.nheads} (batch, head) streams over all "
                         f"{wl.seqlen} tokens ({t:.1f} s), extrapolated to the whole batch"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
            "config": fwd_config(wl), "path": plan["path"],
            "roofline": {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                         "frac": achieved / peak, "traffic": measured_traffic(wl, plan["path"]),
                         "kernel": ("%s (the whole call: one launch after a status-word memset)" % tc_kernel(wl)
                                    if plan["path"] == "tcgen05" else
                                    "whole ssd_fwd call (%d launches)" % plan["kernels"]),
                         "peak_source": src, "alg_bytes": nbytes, "alg_flops": flops,
                         "roofline_tokens_per_s": tokens / t_roof, "frac_of_roofline_time": t_roof / (ms * 1e-3)},
            "cpu_baseline": cpu,
            "e2e": {"value": tokens * ws / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": plan["kernels"] * args.steps,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

"""Throughput of the chunked gated delta rule (prefill) and the decode step on B200.

One bench step = one gdn_chunk_fwd over the long-context prefill workload
(2 sequences x 32768 tokens, Nqk = 16, Nv = 32, Dk = Dv = 128, chunk 64,
bf16 q/k/v/out, fp32 g/beta/state, zero initial state), inputs resident in HBM.
The decode workload (256 sequences x 1024 steps, same heads, fp32 state
[256, 32, 128, 128] carried in place) is timed in the same run and reported
under "decode".

Prints ONE JSON line on rank 0.  Multi-GPU runs are independent replicas (each
rank owns its own sequences; no collective on the data path): weak scaling.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--no-decode] [--no-e2e] [--no-cpu-baseline]
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDN chunked-fwd tokens/s (Nv=32,D=128) & decode tok/s; % of B200 roofline"
PREFILL = "long_bf16_nv32"
DECODE = "decode_bf16_nv32"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# --------------------------------------------------------------------------- accounting
def prefill_bytes(T, nqk, nv, dk, dv, n, esz, s0=False, sf=True):
    """Algorithmic bytes of one gdn_chunk_fwd: inputs read once, outputs written once."""
    b = T * nqk * dk * esz * 2 + T * nv * dv * esz * 2 + T * nv * 4 * 2 + (n + 1) * 4
    b += (n * nv * dk * dv * 4) * (int(s0) + int(sf))
    return b


def prefill_flops(T_per_seq, n, nv, C, D):
    """(dense, triangular) FLOPs: per chunk-head 10C^2D + 6CD^2 + C^3/3, and 5C^2D + 6CD^2 + C^3/3."""
    chunks = n * nv * ((T_per_seq + C - 1) // C)
    dense = 10 * C * C * D + 6 * C * D * D + C ** 3 / 3
    tri = 5 * C * C * D + 6 * C * D * D + C ** 3 / 3
    return chunks * dense, chunks * tri


def decode_bytes(n, nqk, nv, dk, dv, esz):
    return n * nv * dk * dv * 4 * 2 + n * (2 * nqk * dk + 2 * nv * dv) * esz + n * nv * 4 * 2


# DRAM traffic per launch from an ncu capture (profiles/traffic.json), valid
# only while the kernel's sources hash to the value recorded with it.
KERNEL_SOURCES = {
    "chunk_fwd_tc": ["chunk_tc.cu", "sm100_ptx.cuh", "gdn_common.cuh"],
    "recurrent_step": ["decode_step.cu", "gdn_common.cuh"],
}


def source_hash(kernel):
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "gated_deltanet_chunk_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def recorded_traffic(kernel, units):
    """Bytes per launch for `units` (tokens or sequences), or None if no capture matches the sources."""
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))[kernel]
    except Exception:
        return None
    if rec.get("source_sha256") != source_hash(kernel):
        return None
    return rec["bytes_per_unit"] * units


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running (read-only)."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index, period=0.02):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period, self.index = period, index
        self._stop = threading.Event()
        self._thread = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        except Exception:
            self._nv = None
        return self

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                mask = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        return {"sm_mhz": (statistics.median(self.samples) if self.samples else None),
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# --------------------------------------------------------------------------- distributed
def dist_setup(args, backend="nccl"):
    """One process per GPU: rank, world size and local rank from the launcher's
    environment; a process group (NCCL over NVLink by default; gloo for the CPU
    tests of this plumbing) when there is more than one rank."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return world, rank, local  # rank 0 alone runs the CPU oracle; no process group
    if backend == "nccl":
        torch.cuda.set_device(local if world > 1 else 0)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def job_throughput(units_per_rank, world, steps, total_ms):
    """Whole-job units/s: every rank's units over the slowest rank's time (weak scaling)."""
    return units_per_rank * world * steps / (total_ms / 1e3)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world, device=None):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], device=device or "cpu", dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------------------- CPU oracle timing
def time_oracle(w, T_sample, heads=None):
    """Wall time of the fp64 oracle over the first T_sample tokens of each sequence."""
    import torch

    import oracle
    cu = w["cu_seqlens"].tolist()
    idx = torch.cat([torch.arange(cu[n], min(cu[n] + T_sample, cu[n + 1])) for n in range(len(cu) - 1)])
    lens = [min(T_sample, cu[n + 1] - cu[n]) for n in range(len(cu) - 1)]
    sub = {k: w[k][idx] for k in ("q", "k", "v", "g", "beta")}
    cus = torch.tensor([0] + list(torch.cumsum(torch.tensor(lens), 0).tolist()), dtype=torch.int32)
    # conversion to fp64 arrays happens before the clock starts
    q, k, v, g, beta = (oracle._f64(sub[x]) for x in ("q", "k", "v", "g", "beta"))
    t0 = time.perf_counter()
    oracle.recurrent(q, k, v, g, beta, None, cus)
    dt = time.perf_counter() - t0
    return sum(lens), dt


# --------------------------------------------------------------------------- main
def time_steps(fn, warmup, steps, stream, world, dev):
    """Device time per call of ``fn`` (CUDA events on ``stream``, max over ranks), after warm-up."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize(dev)
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        fn()
    b.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    return max_over_ranks(a.elapsed_time(b), world, dev) / steps


def time_graph(calls, replays, warmup, stream, world, dev):
    """Device time per call of the closures ``calls``, captured once in a CUDA graph and replayed
    ``replays`` times: short kernels are then timed without the host's per-call launch cost."""
    import torch
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        for f in calls:  # eager once on a side stream before capture
            f()
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for f in calls:
            f()
    ms = time_steps(g.replay, warmup, replays, stream, world, dev)
    del g
    return ms / len(calls)


def hbm_line(ms, byts, peaks, peak_src, **extra):
    gbs = byts / (ms / 1e3) / 1e9
    r = {"ms_per_step": ms, "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"],
                                         "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                                         "peak_source": peak_src, "alg_bytes_per_launch": byts}}
    r.update(extra)
    return r


def run_ours(args, world, rank, local):
    import torch

    import gated_deltanet_chunk_b200 as gdn
    import workloads as W

    dev = torch.device("cuda", local)
    peaks, peak_src = load_peaks()
    if args.no_prefill:  # profiling helper: the decode workload alone
        stream = torch.cuda.current_stream(dev)
        return {"metric": METRIC, "decode": run_decode(args, world, rank, dev, stream, peaks, peak_src)}
    wl = W.WORKLOADS[PREFILL]
    over = {"seq_len": args.seq_len} if args.seq_len else {}
    host = W.make_workload(PREFILL, seed=2 + rank, **over)  # each rank: its own sequences
    n, T, nqk, nv, D, C = wl.num_seqs, host["T"], wl.nqk, wl.nv, wl.d, wl.chunk
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in host.items()}
    out = torch.empty(T, nv, D, dtype=torch.bfloat16, device=dev)
    sf = torch.empty(n, nv, D, D, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        gdn.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], None, None, chunk_size=C,
                      out=out, final_state=sf, num_seqs=n, kernel=args.kernel)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize(dev)
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for i in range(args.steps):
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
    total_ms = max_over_ranks(t_start.elapsed_time(t_end), world, dev)
    per_launch_ms = [a.elapsed_time(b) for a, b in evs]
    kern_ms = statistics.mean(per_launch_ms)
    ms_per_step = total_ms / args.steps
    value = job_throughput(T, world, args.steps, total_ms)

    bytes_alg = prefill_bytes(T, nqk, nv, D, D, n, 2, s0=False, sf=True)
    fl_dense, fl_tri = prefill_flops(T // n, n, nv, C, D)
    achieved_gbs = bytes_alg / (kern_ms / 1e3) / 1e9
    peak_key = "hbm_gbs"
    res = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded; workloads/)",
        "config": {"workload": PREFILL, "num_seqs": n, "seq_len": T // n, "nqk": nqk, "nv": nv,
                   "dk": D, "dv": D, "chunk": C, "io": "bf16", "state": "fp32",
                   "initial_state": "zeros", "l2": "inputs 1.63 GB > 126 MB L2; no flush",
                   "parallelism": "replicas x%d" % world},
        "gpu_launches": args.steps,
        "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": peaks[peak_key],
                     "unit": "GB/s", "frac": achieved_gbs / peaks[peak_key],
                     "traffic": recorded_traffic("chunk_fwd_tc", T),
                     "peak_source": peak_src, "alg_bytes_per_launch": bytes_alg,
                     "kernel_ms": kern_ms,
                     "tensor_tflops_tri": fl_tri / (kern_ms / 1e3) / 1e12,
                     "tensor_frac_tri": fl_tri / (kern_ms / 1e3) / 1e12 / peaks["bf16_tflops"],
                     "flops_tri_per_launch": fl_tri, "flops_dense_per_launch": fl_dense,
                     "roofline_time_ms": max(bytes_alg / (peaks["hbm_gbs"] * 1e9),
                                             fl_tri / (peaks["bf16_tflops"] * 1e12)) * 1e3},
        "clocks": clk.summary(),
    }
    # the same workload with the gate formed in-kernel from the raw projections
    if not args.no_gated:
        ga = {k_: host[k_].to(dev) for k_ in ("a", "b", "A_log", "dt_bias")}

        def gstep():
            gdn.chunk_fwd_gated(d["q"], d["k"], d["v"], ga["a"], ga["b"], ga["A_log"], ga["dt_bias"],
                                None, None, chunk_size=C, out=out, final_state=sf, num_seqs=n)

        for _ in range(args.warmup):
            gstep()
        torch.cuda.synchronize(dev)
        barrier(world)
        a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a_.record(stream)
        for _ in range(args.steps):
            gstep()
        b_.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
        g_ms = max_over_ranks(a_.elapsed_time(b_), world, dev) / args.steps
        g_bytes = bytes_alg + 2 * nv * 4  # a, b replace g, beta; plus A_log, dt_bias
        res["gated"] = {"value": T * world / (g_ms / 1e3), "unit": "tokens/s", "ms_per_step": g_ms,
                        "call": "gdn_chunk_fwd_gated", "gpu_launches": args.steps,
                        "roofline": {"bound": "hbm", "achieved": g_bytes / (g_ms / 1e3) / 1e9,
                                     "peak": peaks[peak_key], "unit": "GB/s",
                                     "frac": g_bytes / (g_ms / 1e3) / 1e9 / peaks[peak_key],
                                     "traffic": None, "peak_source": peak_src,
                                     "alg_bytes_per_launch": g_bytes}}
        del ga
    # the varlen workload: 32 packed sequences of U[100, 16384] tokens with
    # initial states (the configuration the parity tests sample by heads)
    if not args.no_varlen:
        wv = W.make_workload("varlen_bf16_nv32", seed=3 + rank, device=str(dev))
        nvs, Tv = wv["num_seqs"], wv["T"]
        ov = torch.empty(Tv, nv, D, dtype=torch.bfloat16, device=dev)
        sv = torch.empty_like(wv["initial_state"])

        def vstep():
            gdn.chunk_fwd(wv["q"], wv["k"], wv["v"], wv["g"], wv["beta"], wv["initial_state"], wv["cu_seqlens"],
                          chunk_size=C, out=ov, final_state=sv, kernel=args.kernel)

        v_ms = time_steps(vstep, args.warmup, max(3, args.steps // 4), stream, world, dev)
        vb = prefill_bytes(Tv, nqk, nv, D, D, nvs, 2, s0=True, sf=True)
        res["varlen"] = hbm_line(v_ms, vb, peaks, peak_src, value=Tv * world / (v_ms / 1e3), unit="tokens/s",
                                 workload="varlen_bf16_nv32", num_seqs=nvs, tokens=Tv,
                                 call="gdn_chunk_fwd (cu_seqlens, initial and final state)",
                                 gpu_launches=max(3, args.steps // 4))
        del wv, ov, sv
    # the two fp32 configurations (1 x 256 tokens, D 64, chunk 64; 4 x 4096
    # tokens, Nqk 4, Nv 8, D 128, chunk 128, initial states), each against the
    # HBM roofline and against the TF32 tensor peak measured here
    if not args.no_fp32:
        tf32 = measure_tf32_peak(dev)
        res["tf32_peak_tflops"] = tf32
        for name in ("tiny_f32_d64", "batch_f32_d128"):
            res[name] = run_fp32_config(name, args, world, rank, dev, stream, peaks, peak_src, tf32)
    # the same workload with the gated RMSNorm epilogue fused into the output
    # stores (gdn_chunk_fwd_ex), and the epilogue on its own (gdn_gated_rmsnorm)
    if not args.no_norm:
        z, nw = W.make_norm_inputs((T, nv, D), "bf16", seed=2 + rank, device=str(dev))

        def nstep():
            gdn.chunk_fwd_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], None, None, chunk_size=C, out=out,
                             final_state=sf, num_seqs=n, norm_z=z, norm_weight=nw, norm_eps=1e-6)

        n_ms = time_steps(nstep, args.warmup, args.steps, stream, world, dev)
        zb = T * nv * D * 2 + D * 4
        res["normed"] = hbm_line(n_ms, bytes_alg + zb, peaks, peak_src, value=T * world / (n_ms / 1e3),
                                 unit="tokens/s", call="gdn_chunk_fwd_ex (norm_z): chunk kernel + norm pass",
                                 gpu_launches=2 * args.steps)
        y = torch.empty_like(out)
        r_ms = time_steps(lambda: gdn.gated_rmsnorm(out, z, nw, 1e-6, out=y), args.warmup, args.steps,
                          stream, world, dev)
        res["gated_rmsnorm"] = hbm_line(r_ms, 3 * T * nv * D * 2 + D * 4, peaks, peak_src,
                                        value=T * world / (r_ms / 1e3), unit="tokens/s",
                                        call="gdn_gated_rmsnorm", rows=T * nv, dim=D,
                                        gpu_launches=args.steps)
        del z, y
    # causal conv1d + SiLU producing q, k, v from the packed projection, on the
    # same tokens (gdn_qkv_conv_fwd with the final conv_state)
    if not args.no_conv:
        cv = W.make_conv_inputs(T, nqk, nv, D, D, 4, "bf16", seed=2 + rank, device=str(dev))
        cq, ck, cvv = torch.empty_like(d["q"]), torch.empty_like(d["k"]), torch.empty_like(d["v"])
        cst = torch.empty(n, cv["C"], 4, dtype=torch.bfloat16, device=dev)

        def cstep():
            gdn.qkv_conv_fwd(cv["x"], cv["weight"], nqk, nv, D, D, bias=cv["bias"], num_seqs=n, state_out=cst)

        c_ms = time_steps(cstep, args.warmup, args.steps, stream, world, dev)
        cb = 2 * T * cv["C"] * 2 + cv["C"] * (4 + 1) * 4 + n * cv["C"] * 4 * 2
        res["conv"] = hbm_line(c_ms, cb, peaks, peak_src, value=T * world / (c_ms / 1e3), unit="tokens/s",
                               call="gdn_qkv_conv_fwd", channels=cv["C"], taps=4, gpu_launches=2 * args.steps)
        del cv, cq, ck, cvv, cst
    # e2e: the same call fed from pinned host buffers, copies inside the timed
    # region: every step copies its inputs in and its out and final state back.
    # Steps are pipelined the way a serving loop would run them: the inputs of
    # step i + 1 go in on one stream and the results of step i - 1 come back on
    # another while step i computes (two device buffer sets).
    if not args.no_e2e:
        keys = ("q", "k", "v", "g", "beta")
        hp = {k: host[k].pin_memory() for k in keys}
        ho = torch.empty(T, nv, D, dtype=torch.bfloat16).pin_memory()
        hs = torch.empty(n, nv, D, D, dtype=torch.float32).pin_memory()
        bi = sum(t.numel() * t.element_size() for t in hp.values())
        bo = ho.numel() * 2 + hs.numel() * 4
        din = [{k: torch.empty_like(d[k]) for k in keys} for _ in range(2)]
        dout = [(torch.empty_like(out), torch.empty_like(sf)) for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()
        e_steps = max(3, min(args.steps, 10))

        def run_pipelined(nsteps, t_first=None, t_last=None):
            e_in, e_cmp, e_out = [ev() for _ in range(nsteps)], [ev() for _ in range(nsteps)], [ev() for _ in range(nsteps)]
            if t_first is not None:
                t_first.record(s_in)
            for i in range(nsteps + 1):
                if i < nsteps:  # inputs of step i into set i % 2, once step i - 2 has used it
                    with torch.cuda.stream(s_in):
                        if i >= 2:
                            s_in.wait_event(e_cmp[i - 2])
                        for k in keys:
                            din[i % 2][k].copy_(hp[k], non_blocking=True)
                        e_in[i].record(s_in)
                if i >= 1:  # step i - 1: compute, then its results out
                    j = i - 1
                    stream.wait_event(e_in[j])
                    if j >= 2:
                        stream.wait_event(e_out[j - 2])  # its output set has been read back
                    x = din[j % 2]
                    gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None, None, chunk_size=C,
                                  out=dout[j % 2][0], final_state=dout[j % 2][1], num_seqs=n)
                    e_cmp[j].record(stream)
                    with torch.cuda.stream(s_out):
                        s_out.wait_event(e_cmp[j])
                        ho.copy_(dout[j % 2][0], non_blocking=True)
                        hs.copy_(dout[j % 2][1], non_blocking=True)
                        e_out[j].record(s_out)
            if t_last is not None:
                t_last.record(s_out)

        run_pipelined(2)
        torch.cuda.synchronize(dev)
        barrier(world)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        run_pipelined(e_steps, a, b)
        torch.cuda.synchronize(dev)
        barrier(world)
        e_ms = max_over_ranks(a.elapsed_time(b), world, dev)
        res["e2e"] = {"value": T * world * e_steps / (e_ms / 1e3), "unit": "tokens/s",
                      "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "steps": e_steps,
                      "pipelined": "inputs of step i+1 in and results of step i-1 out while step i computes"}
        del din, dout
    del d
    torch.cuda.empty_cache()
    if not args.no_decode:
        res["decode"] = run_decode(args, world, rank, dev, stream, peaks, peak_src)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        t_sample = args.cpu_sample_tokens or T // n
        tok, dt = time_oracle(host, t_sample)
        res["cpu_baseline"] = {"value": tok / dt, "unit": "tokens/s", "cores": oracle.num_threads(),
                               "kind": "oracle",
                               "sample": "fp64 token loop over the first %d tokens of each of the %d "
                                         "sequences, all %d v-heads (%.1f s wall)"
                                         % (t_sample, n, nv, dt)}
    return res


def measure_tf32_peak(dev, n=8192, reps=10):
    """Dense fp32-in / fp32-out matmul throughput with TF32 tensor cores (torch, best of ``reps``, CUDA
    events): the denominator of the fp32 configurations' tensor roofline (TFLOP/s)."""
    import torch
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = True
    try:
        a = torch.randn(n, n, device=dev)
        b = torch.randn(n, n, device=dev)
        c = torch.empty(n, n, device=dev)
        best = float("inf")
        for _ in range(3):
            torch.matmul(a, b, out=c)
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch.matmul(a, b, out=c)
            e1.record()
            torch.cuda.synchronize(dev)
            best = min(best, e0.elapsed_time(e1))
        del a, b, c
        return 2.0 * n ** 3 / (best / 1e3) / 1e12
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev


def run_fp32_config(name, args, world, rank, dev, stream, peaks, peak_src, tf32_tflops):
    """One fp32 configuration: device time per gdn_chunk_fwd (CUDA events), tokens/s and both roofline terms."""
    import torch

    import gated_deltanet_chunk_b200 as gdn
    import workloads as W
    wl = W.WORKLOADS[name]
    host = W.make_workload(name, seed=W.WORKLOAD_ORDER.index(name) + 10 * rank)
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in host.items()}
    n, T = wl.num_seqs, host["T"]
    out = torch.empty(T, wl.nv, wl.d, dtype=torch.float32, device=dev)
    sf = torch.empty(n, wl.nv, wl.d, wl.d, dtype=torch.float32, device=dev)

    def step():
        gdn.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["initial_state"], d["cu_seqlens"],
                      chunk_size=wl.chunk, out=out, final_state=sf, kernel=args.kernel)

    steps = max(10, args.steps)
    ms = time_steps(step, args.warmup, steps, stream, world, dev)
    byts = prefill_bytes(T, wl.nqk, wl.nv, wl.d, wl.d, n, 4, s0=wl.init_state, sf=True)
    _, fl_tri = prefill_flops(T // n, n, wl.nv, wl.chunk, wl.d)
    t_bytes = byts / (peaks["hbm_gbs"] * 1e9)
    t_flops = fl_tri / (tf32_tflops * 1e12)
    gbs = byts / (ms / 1e3) / 1e9
    return {"value": T * world / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms, "workload": name,
            "num_seqs": n, "seq_len": T // n, "nqk": wl.nqk, "nv": wl.nv, "d": wl.d, "chunk": wl.chunk,
            "io": "f32", "initial_state": "random" if wl.init_state else "zeros",
            "call": "gdn_chunk_fwd", "gpu_launches": steps,
            "l2": "inputs below L2 size: repeated launches re-read them from L2 (an upper bound on speed)",
            "roofline": {"bound": "hbm" if t_bytes >= t_flops else "tensor",
                         "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": max(t_bytes, t_flops) / (ms / 1e3), "traffic": None, "peak_source": peak_src,
                         "alg_bytes_per_launch": byts, "flops_tri_per_launch": fl_tri,
                         "tf32_peak_tflops_measured": tf32_tflops,
                         "roofline_time_ms": max(t_bytes, t_flops) * 1e3}}


def run_decode(args, world, rank, dev, stream, peaks, peak_src):
    import torch

    import gated_deltanet_chunk_b200 as gdn
    import workloads as W
    wl = W.WORKLOADS[DECODE]
    steps = args.decode_steps or wl.steps
    d = W.make_decode(num_seqs=wl.num_seqs, steps=steps, nqk=wl.nqk, nv=wl.nv, d=wl.d, io=wl.io,
                      seed=4 + rank, device=str(dev))
    state = d["initial_state"]
    out = torch.empty(wl.num_seqs, wl.nv, wl.d, dtype=torch.bfloat16, device=dev)

    def run(n_steps):
        for t in range(n_steps):
            gdn.recurrent_step(d["q"][t], d["k"][t], d["v"][t], d["g"][t], d["beta"][t], state, out=out)

    run(min(steps, 32))
    torch.cuda.synchronize(dev)
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    run(steps)
    b.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    ms = max_over_ranks(a.elapsed_time(b), world, dev)
    per_step_ms = ms / steps
    byts = decode_bytes(wl.num_seqs, wl.nqk, wl.nv, wl.d, wl.d, 2)
    gbs = byts / (per_step_ms / 1e3) / 1e9
    res = {"value": wl.num_seqs * steps * world / (ms / 1e3), "unit": "tokens/s",
           "workload": DECODE, "steps": steps, "ms_per_step": per_step_ms, "gpu_launches": steps,
           "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": gbs / peaks["hbm_gbs"], "traffic": recorded_traffic("recurrent_step", wl.num_seqs),
                        "peak_source": peak_src,
                        "alg_bytes_per_launch": byts}}
    if not args.no_slots:
        # the same decode with the states in a 2x larger pool, rows chosen by a permutation
        P = 2 * wl.num_seqs
        gen = torch.Generator(device="cpu").manual_seed(7)
        ids = torch.randperm(P, generator=gen)[: wl.num_seqs].to(torch.int32).to(dev)
        pool = torch.zeros(P, wl.nv, wl.d, wl.d, dtype=torch.float32, device=dev)
        pool[ids.long()] = state

        def run_slots(n_steps):
            for t in range(n_steps):
                gdn.recurrent_step_slots(d["q"][t], d["k"][t], d["v"][t], d["g"][t], d["beta"][t],
                                         pool, ids, out=out)

        run_slots(min(steps, 32))
        torch.cuda.synchronize(dev)
        barrier(world)
        a.record(stream)
        run_slots(steps)
        b.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
        sms = max_over_ranks(a.elapsed_time(b), world, dev) / steps
        sb = byts + wl.num_seqs * 4
        res["slots"] = {"ms_per_step": sms, "value": wl.num_seqs * world / (sms / 1e3), "unit": "tokens/s",
                        "call": "gdn_recurrent_step_slots", "pool_rows": P, "gpu_launches": steps,
                        "roofline": {"bound": "hbm", "achieved": sb / (sms / 1e3) / 1e9,
                                     "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                     "frac": sb / (sms / 1e3) / 1e9 / peaks["hbm_gbs"], "traffic": None,
                                     "peak_source": peak_src, "alg_bytes_per_launch": sb}}
        del pool
    if not args.no_gated:
        def run_gated(n_steps):
            for t in range(n_steps):
                gdn.recurrent_step_gated(d["q"][t], d["k"][t], d["v"][t], d["a"][t], d["b"][t],
                                         d["A_log"], d["dt_bias"], state, out=out)

        run_gated(min(steps, 32))
        torch.cuda.synchronize(dev)
        barrier(world)
        a.record(stream)
        run_gated(steps)
        b.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
        gms = max_over_ranks(a.elapsed_time(b), world, dev) / steps
        gb = byts + 2 * wl.nv * 4
        res["gated"] = {"ms_per_step": gms, "value": wl.num_seqs * world / (gms / 1e3), "unit": "tokens/s",
                        "call": "gdn_recurrent_step_gated", "gpu_launches": steps,
                        "roofline": {"bound": "hbm", "achieved": gb / (gms / 1e3) / 1e9,
                                     "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                     "frac": gb / (gms / 1e3) / 1e9 / peaks["hbm_gbs"], "traffic": None,
                                     "peak_source": peak_src, "alg_bytes_per_launch": gb}}
    if not args.no_conv:
        # the conv update that produces each step's q, k, v (in-place conv_state), then the step
        cv = W.make_conv_inputs(wl.num_seqs, wl.nqk, wl.nv, wl.d, wl.d, 4, "bf16", seed=4 + rank,
                                num_states=wl.num_seqs, device=str(dev))
        qo, ko, vo = (torch.empty_like(d["q"][0]), torch.empty_like(d["k"][0]), torch.empty_like(d["v"][0]))

        def conv_only():
            gdn.qkv_conv_update(cv["x"], cv["weight"], cv["state"], wl.nqk, wl.nv, wl.d, wl.d, bias=cv["bias"],
                                out=(qo, ko, vo))

        it = [0]

        def conv_then_step():
            conv_only()
            t = it[0] % steps
            it[0] += 1
            gdn.recurrent_step(qo, ko, vo, d["g"][t], d["beta"][t], state, out=out)

        # the update alone is a few microseconds: time it through a CUDA graph (no host launch cost per
        # call) that cycles over 8 input / state / output sets (200 MB > L2), so every call reads HBM
        sets = [W.make_conv_inputs(wl.num_seqs, wl.nqk, wl.nv, wl.d, wl.d, 4, "bf16", seed=40 + 8 * rank + i,
                                   num_states=wl.num_seqs, device=str(dev)) for i in range(8)]
        outs = [(torch.empty_like(qo), torch.empty_like(ko), torch.empty_like(vo)) for _ in range(8)]
        calls = [(lambda c=c, o=o: gdn.qkv_conv_update(c["x"], c["weight"], c["state"], wl.nqk, wl.nv, wl.d,
                                                       wl.d, bias=c["bias"], out=o))
                 for c, o in zip(sets, outs)] * 4
        replays = max(1, steps // len(calls))
        cu_ms = time_graph(calls, replays, 3, stream, world, dev)
        del sets, outs, calls
        cs_ms = time_steps(conv_then_step, 32, steps, stream, world, dev)
        C = cv["C"]
        ub = wl.num_seqs * C * (2 + 2 + 2 * 4 * 2) + C * 5 * 4
        res["conv_update"] = hbm_line(cu_ms, ub, peaks, peak_src, call="gdn_qkv_conv_update", channels=C,
                                      gpu_launches=replays * 32, timing="CUDA graph of 32 calls over 8 sets "
                                      "(200 MB > L2), replayed")
        res["conv_then_step"] = hbm_line(cs_ms, byts + ub, peaks, peak_src,
                                         value=wl.num_seqs * world / (cs_ms / 1e3), unit="tokens/s",
                                         call="gdn_qkv_conv_update + gdn_recurrent_step", gpu_launches=2 * steps)
        it[0] = 0

        def conv_fused():
            t = it[0] % steps
            it[0] += 1
            gdn.recurrent_step_ex(None, None, None, d["g"][t], d["beta"][t], state, out=out, conv_x=cv["x"],
                                  conv_state=cv["state"], conv_weight=cv["weight"], conv_bias=cv["bias"],
                                  shapes=(wl.nqk, wl.nv, wl.d, wl.d))

        cf_ms = time_steps(conv_fused, 32, steps, stream, world, dev)
        # the step's bytes without q, k, v, plus the projection, the conv windows and taps
        qkv = wl.num_seqs * (2 * wl.nqk + wl.nv) * wl.d * 2
        fb = byts - qkv + wl.num_seqs * C * (2 + 2 * 4 * 2) + C * 5 * 4
        res["conv_fused"] = hbm_line(cf_ms, fb, peaks, peak_src, value=wl.num_seqs * world / (cf_ms / 1e3),
                                     unit="tokens/s", call="gdn_recurrent_step_ex (conv_x)", gpu_launches=steps)
        del cv
    if not args.no_norm:
        z, nw = W.make_norm_inputs((steps, wl.num_seqs, wl.nv, wl.d), "bf16", seed=4 + rank, device=str(dev))
        it = [0]

        def run_normed():
            t = it[0] % steps
            it[0] += 1
            gdn.recurrent_step_ex(d["q"][t], d["k"][t], d["v"][t], d["g"][t], d["beta"][t], state, out=out,
                                  norm_z=z[t], norm_weight=nw, norm_eps=1e-6)

        nms = time_steps(run_normed, min(steps, 32), steps, stream, world, dev)
        nb = byts + wl.num_seqs * wl.nv * wl.d * 2 + wl.d * 4
        res["normed"] = hbm_line(nms, nb, peaks, peak_src, value=wl.num_seqs * world / (nms / 1e3),
                                 unit="tokens/s", call="gdn_recurrent_step_ex (norm_z)", gpu_launches=steps)
        del z
    return res


def run_reference(args, world, rank):
    """The fp64 CPU oracle as the reference arm, on a bounded sample of the same workload."""
    import oracle
    import workloads as W
    if rank != 0:
        return None
    wl = W.WORKLOADS[PREFILL]
    host = W.make_workload(PREFILL, seed=2)
    for _ in range(args.warmup):
        time_oracle(host, args.ref_sample_tokens)
    tot_tok, tot_s = 0, 0.0
    for _ in range(args.steps):
        tok, dt = time_oracle(host, args.ref_sample_tokens)
        tot_tok += tok
        tot_s += dt
    value = tot_tok / tot_s
    sample = ("fp64 token loop over the first %d tokens of each of the %d sequences, all %d v-heads, "
              "per step" % (args.ref_sample_tokens, wl.num_seqs, wl.nv))
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_s / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded; workloads/)",
            "config": {"workload": PREFILL, "num_seqs": wl.num_seqs, "seq_len": wl.seq_len,
                       "nqk": wl.nqk, "nv": wl.nv, "dk": wl.d, "dv": wl.d, "chunk": wl.chunk,
                       "io": "bf16", "state": "fp32", "initial_state": "zeros",
                       "l2": "host run (no GPU cache involved)", "parallelism": "host cores",
                       "sample_tokens_per_seq": args.ref_sample_tokens},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="time only the decode workload")
    ap.add_argument("--seq-len", type=int, default=0,
                    help="override the prefill sequence length (profiling of smaller cases)")
    ap.add_argument("--decode-steps", type=int, default=0,
                    help="override the number of decode steps (profiling of smaller cases)")
    ap.add_argument("--kernel", choices=["auto", "simt", "tc"], default="auto",
                    help="prefill kernel selection passed to gdn_chunk_fwd (default: auto)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-gated", action="store_true", help="skip the fused-gate prefill and decode lines")
    ap.add_argument("--no-slots", action="store_true", help="skip the slot-indexed decode line")
    ap.add_argument("--no-varlen", action="store_true", help="skip the varlen prefill line")
    ap.add_argument("--no-fp32", action="store_true",
                    help="skip the lines of the two fp32 configurations (and the TF32 peak)")
    ap.add_argument("--no-conv", action="store_true",
                    help="skip the causal-conv lines (prefill conv, decode conv update)")
    ap.add_argument("--no-norm", action="store_true",
                    help="skip the gated-RMSNorm lines (fused prefill and decode, standalone epilogue)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-tokens", type=int, default=0,
                    help="oracle sample per sequence for cpu_baseline (default: the whole workload)")
    ap.add_argument("--ref-sample-tokens", type=int, default=512)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        res = run_reference(args, world, rank)
    else:
        res = run_ours(args, world, rank, local)
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)
    if world > 1 and args.impl == "ours":
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

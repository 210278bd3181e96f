"""Benchmark of the SVDQuant W4A4 linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference]

One step = the whole hot path over one batch: svdq_quantize_act (smoothing,
INT4 codes, scales, down-projection) then svdq_linear (W4A4 tensor-core
product, rescale, up-projection, bias) for the FLUX-like joint-attention QKV
projection (M=4608, K=3072, N=9216, r=32) on seeded synthetic inputs.
Inputs are resident in HBM when the timed region starts; L2 is flushed
(a 256 MiB write) before every timed step, outside the step's CUDA events.

Metric: effective TOPS = 2 M N K / step time (the main product's op count,
as the workload defines it), summed over ranks.  Under torchrun each rank
runs its own replica of the workload (no exchange: token rows are
independent), so scaling is weak.

--impl reference times the CPU oracle (NumPy fp64) on a bounded sample of
rows of the same workload on the host cores and prints the same line with
"impl": "reference".
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "svdq_linear effective TOPS (2MNK/s) at FLUX-like shapes; % int8 roofline"
# minimum span of the clock record around the timed steps (seconds)
CLOCK_WINDOW_S = 0.6

# DRAM bytes (read + write) of one svdq_linear launch on this workload, from a
# one-kernel, one-launch ncu capture (dram__bytes_read.sum +
# dram__bytes_write.sum), valid only for the kernel sources it was taken on
# (SHA-1 over the files below); null otherwise.
LINEAR_SOURCES = ("w4a4_quantized_gemm_smooth_b200/csrc/linear_ws.cu",
                  "w4a4_quantized_gemm_smooth_b200/csrc/gemm_common.cuh",
                  "w4a4_quantized_gemm_smooth_b200/csrc/ptx.cuh",
                  "w4a4_quantized_gemm_smooth_b200/csrc/svdq_internal.h")
LINEAR_TRAFFIC = {"sources_sha1": "71e0331c3d32f46caa1e4d41ad4ec2feb02263b2",
                  "workload": "flux_qkv", "bytes": 26641408 + 33591808}


def _linear_traffic(workload):
    import hashlib
    h = hashlib.sha1()
    try:
        for f in LINEAR_SOURCES:
            with open(os.path.join(ROOT, f), "rb") as fh:
                h.update(fh.read())
    except OSError:
        return None
    if h.hexdigest() != LINEAR_TRAFFIC["sources_sha1"] or workload != LINEAR_TRAFFIC["workload"]:
        return None
    return LINEAR_TRAFFIC["bytes"]


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return (float(pk["bf16_tflops"]), float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])),
                float(pk["hbm_gbs"]), "measured")
    except Exception:
        return 1590.0, 1400.0, 6650.0, "fallback"


def _workload(name):
    specs = dict(synth.WORKLOADS)
    specs.update({p.name: p for p in synth.pixart_points()})
    if name not in specs:
        raise SystemExit(f"unknown workload {name}; choose from {sorted(specs)}")
    return specs[name]


def _config(spec, ws):
    """The workload description shared by both arms' JSON lines."""
    r = spec.rank + spec.lora_rank
    return {"workload": f"{spec.name} M={spec.M} K={spec.K} N={spec.N} r={r}", "M": spec.M,
            "K": spec.K, "N": spec.N, "rank": r, "group": 64, "parallelism": f"replicas x{ws}",
            "l2": "flushed (256 MiB write) before every step"}


def max_over_ranks(values, dist=None, device="cpu"):
    """Element-wise max of per-rank timings over all ranks (every rank gets
    the result).  `dist` is torch.distributed when a process group is up."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist is not None and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_tops(ops_per_rank, world_size, seconds):
    """Whole-job throughput: every rank's work over the slowest rank's time."""
    return world_size * ops_per_rank / seconds / 1e12


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        # raw samples: $SVDQ_CLOCKS_DIR if set, else the system temp directory
        import tempfile
        d = os.environ.get("SVDQ_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(d, f"svdq_clocks_gpu{gpu_index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def mark(self, which):
        """Wall-clock bounds of the timed region (samples outside are dropped)."""
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        import datetime
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    rows.append((ts, float(parts[2]), float(parts[3]),
                                 {nm for nm, v in zip(names, parts[6:10]) if v.lower() == "active"}))
                except ValueError:
                    continue
        t0, t1 = getattr(self, "t0", None), getattr(self, "t1", None)
        inside = [r for r in rows if t0 is not None and t1 is not None and t0 <= r[0] <= t1]
        use = inside or rows
        if not use:
            return None
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": max(r[2] for r in use),
                "samples": len(use), "in_timed_region": bool(inside),
                "reasons": sorted(set().union(*(r[3] for r in use)))}


# --------------------------------------------------------------------------
# CPU oracle timing (the reported baseline and the reference arm)
# --------------------------------------------------------------------------
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def cpu_oracle_setup(spec, rows=512, cols=2048):
    """Oracle pack of a column sample of the layer (cols output channels, all
    K inputs, same rank), plus a row sample of X.  Untimed."""
    import oracle
    L = synth.make_layer(spec)
    Xs = L.X[:rows]
    a = oracle.calib_absmax(oracle.bf16_bits_to_f64(L.X))
    p = oracle.pack_weights(L.W[:cols], a, spec.rank, bias_bits=L.b[:cols], svd="leading")
    return dict(X=Xs, p=p, rows=rows, cols=cols, K=spec.K,
                sample=f"{rows} rows x {cols} output channels of {spec.name} "
                       f"(K={spec.K}, r={spec.rank}); oracle = NumPy fp64")


def cpu_oracle_step(st):
    import oracle
    p = st["p"]
    t0 = time.perf_counter()
    xc, s_x, Z, _ = oracle.quantize_act(st["X"], p["inv_lambda"], p["L1b"])
    oracle.linear(xc, s_x, Z, p["wcodes"], p["s_w"], p["L2b"], p["bias"])
    return time.perf_counter() - t0


def cpu_baseline(spec, reps=3):
    """The oracle on the host's cores (BLAS threads as configured), and the
    same sample on one thread."""
    st = cpu_oracle_setup(spec)
    cpu_oracle_step(st)
    ts = [cpu_oracle_step(st) for _ in range(reps)]
    t = statistics.median(ts)
    ops = 2.0 * st["rows"] * st["cols"] * st["K"]
    out = {"value": ops / t / 1e12, "unit": "TOPS", "cores": _blas_threads(),
           "kind": "oracle", "sample": st["sample"], "seconds_per_sample": t}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1, user_api="blas"):
            t1 = cpu_oracle_step(st)
        out["one_thread"] = {"value": ops / t1 / 1e12, "unit": "TOPS", "cores": 1,
                             "seconds_per_sample": t1}
    except Exception:
        pass
    return out


def run_reference(args, spec):
    ws, rank, _ = _dist()
    if rank != 0:
        return
    st = cpu_oracle_setup(spec)
    for _ in range(args.warmup):
        cpu_oracle_step(st)
    ts = [cpu_oracle_step(st) for _ in range(args.steps)]
    ops = 2.0 * st["rows"] * st["cols"] * st["K"]
    v = ops * len(ts) / sum(ts) / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "TOPS", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(ts) / len(ts),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": _config(spec, ws),
        "cpu_baseline": {"value": v, "unit": "TOPS", "cores": _blas_threads(),
                         "kind": "oracle", "sample": st["sample"]},
        "e2e": {"value": v, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------
def _to_dev(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _time_steps(fn, steps, flush, stream, per_step=False):
    """Per-step CUDA events on the launching stream; `flush` (a buffer larger
    than L2, or None for an L2-warm run) is written before every step,
    outside the events.  Returns per-phase totals in ms, or per-step phase
    times when per_step."""
    import torch
    evs = []
    for i in range(steps):
        if flush is not None:
            flush.fill_(i & 0xFF)
        marks = [torch.cuda.Event(enable_timing=True) for _ in range(fn.n_phases + 1)]
        fn(marks, stream)
        evs.append(marks)
    torch.cuda.synchronize()
    rows = [[m[j].elapsed_time(m[j + 1]) for j in range(fn.n_phases)] for m in evs]
    if per_step:
        return rows
    return [sum(r[j] for r in rows) for j in range(fn.n_phases)]   # ms


def _dist_stats(xs):
    """Median, 10th and 90th percentile (µs) of per-step times given in ms."""
    v = np.asarray(xs, dtype=np.float64) * 1e3
    return {"median_us": float(np.median(v)), "p10_us": float(np.percentile(v, 10)),
            "p90_us": float(np.percentile(v, 90))}


class _Step:
    """quantize_act then linear, with an event between the two kernels.  With
    a workspace the product is svdq_linear_splitk at the automatic split
    (batches whose output tiles cannot fill the GPU)."""
    n_phases = 2

    def __init__(self, S, w, X, bufs, epi, workspace=None):
        self.S, self.w, self.X, self.epi = S, w, X, epi
        self.xq, self.s_x, self.Z, self.Y = bufs
        self.ws = workspace

    def __call__(self, marks, stream):
        S = self.S
        marks[0].record(stream)
        S.svdq_quantize_act(self.w, self.X, self.xq, self.s_x, self.Z, stream)
        marks[1].record(stream)
        if self.ws is None:
            S.svdq_linear(self.w, self.xq, self.s_x, self.Z, self.Y, self.epi, stream)
        else:
            S.svdq_linear_splitk(self.w, self.xq, self.s_x, self.Z, self.Y, self.ws, 0, self.epi,
                                 stream)
        marks[2].record(stream)


class _StepW8(_Step):
    """The W8A8 comparator: quantize_act_w8a8 then linear_w8a8."""

    def __call__(self, marks, stream):
        S = self.S
        marks[0].record(stream)
        S.svdq_quantize_act_w8a8(self.w, self.X, self.xq, self.s_x, self.Z, stream)
        marks[1].record(stream)
        S.svdq_linear_w8a8(self.w, self.xq, self.s_x, self.Z, self.Y, self.epi, stream)
        marks[2].record(stream)


# Rank of the W8A8 comparator: the eight-bit setting's rank (review section 8).
W8A8_RANK = 16


def _time_w8a8(S, spec, L, a, X, flush, stream, steps, int8_peak):
    """The same workload through the W8A8 comparator (int8 operands, one
    scale per token / output channel, rank 16): per-kernel times and the
    GEMM's fraction of the int8 peak."""
    w8 = S.svdq_pack_weights_w8a8(L.W, a, W8A8_RANK, bias_bits=L.b)
    lin8 = S.W8A8Linear(w8)
    step8 = _StepW8(S, w8, X, lin8.buffers(spec.M), S.EPI_NONE)
    _time_steps(step8, 3, flush, stream)
    t_act, t_lin = (v / steps for v in _time_steps(step8, steps, flush, stream))
    S.svdq_get_device_error(w8)
    w8.free()
    ops = 2.0 * spec.M * spec.N * spec.K
    tops = ops / (t_lin * 1e-3) / 1e12
    return {"rank": W8A8_RANK, "ms_per_step": t_act + t_lin, "act_ms": t_act,
            "linear_ms": t_lin, "layer_tops": ops / ((t_act + t_lin) * 1e-3) / 1e12,
            "linear_tops": tops, "linear_frac_int8": tops / int8_peak}


class _StepF4(_Step):
    """The NVFP4 variant: quantize_act_nvfp4 then linear_nvfp4."""

    def __init__(self, S, w, X, bufs, epi):
        self.S, self.w, self.X, self.epi = S, w, X, epi
        self.xq, self.sfa, self.s_x, self.Z, self.Y = bufs

    def __call__(self, marks, stream):
        S = self.S
        marks[0].record(stream)
        S.svdq_quantize_act_nvfp4(self.w, self.X, self.xq, self.sfa, self.s_x, self.Z, stream)
        marks[1].record(stream)
        S.svdq_linear_nvfp4(self.w, self.xq, self.sfa, self.s_x, self.Z, self.Y, self.epi, stream)
        marks[2].record(stream)


def _time_nvfp4(S, spec, L, a, X, flush, stream, steps, fp4_peak):
    """The same workload through the NVFP4 variant (same rank): per-kernel
    times and the GEMM's fraction of the FP4 peak."""
    w4 = S.svdq_pack_weights_nvfp4(L.W, a, spec.rank, bias_bits=L.b)
    lin = S.NVFP4Linear(w4)
    step = _StepF4(S, w4, X, lin.buffers(spec.M), S.EPI_NONE)
    _time_steps(step, 3, flush, stream)
    t_act, t_lin = (v / steps for v in _time_steps(step, steps, flush, stream))
    S.svdq_get_device_error(w4)
    w4.free()
    ops = 2.0 * spec.M * spec.N * spec.K
    tops = ops / (t_lin * 1e-3) / 1e12
    return {"rank": spec.rank, "ms_per_step": t_act + t_lin, "act_ms": t_act, "linear_ms": t_lin,
            "layer_tops": ops / ((t_act + t_lin) * 1e-3) / 1e12, "linear_tflops": tops,
            "linear_frac_fp4": tops / fp4_peak,
            "peak_source": "measured bf16 burst x 4 (fp4/bf16 nominal ratio)"}


class _StepPair:
    """The feed-forward pair fc2(GELU(fc1(X))): fused (fc1's epilogue emits
    fc2's activation side) or unfused (fc1 stores H, fc2's activation pass
    reads it), with an event between the kernels."""

    def __init__(self, S, mlp, X, fused):
        self.S, self.mlp, self.X, self.fused = S, mlp, X, fused
        self.n_phases = 3 if fused else 4

    def __call__(self, marks, stream):
        S, m = self.S, self.mlp
        a, b = m.fc1, m.fc2
        marks[0].record(stream)
        S.svdq_quantize_act(a.w, self.X, a.xq, a.s_x, a.Z, stream)
        marks[1].record(stream)
        if self.fused:
            S.svdq_linear_quantize_next(a.w, b.w, a.xq, a.s_x, a.Z, b.xq, b.s_x, b.Z, m.ws,
                                        S.EPI_GELU, stream)
        else:
            S.svdq_linear(a.w, a.xq, a.s_x, a.Z, m.H, S.EPI_GELU, stream)
            marks[2].record(stream)
            S.svdq_quantize_act(b.w, m.H, b.xq, b.s_x, b.Z, stream)
        marks[-2].record(stream)
        S.svdq_linear(b.w, b.xq, b.s_x, b.Z, b.Y, S.EPI_NONE, stream)
        marks[-1].record(stream)


def _time_mlp_pair(S, flush, stream, steps):
    """The FLUX feed-forward pair (fc1 3072 -> 12288, GELU, fc2 12288 -> 3072,
    rank 32, 4608 tokens) with and without the cross-layer fusion.  fc2 is
    calibrated on fc1's output."""
    import torch
    s1, s2 = synth.WORKLOADS["flux_mlp_fc1"], synth.WORKLOADS["flux_mlp_fc2"]
    L1, L2 = synth.make_layer(s1), synth.make_layer(s2)
    w1 = S.svdq_pack_weights(L1.W, S.svdq_calib_absmax(L1.X), s1.rank, bias_bits=L1.b)
    X = _to_dev(L1.X)
    H = S.SVDQLinear(w1, S.EPI_GELU)(X)
    torch.cuda.synchronize()
    Hb = H.cpu().view(torch.int16).numpy().view(np.uint16)
    w2 = S.svdq_pack_weights(L2.W, S.svdq_calib_absmax(Hb), s2.rank, bias_bits=L2.b)
    mlp = S.SVDQMLP(w1, w2)
    mlp.buffers(s1.M)
    out = {"workload": "flux_mlp_fc1 -> GELU -> flux_mlp_fc2", "M": s1.M,
           "dims": [s1.K, s1.N, s2.N], "rank": [s1.rank, s2.rank]}
    for fused in (False, True):
        st = _StepPair(S, mlp, X, fused)
        _time_steps(st, 3, flush, stream)
        ph = [v / steps for v in _time_steps(st, steps, flush, stream)]
        key = "fused" if fused else "unfused"
        out[key + "_ms"] = sum(ph)
        out[key + "_phases_ms"] = ph
    S.svdq_get_device_error(w1)
    S.svdq_get_device_error(w2)
    ops = 2.0 * s1.M * (s1.K * s1.N + s2.K * s2.N)
    out["phases"] = {"unfused": ["act fc1", "fc1 -> H", "act fc2", "fc2"],
                     "fused": ["act fc1", "fc1 -> fc2 codes, scales, Z", "fc2"]}
    out["pair_tops_unfused"] = ops / (out["unfused_ms"] * 1e-3) / 1e12
    out["pair_tops_fused"] = ops / (out["fused_ms"] * 1e-3) / 1e12
    out["saving"] = 1.0 - out["fused_ms"] / out["unfused_ms"]
    w1.free()
    w2.free()
    return out


def _time_e2e(S, w, Xh, Yh, Xd, bufs, epi, steps, workspace=None):
    """Public API end to end, as a serving loop: every step copies its X from
    pinned host memory to the device, runs svdq_quantize_act and svdq_linear,
    and copies its Y back to pinned host memory.  Uploads, compute and
    downloads run on three streams with two device buffer sets, so step k's
    compute overlaps step k+1's upload and step k-1's download; all copies of
    all steps lie inside the timed region (first upload to last download)."""
    import torch
    up, comp, down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    nb = len(Xd)
    ev_up = [torch.cuda.Event() for _ in range(nb)]     # X of buffer set b uploaded
    ev_cp = [torch.cuda.Event() for _ in range(nb)]     # Y of set b computed
    ev_dn = [torch.cuda.Event() for _ in range(nb)]     # Y of set b downloaded
    ev_xr = [torch.cuda.Event() for _ in range(nb)]     # X of set b consumed
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(up)
    for k in range(steps):
        b = k % nb
        xq, s_x, Z, Y = bufs[b]
        if k >= nb:
            up.wait_event(ev_xr[b])
        with torch.cuda.stream(up):
            Xd[b].copy_(Xh[k % len(Xh)], non_blocking=True)
        ev_up[b].record(up)
        comp.wait_event(ev_up[b])
        if k >= nb:
            comp.wait_event(ev_dn[b])          # Y of set b downloaded before it is rewritten
        S.svdq_quantize_act(w, Xd[b], xq, s_x, Z, comp)
        ev_xr[b].record(comp)
        if workspace is None:
            S.svdq_linear(w, xq, s_x, Z, Y, epi, comp)
        else:       # one compute stream: the split-K workspace is reused in order
            S.svdq_linear_splitk(w, xq, s_x, Z, Y, workspace, 0, epi, comp)
        ev_cp[b].record(comp)
        down.wait_event(ev_cp[b])
        with torch.cuda.stream(down):
            Yh[k % len(Yh)].copy_(Y, non_blocking=True)
        ev_dn[b].record(down)
    t1.record(down)
    torch.cuda.synchronize()
    return t0.elapsed_time(t1)   # ms


def _time_e2e_host(S, w, Xh, Yh, epi, steps):
    """Public API end to end through the C-ABI call with host buffers
    (svdq_linear_host), as a serving loop: every step is one call that
    copies its X from pinned host memory, runs both kernels and copies its Y
    back to pinned host memory.  Steps rotate over len(Yh) streams, each with
    its own device workspace and host Y, so one step's copies overlap the
    other steps' copies and kernels; all copies of all steps lie inside the
    timed region."""
    import torch
    M = Xh[0].shape[0]
    n = len(Yh)
    streams = [torch.cuda.Stream() for _ in range(n)]
    wsp = [torch.empty(S.svdq_linear_host_workspace(w, M), dtype=torch.uint8, device="cuda")
           for _ in range(n)]
    cur = torch.cuda.current_stream()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    done = [torch.cuda.Event() for _ in range(n)]
    torch.cuda.synchronize()
    t0.record(cur)
    for st in streams:
        st.wait_event(t0)
    for k in range(steps):
        i = k % n
        S.svdq_linear_host(w, Xh[k % len(Xh)], Yh[i], wsp[i], epi, streams[i])
    for i in range(n):
        done[i].record(streams[i])
        cur.wait_event(done[i])
    t1.record(cur)
    torch.cuda.synchronize()
    return t0.elapsed_time(t1)   # ms


def _act_bytes(M, K, r):
    """Algorithmic HBM bytes of one svdq_quantize_act launch: read X (bf16),
    write codes (K/2 per token), scales (4 per token-group) and Z (bf16),
    read inv_lambda and L1 once."""
    return 2 * M * K + M * K // 2 + 4 * M * (K // 64) + 2 * M * r + 4 * K + 2 * K * r


def run_ours(args, spec):
    ws, rank, local = _dist()
    if ws > 1 and "OMP_NUM_THREADS" not in os.environ:
        # one process per GPU share the host: split its cores for the host packs
        lws = int(os.environ.get("LOCAL_WORLD_SIZE", ws))
        os.environ["OMP_NUM_THREADS"] = str(max(1, (os.cpu_count() or 1) // max(lws, 1)))
    import torch
    import w4a4_quantized_gemm_smooth_b200 as S

    torch.cuda.set_device(local)
    dist = None
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    M, K, N, r = spec.M, spec.K, spec.N, spec.rank + spec.lora_rank
    L = synth.make_layer(spec)
    a = S.svdq_calib_absmax(L.X)
    w = S.svdq_pack_weights(L.W, a, spec.rank, bias_bits=L.b, lora_A_bits=L.A,
                            lora_B_bits=L.B)
    w0 = S.svdq_pack_weights(L.W, a, 0, bias_bits=L.b)        # same layer without the branch
    X = _to_dev(L.X)
    lin, lin0 = S.SVDQLinear(w), S.SVDQLinear(w0)
    bufs, bufs0 = lin.buffers(M), lin0.buffers(M)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    # split-K at the automatic split when the output tiles cannot fill the
    # GPU (the library picks the split; 1 means the plain kernel)
    splitk = S.svdq_linear_splitk_workspace(w, M, 0) > S.svdq_linear_splitk_workspace(w, M, 1)
    wsb = wsb0 = None
    if splitk:
        wsb = torch.empty(S.svdq_linear_splitk_workspace(w, M, 0), dtype=torch.uint8, device="cuda")
        wsb0 = torch.empty(S.svdq_linear_splitk_workspace(w0, M, 0), dtype=torch.uint8,
                           device="cuda")
    step = _Step(S, w, X, bufs, S.EPI_NONE, wsb)
    step0 = _Step(S, w0, X, bufs0, S.EPI_NONE, wsb0)
    # e2e: two pinned host batches in, two out; two device buffer sets
    Xh = [torch.empty((M, K), dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
    for xh in Xh:
        xh.copy_(X.cpu())
    Yh = [torch.empty((M, N), dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
    Xd = [torch.empty_like(X) for _ in range(2)]
    e2e_bufs = [lin.buffers(M) for _ in range(2)]

    _time_steps(step, max(args.warmup, 3), flush, stream)
    barrier()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.2)                      # sampler up before the timed region
    barrier()
    clocks.mark("t0")
    t_wall0 = time.time()
    rows = _time_steps(step, args.steps, flush, stream, per_step=True)
    barrier()
    clocks.mark("t_timed")
    # clock window: untimed steps of the same workload until the sampled span
    # reaches CLOCK_WINDOW_S, so that the clock record holds samples under
    # this load even when the timed steps end within one sampling interval
    n_more = 0
    while time.time() - t_wall0 < CLOCK_WINDOW_S and n_more < 100000:
        _time_steps(step, 8, flush, stream)
        n_more += 8
    barrier()
    clocks.mark("t1")
    clk = clocks.stop()
    if clk is not None:
        clk["window"] = (f"the {args.steps} timed steps plus {n_more} untimed steps of the same "
                         f"workload ({time.time() - t_wall0:.2f} s)")
    S.svdq_get_device_error(w)
    t_act = sum(r[0] for r in rows)
    t_lin = sum(r[1] for r in rows)

    # L2-warm: the same steps without the flush
    rows_warm = _time_steps(step, args.steps, None, stream, per_step=True)
    # same kernels without the low-rank branch (overhead), and end to end
    _time_steps(step0, 3, flush, stream)
    t_act0, t_lin0 = _time_steps(step0, args.steps, flush, stream)
    if wsb is None:
        # the C-ABI call with host buffers; three streams
        e2e_api = "svdq_linear_host"
        Yh3 = Yh + [torch.empty((M, N), dtype=torch.bfloat16, pin_memory=True)]
        _time_e2e_host(S, w, Xh, Yh3, S.EPI_NONE, max(args.warmup, 3))
        t_e2e = _time_e2e_host(S, w, Xh, Yh3, S.EPI_NONE, args.steps)
    else:
        # split-K product: device calls with the copies on their own streams
        e2e_api = "svdq_quantize_act + svdq_linear_splitk, torch copies"
        _time_e2e(S, w, Xh, Yh, Xd, e2e_bufs, S.EPI_NONE, max(args.warmup, 3), wsb)
        t_e2e = _time_e2e(S, w, Xh, Yh, Xd, e2e_bufs, S.EPI_NONE, args.steps, wsb)
    S.svdq_get_device_error(w0)

    tt = max_over_ranks([t_act + t_lin, t_lin, t_act, t_e2e], dist, "cuda")
    t_step_ms, t_lin_ms, t_act_ms, t_e2e_ms = (v / args.steps for v in tt)
    ops = 2.0 * M * N * K
    value = job_tops(ops, ws, t_step_ms * 1e-3)
    bf16_burst, bf16_sust, hbm, which = _peaks()
    int8_peak = 2.0 * bf16_burst          # int8 dense = 2 x bf16 dense (nominal ratio)
    lin_tops = ops / (t_lin_ms * 1e-3) / 1e12
    act_gbs = _act_bytes(M, K, r) / (t_act_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic",
        "config": _config(spec, ws),
        "roofline": {"bound": "tensor", "achieved": lin_tops, "peak": int8_peak,
                     "unit": "TFLOP/s", "frac": lin_tops / int8_peak,
                     "traffic": _linear_traffic(spec.name),
                     "kernel": "svdq_linear", "peak_source":
                     f"{which} bf16 burst {bf16_burst} x 2 (int8/bf16 nominal ratio)"},
        "act_quant": {"ms": t_act_ms, "achieved_gbs": act_gbs, "peak_gbs": hbm,
                      "frac": act_gbs / hbm, "bytes": _act_bytes(M, K, r)},
        "linear_ms": t_lin_ms,
        "lowrank_overhead": {"linear": t_lin_ms / (t_lin0 / args.steps) - 1.0,
                             "layer": t_step_ms / ((t_act0 + t_lin0) / args.steps) - 1.0},
        "e2e": {"value": job_tops(ops, ws, t_e2e_ms * 1e-3), "unit": "TOPS",
                "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2,
                "api": e2e_api},
        "gpu_launches": 2 * args.steps,
        "clocks": clk,
        "product": "svdq_linear_splitk (automatic split)" if splitk else "svdq_linear",
        "variability": {"l2_flushed": {"act": _dist_stats([r[0] for r in rows]),
                                       "linear": _dist_stats([r[1] for r in rows]),
                                       "step": _dist_stats([r[0] + r[1] for r in rows])},
                        "l2_warm": {"act": _dist_stats([r[0] for r in rows_warm]),
                                    "linear": _dist_stats([r[1] for r in rows_warm]),
                                    "step": _dist_stats([r[0] + r[1] for r in rows_warm])}},
    }
    # the comparisons below are single-GPU diagnostics, timed after the
    # headline steps; a multi-GPU run reports the headline only
    extras = ws == 1
    if extras and not args.no_w8a8:
        line["w8a8_comparator"] = _time_w8a8(S, spec, L, a, X, flush, stream, args.steps,
                                             int8_peak)
    if extras and not args.no_nvfp4:
        line["nvfp4_variant"] = _time_nvfp4(S, spec, L, a, X, flush, stream, args.steps,
                                            4.0 * bf16_burst)
    if extras and args.mlp_pair:
        line["cross_layer_fusion"] = _time_mlp_pair(S, flush, stream, args.steps)
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:      # at N = 1 only
        line["cpu_baseline"] = cpu_baseline(spec)
    if rank == 0:
        print(json.dumps(line), flush=True)
    w.free()
    w0.free()
    if dist is not None:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="flux_qkv",
                    help="a name of synth.WORKLOADS or of synth.pixart_points()")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-w8a8", action="store_true",
                    help="skip the W8A8 comparator's timing")
    ap.add_argument("--no-nvfp4", action="store_true",
                    help="skip the NVFP4 variant's timing")
    ap.add_argument("--no-mlp-pair", action="store_true",
                    help="skip the FLUX feed-forward pair (with and without the cross-layer "
                         "fusion)")
    ap.add_argument("--mlp-pair", action="store_true", help=argparse.SUPPRESS)   # the default
    args = ap.parse_args()
    args.mlp_pair = not args.no_mlp_pair
    spec = _workload(args.workload)
    if args.impl == "reference":
        run_reference(args, spec)
    else:
        run_ours(args, spec)


if __name__ == "__main__":
    main()

"""Benchmark of the S4 DPLR forward hot path on B200: kernel generation
(Cauchy/Woodbury spectrum + inverse real FFT + the spectrum of the
zero-padded kernel) followed by the zero-padded causal FFT convolution.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--config 3]

Prints one JSON line. The headline is the workload named by --config
(default 3: H=256, N=64, L=16384, batch 8, the largest DPLR workload); the
metric is (batch * H * L) output elements per second of the whole forward.
The line carries the roofline of the dominant kernel (the convolution, bound
by HBM), the Cauchy stage's fraction of the FP32 peak, the end-to-end number
through the public API with host buffers, clocks sampled during the timed
region, the S4Block, backward, decode and set-up variants of the same layer,
and, under "configs", the forward of every workload (1-5) with its own
roofline and Cauchy figures. The CPU-baseline leg times the fp64 oracle on a
bounded sample of each workload and reports, next to it, the parity of the
GPU results on that same sample.

Multi-GPU (torchrun, one process per GPU): weak scaling, each rank owns its
own H-slice of channels (a different seed per rank); the channels are
independent SSMs, so there is no data-path collective. The timed region is
bracketed by barriers and the reported time is the max over ranks. Only the
headline workload runs then.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import s4inputs  # noqa: E402

METRIC = "S4 fwd (batch·H·L) elems/s; Cauchy FP32 % peak; FFT-conv HBM GB/s % peak"
UNIT = "elem/s"
FALLBACK_HBM_GBS = 6650.0
SM_COUNT = 148
FP32_LANES_PER_SM = 128
NOMINAL_SM_MHZ = 1965.0
# algorithmic FP32 work of the Cauchy stage per (frequency, mode pair): the
# scaled denominator (2 mul, 1 add/fma, 2 fma for |q|^2 -> 8 flop incl. the
# two products by 1/|q|^2) and four complex Cauchy sums as 16 FMAs (32 flop)
CAUCHY_FLOP_PER_TERM = 40
VANDERMONDE_FLOP_PER_TERM = 4
E2E_CHUNKS = 2     # row-pair chunks of the host-buffer pipeline
E2E_INFLIGHT = 2   # consecutive end-to-end steps in flight
# S4Block projection per (b, t) element of the output: 2 dot products of
# length H (value and gate rows of W) = 4 H flop per output element; HBM
# bytes: read y and x, write out
BLOCK_FLOP_PER_ELEM = lambda H: 4 * H   # noqa: E731
BLOCK_PROJ_BYTES_PER_ELEM = 12
# the sources each workload's convolution kernel is built from (L <= 8192:
# the one-CTA pair kernel; L = 16384: the cluster of two; longer: the
# cluster split), hashed to tell whether a recorded ncu figure still holds
_CONV_COMMON = ["common.cuh", "fft.cuh", "pairs.cuh", "cluster.cuh"]
KERNEL_SOURCES = {1: _CONV_COMMON + ["spectral.cu"], 2: _CONV_COMMON + ["spectral.cu"],
                  3: _CONV_COMMON + ["quad.cuh", "quad.cu"], 4: _CONV_COMMON + ["spectral.cu"],
                  5: _CONV_COMMON + ["spectral.cu"]}
# DRAM traffic of one convolution launch per workload, from committed ncu
# summaries (reported only while the convolution's sources are unchanged)
TRAFFIC_FILES = {
    2: os.path.join(ROOT, "profiles", "fftconv_h256_l4096_b16_traffic.txt"),
    3: os.path.join(ROOT, "profiles", "fftconv_h256_l16384_b8_traffic.txt"),
    4: os.path.join(ROOT, "profiles", "fftconv_h64_l65536_b4_traffic.txt"),
}
# channels of each workload the CPU leg runs the oracle on (every row, every
# output), sized to a few seconds of fp64 work on the host
ORACLE_CHANNELS = {1: 4, 2: 16, 3: 4, 4: 2, 5: 8}
# the headline workload's CPU baseline runs more of them, in chunks of the
# above, until about CPU_BUDGET_S seconds of oracle work are spent
HEAD_SAMPLE_CHANNELS = 64
CPU_BUDGET_S = 10.0


# ----------------------------------------------------------------- helpers --
def peaks():
    """(HBM GB/s, SM MHz for the derived FP32 peak, source): the measured copy
    bandwidth from MEASURED_PEAKS.json when the file has a usable one, else
    the fallback figure, labelled as such."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")

    def number(v):
        if isinstance(v, dict):   # {"value": ...} style entries
            v = v.get("value")
        try:
            v = float(v)
        except (TypeError, ValueError):
            return None
        return v if v > 0 else None

    try:
        with open(p) as f:
            d = json.load(f)
    except (OSError, ValueError):
        d = None
    if isinstance(d, dict) and number(d.get("hbm_gbs")) is not None:
        mhz = number(d.get("sm_max_mhz")) or NOMINAL_SM_MHZ
        return number(d["hbm_gbs"]), mhz, "measured"
    return FALLBACK_HBM_GBS, NOMINAL_SM_MHZ, "fallback"


def kernel_source_hash(cfg):
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[cfg]:
        with open(os.path.join(ROOT, "structured_state_space_dplr_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(cfg):
    """dram bytes per launch of the convolution kernel of workload cfg from
    the committed ncu summary, if it was taken on the current kernel source;
    else None."""
    path = TRAFFIC_FILES.get(cfg)
    if path is None or not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
    if vals.get("kernel_source_sha256_16") != kernel_source_hash(cfg):
        return None
    try:
        return float(vals["dram_bytes_per_launch_full_size"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r for r in csv.reader(io.StringIO(out)) if len(r) >= 9]
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1])); smax.append(float(r[2]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons)}


def physical_gpu(local_rank):
    """nvidia-smi id of this process's device (CUDA_VISIBLE_DEVICES aware)."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [v.strip() for v in vis.split(",") if v.strip()]
    if local_rank < len(ids):
        return ids[local_rank]
    return str(local_rank)


# ------------------------------------------------------------ multi-rank ----
def rank_shard(cfg, rank, world):
    """Weak scaling by channel: rank r owns channels [r H, (r + 1) H) of a
    layer with world * H channels (its inputs drawn with seed r). The
    channels are independent SSMs, so no data crosses ranks."""
    H = s4inputs.CONFIGS[cfg]["H"]
    return {"seed": rank, "channel_begin": rank * H, "channel_end": (rank + 1) * H}


def max_over_ranks(values, dist=None, device=None):
    """Element-wise max of per-rank timings (all ranks get the result)."""
    if dist is None:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(elements_per_rank_step, world, steps, max_ms):
    """Whole-job elements per second: all ranks' elements over the slowest rank's time."""
    return elements_per_rank_step * world * steps / (max_ms * 1e-3)


# ------------------------------------------------------------- workload -----
def workload(cfg, seed):
    c = s4inputs.CONFIGS[cfg]
    return s4inputs.make_inputs(cfg, seed=seed), c


def algorithmic(c):
    H, L, Bt, Nh = c["H"], c["L"], c["Bt"], c["N"] // 2
    return {
        "elements": Bt * H * L,
        # the convolution launch: read u, write y, read the kernel spectrum
        # (H x 2L complex fp32); K itself is not read by it
        "conv_bytes": 8 * Bt * H * L + 16 * H * L,
        # Cauchy sums: per (channel, frequency j < L/2, mode pair); Vandermonde:
        # 2 FMAs per (channel, k, stored mode)
        "kernel_flop": (VANDERMONDE_FLOP_PER_TERM * H * L * Nh if c["kind"] == "s4d"
                        else CAUCHY_FLOP_PER_TERM * H * (L // 2) * Nh),
    }


def conv_kernel_name(L):
    if L <= 8192:
        return "k_fftconv_pair"
    if L == 16384:
        return "k_fftconv_quad"
    return "k_fftconv (cluster of 16)"


def graph_kernel_nodes(g):
    """Kernel nodes of a captured torch CUDA graph (kept with keep_graph=True):
    the launches one replay issues."""
    from cuda.bindings import runtime as rt
    graph = rt.cudaGraph_t(init_value=g.raw_cuda_graph())
    err, _, n = rt.cudaGraphGetNodes(graph, 0)
    if err != rt.cudaError_t.cudaSuccess:
        raise RuntimeError(f"cudaGraphGetNodes: {err}")
    err, nodes, n = rt.cudaGraphGetNodes(graph, n)
    if err != rt.cudaError_t.cudaSuccess:
        raise RuntimeError(f"cudaGraphGetNodes: {err}")
    count = 0
    for nd in nodes[:n]:
        err, kind = rt.cudaGraphNodeGetType(nd)
        if err != rt.cudaError_t.cudaSuccess:
            raise RuntimeError(f"cudaGraphNodeGetType: {err}")
        count += kind == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel
    return count


def launches_per_step(c):
    """Kernel launches of one forward step (generation + convolution)."""
    L = c["L"]
    if c["kind"] == "s4d":
        gen = 2                               # Vandermonde, spectrum
    elif L <= 8192:
        gen = 1                               # k_kgen (Cauchy, inverse, spectrum)
    elif L == 16384:
        gen = 2                               # k_cauchy, k_kspec_quad_pair
    else:
        gen = 3                               # k_cauchy, k_irfft, k_kspec_cl
    return gen + 1


# --------------------------------------------------------------- GPU arm ----
def forward_case(s4, torch, dev, cfg, seed, steps, warmup, flags, dist=None, clock_gpu=None, keep=False,
                 keep_head_sample=False):
    """The forward of workload cfg: each stage of each rotating input set
    captured once as a CUDA graph and replayed; per-stage CUDA events over
    `steps` timed steps; then the FP32-bound kernel stage alone. Returns the
    record, the parity sample (K and y of the first ORACLE_CHANNELS channels)
    and, if keep, the device buffers for the headline's extra measurements."""
    inp, c = workload(cfg, seed)
    H, L, Bt = c["H"], c["L"], c["Bt"]
    alg = algorithmic(c)
    s4d = c["kind"] == "s4d"
    names = (["A", "B", "C"] if s4d else ["Lambda", "P", "Q", "B", "C"]) + ["log_dt", "D", "u"]
    base = {k: torch.from_numpy(np.ascontiguousarray(inp[k])).to(dev) for k in names}
    ws_bytes = s4.fft_conv_workspace_size(H, L)
    # rotating input sets: consecutive steps touch different memory, together
    # well above the 126 MB L2, so every step reads its inputs from HBM
    set_bytes = (2 * Bt * H * L + H * L) * 4 + ws_bytes
    nsets = max(2, math.ceil(3 * 126e6 / set_bytes) + 1)
    sets = []
    for i in range(nsets):
        s = {k: v.clone() for k, v in base.items()}
        s["K"] = torch.empty(H, L, device=dev)
        s["y"] = torch.empty(Bt, H, L, device=dev)
        s["ws"] = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        sets.append(s)
    del base

    def gen_stage(s):
        if s4d:   # S4D: Vandermonde kernel, then the spectrum of K + D delta_0
            s4.s4d_kernel_vandermonde(s["A"], s["B"], s["C"], s["log_dt"], L, out=s["K"], flags=flags)
            s4.fft_conv_prepare(s["K"], s["D"], workspace=s["ws"])
        else:     # S4 DPLR: s4_kernel_dplr_prepare
            s4.kernel_dplr_prepare(s["Lambda"], s["P"], s["Q"], s["B"], s["C"], s["log_dt"], s["D"], L,
                                   K=s["K"], workspace=s["ws"], flags=flags)

    def conv_stage(s):
        s4.fft_conv_apply(s["u"], s["ws"], out=s["y"])

    def kernel_only(s):   # the FP32-bound kernel stage alone: Cauchy sums or Vandermonde
        if s4d:
            s4.s4d_kernel_vandermonde(s["A"], s["B"], s["C"], s["log_dt"], L, out=s["K"])
        else:
            s4.dplr_spectrum(s["Lambda"], s["P"], s["Q"], s["B"], s["C"], s["log_dt"], L, out=s["K"])

    for i in range(warmup):
        gen_stage(sets[i % nsets])
        conv_stage(sets[i % nsets])
    torch.cuda.synchronize()
    if int(flags.item()) != 0:
        raise RuntimeError(f"kernel flags set: {int(flags.item())}")

    gen_graphs, conv_graphs = [], []
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        for s in sets:
            g1, g2 = torch.cuda.CUDAGraph(keep_graph=True), torch.cuda.CUDAGraph(keep_graph=True)
            with torch.cuda.graph(g1, stream=cap):
                gen_stage(s)
            with torch.cuda.graph(g2, stream=cap):
                conv_stage(s)
            gen_graphs.append(g1)
            conv_graphs.append(g2)
    torch.cuda.current_stream().wait_stream(cap)
    launches = graph_kernel_nodes(gen_graphs[0]) + graph_kernel_nodes(conv_graphs[0])
    for g in gen_graphs + conv_graphs:
        g.instantiate()
    for i in range(warmup):
        gen_graphs[i % nsets].replay()
        conv_graphs[i % nsets].replay()
    torch.cuda.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(clock_gpu) if clock_gpu is not None else None
    if clocks is not None:
        clocks.start()
        time.sleep(0.3)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t0.record()
    for i in range(steps):
        ev = evs[i]
        ev[0].record()
        gen_graphs[i % nsets].replay()
        ev[1].record()
        conv_graphs[i % nsets].replay()
        ev[2].record()
    t1.record()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clk = clocks.stop() if clocks is not None else None
    ms = t0.elapsed_time(t1)
    stage = [sum(e[j].elapsed_time(e[j + 1]) for e in evs) / steps for j in range(2)]
    if dist is not None:
        del gen_graphs, conv_graphs

    # parity sample (before the kernel-only stage overwrites K): K and y of
    # the channels the CPU leg will run the oracle on
    nch = min(H, HEAD_SAMPLE_CHANNELS if keep_head_sample else ORACLE_CHANNELS[cfg])
    sample = {"K": sets[0]["K"][:nch].cpu().numpy(), "y": sets[0]["y"][:, :nch, :].cpu().numpy(),
              "inp": {k: (v[:, :nch, :] if k == "u" else v[:nch]) if isinstance(v, np.ndarray) else v
                      for k, v in inp.items()}}
    sample["inp"]["H"] = nch

    # the FP32-bound kernel stage alone (Cauchy sums / Vandermonde), timed
    # separately for its FP32 roofline
    cev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    for i in range(warmup):
        kernel_only(sets[i % nsets])
    torch.cuda.synchronize()
    cev[0].record()
    for i in range(steps):
        kernel_only(sets[i % nsets])
    cev[1].record()
    torch.cuda.synchronize()
    stage.append(cev[0].elapsed_time(cev[1]) / steps)

    rec = {"c": c, "alg": alg, "ms": ms, "stage": stage, "clocks": clk, "nsets": nsets, "set_bytes": set_bytes,
           "launches": launches, "inp": inp if keep else None, "sets": sets if keep else None, "names": names}
    if not keep:
        del sets
        torch.cuda.empty_cache()
    return rec, sample


def forward_record(rec, steps, world, hbm, fp32_peak, sm_max_mhz, peak_src, with_traffic=True):
    """The JSON figures of one forward_case."""
    c, alg, stage = rec["c"], rec["alg"], rec["stage"]
    H, L, Bt = c["H"], c["L"], c["Bt"]
    s4d = c["kind"] == "s4d"
    cfg = next(k for k, v in s4inputs.CONFIGS.items() if v["name"] == c["name"])
    conv_gbs = alg["conv_bytes"] / (stage[1] * 1e-3) / 1e9
    cauchy_tflops = alg["kernel_flop"] / (stage[2] * 1e-3) / 1e12
    cauchy = {"kernel": ("k_vandermonde_tc" if L % 8192 == 0 else "k_vandermonde") if s4d else "k_cauchy",
              "bound": "alu", "achieved": cauchy_tflops, "peak": fp32_peak, "unit": "TFLOP/s",
              "frac": cauchy_tflops / fp32_peak,
              "peak_derivation": f"{SM_COUNT} SM x {FP32_LANES_PER_SM} FP32 lanes x 2 x {sm_max_mhz:.0f} MHz",
              "algorithmic_flop": alg["kernel_flop"]}
    if s4d and L % 8192 == 0:
        cauchy["note"] = ("the Vandermonde product runs on the tensor cores (3 tf32 products); achieved is the "
                          "algorithmic FP32-equivalent rate (2 FMAs per term) against the CUDA-core FP32 peak")
    if not s4d:
        if L <= 8192:
            # the forward runs the Cauchy sums inside k_kgen, fused with the
            # inverse transform and the spectrum: its whole launch time is
            # charged to the Cauchy FLOPs (a lower bound on the fraction)
            t = alg["kernel_flop"] / (stage[0] * 1e-3) / 1e12
            cauchy["in_forward"] = {"kernel": "k_kgen", "achieved": t, "frac": t / fp32_peak,
                                    "note": "Cauchy FLOPs over the whole k_kgen launch (which also runs "
                                            "the length-L inverse and the length-2L forward transforms)"}
        else:
            cauchy["in_forward"] = {"kernel": "k_cauchy", "achieved": cauchy_tflops,
                                    "frac": cauchy_tflops / fp32_peak,
                                    "note": "the forward's generation launches this same kernel"}
    traffic = recorded_traffic(cfg) if with_traffic else None
    return {
        "value": job_throughput(alg["elements"], world, steps, rec["ms"]),
        "unit": UNIT,
        "ms_per_step": rec["ms"] / steps,
        "stages_ms": {"kernel_and_spectrum": stage[0], "fft_conv": stage[1],
                      ("vandermonde_alone" if s4d else "cauchy_spectrum_alone"): stage[2]},
        "roofline": {"kernel": conv_kernel_name(L), "bound": "hbm", "achieved": conv_gbs, "peak": hbm,
                     "unit": "GB/s", "frac": conv_gbs / hbm, "traffic": traffic, "peak_source": peak_src,
                     "algorithmic_bytes": alg["conv_bytes"],
                     "algorithmic_bytes_formula": "8*Bt*H*L (u read, y written) + 16*H*L (spectrum read)"},
        "cauchy": cauchy,
        "gpu_launches_per_step": rec["launches"],
    }


def torch_fft_context(s4, torch, sets, nsets, c, steps, warmup, flags, lib_conv_us):
    """Context beside the library's convolution (feeds no value of this line):
    the same convolution as the pages write it, with torch.fft (cuFFT) on the
    same device and rotating inputs, y = irfft(rfft(u, 2L) rfft(K, 2L))[:L] + D u,
    timed with CUDA events -- once with rfft(K) precomputed (the library's
    apply stage also starts from a stored spectrum) and once per call as the
    pages' fft_conv does -- and its largest difference from the library's y."""
    L, n = c["L"], 2 * c["L"]
    s4d = c["kind"] == "s4d"
    for s in sets:   # K as the forward produced it (the kernel-only timing left its own data there)
        if s4d:
            s4.s4d_kernel_vandermonde(s["A"], s["B"], s["C"], s["log_dt"], L, out=s["K"])
        else:
            s4.kernel_dplr_prepare(s["Lambda"], s["P"], s["Q"], s["B"], s["C"], s["log_dt"], s["D"], L,
                                   K=s["K"], workspace=s["ws"], flags=flags)
    kf = [torch.fft.rfft(s["K"], n=n) for s in sets]

    def conv(i, with_kernel_fft):
        s = sets[i % nsets]
        k = torch.fft.rfft(s["K"], n=n) if with_kernel_fft else kf[i % nsets]
        y = torch.fft.irfft(torch.fft.rfft(s["u"], n=n) * k, n=n)[..., :L]
        return y + s["D"][:, None] * s["u"]

    out = {}
    for key, wk in (("torch_fft_conv_us", False), ("torch_fft_conv_with_kernel_fft_us", True)):
        for i in range(warmup):
            conv(i, wk)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(steps):
            conv(i, wk)
        e1.record()
        torch.cuda.synchronize()
        out[key] = e0.elapsed_time(e1) * 1e3 / steps
    ref = conv(0, False)
    s4.fft_conv_apply(sets[0]["u"], sets[0]["ws"], out=sets[0]["y"])
    torch.cuda.synchronize()
    out["max_abs_diff_over_max_abs_y"] = float((ref - sets[0]["y"]).abs().max() / sets[0]["y"].abs().max())
    out["library_fft_conv_us"] = lib_conv_us
    out["note"] = ("torch.fft (cuFFT) in fp32 on the same inputs; the library's convolution is "
                   "s4_fft_conv_apply from the spectrum its generation stage stored")
    del kf
    torch.cuda.empty_cache()
    return out


def torch_dplr_kernel(torch, d, L, chunk=32):
    """The DPLR kernel as the pages write it, with torch complex64 tensors (on
    whatever device d's tensors are): at the roots of unity z_j (j < L/2),
    g_j = (2/dt)(1 - z_j)/(1 + z_j); the four Cauchy sums over all N = 2 Nh
    modes (the stored ones and their conjugates) of v / (g - lambda) for
    v = C B, C P, conj(Q) B, conj(Q) P; K_hat = 2/(1 + z) (k00 - k01 k10 /
    (1 + k11)); the Nyquist bin from its limit dt sum Re(C B); K =
    irfft(K_hat, L). Channels in chunks of `chunk` to bound the
    (chunk, L/2, N) intermediates."""
    import math
    lam, C, B, P, Q = (d[k] for k in ("Lambda", "C", "B", "P", "Q"))
    H = lam.shape[0]
    jj = torch.arange(L // 2, device=lam.device, dtype=torch.float32)
    z = torch.polar(torch.ones_like(jj), -2.0 * math.pi * jj / L)
    dt = torch.exp(d["log_dt"])
    Ks = []
    for h0 in range(0, H, chunk):
        hs = slice(h0, min(H, h0 + chunk))
        lm = torch.cat([lam[hs], lam[hs].conj()], dim=1)                       # [hc, N]
        V = torch.stack([C[hs] * B[hs], C[hs] * P[hs], Q[hs].conj() * B[hs], Q[hs].conj() * P[hs]], 1)
        V = torch.cat([V, V.conj()], dim=2)                                      # [hc, 4, N]
        g = (2.0 / dt[hs])[:, None] * ((1 - z) / (1 + z))[None, :]              # [hc, L/2]
        r = 1.0 / (g[:, :, None] - lm[:, None, :])                              # [hc, L/2, N]
        k = torch.einsum("hjn,hvn->hvj", r, V)                                  # [hc, 4, L/2]
        kh = (2.0 / (1 + z))[None, :] * (k[:, 0] - k[:, 1] * k[:, 2] / (1 + k[:, 3]))
        nyq = dt[hs] * (C[hs] * B[hs]).real.sum(1)
        kh = torch.cat([kh, nyq.to(kh.dtype)[:, None]], dim=1)                   # [hc, L/2 + 1]
        Ks.append(torch.fft.irfft(kh, n=L))
    return torch.cat(Ks, 0)


def torch_generation_context(torch, d, c, steps, warmup, lib_gen_us, chunk=32):
    """Context beside the library's kernel generation (feeds no value of this
    line): torch_dplr_kernel on the same device and parameters, timed with
    CUDA events, and K's largest per-channel difference from the library's K
    (d["K"])."""
    L = c["L"]
    for _ in range(warmup):
        torch_dplr_kernel(torch, d, L, chunk)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        torch_dplr_kernel(torch, d, L, chunk)
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / steps
    K = torch_dplr_kernel(torch, d, L, chunk)
    err = float(((K - d["K"]).abs().max(dim=1).values / d["K"].abs().max(dim=1).values).max())
    torch.cuda.empty_cache()
    return {"torch_generation_us": us, "library_generation_us": lib_gen_us,
            "max_per_channel_rel_diff_of_K": err,
            "note": f"torch complex64 Cauchy sums + Woodbury + 2/(1+z) + irfft, {chunk} channels per chunk; "
                    "the library's generation is s4_kernel_dplr_prepare (K and the convolution spectrum)"}


def block_case(s4, torch, dev, sets, nsets, H, seed, steps, warmup, flags):
    """The S4Block around the layer: channel layer norm -> the layer's
    convolution (the prepared spectrum) -> GLU projection + residual, over the
    rotating input sets (x = the set's u)."""
    bp = s4inputs.block_params(seed, H)
    bdev = {k: torch.from_numpy(bp[k]).to(dev) for k in ("gamma", "beta", "W", "bias")}
    glu_ws = s4.glu_projection_prepare(bdev["W"])
    bz = [torch.empty_like(s["u"]) for s in sets]
    bo = [torch.empty_like(s["u"]) for s in sets]

    def blk(i, ev=None):
        s, j = sets[i % nsets], i % nsets
        if ev is not None:
            ev[0].record()
        s4.layernorm_channels(s["u"], bdev["gamma"], bdev["beta"], bp["eps"], out=bz[j])
        if ev is not None:
            ev[1].record()
        s4.fft_conv_apply(bz[j], s["ws"], out=s["y"])
        if ev is not None:
            ev[2].record()
        s4.glu_projection_residual(s["y"], s["u"], bdev["bias"], glu_ws, out=bo[j], flags=flags)
        if ev is not None:
            ev[3].record()

    for i in range(warmup):
        blk(i)
    torch.cuda.synchronize()
    bev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for i in range(steps):
        blk(i, bev[i])
    torch.cuda.synchronize()
    if int(flags.item()) != 0:
        raise RuntimeError(f"kernel flags set in the block: {int(flags.item())}")
    kst = [sum(e[j].elapsed_time(e[j + 1]) for e in bev) / steps for j in range(3)]
    del bz, bo
    return kst


def block_record(kst, alg, H):
    ktot = sum(kst)
    proj_s = kst[2] * 1e-3
    return {"metric": "S4Block forward (batch*H*L) elems/s", "value": alg["elements"] / (ktot * 1e-3),
            "ms_per_step": ktot,
            "stages_us": {"layernorm": kst[0] * 1e3, "conv": kst[1] * 1e3, "glu_projection_residual": kst[2] * 1e3},
            "glu_projection": {
                "tflops": BLOCK_FLOP_PER_ELEM(H) * alg["elements"] / proj_s / 1e12,
                "tensor_tflops_issued": 3 * BLOCK_FLOP_PER_ELEM(H) * alg["elements"] / proj_s / 1e12,
                "gbs": BLOCK_PROJ_BYTES_PER_ELEM * alg["elements"] / proj_s / 1e9,
                "operands": "fp32 split into bf16 hi/lo, 3 products (tcgen05 kind::f16), fp32 accumulate"},
            "layernorm_gbs": 8 * alg["elements"] / (kst[0] * 1e-3) / 1e9,
            "calls": "s4_layernorm_channels + s4_fft_conv_apply + s4_glu_projection_residual, one launch each"}


def run_gpu(args, rank, world, local_rank):
    import torch
    import structured_state_space_dplr_b200 as s4

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    hbm, sm_max_mhz, peak_src = peaks()
    fp32_peak = SM_COUNT * FP32_LANES_PER_SM * 2 * sm_max_mhz * 1e6 / 1e12
    cfg = args.config
    shard = rank_shard(cfg, rank, world)
    flags = torch.zeros(1, dtype=torch.int32, device=dev)

    # ---- the headline workload (timed region: barriers, max over ranks, clocks)
    rec, head_sample = forward_case(s4, torch, dev, cfg, shard["seed"], args.steps, args.warmup, flags, dist=dist,
                                    clock_gpu=physical_gpu(local_rank), keep=True, keep_head_sample=rank == 0)
    c, alg, inp, sets, nsets, names = rec["c"], rec["alg"], rec["inp"], rec["sets"], rec["nsets"], rec["names"]
    H, L, Bt = c["H"], c["L"], c["Bt"]
    s4d = c["kind"] == "s4d"
    ms = rec["ms"]

    # ---- end to end through the public API with host buffers (pinned):
    # every step uploads that step's batch u and downloads its output y; the
    # layer's parameters are resident on the device (uploaded once, as a
    # model's weights are)
    # E2E_INFLIGHT consecutive steps overlap (one step's downloads with the
    # next one's uploads), each on its own stream with its own device buffers
    # and host output, as a serving loop over a stream of batches runs
    host = {k: torch.from_numpy(np.ascontiguousarray(inp[k])).pin_memory() for k in names}
    esets = [sets[i % nsets] for i in range(E2E_INFLIGHT)]
    y_hosts = [torch.empty(Bt, H, L, dtype=torch.float32).pin_memory() for _ in esets]
    e2e_streams = [torch.cuda.Stream() for _ in esets]
    for ds in esets:
        for k in names:
            if k != "u":
                ds[k].copy_(host[k])
    h2d = host["u"].numel() * 4
    d2h = y_hosts[0].numel() * 4

    def e2e_step(i):
        ds, y_host = esets[i % E2E_INFLIGHT], y_hosts[i % E2E_INFLIGHT]
        with torch.cuda.stream(e2e_streams[i % E2E_INFLIGHT]):
            if s4d:
                K = s4.s4d_kernel_vandermonde(ds["A"], ds["B"], ds["C"], ds["log_dt"], L, out=ds["K"])
                s4.fft_conv_host(host["u"], K, ds["D"], y_host=y_host, u_dev=ds["u"], y_dev=ds["y"],
                                 workspace=ds["ws"], chunks=E2E_CHUNKS)
            else:
                s4.forward_dplr_host(host["u"], ds["Lambda"], ds["P"], ds["Q"], ds["B"], ds["C"],
                                     ds["log_dt"], ds["D"], y_host=y_host, K=ds["K"], u_dev=ds["u"],
                                     y_dev=ds["y"], workspace=ds["ws"], chunks=E2E_CHUNKS)

    def e2e_steps(n):
        cur = torch.cuda.current_stream()
        for st in e2e_streams:
            st.wait_stream(cur)
        for i in range(n):
            e2e_step(i)
        for st in e2e_streams:
            cur.wait_stream(st)

    e2e_ms = float("nan")
    if not args.no_e2e:
        e2e_steps(max(E2E_INFLIGHT, args.warmup))
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if dist is not None:
            dist.barrier()
        e0.record()
        e2e_steps(args.steps)
        e1.record()
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1)

    # ---- backward pass of the same layer: du by the adjoint convolution, dK
    # and dD by the batch correlation, and the parameter gradients through the
    # kernel; dy is another input set's u
    d, dy = sets[0], sets[1 % nsets]["u"]
    du = torch.empty_like(dy)
    gK = torch.empty(H, L, device=dev)
    gD = torch.empty(H, device=dev)
    gws = torch.empty(s4.fft_conv_kernel_grad_workspace_size(H, L), dtype=torch.uint8, device=dev)
    kneed = s4.kernel_dplr_backward_workspace_size(H, L)
    kws = torch.empty(kneed, dtype=torch.uint8, device=dev) if kneed > 0 else None

    def bwd(ev=None):
        if ev is not None:
            ev[0].record()
        s4.fft_conv_apply_adjoint(dy, d["ws"], out=du)
        if ev is not None:
            ev[1].record()
        s4.fft_conv_kernel_grad(d["u"], dy, dK=gK, dD=gD, workspace=gws)
        if ev is not None:
            ev[2].record()
        if s4d:
            s4.s4d_kernel_vandermonde_backward(d["A"], d["B"], d["C"], d["log_dt"], gK)
        else:
            s4.kernel_dplr_backward(d["Lambda"], d["P"], d["Q"], d["B"], d["C"], d["log_dt"], gK,
                                    workspace=kws)
        if ev is not None:
            ev[3].record()

    for _ in range(max(1, args.warmup)):
        bwd()
    torch.cuda.synchronize()
    bev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for i in range(args.steps):
        bwd(bev[i])
    torch.cuda.synchronize()
    bst = [sum(e[j].elapsed_time(e[j + 1]) for e in bev) / args.steps for j in range(3)]
    total = sum(bst)
    backward = {"metric": "S4 layer backward (batch*H*L) elems/s", "value": alg["elements"] / (total * 1e-3),
                "ms_per_step": total,
                "stages_ms": {"du_adjoint_conv": bst[0], "dK_dD_batch_correlation": bst[1],
                              "kernel_param_grads": bst[2]},
                "calls": "s4_fft_conv_apply_adjoint (1 launch) + s4_fft_conv_kernel_grad ("
                         + ("1 launch" if L <= 8192
                            else f"{3 * ((Bt + 1) // 2) + 1} launches: per batch row pair spectrum, adjoint "
                             "convolution, accumulate")
                         + ")" + (" + s4d_kernel_vandermonde_backward (1 launch)" if s4d
                                  else " + s4_kernel_dplr_backward_ws ("
                                  + ("1 launch" if L <= 16384 else "4 launches: four-step DFT, sliced gradients, assembly") + ")")}
    del du, gK, gD, gws, kws

    # ---- the S4Block around the same layer
    block = block_record(block_case(s4, torch, dev, sets, nsets, H, shard["seed"], args.steps, args.warmup, flags),
                         alg, H)

    # ---- context: the same convolution through torch.fft (cuFFT)
    torch_fft = None
    if not args.headline_only:
        try:
            torch_fft = torch_fft_context(s4, torch, sets, nsets, c, args.steps, args.warmup, flags,
                                          rec["stage"][1] * 1e3)
            if not s4d:
                torch_fft["generation"] = torch_generation_context(torch, sets[0], c, args.steps, args.warmup,
                                                                   rec["stage"][0] * 1e3)
        except Exception as exc:   # noqa: BLE001 - reported, the main line stands
            torch_fft = {"error": f"{type(exc).__name__}: {exc}"}

    # ---- recurrent view (decode): up to 1024 tokens from a zero state, as
    # one s4_recurrent_scan and as single-token steps replayed from a graph
    d = sets[0]
    if s4d:
        Ab, Bb = s4.s4d_discretize_zoh(d["A"], d["B"], d["log_dt"])
        step_kind = "diagonal ZOH (S4D), O(Nh) per token"
    else:
        Ab, Bb = s4.dplr_discretize_structured(d["Lambda"], d["P"], d["Q"], d["B"], d["log_dt"])
        step_kind = "structured bilinear DPLR (diagonal + rank 1), O(Nh) per token"
    T = min(1024, L)
    x = torch.zeros(Bt, H, c["N"] // 2, dtype=torch.complex64, device=dev)
    u_tok = d["u"][:, :, :T].contiguous()
    y_tok = torch.empty_like(u_tok)
    u_cols = [u_tok[:, :, k].contiguous() for k in range(T)]
    y_col = torch.empty(Bt, H, device=dev)
    g_steps = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        s4.recurrent_step(Ab, Bb, d["C"], d["D"], x, u_cols[0], out=y_col)   # warm-up outside capture
        with torch.cuda.graph(g_steps, stream=cap):
            for k in range(T):
                s4.recurrent_step(Ab, Bb, d["C"], d["D"], x, u_cols[k], out=y_col)
    torch.cuda.current_stream().wait_stream(cap)
    for _ in range(2):
        s4.recurrent_scan(Ab, Bb, d["C"], d["D"], x, u_tok, out=y_tok)
        g_steps.replay()
    torch.cuda.synchronize()
    e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    e[0].record()
    s4.recurrent_scan(Ab, Bb, d["C"], d["D"], x, u_tok, out=y_tok)
    e[1].record()
    e[2].record()
    g_steps.replay()
    e[3].record()
    torch.cuda.synchronize()
    decode = {"tokens": T, "batch": Bt, "H": H, "state": c["N"] // 2, "step": step_kind,
              "scan_us_per_token": e[0].elapsed_time(e[1]) * 1e3 / T,
              "step_us_per_token": e[2].elapsed_time(e[3]) * 1e3 / T,
              "step_launch": f"{T} s4_recurrent_step launches replayed from one CUDA graph"}
    del g_steps, u_cols

    # ---- the set-up variants of the DPLR layer (timed once per call, not per
    # batch): the ZOH discretisation and its truncated kernel (fp64 matrix
    # exponential per channel, Nh <= 32), and C~ = C (I - Abar^L) with the
    # truncated kernel from the Cauchy path. A failure here is reported in
    # the line, never fatal to it.
    variants = None
    if not s4d and c["N"] // 2 <= 32:
        try:
            pk = [d[k] for k in ("Lambda", "P", "Q", "B", "C", "log_dt")]
            Kz = torch.empty(H, L, device=dev)

            def timed(fn, reps=3):
                fn()
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                for _ in range(reps):
                    fn()
                e1.record()
                torch.cuda.synchronize()
                return e0.elapsed_time(e1) * 1e3 / reps

            def ct_kernel():
                Ct = s4.dplr_ctilde(d["Lambda"], d["P"], d["Q"], d["C"], d["log_dt"], L)
                s4.kernel_dplr(d["Lambda"], d["P"], d["Q"], d["B"], Ct, d["log_dt"], L, out=Kz)

            variants = {
                "zoh_kernel_us": timed(lambda: s4.kernel_dplr_zoh(*pk, L, out=Kz)),
                "zoh_discretize_us": timed(lambda: s4.dplr_discretize_zoh(*pk)),
                "ctilde_truncated_kernel_us": timed(ct_kernel),
                "calls": "s4_kernel_dplr_zoh; s4_dplr_discretize_zoh; s4_dplr_ctilde + s4_kernel_dplr"}
            del Kz
        except Exception as exc:   # noqa: BLE001 - reported, the main line stands
            variants = {"error": f"{type(exc).__name__}: {exc}"}

    times = max_over_ranks([ms, e2e_ms] + rec["stage"], dist, dev)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    ms, e2e_ms = times[0], times[1]
    rec["ms"], rec["stage"] = ms, times[2:]
    del sets, esets, d, rec["sets"]
    torch.cuda.empty_cache()
    if rank != 0:
        return None

    head = forward_record(rec, args.steps, world, hbm, fp32_peak, sm_max_mhz, peak_src)
    samples = {cfg: head_sample}
    line = {
        "metric": METRIC,
        "value": head["value"],
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": ("synthetic (S4D-Lin parameters, seeded inputs)" if s4d else
                 "synthetic (seeded HiPPO-LegS DPLR parameters, seeded inputs)"),
        "config": {"workload": c["name"], "H": H, "N": c["N"], "L": L, "batch": Bt,
                   "global_batch": Bt * world, "dt_range": [c["dt_min"], c["dt_max"]],
                   "parallelism": f"channel shard x{world}, no collective",
                   "launch": ("per step: s4d_kernel_vandermonde + s4_fft_conv_prepare" if s4d
                              else "per step: s4_kernel_dplr_prepare")
                             + " + s4_fft_conv_apply, each stage replayed from a CUDA graph",
                   "l2": f"{nsets} rotating input sets of {rec['set_bytes'] / 1e6:.0f} MB (> 126 MB L2)"},
        "stages_ms": head["stages_ms"],
        "roofline": head["roofline"],
        "cauchy": head["cauchy"],
        "e2e": None if args.no_e2e else {"value": job_throughput(alg["elements"], world, args.steps, e2e_ms),
                                         "unit": UNIT,
                                         "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                                         "call": ("s4d_kernel_vandermonde + s4_fft_conv_host" if s4d
                                                  else "s4_forward_dplr_host")
                                         + f", pinned host u/y, {E2E_CHUNKS} row-pair chunks, "
                                           f"{E2E_INFLIGHT} steps in flight (own stream, device buffers and host "
                                           "output each); the layer's parameters resident on the device"},
        "gpu_launches": rec["launches"] * args.steps,
        "gpu_launches_source": "kernel nodes of the captured generation and convolution graphs, x steps",
        "decode": decode,
        "variants": variants,
        "backward": backward,
        "block": block,
        "torch_fft_context": torch_fft,
        "clocks": rec["clocks"],
    }

    # ---- every workload's forward (single GPU only): its own roofline,
    # Cauchy figures and S4Block, outside the headline's timed region
    if world == 1 and not args.headline_only:
        configs = {}
        for k in sorted(s4inputs.CONFIGS):
            if k == cfg:
                sub = dict(head)
                sub["block_us"] = block["stages_us"]
            else:
                r, smp = forward_case(s4, torch, dev, k, 0, args.steps, args.warmup, flags, keep=True)
                sub = forward_record(r, args.steps, 1, hbm, fp32_peak, sm_max_mhz, peak_src)
                kc = r["c"]
                sub["block_us"] = block_record(
                    block_case(s4, torch, dev, r["sets"], r["nsets"], kc["H"], 0, args.steps, args.warmup, flags),
                    r["alg"], kc["H"])["stages_us"]
                del r
                torch.cuda.empty_cache()
                samples[k] = smp
            kc = s4inputs.CONFIGS[k]
            sub = {"workload": kc["name"], "H": kc["H"], "L": kc["L"], "batch": kc["Bt"], **sub}
            configs[str(k)] = sub
        line["configs"] = configs

    if world == 1 and not args.no_cpu_baseline:
        base = cpu_baseline_and_parity(samples, head=cfg)
        line["cpu_baseline"] = base[cfg]
        line["parity"] = base[cfg]["parity"]
        if "configs" in line:
            for k, b in base.items():
                line["configs"][str(k)]["cpu_baseline"] = b
                line["configs"][str(k)]["parity"] = b["parity"]
    return line


# ------------------------------------------------------- oracle (CPU) arm ---
def oracle_sample(inp, channels):
    """fp64 oracle forward for all rows of the given channels: the kernel
    (dense powers / the Vandermonde sum) and every output of the direct
    O(L^2) sum. Returns (K [len(channels), L], y [Bt, len(channels), L])."""
    from oracle import workloads
    if inp["kind"] == "s4d":
        K = workloads.s4d_kernel(inp, channels=channels)
    else:
        K = workloads.dplr_kernel(inp, channels=channels)
    rows = [(b, h) for b in range(inp["Bt"]) for h in channels]
    Krows = [K[list(channels).index(h)] for _, h in rows]
    y = workloads.conv_rows_at(inp, Krows, rows, np.arange(inp["L"]))
    return K, y.reshape(inp["Bt"], len(channels), inp["L"])


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline_and_parity(samples, head=None, budget_s=CPU_BUDGET_S):
    """The fp64 oracle on the host cores, per workload, on its first
    channels (all rows, every output): its throughput (the CPU baseline) and
    the GPU results' error on that same sample. Each workload runs one chunk
    of ORACLE_CHANNELS channels; the headline workload runs chunks until
    about budget_s seconds are spent or its sampled channels run out."""
    os.environ.setdefault("OMP_NUM_THREADS", str(cpu_cores()))
    out = {}
    for cfg, smp in samples.items():
        inp, c = smp["inp"], s4inputs.CONFIGS[cfg]
        avail, chunk = smp["K"].shape[0], ORACLE_CHANNELS[cfg]
        Ks, ys, dt, nch = [], [], 0.0, 0
        while nch < avail and (nch == 0 or (cfg == head and dt < budget_s)):
            ch = list(range(nch, min(nch + chunk, avail)))
            t = time.perf_counter()
            Kc, yc = oracle_sample(inp, ch)
            dt += time.perf_counter() - t
            Ks.append(Kc)
            ys.append(yc)
            nch += len(ch)
        Kr, yr = np.concatenate(Ks, axis=0), np.concatenate(ys, axis=1)
        elems = c["Bt"] * nch * c["L"]
        Kg = smp["K"][:nch].astype(np.float64)
        yg = smp["y"][:, :nch].astype(np.float64)
        k_err = max(float(np.abs(Kg[i] - Kr[i]).max() / np.abs(Kr[i]).max()) for i in range(nch))
        y_rel = float(np.linalg.norm(yg - yr) / np.linalg.norm(yr))
        worst = max(float(np.linalg.norm(yg[b, i] - yr[b, i]) / np.linalg.norm(yr[b, i]))
                    for b in range(c["Bt"]) for i in range(nch))
        out[cfg] = {"value": elems / dt, "unit": UNIT, "cores": int(os.environ["OMP_NUM_THREADS"]),
                    "kind": "oracle",
                    "sample": f"channels 0..{nch - 1} of {c['H']} (all {c['Bt']} rows, every output): fp64 "
                              f"{'Vandermonde' if c['kind'] == 's4d' else 'dense-power aliased'} kernel + "
                              f"direct O(L^2) convolution, {dt:.1f} s",
                    "parity": {"kernel_max_rel_err": k_err, "y_rel_l2": y_rel, "y_worst_row_rel_l2": worst,
                               "tolerances": {"kernel": 1e-4, "y": 2e-4},
                               "sample": f"channels 0..{nch - 1}, all rows, every output, vs the fp64 oracle"}}
    return out


def reference_chunk(c):
    """Channels per reference step: about 1e9 multiply-adds of direct sum."""
    per_channel = c["Bt"] * c["L"] * c["L"] / 2
    return max(1, min(c["H"], int(round(1e9 / per_channel))))


def run_reference(args):
    os.environ.setdefault("OMP_NUM_THREADS", str(cpu_cores()))
    inp, c = workload(args.config, seed=0)
    chunk = reference_chunk(c)
    for i in range(args.warmup):
        oracle_sample(inp, list(range(chunk)))
    t = time.perf_counter()
    elems = 0
    for i in range(args.steps):
        h0 = (i * chunk) % c["H"]
        ch = list(range(h0, min(h0 + chunk, c["H"])))
        oracle_sample(inp, ch)
        elems += c["Bt"] * len(ch) * c["L"]
    dt = time.perf_counter() - t
    v = elems / dt
    return {
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": ("synthetic (S4D-Lin parameters, seeded inputs)" if c["kind"] == "s4d" else
                 "synthetic (seeded HiPPO-LegS DPLR parameters, seeded inputs)"),
        "config": {"workload": c["name"], "H": c["H"], "N": c["N"], "L": c["L"], "batch": c["Bt"]},
        "cpu_baseline": {"value": v, "unit": UNIT, "kind": "oracle", "cores": int(os.environ["OMP_NUM_THREADS"]),
                         "sample": f"each step: {chunk} channel(s) x {c['Bt']} rows of the workload, every "
                                   "output: fp64 kernel by dense powers / the Vandermonde sum + direct O(L^2) "
                                   "convolution"},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", type=int, default=3, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--headline-only", action="store_true", help="skip the other workloads' sub-records")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end loop")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    line = run_gpu(args, rank, world, local_rank)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()

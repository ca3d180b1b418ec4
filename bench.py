#!/usr/bin/env python
"""Benchmark of the fused attention forward hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass of the path over one batch of synthetic input.  The
headline workload is causal MHA prefill, B=2, H=16, S=2048, d=128 (bf16
in, fp32 accumulate, fp32 out), reported in TFLOP/s with the causal-halved
count 4*B*H*S*S*d/2.  The other workloads of this path are timed in the
same run and reported under "workloads":
- tiny full prefill and GQA d=256 prefill;
- prefill with every score modifier;
- the (192,128), (192,192) and (320,256) head-size pairs;
- prefill over q8_0 K/V (the pre-pass plus prefill);
- chunked prefill over the paged cache;
- paged GQA decode, over bf16, q8_0, q4_0 and FP8 E4M3 caches;
- latent sparse decode;
- the MLA decode tail.
More workloads run alone with --only NAME (prefill over FP8 K/V, the
dequant kernels, latent prefill).

Timing: inputs already resident in HBM; several copies of every input are
rotated so that consecutive steps never find their operands in L2; steps are
captured in a CUDA graph and the K timed steps are bracketed by CUDA events
on the launching stream, with a barrier and a device synchronise on both
sides; the time is the max over ranks.  nvidia-smi clocks are sampled while
the timed region runs.  "e2e" repeats the headline through the public API
with pinned host buffers, host<->device copies inside the timed region,
steps pipelined over two buffer sets (uploads, compute and downloads on
their own streams).

Multi-GPU (torchrun): every rank runs its own replica of the workload (the
path has no exchange step), value = all ranks' work / max time ("weak").

--impl reference times the CPU fp64 oracle (the only other implementation
of this path) on a bounded sample of the same workload, rank 0 only.
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

METRIC = "attention TFLOP/s & % dense BF16 peak (prefill); decode HBM GB/s, 1×B200"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# dram__bytes_read.sum + dram__bytes_write.sum per launch from ncu, with the
# profile summary it comes from; None until a capture of the current kernel.
NCU_TRAFFIC = {
    # dram__bytes_read.sum + dram__bytes_write.sum of one launch; the summary
    # under profiles/ named for the kernel and workload gives the capture.
    "causal_mha_b2_h16_s2048_d128": 54526208,
    "gqa_full_b1_hq32_hkv8_s4096_d256": 215944192,
    "causal_mha_mods_b2_h16_s2048_d128": 58342656,
    "paged_gqa_b64_hq32_hkv8_d128_bs64": 1236043776,
    "paged_gqa_q8_0kv_b64_hq32_hkv8_d128_bs64": 658865408,
    "latent_sparse_t32_hq128_dk576_dv512_top2048": 45273088,
    "causal_mha_b2_h16_s2048_dk192_dv128": 72717056,
    "causal_gqa_b2_hq16_hkv4_s2048_dk192_dv192": 39777792,
    "kv_dequant causal_mha_q8_0kv_b2_h16_s2048_d128": 17835776,
    "kv_dequant causal_mha_fp8kv_b2_h16_s2048_d128": 16799744,
    "paged_prefill_gqa_b16_hq32_hkv8_sq512_d128_bs64": 417585664,
    "mla_tail_t32_hq128_r512_v128_hidden7168": 257049088,
    "causal_gqa_b1_hq16_hkv4_s4096_dk320_dv256": 78919168,
    "paged_gqa_fp8kv_b64_hq32_hkv8_d128_bs64": 620406528,
    "paged_gqa_q4_0kv_b64_hq32_hkv8_d128_bs64": 351211008,
    "causal_mqa_b1_hq16_hkv1_s4096_dk576_dv512": 167481088,
}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-secondary", action="store_true", help="only the headline workload")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", default=None,
                    help="time one named workload alone (for profiling), e.g. causal_mha_b2_h16_s2048_d128")
    ap.add_argument("--eager", action="store_true", help="with --only: launch every step eagerly (no CUDA graph)")
    ap.add_argument("--soak-s", type=float, default=0.25,
                    help="untimed replays before each headline region, in seconds (0 under a profiler)")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks --

class ClockSampler:
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self, t_from=None, t_to=None):
        """Summary of the samples taken between host times t_from and t_to."""
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        sm = []
        mx = None
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                ts = time.mktime(time.strptime(r[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                ts += float("0." + r[0].split(".")[1]) if "." in r[0] else 0.0
            except Exception:
                ts = None
            if t_from is not None and ts is not None and not (t_from - 0.05 <= ts <= t_to + 0.05):
                continue
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------- helpers --

def rotation_copies(footprint_bytes, l2_bytes, cap=64):
    """Copies of the inputs so that one cycle spans > 2x L2."""
    return int(max(1, min(cap, math.ceil(2.0 * l2_bytes / max(footprint_bytes, 1)) + 1)))


def time_graph(torch, launch, n_copies, K, W, dist=None, window=None):
    """Capture one graph that runs `per_graph` steps (cycling over the input
    copies), then time K steps.  Returns (ms_total, steps); if `window` is a
    list, the host times around the timed region are appended to it."""
    stream = torch.cuda.Stream()
    per_graph = n_copies * max(1, min(50, K) // n_copies)
    with torch.cuda.stream(stream):
        for i in range(max(W, 1)):
            launch(i % n_copies)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(per_graph):
            launch(i % n_copies)
    reps, rem = divmod(K, per_graph)
    with torch.cuda.stream(stream):
        g.replay()  # graph warm-up
    stream.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_host0 = time.time()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        for i in range(rem):
            launch(i % n_copies)
        e1.record(stream)
    stream.synchronize()
    torch.cuda.synchronize()
    if window is not None:
        window += [t_host0, time.time()]
    if dist is not None:
        dist.barrier()
    ms = e0.elapsed_time(e1)
    del g
    return ms, K


def time_graph_repeats(torch, launch, n_copies, K, W, dist=None, repeats=5, soak_s=0.25, window=None):
    """The headline's timing: capture one graph, then `repeats` timed
    regions of exactly K steps each (CUDA events on the launching stream,
    barrier + device synchronise on both sides), each region preceded by
    about soak_s of untimed replays so that the clocks sampled around the
    regions are the clocks under this load.  Returns the per-region times
    (ms, max over ranks) and the graph, kept for latency probes."""
    stream = torch.cuda.Stream()
    per_graph = n_copies * max(1, min(50, K) // n_copies)
    with torch.cuda.stream(stream):
        for i in range(max(W, 1)):
            launch(i % n_copies)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(per_graph):
            launch(i % n_copies)
    reps, rem = divmod(K, per_graph)
    with torch.cuda.stream(stream):
        g.replay()  # graph warm-up
    stream.synchronize()
    # replays needed for ~soak_s, from one timed replay
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        g.replay()
        e1.record(stream)
    stream.synchronize()
    n_soak = int(max(0, min(20000, soak_s * 1e3 / max(e0.elapsed_time(e1), 1e-3))))
    out = []
    t_host0 = time.time()
    for r in range(repeats):
        with torch.cuda.stream(stream):
            for _ in range(n_soak):
                g.replay()
        stream.synchronize()
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            for i in range(rem):
                launch(i % n_copies)
            e1.record(stream)
        stream.synchronize()
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        out.append(max_over_ranks(torch, dist, e0.elapsed_time(e1)))
    if window is not None:
        window += [t_host0, time.time()]
    del g
    return out


def step_latency_us(torch, launch, n_copies, n=21):
    """Device time of ONE step, graph-launched (one single-step graph per
    input copy, copies rotated so the operands are not in L2): median of n."""
    stream = torch.cuda.Stream()
    graphs = []
    for i in range(n_copies):
        with torch.cuda.stream(stream):
            launch(i)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            launch(i)
        graphs.append(g)
    ts = []
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for r in range(n + 1):
        with torch.cuda.stream(stream):
            e0.record(stream)
            graphs[r % n_copies].replay()
            e1.record(stream)
        stream.synchronize()
        if r:
            ts.append(e0.elapsed_time(e1) * 1e3)
    del graphs
    return round(statistics.median(ts), 2)


def max_over_ranks(torch, dist, x, device="cuda"):
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(torch, dist, x, device="cuda"):
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# --------------------------------------------------------------- workloads --

def prefill_workload(torch, fa, W_, c, l2):
    q0, k0, v0 = W_.prefill_inputs(c)
    mods = c.name == W_.MODS_C2.name  # every score modifier on: ALiBi distance mask, softcap, sinks
    m0 = W_.distance_mask(c.Sq, c.Sk, causal=True) if mods else None
    s0 = W_.random_sinks(c.Hq, seed=c.seed) if mods else None
    foot = (q0.numel() + k0.numel() + v0.numel()) * 2 + c.B * c.Hq * c.Sq * (c.dv * 4 + 4)
    if mods:
        foot += m0.numel() * 2
    n = rotation_copies(foot, l2)
    bufs = []
    for i in range(n):
        q, k, v = q0.cuda(), k0.cuda(), v0.cuda()
        o = torch.empty(c.B, c.Hq, c.Sq, c.dv, device="cuda")
        lse = torch.empty(c.B, c.Hq, c.Sq, device="cuda")
        extra = (m0.cuda(), s0.cuda()) if mods else (None, None)
        bufs.append((q, k, v, o, lse) + extra)
    import ctypes
    lib = fa.load()
    if mods:
        params = [fa.fwd_params(q, k, v, o, lse, c.scale, c.causal, mask=m, max_bias=W_.MODS_C2_MAX_BIAS,
                                softcap=W_.MODS_C2_SOFTCAP, sinks=sk) for (q, k, v, o, lse, m, sk) in bufs]
    else:
        params = [fa.fwd_params(q, k, v, o, lse, c.scale, c.causal) for (q, k, v, o, lse, _, _) in bufs]

    def launch(i):
        st = lib.fa_fwd(ctypes.byref(params[i]), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        if st != 0:
            raise RuntimeError(lib.fa_last_error().decode())

    launch.keep = bufs  # the launches hold raw pointers into these tensors
    return launch, n, foot, 1


def quant_prefill_workload(torch, fa, W_, c, qtype, l2, dequant_only=False):
    """Prefill over quantised K/V the pages' way: one fa_kv_dequant_n launch
    (K rows and V rows) into bf16 buffers, then fa_fwd.  With dequant_only,
    the step is the dequant launch alone (its HBM roofline)."""
    import ctypes
    q0 = W_.randn_bf16((c.B, c.Hq, c.Sq, c.dk), 1000 + c.seed)
    kb0 = W_.random_quant_rows((c.B, c.Hkv, c.Sk), c.dk, qtype, c.seed)
    vb0 = W_.random_quant_rows((c.B, c.Hkv, c.Sk), c.dv, qtype, c.seed + 100)
    kv_scale = W_.FP8_SCALE if qtype == "fp8_e4m3" else 1.0
    kv_bf16 = c.B * c.Hkv * c.Sk * (c.dk + c.dv) * 2
    dq_bytes = kb0.numel() + vb0.numel() + kv_bf16  # quantised blocks read + bf16 rows written
    foot = q0.numel() * 2 + dq_bytes + c.B * c.Hq * c.Sq * (c.dv * 4 + 4)
    n = rotation_copies(foot, l2)
    lib = fa.load()
    bufs, params = [], []
    for i in range(n):
        q, kb, vb = q0.cuda(), kb0.cuda(), vb0.cuda()
        kbuf = torch.empty(c.B, c.Hkv, c.Sk, c.dk, device="cuda", dtype=torch.bfloat16)
        vbuf = torch.empty(c.B, c.Hkv, c.Sk, c.dv, device="cuda", dtype=torch.bfloat16)
        o = torch.empty(c.B, c.Hq, c.Sq, c.dv, device="cuda")
        lse = torch.empty(c.B, c.Hq, c.Sq, device="cuda")
        bufs.append((q, kb, vb, kbuf, vbuf, o, lse))
        pkv = (fa.KvDequantParams * 2)(
            fa.kv_dequant_params(kb.view(-1, kb.shape[-1]), qtype, c.dk, kbuf.view(-1, c.dk), kv_scale),
            fa.kv_dequant_params(vb.view(-1, vb.shape[-1]), qtype, c.dv, vbuf.view(-1, c.dv), kv_scale))
        pf = fa.fwd_params(q, kbuf, vbuf, o, lse, c.scale, c.causal)
        params.append((pkv, pf))

    def launch(i):
        st_ = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        pkv, pf = params[i]
        st = lib.fa_kv_dequant_n(pkv, 2, st_)
        if st == 0 and not dequant_only:
            st = lib.fa_fwd(ctypes.byref(pf), st_)
        if st != 0:
            raise RuntimeError(lib.fa_last_error().decode())

    launch.keep = bufs
    return launch, n, dq_bytes, 1 if dequant_only else 2


def paged_prefill_workload(torch, fa, W_, c, l2):
    """Chunked prefill over the paged cache: one fa_prefill_paged per step."""
    import ctypes
    q0, kc0, vc0, table0, sl0 = W_.paged_prefill_inputs(c)
    foot = (q0.numel() + kc0.numel() + vc0.numel()) * 2 + c.B * c.Hq * c.Sq * (c.d * 4 + 4)
    n = rotation_copies(foot, l2)
    lib = fa.load()
    bufs, params = [], []
    for i in range(n):
        q, kc, vc, tb, sl = q0.cuda(), kc0.cuda(), vc0.cuda(), table0.cuda(), sl0.cuda()
        o = torch.empty(c.B, c.Hq, c.Sq, c.d, device="cuda")
        lse = torch.empty(c.B, c.Hq, c.Sq, device="cuda")
        bufs.append((q, kc, vc, tb, sl, o, lse))
        params.append(fa.prefill_paged_params(q, kc, vc, tb, sl, o, lse, c.scale, c.causal))

    def launch(i):
        st = lib.fa_prefill_paged(ctypes.byref(params[i]), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        if st != 0:
            raise RuntimeError(lib.fa_last_error().decode())

    launch.keep = bufs
    return launch, n, c.flops(sl0), 1


def mla_tail_workload(torch, fa, W_, c, l2):
    """The MLA decode tail: one fa_mla_tail (out-absorb GEMM, o-projection
    GEMM, split reduce) per step."""
    import ctypes
    o0, wa0, wo0 = W_.mla_tail_inputs(c)
    foot = c.bytes
    n = rotation_copies(foot, l2)
    lib = fa.load()
    bufs, params = [], []
    for i in range(n):
        o, wa, wo = o0.cuda(), wa0.cuda(), wo0.cuda()
        y = torch.empty(c.T, c.Hd, device="cuda")
        ws = torch.empty(max(fa.mla_tail_workspace_bytes(o, wa, wo), 256), device="cuda", dtype=torch.uint8)
        bufs.append((o, wa, wo, y, ws))
        params.append(fa.mla_tail_params(o, wa, wo, y, 0, ws))

    def launch(i):
        st = lib.fa_mla_tail(ctypes.byref(params[i]), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        if st != 0:
            raise RuntimeError(lib.fa_last_error().decode())

    launch.keep = bufs
    return launch, n, c.bytes, 3


def latent_prefill_workload(torch, fa, W_, c, l2):
    """MLA prefill in latent space: one contiguous-row fa_decode_gather per
    step (+ its LSE combine)."""
    import ctypes
    q0, r0 = W_.latent_prefill_inputs(c)
    foot = (q0.numel() + r0.numel()) * 2 + c.Sq * c.Hq * (512 * 4 + 4)
    n = rotation_copies(foot, l2)
    lib = fa.load()
    bufs, params = [], []
    for i in range(n):
        q, rows = q0.cuda(), r0.cuda()
        qpos = torch.arange(c.Sk - c.Sq, c.Sk, device="cuda", dtype=torch.int32) if c.causal else None
        o = torch.empty(c.Sq, c.Hq, 512, device="cuda")
        lse = torch.empty(c.Sq, c.Hq, device="cuda")
        ws = torch.empty(max(fa.gather_workspace_bytes(q, rows, None, 0, topk=c.Sk, dk=c.dk), 256), device="cuda",
                         dtype=torch.uint8)
        bufs.append((q, rows, qpos, o, lse, ws))
        params.append(fa.gather_params(q, rows, None, None, qpos, o, lse, 1.0 / math.sqrt(c.dk), 0, ws, topk=c.Sk,
                                       dk=c.dk, v_offset=64 if c.dk == 576 else 0))

    def launch(i):
        st = lib.fa_decode_gather(ctypes.byref(params[i]), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        if st != 0:
            raise RuntimeError(lib.fa_last_error().decode())

    launch.keep = bufs
    return launch, n, c.flops, 2


def paged_workload(torch, fa, W_, c, l2, q8=False, fp8=False, q4=False):
    """Paged decode (decode kernel + LSE combine per step); q8 / q4 / fp8:
    the caches hold q8_0 rows, q4_0 rows or fp8 e4m3 bytes, converted inside
    the decode kernel."""
    q0, kc0, vc0, tb0, sl0 = W_.paged_inputs(c)
    if q8:
        kc0, vc0 = W_.paged_q8_caches(c, kc0.shape[0])
    elif q4:
        kc0, vc0 = W_.paged_q4_caches(c, kc0.shape[0])
    elif fp8:
        kc0, vc0 = W_.paged_fp8_caches(c, kc0.shape[0])
    byts = W_.paged_bytes(c, sl0, tb0.shape[1], q8=q8, fp8=fp8, q4=q4)
    foot = (kc0.numel() + vc0.numel()) * kc0.element_size()
    n = rotation_copies(foot, l2)
    import ctypes
    lib = fa.load()
    bufs, params = [], []
    for i in range(n):
        q, kc, vc, tb, sl = q0.cuda(), kc0.cuda(), vc0.cuda(), tb0.cuda(), sl0.cuda()
        o = torch.empty(c.B, c.Hq, c.dv, device="cuda")
        lse = torch.empty(c.B, c.Hq, device="cuda")
        nws = fa.paged_workspace_bytes(q, kc, vc, tb, sl, 0)
        ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
        bufs.append((q, kc, vc, tb, sl, o, lse, ws))
        params.append(fa.paged_params(q, kc, vc, tb, sl, o, lse, c.scale, 0, ws,
                                      kv_type="fp8_e4m3" if fp8 else None, k_scale=W_.FP8_SCALE,
                                      v_scale=W_.FP8_SCALE))

    def launch(i):
        st = lib.fa_decode_paged(ctypes.byref(params[i]), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        if st != 0:
            raise RuntimeError(lib.fa_last_error().decode())

    launch.keep = bufs  # the launches hold raw pointers into these tensors
    return launch, n, byts, 2


def latent_workload(torch, fa, W_, c, l2):
    q0, rows0, idx0, qpos0 = W_.latent_inputs(c)
    nvis = W_.latent_visible(idx0, qpos0)
    byts = W_.latent_bytes(c, nvis)
    flops = W_.latent_flops(c, nvis)
    n = rotation_copies(byts, l2)
    import ctypes
    lib = fa.load()
    bufs, params = [], []
    for i in range(n):
        q, rows, idx, qpos = q0.cuda(), rows0.cuda(), idx0.cuda(), qpos0.cuda()
        o = torch.empty(c.T, c.Hq, c.dv, device="cuda")
        lse = torch.empty(c.T, c.Hq, device="cuda")
        nws = fa.gather_workspace_bytes(q, rows, idx, 0)
        ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
        bufs.append((q, rows, idx, qpos, o, lse, ws))
        params.append(fa.gather_params(q, rows, idx, None, qpos, o, lse, c.scale, 0, ws))

    def launch(i):
        st = lib.fa_decode_gather(ctypes.byref(params[i]), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        if st != 0:
            raise RuntimeError(lib.fa_last_error().decode())

    launch.keep = bufs  # the launches hold raw pointers into these tensors
    return launch, n, (byts, flops), 2


HBM_SPEC_GBS = 8000.0  # B200 HBM3e, nominal (the ~8 TB/s the decode target is stated against)


def roofline(bound, achieved, peak, unit, traffic):
    r = {"bound": bound, "achieved": round(achieved, 2), "peak": peak, "unit": unit,
         "frac": round(achieved / peak, 4), "traffic": traffic}
    if bound == "tensor":
        # the long-loop cuBLAS figure, for kernels timed under sustained load
        # (the headline's regions follow a quarter second of replays)
        pk, _ = load_peaks()
        r["peak_sustained"] = pk["bf16_tflops_sustained"]
        r["frac_sustained"] = round(achieved / pk["bf16_tflops_sustained"], 4)
    if bound == "hbm":
        # the measured peak is a copy (half reads, half writes); a read-mostly
        # kernel can pass it, so the nominal figure is given beside it
        r["peak_spec"] = HBM_SPEC_GBS
        r["frac_of_spec"] = round(achieved / HBM_SPEC_GBS, 4)
        if achieved > peak:
            r["note"] = "above the measured copy bandwidth (a copy is half writes); see frac_of_spec"
    return r


# ------------------------------------------------------------ CPU baseline --

def cpu_baseline_prefill(c, budget_s=10.0, max_s=30.0, max_slices=None):
    """Time the fp64 oracle on whole (batch, head) slices of the workload
    (all query rows, causal mask as in the workload) until ~budget_s."""
    import numpy as np

    import oracle
    from attention_attn_fwd_11_b200 import workloads as W_

    q, k, v = W_.prefill_inputs(c)
    qb, kb, vb = W_.bits(q), W_.bits(k), W_.bits(v)
    grp = c.Hq // c.Hkv
    slices = [(b, h) for b in range(c.B) for h in range(c.Hq)]
    if max_slices:
        slices = slices[:max_slices]
    done, t0 = 0, time.perf_counter()
    for (b, h) in slices:
        oracle.attention(np.ascontiguousarray(qb[b:b + 1, h:h + 1]), np.ascontiguousarray(kb[b:b + 1, h // grp:h // grp + 1]),
                         np.ascontiguousarray(vb[b:b + 1, h // grp:h // grp + 1]), c.scale, c.causal)
        done += 1
        el = time.perf_counter() - t0
        if el >= budget_s or el >= max_s:
            break
    el = time.perf_counter() - t0
    flops = c.flops * done / len([(b, h) for b in range(c.B) for h in range(c.Hq)])
    return {"value": round(flops / el / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "%d of %d (batch, head) slices, all %d query rows each, %.1f s" % (done, c.B * c.Hq, c.Sq, el)}


def cpu_baseline_prefill_rows(c, n_rows=64, seed=0):
    """Full (non-causal) prefill: every (batch, head) on a seeded sample of
    n_rows query rows.  Rows are independent, so the sampled rows are the
    exact oracle rows; the rate is extrapolated by FLOPs."""
    import numpy as np

    import oracle
    from attention_attn_fwd_11_b200 import workloads as W_

    assert not c.causal
    q, k, v = W_.prefill_inputs(c)
    rows = np.sort(np.random.default_rng(seed).choice(c.Sq, n_rows, replace=False))
    qb = np.ascontiguousarray(W_.bits(q)[:, :, rows])
    kb, vb = W_.bits(k), W_.bits(v)
    grp = c.Hq // c.Hkv
    t0 = time.perf_counter()
    for h in range(c.Hq):
        oracle.attention(np.ascontiguousarray(qb[:, h:h + 1]), np.ascontiguousarray(kb[:, h // grp:h // grp + 1]),
                         np.ascontiguousarray(vb[:, h // grp:h // grp + 1]), c.scale, False)
    el = time.perf_counter() - t0
    flops = c.flops * n_rows / c.Sq
    return {"value": round(flops / el / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "%d of %d query rows (seeded) of every (batch, head), %.1f s; rate extrapolated by FLOPs" % (
                n_rows, c.Sq, el)}


def cpu_baseline_paged(c, budget_s=6.0):
    """Paged decode: whole sequences, one at a time, until ~budget_s;
    GB/s of the sampled sequences' algorithmic bytes."""
    import oracle
    from attention_attn_fwd_11_b200 import workloads as W_

    q, kc, vc, tb, sl = W_.paged_inputs(c)
    qb, kb, vb = W_.bits(q), W_.bits(kc), W_.bits(vc)
    tbn, sln = tb.numpy(), sl.numpy()
    done, byts, t0 = 0, 0, time.perf_counter()
    for b in range(c.B):
        oracle.decode_paged(qb[b:b + 1], kb, vb, tbn[b:b + 1], sln[b:b + 1], c.scale)
        n = int(sln[b])
        byts += n * c.Hkv * (c.dk + c.dv) * 2 + (n + c.block_size - 1) // c.block_size * 4 + 4 + \
            c.Hq * (c.dk * 2 + c.dv * 4 + 4)
        done += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    el = time.perf_counter() - t0
    return {"value": round(byts / el / 1e9, 4), "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "%d of %d sequences, %.1f s" % (done, c.B, el)}


def cpu_baseline_latent(c, budget_s=6.0):
    """Latent sparse decode: whole tokens, one at a time, until ~budget_s;
    GB/s of the sampled tokens' algorithmic bytes."""
    import oracle
    from attention_attn_fwd_11_b200 import workloads as W_

    q, rows, idx, qpos = W_.latent_inputs(c)
    qb, rb = W_.bits(q), W_.bits(rows)
    idn, qpn = idx.numpy(), qpos.numpy()
    done, byts, t0 = 0, 0, time.perf_counter()
    for t in range(c.T):
        oracle.decode_latent(qb[t:t + 1], rb, idn[t:t + 1], c.scale, c.dk, c.dv, c.v_offset, None, qpn[t:t + 1])
        nvis = W_.latent_visible(idx[t:t + 1], qpos[t:t + 1])
        byts += nvis * max(c.dk, c.v_offset + c.dv) * 2 + c.topk * 4 + 4 + c.Hq * (c.dk * 2 + c.dv * 4 + 4)
        done += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    el = time.perf_counter() - t0
    return {"value": round(byts / el / 1e9, 4), "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "%d of %d tokens, %.1f s" % (done, c.T, el)}


# -------------------------------------------------------------------- main --

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from attention_attn_fwd_11_b200 import workloads as W_

    c = W_.CAUSAL_MHA
    import numpy as np

    import oracle

    q, k, v = W_.prefill_inputs(c)
    qb, kb, vb = W_.bits(q), W_.bits(k), W_.bits(v)
    slices = [(b, h) for b in range(c.B) for h in range(c.Hq)]

    def step(i):
        b, h = slices[i % len(slices)]
        oracle.attention(np.ascontiguousarray(qb[b:b + 1, h:h + 1]), np.ascontiguousarray(kb[b:b + 1, h:h + 1]),
                         np.ascontiguousarray(vb[b:b + 1, h:h + 1]), c.scale, c.causal)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    el = time.perf_counter() - t0
    flops = c.flops / len(slices) * args.steps
    val = flops / el / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": round(val, 6), "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el * 1e3 / max(args.steps, 1), 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": c.name, "B": c.B, "Hq": c.Hq, "Hkv": c.Hkv, "Sq": c.Sq, "Sk": c.Sk, "d": c.dk,
                       "causal": c.causal, "step": "one (batch, head) slice of the workload, all query rows"},
            "cpu_baseline": {"value": round(val, 6), "unit": "TFLOP/s", "kind": "oracle",
                             "cores": oracle.num_threads(),
                             "sample": "one (batch, head) slice per step (1/%d of the workload)" % len(slices)},
            "e2e": {"value": round(val, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_only(args):
    """One workload alone, eager or graph-launched: the command the ncu
    profiles under profiles/ were taken with."""
    import torch

    from attention_attn_fwd_11_b200 import fa
    from attention_attn_fwd_11_b200 import workloads as W_

    torch.cuda.set_device(0)
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    table = {c.name: c for c in (W_.TINY_FULL, W_.CAUSAL_MHA, W_.GQA_FULL, W_.MODS_C2, W_.CAUSAL_DK192,
                                 W_.CAUSAL_DK192_DV192, W_.CAUSAL_DK320, W_.CAUSAL_DK576, W_.CAUSAL_DK512,
                                 W_.PAGED_GQA, W_.LATENT_SPARSE,
                                 W_.QUANT_C2, W_.PAGED_PREFILL, W_.MLA_TAIL)}
    table[W_.PAGED_Q8_NAME] = W_.PAGED_GQA
    table[W_.PAGED_FP8_NAME] = W_.PAGED_GQA
    table[W_.PAGED_Q4_NAME] = W_.PAGED_GQA
    table[W_.LATENT_PREFILL.name] = W_.LATENT_PREFILL
    table[W_.LATENT_PREFILL_512.name] = W_.LATENT_PREFILL_512
    table["kv_dequant_" + W_.QUANT_C2.name] = W_.QUANT_C2
    table[W_.FP8_C2.name] = W_.FP8_C2
    table["kv_dequant_" + W_.FP8_C2.name] = W_.FP8_C2
    if args.only not in table:
        raise SystemExit("unknown workload %r; one of %s" % (args.only, sorted(table)))
    c = table[args.only]
    if c is W_.QUANT_C2 or c is W_.FP8_C2:
        only_dq = args.only.startswith("kv_dequant_")
        qt = W_.QUANT_C2_TYPE if c is W_.QUANT_C2 else "fp8_e4m3"
        launch, n, work, kpl = quant_prefill_workload(torch, fa, W_, c, qt, l2, dequant_only=only_dq)
        unit, amount = ("GB/s", work / 1e9) if only_dq else ("TFLOP/s", c.flops / 1e12)
    elif isinstance(c, W_.PrefillCase):
        launch, n, work, kpl = prefill_workload(torch, fa, W_, c, l2)
        unit, amount = "TFLOP/s", c.flops / 1e12
    elif isinstance(c, W_.LatentPrefillCase):
        launch, n, work, kpl = latent_prefill_workload(torch, fa, W_, c, l2)
        unit, amount = "TFLOP/s", work / 1e12
    elif isinstance(c, W_.MlaTailCase):
        launch, n, work, kpl = mla_tail_workload(torch, fa, W_, c, l2)
        unit, amount = "GB/s", work / 1e9
    elif isinstance(c, W_.PagedPrefillCase):
        launch, n, work, kpl = paged_prefill_workload(torch, fa, W_, c, l2)
        unit, amount = "TFLOP/s", work / 1e12
    elif isinstance(c, W_.PagedCase):
        launch, n, work, kpl = paged_workload(torch, fa, W_, c, l2, q8=args.only == W_.PAGED_Q8_NAME,
                                              fp8=args.only == W_.PAGED_FP8_NAME, q4=args.only == W_.PAGED_Q4_NAME)
        unit, amount = "GB/s", work / 1e9
    else:
        launch, n, work, kpl = latent_workload(torch, fa, W_, c, l2)
        unit, amount = "GB/s", work[0] / 1e9
    if args.eager:
        s = torch.cuda.Stream()
        with torch.cuda.stream(s):
            for i in range(args.warmup):
                launch(i % n)
            s.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            for i in range(args.steps):
                launch(i % n)
            e1.record(s)
        s.synchronize()
        ms = e0.elapsed_time(e1)
    else:
        ms, _ = time_graph(torch, launch, n, args.steps, max(args.warmup, 1))
    assert fa.device_error() == 0
    per = ms / max(args.steps, 1)
    print(json.dumps({"workload": c.name, "steps": args.steps, "ms_per_step": round(per, 5),
                      "value": round(amount / (per * 1e-3), 2), "unit": unit, "l2_copies": n,
                      "eager": bool(args.eager)}), flush=True)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.only:
        return run_only(args)

    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist_

        torch.cuda.set_device(local)
        dist_.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=torch.device("cuda", local))
        dist = dist_
    else:
        torch.cuda.set_device(0)
    from attention_attn_fwd_11_b200 import fa
    from attention_attn_fwd_11_b200 import workloads as W_

    fa.load()
    peaks, peak_src = load_peaks()
    l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
    K, Wm = args.steps, max(args.warmup, 3)
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    phys = int(vis.split(",")[local]) if vis and vis.split(",")[local].strip().isdigit() else local

    # ---- headline: causal MHA prefill ----
    c = W_.CAUSAL_MHA
    launch, ncopy, foot, kpl = prefill_workload(torch, fa, W_, c, l2)
    sampler = ClockSampler(phys)
    sampler.start()
    time.sleep(0.3)
    win = []
    R = 5
    region_ms = time_graph_repeats(torch, launch, ncopy, K, Wm, dist, repeats=R, soak_s=args.soak_s, window=win)
    clocks = sampler.stop(win[0], win[1])
    clocks["window_s"] = round(win[1] - win[0], 3)
    clocks["note"] = "samples over the %d timed regions and the untimed replays between them" % R
    # the line's value is the median region: ms_per_step * steps = that region's time
    ms = statistics.median(region_ms)
    steps = K
    total_flops = sum_over_ranks(torch, dist, c.flops * steps)
    value = total_flops / (ms * 1e-3) / 1e12
    per_launch_ms = ms / steps
    achieved = c.flops / (per_launch_ms * 1e-3) / 1e12
    latency = step_latency_us(torch, launch, ncopy)
    assert fa.device_error() == 0, "device error during the timed region"
    region_vals = sorted(c.flops * K / (m * 1e-3) / 1e12 * (world if dist is not None else 1) for m in region_ms)

    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": steps,
        "warmup": Wm, "ms_per_step": round(per_launch_ms, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16)",
        "config": {"workload": c.name, "B": c.B, "Hq": c.Hq, "Hkv": c.Hkv, "Sq": c.Sq, "Sk": c.Sk, "d": c.dk,
                   "causal": c.causal, "out": "fp32 O + fp32 LSE",
                   "l2": "%d rotating input copies (%.0f MB per step, L2 %.0f MB)" % (ncopy, foot / 1e6, l2 / 1e6),
                   "timing": "CUDA graph replay, CUDA events on the launching stream",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "roofline": roofline("tensor", achieved, peaks["bf16_tflops"], "TFLOP/s", NCU_TRAFFIC.get(c.name)),
        "peak_source": peak_src + " (bf16_tflops burst; kernel timed alone)",
        "gpu_launches": R * steps * kpl,
        "repeats": {"regions": R, "steps_per_region": K, "value": "median region",
                    "ms_per_region": [round(m, 4) for m in region_ms],
                    "min": round(region_vals[0], 2), "max": round(region_vals[-1], 2),
                    "spread_pct": round(100.0 * (region_vals[-1] - region_vals[0]) / region_vals[len(region_vals) // 2], 2)},
        "latency_us": latency,
        "latency_note": "one step (prefill kernel), graph-launched, cold inputs: median of 21",
        "clocks": clocks,
    }

    # ---- e2e through the public API with pinned host buffers ----
    # Every step copies its Q, K, V from pinned host memory, runs fa.fwd and
    # copies O and the LSE back to pinned host memory.  Steps are pipelined
    # the way a serving loop runs them: two device buffer sets, uploads on
    # one copy stream and downloads on another, so the upload of step i + 1
    # and the download of step i - 1 overlap the compute of step i (PCIe is
    # full duplex).  Events order each buffer set's reuse.
    q0, k0, v0 = W_.prefill_inputs(c)
    hq, hk, hv = q0.pin_memory(), k0.pin_memory(), v0.pin_memory()
    ho = [torch.empty(c.B, c.Hq, c.Sq, c.dv).pin_memory() for _ in range(2)]
    hl = [torch.empty(c.B, c.Hq, c.Sq).pin_memory() for _ in range(2)]
    dev = [dict(q=torch.empty_like(q0, device="cuda"), k=torch.empty_like(k0, device="cuda"),
                v=torch.empty_like(v0, device="cuda"), o=torch.empty(c.B, c.Hq, c.Sq, c.dv, device="cuda"),
                lse=torch.empty(c.B, c.Hq, c.Sq, device="cuda")) for _ in range(2)]
    s_up, s_cmp, s_dn = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_up = [torch.cuda.Event() for _ in range(2)]     # inputs of set j landed
    ev_cmp = [torch.cuda.Event() for _ in range(2)]    # compute on set j done
    ev_dn = [torch.cuda.Event() for _ in range(2)]     # outputs of set j read back
    Ke = max(3, min(K, 30))

    def e2e_step(i):
        j = i % 2
        d = dev[j]
        with torch.cuda.stream(s_up):
            s_up.wait_event(ev_cmp[j])  # the compute of step i - 2 has read set j
            d["q"].copy_(hq, non_blocking=True)
            d["k"].copy_(hk, non_blocking=True)
            d["v"].copy_(hv, non_blocking=True)
            ev_up[j].record(s_up)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_up[j])
            s_cmp.wait_event(ev_dn[j])  # the download of step i - 2 has read O of set j
            fa.fwd(d["q"], d["k"], d["v"], scale=c.scale, causal=c.causal, out=d["o"], lse=d["lse"])
            ev_cmp[j].record(s_cmp)
        with torch.cuda.stream(s_dn):
            s_dn.wait_event(ev_cmp[j])
            ho[j].copy_(d["o"], non_blocking=True)
            hl[j].copy_(d["lse"], non_blocking=True)
            ev_dn[j].record(s_dn)

    for i in range(Wm):
        e2e_step(i)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_up)
    s_cmp.wait_event(e0)
    s_dn.wait_event(e0)
    for i in range(Ke):
        e2e_step(i)
    # the timed region ends once the last step's outputs are on the host
    s_up.wait_stream(s_dn)
    e1.record(s_up)
    torch.cuda.synchronize()
    ems = max_over_ranks(torch, dist, e0.elapsed_time(e1))
    e2e_val = sum_over_ranks(torch, dist, c.flops * Ke) / (ems * 1e-3) / 1e12
    result["e2e"] = {"value": round(e2e_val, 3), "unit": "TFLOP/s",
                     "h2d_bytes_per_step": int((q0.numel() + k0.numel() + v0.numel()) * 2),
                     "d2h_bytes_per_step": int(c.B * c.Hq * c.Sq * (c.dv + 1) * 4), "steps": Ke,
                     "pipelining": "two buffer sets; uploads, compute and downloads on three streams"}
    result["gpu_launches"] += Ke  # the e2e steps launch the prefill kernel too
    del hq, hk, hv, ho, hl, dev

    # ---- the path's other workloads ----
    if not args.no_secondary:
        wl = {}
        Ks = 200
        for cc in (W_.TINY_FULL, W_.GQA_FULL, W_.MODS_C2, W_.CAUSAL_DK192, W_.CAUSAL_DK192_DV192,
                   W_.CAUSAL_DK320, W_.CAUSAL_DK576):
            launch, ncopy, foot, kpl = prefill_workload(torch, fa, W_, cc, l2)
            ms2, st2 = time_graph(torch, launch, ncopy, Ks, Wm, dist)
            ms2 = max_over_ranks(torch, dist, ms2)
            per = ms2 / st2
            ach = cc.flops / (per * 1e-3) / 1e12
            wl[cc.name] = {"value": round(sum_over_ranks(torch, dist, cc.flops * st2) / (ms2 * 1e-3) / 1e12, 2),
                           "unit": "TFLOP/s", "ms_per_step": round(per, 5), "steps": st2, "l2_copies": ncopy,
                           "roofline": roofline("tensor", ach, peaks["bf16_tflops"], "TFLOP/s",
                                                NCU_TRAFFIC.get(cc.name))}
            result["gpu_launches"] += st2 * kpl
            del launch
        # prefill over q8_0 K/V: two dequant launches + fa_fwd per step
        qc = W_.QUANT_C2
        launch, ncopy, dq_bytes, kpl = quant_prefill_workload(torch, fa, W_, qc, W_.QUANT_C2_TYPE, l2)
        ms2, st2 = time_graph(torch, launch, ncopy, Ks, Wm, dist)
        ms2 = max_over_ranks(torch, dist, ms2)
        per = ms2 / st2
        result["gpu_launches"] += st2 * kpl
        del launch
        launch, ncopy_d, _, kpl_d = quant_prefill_workload(torch, fa, W_, qc, W_.QUANT_C2_TYPE, l2, dequant_only=True)
        msd, std_ = time_graph(torch, launch, ncopy_d, Ks, Wm, dist)
        msd = max_over_ranks(torch, dist, msd)
        perd = msd / std_
        result["gpu_launches"] += std_ * kpl_d
        del launch
        wl[qc.name] = {"value": round(sum_over_ranks(torch, dist, qc.flops * st2) / (ms2 * 1e-3) / 1e12, 2),
                       "unit": "TFLOP/s", "ms_per_step": round(per, 5), "steps": st2, "l2_copies": ncopy,
                       "kernels": "kv_dequant (%s K and V rows -> bf16, one launch) + prefill" % W_.QUANT_C2_TYPE,
                       "dequant": {"ms_per_step": round(perd, 5), "bytes_per_step": dq_bytes,
                                   "roofline": roofline("hbm", dq_bytes / (perd * 1e-3) / 1e9, peaks["hbm_gbs"],
                                                        "GB/s", NCU_TRAFFIC.get("kv_dequant " + qc.name))}}
        # chunked prefill over the paged cache
        ppc = W_.PAGED_PREFILL
        launch, ncopy, pflops, kpl = paged_prefill_workload(torch, fa, W_, ppc, l2)
        ms2, st2 = time_graph(torch, launch, ncopy, Ks, Wm, dist)
        ms2 = max_over_ranks(torch, dist, ms2)
        per = ms2 / st2
        ach = pflops / (per * 1e-3) / 1e12
        wl[ppc.name] = {"value": round(sum_over_ranks(torch, dist, pflops * st2) / (ms2 * 1e-3) / 1e12, 2),
                        "unit": "TFLOP/s", "ms_per_step": round(per, 5), "steps": st2, "l2_copies": ncopy,
                        "flops_per_step": pflops,
                        "roofline": roofline("tensor", ach, peaks["bf16_tflops"], "TFLOP/s",
                                             NCU_TRAFFIC.get(ppc.name))}
        result["gpu_launches"] += st2 * kpl
        del launch
        pc = W_.PAGED_GQA
        launch, ncopy, byts, kpl = paged_workload(torch, fa, W_, pc, l2)
        ms2, st2 = time_graph(torch, launch, ncopy, Ks, Wm, dist)
        ms2 = max_over_ranks(torch, dist, ms2)
        per = ms2 / st2
        ach = byts / (per * 1e-3) / 1e9
        wl[pc.name] = {"value": round(sum_over_ranks(torch, dist, byts * st2) / (ms2 * 1e-3) / 1e9, 1), "unit": "GB/s",
                       "ms_per_step": round(per, 5), "steps": st2, "l2_copies": ncopy, "bytes_per_step": byts,
                       "roofline": roofline("hbm", ach, peaks["hbm_gbs"], "GB/s", NCU_TRAFFIC.get(pc.name)),
                       "kernels": "paged decode + LSE combine"}
        result["gpu_launches"] += st2 * kpl
        del launch
        # the same decode over q8_0 caches (dequant prologue in the kernel)
        for qname, qkw in ((W_.PAGED_Q8_NAME, dict(q8=True)), (W_.PAGED_Q4_NAME, dict(q4=True)),
                           (W_.PAGED_FP8_NAME, dict(fp8=True))):
            launch, ncopy, byts, kpl = paged_workload(torch, fa, W_, pc, l2, **qkw)
            ms2, st2 = time_graph(torch, launch, ncopy, Ks, Wm, dist)
            ms2 = max_over_ranks(torch, dist, ms2)
            per = ms2 / st2
            ach = byts / (per * 1e-3) / 1e9
            wl[qname] = {"value": round(sum_over_ranks(torch, dist, byts * st2) / (ms2 * 1e-3) / 1e9, 1),
                         "unit": "GB/s", "ms_per_step": round(per, 5), "steps": st2, "l2_copies": ncopy,
                         "bytes_per_step": byts,
                         "roofline": roofline("hbm", ach, peaks["hbm_gbs"], "GB/s", NCU_TRAFFIC.get(qname)),
                         "kernels": "paged decode with the %s prologue + LSE combine" % (
                             "q8_0" if "q8" in qkw else ("q4_0" if "q4" in qkw else "fp8 e4m3"))}
            result["gpu_launches"] += st2 * kpl
            del launch
        try:
            lc = W_.LATENT_SPARSE
            launch, ncopy, (byts, flops), kpl = latent_workload(torch, fa, W_, lc, l2)
            ms2, st2 = time_graph(torch, launch, ncopy, Ks, Wm, dist)
            ms2 = max_over_ranks(torch, dist, ms2)
            per = ms2 / st2
            ach = byts / (per * 1e-3) / 1e9
            wl[lc.name] = {"value": round(sum_over_ranks(torch, dist, byts * st2) / (ms2 * 1e-3) / 1e9, 1),
                           "unit": "GB/s", "tflops": round(flops / (per * 1e-3) / 1e12, 2),
                           "ms_per_step": round(per, 5), "steps": st2, "l2_copies": ncopy, "bytes_per_step": byts,
                           "roofline": roofline("hbm", ach, peaks["hbm_gbs"], "GB/s", NCU_TRAFFIC.get(lc.name)),
                           "kernels": "latent gather decode + LSE combine"}
            result["gpu_launches"] += st2 * kpl
            del launch
        except Exception as e:  # report, never hide
            wl[W_.LATENT_SPARSE.name] = {"error": str(e)[:200]}
        # MLA decode tail (out-absorb + o-projection)
        mc = W_.MLA_TAIL
        launch, ncopy, byts, kpl = mla_tail_workload(torch, fa, W_, mc, l2)
        ms2, st2 = time_graph(torch, launch, ncopy, Ks, Wm, dist)
        ms2 = max_over_ranks(torch, dist, ms2)
        per = ms2 / st2
        ach = byts / (per * 1e-3) / 1e9
        wl[mc.name] = {"value": round(sum_over_ranks(torch, dist, byts * st2) / (ms2 * 1e-3) / 1e9, 1),
                       "unit": "GB/s", "tflops": round(mc.flops / (per * 1e-3) / 1e12, 2),
                       "ms_per_step": round(per, 5), "steps": st2, "l2_copies": ncopy, "bytes_per_step": byts,
                       "roofline": roofline("hbm", ach, peaks["hbm_gbs"], "GB/s", NCU_TRAFFIC.get(mc.name)),
                       "kernels": "out-absorb GEMM + o-projection GEMM (split K, cluster reduce)"}
        result["gpu_launches"] += st2 * kpl
        del launch
        result["workloads"] = wl
        assert fa.device_error() == 0, "device error in a secondary workload"

    # ---- CPU baseline: the oracle on this host, rank 0 at N = 1 only ----
    if world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline_prefill(c)
        wl = result.get("workloads")
        if wl is not None:  # the five configurations of the path, each beside its GPU number
            for name, fn in ((W_.TINY_FULL.name, lambda: cpu_baseline_prefill(W_.TINY_FULL)),
                             (W_.GQA_FULL.name, lambda: cpu_baseline_prefill_rows(W_.GQA_FULL)),
                             (W_.PAGED_GQA.name, lambda: cpu_baseline_paged(W_.PAGED_GQA)),
                             (W_.LATENT_SPARSE.name, lambda: cpu_baseline_latent(W_.LATENT_SPARSE))):
                if name in wl and "error" not in wl[name]:
                    wl[name]["cpu_baseline"] = fn()

    if rank == 0:
        print(json.dumps(result), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

#!/usr/bin/env python
"""Benchmark of the KDA hot path on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one ``kda_chunk_fwd_prologue`` over the largest length-sweep workload
(B=1, T=65536, H=96, dk=dv=128, bf16 raw q/k/v/z, FP32 beta logits, conv taps and
S0 -> out, S_T): the fused prologue (short conv k=4 + SiLU, gate, beta), the
chunk-local cumsum, A_kk / A_qk / UT / WY and the inter-chunk scan, inputs resident
in HBM.  Its inputs (8 GB) are larger than the 126 MB L2, so no flush is needed
between steps.  Under torchrun every rank runs its own batch (weak scaling, no
collective on the data path); ``value`` is the tokens of all ranks over the
slowest rank's time.

Also measured on rank 0 at N=1 (the ``rows`` object):
  * the prefill workload (B=1, T=4096, H=16), 20 timed calls with its own clock record;
  * the sweep at T=8192 and T=32768;
  * the output epilogue, the backward, the Kimi Linear softplus gate and the split of
    one sequence into four segments, all on the prefill shape;
  * the decode step and the decode step with its prologue (N=256, H=96);
  * the Complex-KDA workload (B=8, T=8192, H=32) next to unsigned KDA of the same shape.
``e2e`` is the same metric through the C ABI with host buffers, copies timed.
``cpu_baseline`` times the FP64 oracle on the host cores on a bounded sample.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import kda_workloads as W  # noqa: E402

METRIC = "chunk_kda fwd tokens/s & % of BF16 roofline; decode step state GB/s vs HBM"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 256 << 20

# algorithmic counts per token-head and per head (d = 128, C = 64): bf16 q,k,v,g,out
# (4*256 + 256 bytes) + bf16 beta; FP32 S0 and S_T per head; FLOPs of the
# triangular intra-chunk products, the three state GEMMs and the C x C inverse
PREFILL_FLOP_PER_TOKEN_HEAD = 5 * 64 * 128 + 6 * 128 * 128 + 64 * 64 / 3


def token_head_bytes(d, elt=2, beta_elt=2):
    return 4 * d * elt + d * elt + beta_elt


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


class ClockSampler:
    """Polls NVML (read-only) for SM clock and clock-event reasons while timing."""

    REASONS = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
               "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
               "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
               "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
               "hw_power_brake": "nvmlClocksEventReasonHwPowerBrakeSlowdown"}

    def __init__(self, device_index):
        self.samples, self.reasons, self.ok = [], set(), False
        self.max_mhz = None
        try:
            import pynvml as N
            N.nvmlInit()
            self.N = N
            self.h = N.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = N.nvmlDeviceGetMaxClockInfo(self.h, N.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
        self._stop = threading.Event()
        self._t = None

    def _sample(self):
        N = self.N
        try:
            self.samples.append(N.nvmlDeviceGetClockInfo(self.h, N.NVML_CLOCK_SM))
            r = N.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            for name, attr in self.REASONS.items():
                if r & getattr(N, attr, 0):
                    self.reasons.add(name)
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._t:
            self._sample()          # one more reading at the end of the timed region
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples)}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import torch.distributed as dist
        from datetime import timedelta
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, ws):
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- the headline workload
HEADLINE_T = W.SWEEP_T[-1]          # T = 65536, the largest length-sweep config
SWEEP_H, SWEEP_D = W.SWEEP["H"], W.SWEEP["dk"]
HEADLINE_WORKLOAD = (f"length sweep with the fused prologue, B=1 T={HEADLINE_T} H={SWEEP_H} dk=dv={SWEEP_D}: "
                     "kda_chunk_fwd_prologue (short conv k=4 + SiLU, bounded gate, beta, chunk_kda fwd)")


def sweep_alg_bytes(T, H=SWEEP_H, d=SWEEP_D):
    """Algorithmic bytes of kda_chunk_fwd_prologue on the sweep workload: per token-head raw
    q, k, v, z and out in bf16 and the FP32 beta logit; per head S0 and S_T (FP32) and the
    conv taps of q, k, v (bf16)."""
    return T * H * (4 * d * 2 + 4 + d * 2) + H * (2 * d * d * 4 + 3 * d * 4 * 2)


def oracle_sweep_sample(heads, tokens, seed):
    """A bounded sample of the sweep workload for the FP64 oracle: `heads` heads x `tokens`
    tokens drawn with the sweep recipe (same distributions and shapes per head; the oracle's
    time does not depend on the values)."""
    import numpy as np
    x = W.prologue_inputs(1, tokens, heads, SWEEP_D, SWEEP_D, dtype=torch.bfloat16,
                          S0_std=W.SWEEP["S0_std"], seed=seed)
    return {n: (None if x[n] is None else x[n].double().numpy()) for n in x}


def run_oracle_sample(smp, threads):
    import oracle
    q, k, v, g, beta = oracle.prologue_np(smp["q_pre"], smp["k_pre"], smp["v_pre"], smp["conv_w"],
                                          smp["z"], smp["A"], smp["b_logit"])
    return oracle.recurrence_c(q, k, v, g, beta, smp["S0"], nthreads=threads)


# ---------------------------------------------------------------- reference arm (the oracle)
def run_reference(args, ws, rank):
    if rank != 0:
        return 0
    heads, tokens = 16, 4096          # a bounded sample of the workload per step
    smp = oracle_sweep_sample(heads, tokens, HEADLINE_T)
    host_cores = os.cpu_count() or 1
    threads = min(host_cores, heads)  # the oracle threads over sequences (heads)
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        run_oracle_sample(smp, threads)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    # the sample is `heads` of the workload's H heads: that many tokens of the whole workload
    tok = tokens * heads / SWEEP_H
    value = tok / statistics.mean(times)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * statistics.mean(times), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": HEADLINE_WORKLOAD + f" (oracle sample: {heads} heads x {tokens} tokens)",
                       "B": 1, "T": HEADLINE_T, "H": SWEEP_H, "dk": SWEEP_D, "dv": SWEEP_D},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "host_cores": host_cores,
                             "kind": "oracle",
                             "sample": f"{heads} of {SWEEP_H} heads x {tokens} tokens of the sweep recipe per "
                                       f"step, prologue and recurrence in FP64 (counted as the {tok:.0f} tokens "
                                       "of the whole workload they are)"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- our arm
def time_calls(fn, reps, flush=None, stream=None):
    """Per-call CUDA-event times (ms) on the current stream, L2 flushed before each."""
    out = []
    for _ in range(reps):
        if flush is not None:
            flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        out.append((a, b))
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in out]


def cpu_baseline_sweep(min_seconds=10.0, max_runs=40):
    """The FP64 oracle (prologue in numpy, recurrence in C threaded over heads) on the host's
    cores, on a bounded sample of the headline workload: 16 heads x 8192 tokens of the sweep
    recipe, run repeatedly until about `min_seconds` of CPU work (at most `max_runs` runs);
    rate = the workload tokens the sample stands for / the time."""
    heads, tokens = 16, 8192
    smp = oracle_sweep_sample(heads, tokens, HEADLINE_T)
    host_cores = os.cpu_count() or 1
    threads = min(host_cores, heads)
    runs, dt = 0, 0.0
    while runs < max_runs and (runs == 0 or dt < min_seconds):
        t0 = time.perf_counter()
        run_oracle_sample(smp, threads)
        dt += time.perf_counter() - t0
        runs += 1
    tok = tokens * heads / SWEEP_H
    return {"value": runs * tok / dt, "unit": UNIT, "cores": threads, "host_cores": host_cores, "kind": "oracle",
            "sample": f"{heads} of {SWEEP_H} heads x {tokens} tokens of the sweep recipe (prologue + recurrence, "
                      f"FP64, one thread per head), run {runs} times; counted as the {tok:.0f} tokens of "
                      "the whole workload each run stands for",
            "seconds": dt, "runs": runs}


def sweep_row(K, T, flush, hbm_peak):
    """a1-a4 on the length-sweep workload (B=1, H=96, d=128, raw inputs through the fused
    prologue) at one T: the call's time and its fraction of the HBM roofline."""
    H, d = 96, 128
    prev = W._DEVICE
    W.set_device("cuda")
    try:
        x = W.sweep_inputs(T)
        args = [x[n] for n in ("q_pre", "k_pre", "v_pre", "conv_w", "z", "A", "b_logit")]
        opts0 = K.make_opts(torch.bfloat16)
        ws = torch.empty(K.kda_prologue_workspace_bytes(1, T, H, d, d, opts0), dtype=torch.uint8,
                         device="cuda")
        out = torch.empty((1, T, H, d), dtype=torch.bfloat16, device="cuda")
        S_T = torch.empty((1, H, d, d), dtype=torch.float32, device="cuda")
        opts = K.make_opts(torch.bfloat16, workspace=ws)
        fn = lambda: K.kda_chunk_fwd_prologue(*args, x["S0"], out, S_T, opts)
        fn()
        ms = statistics.median(time_calls(fn, 3, flush))
        nbytes = T * H * (4 * d * 2 + 4 + d * 2) + H * (2 * d * d * 4 + 3 * d * 4 * 2)
        return {"ms": ms, "tokens_per_s": T / (ms * 1e-3), "token_heads_per_s": T * H / (ms * 1e-3),
                "roofline_bytes": nbytes, "roofline_flops": PREFILL_FLOP_PER_TOKEN_HEAD * T * H,
                "frac_of_hbm_roofline": (nbytes / (ms * 1e-3) / 1e9) / hbm_peak}
    finally:
        W.set_device(prev)
        torch.cuda.empty_cache()


def rows_n1(K, flush, hbm_peak, rows):
    """Per-row measurements beyond the headline (rank 0, N=1), filled into `rows` as they
    finish (a row that fails leaves the earlier ones in place)."""
    W.set_device("cuda")
    try:
        d = 128

        # a2-a4 + the output epilogue (RMSNorm * sigmoid gate) on the prefill workload
        x = W.workload_inputs("prefill")
        Bp, Tp, Hp = x["q"].shape[:3]
        gen = torch.Generator().manual_seed(11)
        gate = torch.randn(x["v"].shape, generator=gen).to(torch.bfloat16).cuda()
        nw = torch.ones(d, dtype=torch.float32, device="cuda")
        o1 = K.make_opts(torch.bfloat16)
        wsg = torch.empty(max(K.kda_chunk_workspace_bytes(Bp, Tp, Hp, d, d, o1), 16), dtype=torch.uint8,
                          device="cuda")
        og = K.make_opts(torch.bfloat16, workspace=wsg)
        outg = torch.empty(x["v"].shape, dtype=torch.bfloat16, device="cuda")
        Sg = torch.empty((Bp, Hp, d, d), dtype=torch.float32, device="cuda")
        fg = lambda: K.kda_chunk_fwd_gated(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], outg, Sg,
                                           gate, nw, 1e-5, og)
        fp = lambda: K.kda_chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], outg, Sg, og)
        fg(); fp()
        ms_g = statistics.median(time_calls(fg, 10, flush))
        ms_p = statistics.median(time_calls(fp, 10, flush))
        rows["prefill_output_epilogue"] = {"ms_gated": ms_g, "ms_plain": ms_p,
                                           "extra_bytes": Bp * Tp * Hp * d * 2,
                                           "note": "kda_chunk_fwd_gated vs kda_chunk_fwd, B=1 T=4096 H=16"}
        del gate, nw, wsg, outg, Sg
        torch.cuda.empty_cache()

        # backward (kda_chunk_bwd) on the prefill workload: FP32 gradients of q, k, v, g, beta, S0
        gr = W.grad_inputs(Bp, Tp, Hp, d, d, dtype=torch.bfloat16, seed=0)
        ob = K.make_opts(torch.bfloat16)
        wsb = torch.empty(K.kda_chunk_bwd_workspace_bytes(Bp, Tp, Hp, d, d, ob), dtype=torch.uint8,
                          device="cuda")
        ob = K.make_opts(torch.bfloat16, workspace=wsb)
        e = lambda *shape: torch.empty(shape, dtype=torch.float32, device="cuda")
        grads = (e(Bp, Tp, Hp, d), e(Bp, Tp, Hp, d), e(Bp, Tp, Hp, d), e(Bp, Tp, Hp, d),
                 e(Bp, Tp, Hp), e(Bp, Hp, d, d))
        fb = lambda: K.kda_chunk_bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], gr["dout"],
                                     gr["dS_T"], *grads, ob)
        fb()
        ms_b = statistics.median(time_calls(fb, 5, flush))
        th = Bp * Tp * Hp
        # in: q, k, v, g, dout (bf16), beta (bf16); out: dq, dk, dv, dg (FP32), dbeta (FP32);
        # per head S0, dS_T in and dS0 out (FP32)
        nb = th * (5 * d * 2 + 2 + 4 * d * 4 + 4) + Bp * Hp * 3 * d * d * 4
        rows["prefill_backward"] = {
            "ms": ms_b, "tokens_per_s": Bp * Tp / (ms_b * 1e-3), "algorithmic_bytes": nb,
            "frac_of_hbm_roofline": (nb / (ms_b * 1e-3) / 1e9) / hbm_peak,
            "workspace_bytes": wsb.numel(),
            "note": "kda_chunk_bwd, B=1 T=4096 H=16 d=128 bf16 in, FP32 gradients out"}
        del gr, wsb, grads
        torch.cuda.empty_cache()

        # Complex-KDA against KDA, forward + backward, at the shape of the CKDA review's Figure 5
        # (BF16, 16 heads, dk = dv = 128, 32k tokens per step): context for the pages' 96-97 %
        fb_ms = {}
        for cplx in (False, True):
            xc = W.chunk_inputs(1, 32768, 16, d, d, dtype=torch.bfloat16, seed=5, complex_gate=cplx)
            gc = W.grad_inputs(1, 32768, 16, d, d, dtype=torch.bfloat16, seed=6)
            ob = K.make_opts(torch.bfloat16, complex_gate=cplx)
            wsc = torch.empty(K.kda_chunk_bwd_workspace_bytes(1, 32768, 16, d, d, ob), dtype=torch.uint8,
                              device="cuda")
            ff = lambda: K.chunk_fwd(xc["q"], xc["k"], xc["v"], xc["g"], xc["beta"], xc["S0"],
                                     complex_gate=cplx)
            fbw = lambda: K.chunk_bwd(xc["q"], xc["k"], xc["v"], xc["g"], xc["beta"], xc["S0"], gc["dout"],
                                      gc["dS_T"], complex_gate=cplx, workspace=wsc)
            ff(); fbw()
            torch.cuda.synchronize()
            t_f = statistics.median(time_calls(ff, 3, flush))
            t_b = statistics.median(time_calls(fbw, 3, flush))
            fb_ms["ckda" if cplx else "kda"] = {"fwd_ms": t_f, "bwd_ms": t_b, "fwd_bwd_ms": t_f + t_b}
            del xc, gc, wsc
            torch.cuda.empty_cache()
        fb_ms["ckda_over_kda_throughput_fwd_bwd"] = fb_ms["kda"]["fwd_bwd_ms"] / fb_ms["ckda"]["fwd_bwd_ms"]
        fb_ms["ckda_over_kda_throughput_fwd"] = fb_ms["kda"]["fwd_ms"] / fb_ms["ckda"]["fwd_ms"]
        fb_ms["note"] = ("B=1 T=32768 H=16 dk=dv=128 bf16, kda_chunk_fwd + kda_chunk_bwd (FP32: sweeps for "
                         "the 8-token boundary values, then all windows in parallel); the pages report "
                         "96-97 % on H100 (context only)")
        rows["complex_kda_fwd_bwd_T32768_H16"] = fb_ms

        # context parallelism over T, emulated on one GPU: the prefill sequence cut into 4
        # segments; each segment's pair (one prep pass, two scans over its records), the fold and
        # the segment's forward from the folded state (a scan over the same records), timed per
        # piece (on R GPUs the ranks run their pieces side by side)
        R = 4
        Ts = Tp // R
        segs = [{n: x[n][:, r * Ts:(r + 1) * Ts].contiguous() for n in ("q", "k", "v", "g", "beta")}
                for r in range(R)]
        op = K.make_opts(torch.bfloat16)
        wsp = torch.empty(K.kda_segment_pair_workspace_bytes(Bp, Ts, Hp, d, d, op), dtype=torch.uint8,
                          device="cuda")
        op = K.make_opts(torch.bfloat16, workspace=wsp)
        Ms = torch.empty((R, Bp, Hp, d, d), dtype=torch.float32, device="cuda")
        Bs = torch.empty((R, Bp, Hp, d, d), dtype=torch.float32, device="cuda")
        fpair = lambda r: K.kda_segment_pair(*(segs[r][n] for n in ("q", "k", "v", "g", "beta")),
                                             Ms[r], Bs[r], op)
        for r in range(R):
            fpair(r)
        ms_pair = statistics.median(time_calls(lambda: fpair(R - 1), 5, flush))
        S_start = torch.empty((Bp, Hp, d, d), dtype=torch.float32, device="cuda")
        fcomb = lambda: K.kda_affine_combine(Ms, Bs, R - 1, x["S0"], S_start)
        fcomb()
        ms_comb = statistics.median(time_calls(fcomb, 5, flush))
        outs = torch.empty((Bp, Ts, Hp, d), dtype=torch.bfloat16, device="cuda")
        Sseg = torch.empty((Bp, Hp, d, d), dtype=torch.float32, device="cuda")
        # wsp holds the last segment's records (its pair was the last call on it)
        fseg = lambda: K.kda_segment_forward(*(segs[R - 1][n] for n in ("q", "k", "v", "g", "beta")),
                                             S_start, outs, Sseg, op)
        fseg()
        ms_seg = statistics.median(time_calls(fseg, 5, flush))
        pair_bytes = R * Bp * Hp * 2 * d * d * 4
        rows["context_parallel_prefill_4_segments"] = {
            "segment_T": Ts, "ms_segment_pair": ms_pair, "ms_fold": ms_comb, "ms_segment_forward": ms_seg,
            "ms_per_rank_compute": ms_pair + ms_comb + ms_seg, "ms_whole_sequence_one_gpu": ms_p,
            "all_gather_bytes": pair_bytes,
            "note": "one GPU, pieces timed separately; per rank = pair + fold of 3 pairs + the segment's "
                    "forward over its 1024 tokens; the all-gather of the pairs (all_gather_bytes) is not "
                    "timed here"}
        del segs, wsp, Ms, Bs, S_start, outs, Sseg
        torch.cuda.empty_cache()

        # unbounded decay (Kimi Linear softplus gate) on the prefill shape: the split tensor-core
        # form with FP32 diagonal blocks (one launch here), beside the bounded gate's time
        xs = W.chunk_inputs(Bp, Tp, Hp, d, d, dtype=torch.bfloat16, seed=0, gate="softplus")
        ou = K.make_opts(torch.bfloat16, unbounded=True)
        wsu = torch.empty(K.kda_chunk_workspace_bytes(Bp, Tp, Hp, d, d, ou), dtype=torch.uint8,
                          device="cuda")
        ou = K.make_opts(torch.bfloat16, unbounded=True, workspace=wsu)
        outu = torch.empty(xs["v"].shape, dtype=torch.bfloat16, device="cuda")
        Su = torch.empty((Bp, Hp, d, d), dtype=torch.float32, device="cuda")
        fu = lambda: K.kda_chunk_fwd(xs["q"], xs["k"], xs["v"], xs["g"], xs["beta"], xs["S0"], outu,
                                     Su, ou)
        fu()
        ms_u = statistics.median(time_calls(fu, 5, flush))
        nbu = th * token_head_bytes(d) + Bp * Hp * 2 * d * d * 4
        ms_b = rows.get("prefill_B1_T4096_H16", {}).get("ms")
        rows["prefill_softplus_gate"] = {
            "ms": ms_u, "tokens_per_s": Bp * Tp / (ms_u * 1e-3),
            "ms_bounded_gate": ms_b,
            "ratio_to_bounded": ms_u / ms_b if ms_b else None,
            "frac_of_hbm_roofline": (nbu / (ms_u * 1e-3) / 1e9) / hbm_peak,
            "note": "kda_chunk_fwd with KDA_UNBOUNDED_DECAY, softplus-gate inputs: split tensor-core "
                    "form, off-diagonal band pairs on tcgen05, diagonal 16-token blocks as FP32 pairs"}
        del x, xs, wsu, outu, Su
        torch.cuda.empty_cache()

        # a5: decode step, N = 256, H = 96, 64 steps with S carried in HBM
        D = W.DECODE
        N, H = D["N"], D["H"]
        S = W.decode_state(N, H, d, d, S_std=D["S_std"])
        A = W.decode_log_scale(H)
        toks = [W.decode_step_inputs(N, H, d, d, s, A=A) for s in range(4)]
        outd = torch.empty((N, H, d), dtype=torch.bfloat16, device="cuda")
        optd = K.make_opts(torch.bfloat16)
        it = [0]

        def dstep():
            t = toks[it[0] % 4]
            it[0] += 1
            K.kda_recurrent_step(t["q"], t["k"], t["v"], t["g"], t["beta"], S, outd, optd)
        for _ in range(3):
            dstep()
        ms = statistics.median(time_calls(dstep, D["steps"]))
        nbytes = N * H * (2 * d * d * 4 + token_head_bytes(d))
        gbs = nbytes / (ms * 1e-3) / 1e9
        rows["decode_step"] = {"ms": ms, "GB_per_s": gbs, "bytes_per_step": nbytes,
                               "frac_of_hbm": gbs / hbm_peak, "steps": D["steps"],
                               "note": "state 3.2 GB > L2, no flush needed"}

        # decode step with the prologue fused in (conv state carried in HBM), same shapes
        par = W.decode_prologue_params(H, d)
        ptoks = [W.decode_prologue_step_inputs(N, H, d, s) for s in range(4)]
        cstate = torch.zeros((N, 3, 3, H * d), dtype=torch.bfloat16, device="cuda")

        def pstep():
            t = ptoks[it[0] % 4]
            it[0] += 1
            K.kda_recurrent_step_prologue(t["q_pre"], t["k_pre"], t["v_pre"], par["conv_w"], cstate,
                                          t["z"], par["A"], t["b_logit"], S, outd, optd)
        for _ in range(3):
            pstep()
        ms = statistics.median(time_calls(pstep, D["steps"]))
        # state read + write, raw q, k, v, z in, out, beta logit, conv state read + write
        nbytes = N * H * (2 * d * d * 4 + 5 * d * 2 + 4 + 2 * 9 * d * 2) + H * 3 * d * 4 * 2
        gbs = nbytes / (ms * 1e-3) / 1e9
        rows["decode_step_prologue"] = {"ms": ms, "GB_per_s": gbs, "bytes_per_step": nbytes,
                                        "frac_of_hbm": gbs / hbm_peak, "steps": D["steps"]}
        del S, toks, outd, ptoks, cstate, par
        torch.cuda.empty_cache()

        # a6: Complex-KDA vs unsigned KDA at B=8, T=8192, H=32
        cfg = W.WORKLOADS["ckda"]
        res = {}
        for cplx in (True, False):
            x = W.chunk_inputs(cfg["B"], cfg["T"], cfg["H"], d, d, dtype=torch.bfloat16,
                               S0_std=cfg["S0_std"], seed=0, complex_gate=cplx)
            o0 = K.make_opts(torch.bfloat16, complex_gate=cplx)
            wsz = K.kda_chunk_workspace_bytes(cfg["B"], cfg["T"], cfg["H"], d, d, o0)
            ws = torch.empty(max(wsz, 16), dtype=torch.uint8, device="cuda")
            o = K.make_opts(torch.bfloat16, complex_gate=cplx, workspace=ws)
            out = torch.empty_like(x["v"])
            S_T = torch.empty((cfg["B"], cfg["H"], d, d), dtype=torch.float32, device="cuda")
            fn = lambda: K.kda_chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], out, S_T, o)
            fn()
            ms = statistics.median(time_calls(fn, 3))
            th = cfg["B"] * cfg["T"] * cfg["H"]
            nbytes = th * token_head_bytes(d) + cfg["B"] * cfg["H"] * 2 * d * d * 4
            res["ckda" if cplx else "kda"] = {
                "ms": ms, "tokens_per_s": cfg["B"] * cfg["T"] / (ms * 1e-3),
                "frac_of_hbm_roofline": (nbytes / (ms * 1e-3) / 1e9) / hbm_peak}
            del x, ws, out, S_T
            torch.cuda.empty_cache()
        res["ckda_over_kda_throughput"] = res["kda"]["ms"] / res["ckda"]["ms"]
        rows["complex_kda_B8_T8192_H32"] = res
    finally:
        W.set_device("cpu")
    return rows


def time_steps(call, steps, sampler=None):
    """`steps` calls, one event pair around each on the current stream; returns the per-call
    device times (ms) and the wall time of the timed region."""
    t0s = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    t1s = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    torch.cuda.synchronize()
    ctx = sampler if sampler is not None else _NullCtx()
    with ctx:
        w0 = time.perf_counter()
        for i in range(steps):
            t0s[i].record()
            call()
            t1s[i].record()
        torch.cuda.synchronize()
        w1 = time.perf_counter()
    return [a.elapsed_time(b) for a, b in zip(t0s, t1s)], w1 - w0


class _NullCtx:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def kernel_times(call, steps, max_launch=4):
    """Launches per call and each launch's mean device time (ms), from calls that record an
    event before every launch (kda_opts.events)."""
    probe = [torch.cuda.Event(enable_timing=True) for _ in range(max_launch + 1)]
    for e in probe:
        e.record()
    torch.cuda.synchronize()
    mark = torch.cuda.Event(enable_timing=True)
    mark.record()
    call(probe)
    torch.cuda.synchronize()
    launches = sum(1 for e in probe[1:] if mark.elapsed_time(e) > 0.0)
    sets = [[torch.cuda.Event(enable_timing=True) for _ in range(max_launch + 1)] for _ in range(steps)]
    for evs in sets:
        for e in evs:
            e.record()
    torch.cuda.synchronize()
    for evs in sets:
        call(evs)
    torch.cuda.synchronize()
    return launches, [statistics.mean(evs[j].elapsed_time(evs[j + 1]) for evs in sets) for j in range(launches)]


def prefill_row(K, flush, hbm_peak, steps=20):
    """The prefill workload (B=1, T=4096, H=16): `steps` timed calls (L2 flushed between them,
    its inputs fit in L2) with their own clock record and per-launch times."""
    cfg = W.WORKLOADS["prefill"]
    B, T, H, d = cfg["B"], cfg["T"], cfg["H"], cfg["dk"]
    x = W.workload_inputs("prefill")
    o0 = K.make_opts(torch.bfloat16)
    wsb = torch.empty(max(K.kda_chunk_workspace_bytes(B, T, H, d, d, o0), 16), dtype=torch.uint8, device="cuda")
    out = torch.empty((B, T, H, d), dtype=torch.bfloat16, device="cuda")
    S_T = torch.empty((B, H, d, d), dtype=torch.float32, device="cuda")

    def call(evs=None):
        o = K.make_opts(torch.bfloat16, workspace=wsb, events=evs)
        K.kda_chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], out, S_T, o)
    for _ in range(3):
        call()
    sampler = ClockSampler(torch.cuda.current_device())
    ms = []
    with sampler:
        for _ in range(steps):
            ms += time_calls(call, 1, flush)
    launches, kms = kernel_times(lambda evs: (flush.zero_(), call(evs)), 5)
    nbytes = B * T * H * token_head_bytes(d) + B * H * 2 * d * d * 4
    med = statistics.median(ms)
    return {"ms": med, "ms_mean": statistics.mean(ms), "tokens_per_s": B * T / (med * 1e-3),
            "frac_of_hbm_roofline": (nbytes / (med * 1e-3) / 1e9) / hbm_peak, "roofline_bytes": nbytes,
            "launches": launches, "kernel_ms": kms, "clocks": sampler.summary(), "steps": steps,
            "note": "kda_chunk_fwd B=1 T=4096 H=16 d=128 bf16; 256 MiB written between calls (inputs fit in L2)"}


def run_ours(args, ws, rank, local):
    import gated_delta_rule_73_b200 as K
    dev = torch.device("cuda", local)
    hbm_peak, tf_peak, peak_kind = peaks()
    T, H, d = HEADLINE_T, SWEEP_H, SWEEP_D
    W.set_device("cuda")
    x = W.sweep_inputs(T, seed=T + rank)       # each rank its own batch
    W.set_device("cpu")
    names = ("q_pre", "k_pre", "v_pre", "conv_w", "z", "A", "b_logit", "S0")
    opts0 = K.make_opts(torch.bfloat16)
    wsz = K.kda_prologue_workspace_bytes(1, T, H, d, d, opts0)
    wsb = torch.empty(max(wsz, 16), dtype=torch.uint8, device=dev)
    out = torch.empty((1, T, H, d), dtype=torch.bfloat16, device=dev)
    S_T = torch.empty((1, H, d, d), dtype=torch.float32, device=dev)

    def call_on(dd, oo, evs=None):
        o = K.make_opts(torch.bfloat16, workspace=wsb, events=evs)
        K.kda_chunk_fwd_prologue(*(dd[n] for n in names[:-1]), dd["S0"], oo[0], oo[1], o)

    def call(evs=None):
        call_on(x, (out, S_T), evs)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    # timed steps: one event pair around each call (the call as a user makes it; the inputs,
    # 8 GB, are far larger than L2, so nothing is flushed between steps)
    sampler = ClockSampler(local)
    barrier(ws)
    step_ms, wall = time_steps(call, args.steps, sampler)
    barrier(ws)
    # per-kernel durations from a second pass with an event before each launch
    launches, mean_k = kernel_times(call, args.steps)
    total_ms = sum(step_ms)
    total_ms_max = max_over_ranks(total_ms, ws)
    ms_per_step = total_ms_max / args.steps
    tokens_per_step = T
    value = ws * tokens_per_step * args.steps / (total_ms_max * 1e-3)

    # roofline of the dominant kernel: the path's algorithmic bytes (every launch of the split
    # form processes every token-head of the call) over its mean duration
    alg_bytes = sweep_alg_bytes(T)
    alg_flops = PREFILL_FLOP_PER_TOKEN_HEAD * T * H
    dom = max(range(launches), key=lambda j: mean_k[j])
    achieved = alg_bytes / (mean_k[dom] * 1e-3) / 1e9
    call_achieved = alg_bytes / (statistics.mean(step_ms) * 1e-3) / 1e9
    kernel_names = SWEEP_KERNELS.get(launches, [None] * launches)
    items = ((T + 63) // 64) * H
    per_item = KERNEL_TRAFFIC_PER_ITEM.get(kernel_names[dom])
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak, "traffic": None if per_item is None else per_item * items,
                "peak_kind": peak_kind, "kernel": kernel_names[dom],
                "algorithmic_bytes_per_step": alg_bytes, "algorithmic_flops_per_step": alg_flops,
                "tensor_frac_of_bf16_peak": alg_flops / (statistics.mean(step_ms) * 1e-3) / 1e12 / tf_peak,
                "kernel_ms": mean_k, "kernel_names": kernel_names, "dominant_launch": dom,
                "whole_call_achieved": call_achieved, "whole_call_frac": call_achieved / hbm_peak,
                "note": "achieved = algorithmic bytes per launch (the whole call's: each launch covers every "
                        "token-head) / the dominant kernel's mean duration (a second pass, an event before "
                        "each launch); whole_call_* = the same bytes / the call's device time; traffic = that "
                        "kernel's DRAM bytes per (chunk, head) item from an ncu capture at T=2048, times the "
                        "items of one launch"}

    # end to end through the C ABI with host buffers (pinned), copies inside the timed region.
    # Every step copies all its inputs host -> device, runs the call and reads out and S_T back.
    # Pipelined as a serving loop would run it: the copy-in of step i+1, the call of step i and
    # the copy-out of step i-1 overlap on three streams, device buffers double-buffered.  The
    # serialised form (copy, call, copy on one stream) is kept beside it.
    host = {n: x[n].cpu().pin_memory() for n in names}
    cs = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    dbuf = [x, {n: torch.empty_like(x[n]) for n in names}]
    obuf = [(out, S_T), (torch.empty_like(out), torch.empty_like(S_T))]
    hout = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    hS = [torch.empty(S_T.shape, dtype=S_T.dtype).pin_memory() for _ in range(2)]
    e2e_steps = min(args.steps, 10)

    def e2e_pipelined(nsteps):
        ev_in = [torch.cuda.Event() for _ in range(nsteps)]
        ev_call = [torch.cuda.Event() for _ in range(nsteps)]
        ev_out = [torch.cuda.Event() for _ in range(nsteps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        t0.record(cs)
        s_in.wait_event(t0)
        s_out.wait_event(t0)
        for i in range(nsteps):
            bi = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_call[i - 2])          # the call of step i-2 read dbuf[bi]
                for n in names:
                    dbuf[bi][n].copy_(host[n], non_blocking=True)
                ev_in[i].record(s_in)
            cs.wait_event(ev_in[i])
            if i >= 2:
                cs.wait_event(ev_out[i - 2])                 # obuf[bi] has been read back
            call_on(dbuf[bi], obuf[bi])
            ev_call[i].record(cs)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_call[i])
                hout[bi].copy_(obuf[bi][0], non_blocking=True)
                hS[bi].copy_(obuf[bi][1], non_blocking=True)
                ev_out[i].record(s_out)
        cs.wait_event(ev_in[nsteps - 1])
        cs.wait_event(ev_out[nsteps - 1])
        t1.record(cs)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    def e2e_step():
        for n in names:
            x[n].copy_(host[n], non_blocking=True)
        call()
        hout[0].copy_(out, non_blocking=True)
        hS[0].copy_(S_T, non_blocking=True)
    e2e_step()
    torch.cuda.synchronize()
    ref_out, ref_S = hout[0].clone(), hS[0].clone()
    e2e_serial_ms = time_calls(e2e_step, e2e_steps)
    e2e_pipelined(3)
    e2e_ms = e2e_pipelined(e2e_steps)
    last = (e2e_steps - 1) % 2
    close = lambda a, b: float((a.float() - b.float()).abs().max()) <= 1e-3 * float(b.float().abs().max())
    e2e_ok = bool(close(hout[last], ref_out) and close(hS[last], ref_S))
    e2e_max = max_over_ranks(e2e_ms, ws)
    e2e_serial_max = max_over_ranks(sum(e2e_serial_ms), ws)
    h2d = sum(host[n].numel() * host[n].element_size() for n in names)
    d2h = hout[0].numel() * hout[0].element_size() + hS[0].numel() * hS[0].element_size()
    e2e = {"value": ws * tokens_per_step * e2e_steps / (e2e_max * 1e-3), "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
           "ms_per_step": e2e_max / e2e_steps, "outputs_match_serial": e2e_ok,
           "serial_value": ws * tokens_per_step * e2e_steps / (e2e_serial_max * 1e-3),
           "note": "pipelined over three streams (copy-in of step i+1, call i, copy-out of step i-1), every "
                   "step's copies inside the timed region; serial_value = one stream; PCIe-bound"}
    del host, dbuf, obuf, hout, hS
    torch.cuda.empty_cache()

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": HEADLINE_WORKLOAD, "B": 1, "T": T, "H": H, "dk": d, "dv": d,
                       "l2": "inputs (8 GB) larger than the 126 MB L2; nothing flushed between steps",
                       "parallelism": f"replicas x{ws}: each rank runs its own batch, no collective"},
            "roofline": roofline, "e2e": e2e, "gpu_launches": launches * args.steps,
            "step_ms_median": statistics.median(step_ms),
            "clocks": sampler.summary(), "wall_s_timed": wall}
    del x, wsb, out, S_T
    torch.cuda.empty_cache()
    if ws == 1 and rank == 0 and not args.no_rows:
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        rows = {}
        try:
            W.set_device("cuda")
            rows["prefill_B1_T4096_H16"] = prefill_row(K, flush, hbm_peak)
        except Exception as e:          # a failed row must not cost the headline its line
            rows["prefill_B1_T4096_H16"] = {"error": f"{type(e).__name__}: {e}"}
        finally:
            W.set_device("cpu")
        try:
            rows_n1(K, flush, hbm_peak, rows)
        except Exception as e:
            rows["error"] = f"{type(e).__name__}: {e}"
        for Ts in W.SWEEP_T[1:-1]:         # T = 8192, 32768 (65536 is the headline)
            try:
                rows[f"sweep_T{Ts}_prologue"] = sweep_row(K, Ts, flush, hbm_peak)
            except Exception as e:
                rows[f"sweep_T{Ts}_prologue"] = {"error": f"{type(e).__name__}: {e}"}
        line["rows"] = rows
        del flush
    if ws == 1 and rank == 0 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline_sweep()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


CASES = ("prefill", "decode", "sweep", "ckda", "bwd", "sweep_plain", "softplus")

# Kernels of kda_chunk_fwd_prologue on the sweep workload (B*H = 96 takes the split form: the
# two-group prep with the fused prologue, then the TMEM scan) by launches per call, and the DRAM
# bytes (read + write) per (chunk, head) item of each from one ncu capture at T = 2048
# (profiles/), None where no capture of the kernel as it stands exists.
SWEEP_KERNELS = {2: ["chunk_prep2_kernel", "chunk_scan3_kernel"], 1: ["chunk_mega2_kernel"]}
# (the prep's figure was taken before its later-band B rows were spread over the item group: a
# change inside the kernel, so no figure is reported for it until it is captured again)
KERNEL_TRAFFIC_PER_ITEM = {"chunk_prep2_kernel": None, "chunk_scan3_kernel": 86_792, "chunk_mega2_kernel": None}


def run_case(args):
    """Run one workload's call a few times and exit (a small case for ncu captures):
    prefill = B=1 T=4096 H=16; decode = N=64 H=96 (800 MB of state);
    sweep = prologue path at T=2048 H=96; sweep_plain = kda_chunk_fwd at B=1 T=2048 H=96;
    softplus = kda_chunk_fwd with the unbounded (softplus) gate at B=1 T=2048 H=96;
    ckda = B=2 T=8192 H=32 signed gate; bwd = kda_chunk_bwd at B=1 T=1024 H=16."""
    import gated_delta_rule_73_b200 as K
    torch.cuda.set_device(0)
    W.set_device("cuda")
    d = 128
    if args.case == "decode":
        N, H = 64, 96
        S = W.decode_state(N, H, d, d)
        t = W.decode_step_inputs(N, H, d, d, 0)
        out = torch.empty((N, H, d), dtype=torch.bfloat16, device="cuda")
        o = K.make_opts(torch.bfloat16)
        fn = lambda: K.kda_recurrent_step(t["q"], t["k"], t["v"], t["g"], t["beta"], S, out, o)
    elif args.case == "bwd":
        x = W.workload_inputs("prefill", T=1024)
        gr = W.grad_inputs(1, 1024, 16, d, d, dtype=torch.bfloat16, seed=0)
        fn = lambda: K.chunk_bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], gr["dout"],
                                 gr["dS_T"])
    elif args.case == "sweep":
        T, H = 2048, 96
        x = W.sweep_inputs(T)
        a = [x[n] for n in ("q_pre", "k_pre", "v_pre", "conv_w", "z", "A", "b_logit")]
        fn = lambda: K.chunk_fwd_prologue(*a, x["S0"])
    elif args.case == "sweep_plain":
        x = W.chunk_inputs(1, 2048, 96, d, d, dtype=torch.bfloat16, seed=0)
        fn = lambda: K.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], fused=False)
    elif args.case == "softplus":
        x = W.chunk_inputs(1, 2048, 96, d, d, dtype=torch.bfloat16, seed=0, gate="softplus")
        fn = lambda: K.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], unbounded=True)
    else:
        if args.case == "prefill":
            x = W.workload_inputs("prefill")
            cplx = False
        else:
            x = W.chunk_inputs(2, 8192, 32, d, d, dtype=torch.bfloat16, seed=0, complex_gate=True)
            cplx = True
        fn = lambda: K.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], complex_gate=cplx)
    for _ in range(args.case_reps):
        fn()
    torch.cuda.synchronize()
    W.set_device("cpu")
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", choices=CASES, default=None,
                    help="run one small workload a few times (for profiler captures) and exit")
    ap.add_argument("--case-reps", type=int, default=3)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-rows", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    args = ap.parse_args()
    if args.case:
        return run_case(args)
    ws, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            return run_reference(args, ws, rank)
        return run_ours(args, ws, rank, local)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())

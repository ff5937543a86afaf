#!/usr/bin/env python3
"""Benchmark of the INT4 W4A16 hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode|prefill|moe|moe_layer|qat|qat_gemm|gemv|quant|zp]

Default workload: the decode GEMV sweep -- W[12288, 4096] BF16 ~ N(0, 0.02^2)
with 0.1 % x20 outliers, group 32, activations X[M, 4096] ~ N(0, 1) for
M in {1, 8, 16, 32}.  One step is one pass of the whole hot path over it:
  1. fake quantization of W (QAT forward, w4_fake_quant),
  2. the STE backward of the gradient into a separate buffer (w4_ste_backward),
  3. real quantization + packing of W (export, w4_quantize_pack),
  4. the W4A16 GEMM for each M (decode, w4a16_gemm).
The metric is the step's algorithmic HBM throughput (GB/s): the bytes each
kernel must move at minimum, summed over the step, divided by the step time.
Every kernel reads inputs that are not resident in L2: W and the gradients
alternate between two copies, the decode GEMMs rotate over eight packed copies
of the weight (each copy is about 28 MB; L2 is 126 MB).

--impl reference times the CPU oracle (plain C, all host cores) on the same
workload and metric; under torchrun only rank 0 runs it.

Multi-GPU (torchrun): each rank runs an independent replica of the workload
(weak scaling; no collective on the data path); time is the max over ranks.
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0

# DRAM bytes (read + write) per launch from one ncu capture of the kernel
# (profiles/ holds the summaries and commands); an entry is used only while the
# kernel's source file is unchanged since the capture.
NCU_TRAFFIC = {
    ("gemm_m16", "decode"): {"bytes": 28523008 + 0, "file": "w4_gemm.cu", "src": "389a57b5497f8f27"},
    ("gemm_m1", "decode"): {"bytes": 28345088 + 0, "file": "w4_gemv.cu", "src": "bee317c18421180b"},
    ("fake_quant", "decode"): {"bytes": 100688640 + 47492864, "file": "w4_quant.cu", "src": "daef7cabc96462d0"},
    ("ste_backward", "decode"): {"bytes": 100670976 + 45220864, "file": "w4_quant.cu", "src": "daef7cabc96462d0"},
    ("quantize_pack", "decode"): {"bytes": 100686848 + 5896448, "file": "w4_quant.cu", "src": "daef7cabc96462d0"},
}


def _src_hash(fname: str) -> str:
    with open(os.path.join(ROOT, "int4_w4a16_b200", "csrc", fname), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def _traffic(kernel: str, workload_key: str):
    e = NCU_TRAFFIC.get((kernel, workload_key))
    if e is None or e["src"] != _src_hash(e["file"]):
        return None
    return e["bytes"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------------------
# Clock sampling during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for name, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(rows)}


# ---------------------------------------------------------------------------
# Decode workload (default bench line)
# ---------------------------------------------------------------------------

class DecodeWorkload:
    name = "decode"

    def __init__(self, device):
        import int4_w4a16_b200 as w4
        self.w4 = w4
        cfg = synth.Decode()
        self.cfg = cfg
        self.N, self.K, self.Ms = cfg.N, cfg.K, cfg.Ms
        N, K = self.N, self.K
        self.W = [cfg.weight(device), synth.normal_bf16((N, K), 0.02, cfg.seed, 1, device,
                                                        outlier_frac=0.001)]
        self.G = [cfg.grads(device), synth.normal_bf16((N, K), 1e-3, cfg.seed, 6, device)]
        self.X = {M: cfg.activations(M, device) for M in self.Ms}
        self.Wdq = torch.empty_like(self.W[0])
        self.dW = torch.empty_like(self.W[0])
        self.Wq = torch.empty((N, K // 8), dtype=torch.int32, device=device)
        self.S = torch.empty((N, K // 32), dtype=torch.bfloat16, device=device)
        # eight packed copies for the decode GEMMs (L2-cold reads)
        self.copies = []
        for i in range(8):
            Wq, S = w4.quantize_pack(self.W[i % 2])
            self.copies.append((Wq, S))
        self.Y = {M: torch.empty((M, N), dtype=torch.bfloat16, device=device) for M in self.Ms}
        self.step_idx = 0
        nk = N * K
        self.kernels = ["fake_quant", "ste_backward", "quantize_pack"] + [f"gemm_m{M}" for M in self.Ms]
        self.bytes = {"fake_quant": 4 * nk, "ste_backward": 4 * nk,
                      "quantize_pack": 2 * nk + nk // 2 + nk // 16}
        self.flops = {}
        for M in self.Ms:
            self.bytes[f"gemm_m{M}"] = nk // 2 + nk // 16 + 2 * M * K + 2 * M * N
            self.flops[f"gemm_m{M}"] = 2 * M * N * K
        self.launches_per_step = 3 + len(self.Ms)

    def step(self, ev=None, gemm_ev=None):
        """One pass; ev (optional) = {kernel: (start_event, end_event)} to record
        around each launch; gemm_ev (optional) = (start, end) recorded once
        around the decode GEMM launches together."""
        w4 = self.w4
        i = self.step_idx
        self.step_idx += 1
        W, G = self.W[i % 2], self.G[i % 2]

        def rec(name, fn):
            if ev is not None:
                ev[name][0].record()
            fn()
            if ev is not None:
                ev[name][1].record()

        rec("fake_quant", lambda: w4.w4_fake_quant(W, self.Wdq))
        rec("ste_backward", lambda: w4.w4_ste_backward(G, self.dW))
        rec("quantize_pack", lambda: w4.w4_quantize_pack(W, self.Wq, self.S))
        if gemm_ev is not None:
            gemm_ev[0].record()
        for j, M in enumerate(self.Ms):
            Wq, S = self.copies[(4 * i + j) % len(self.copies)]
            rec(f"gemm_m{M}", lambda: w4.w4a16_gemm(self.X[M], Wq, S, self.Y[M]))
        if gemm_ev is not None:
            gemm_ev[1].record()

    def e2e_run(self, host, nsteps, start_ev, end_ev):
        """nsteps passes through the public API from pinned host buffers, with
        every step's inputs copied in and its results copied out, pipelined the
        way a serving loop runs: step i + 1's host-to-device copies (one
        stream) and step i - 1's device-to-host copies (another) overlap step
        i's kernels, on two device buffer sets.  start_ev / end_ev bracket all
        of it on the current stream."""
        w4 = self.w4
        dev = self.W[0].device
        comp = torch.cuda.current_stream()
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        if not hasattr(self, "_e2e_bufs"):
            mk = lambda t: torch.empty_like(t)
            self._e2e_bufs = [{"W": mk(self.W[0]), "G": mk(self.G[0]),
                               "X": {M: mk(self.X[M]) for M in self.Ms},
                               "Wdq": mk(self.Wdq), "dW": mk(self.dW), "Wq": mk(self.Wq),
                               "S": mk(self.S), "Y": {M: mk(self.Y[M]) for M in self.Ms}}
                              for _ in range(2)]
        bufs = self._e2e_bufs
        in_ready = [torch.cuda.Event() for _ in range(2)]
        comp_done = [torch.cuda.Event() for _ in range(2)]
        out_done = [torch.cuda.Event() for _ in range(2)]
        start_ev.record(comp)
        s_in.wait_event(start_ev)
        s_out.wait_event(start_ev)
        for i in range(nsteps):
            b = bufs[i % 2]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(comp_done[i % 2])        # step i - 2 read these inputs
                b["W"].copy_(host["W"], non_blocking=True)
                b["G"].copy_(host["G"], non_blocking=True)
                for M in self.Ms:
                    b["X"][M].copy_(host["X"][M], non_blocking=True)
                in_ready[i % 2].record(s_in)
            comp.wait_event(in_ready[i % 2])
            if i >= 2:
                comp.wait_event(out_done[i % 2])             # step i - 2's results copied out
            w4.w4_fake_quant(b["W"], b["Wdq"])
            w4.w4_ste_backward(b["G"], b["dW"])
            w4.w4_quantize_pack(b["W"], b["Wq"], b["S"])
            for M in self.Ms:
                w4.w4a16_gemm(b["X"][M], b["Wq"], b["S"], b["Y"][M])
            comp_done[i % 2].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[i % 2])
                host["Wdq"].copy_(b["Wdq"], non_blocking=True)
                host["dW"].copy_(b["dW"], non_blocking=True)
                host["Wq"].copy_(b["Wq"], non_blocking=True)
                host["S"].copy_(b["S"], non_blocking=True)
                for M in self.Ms:
                    host["Y"][M].copy_(b["Y"][M], non_blocking=True)
                out_done[i % 2].record(s_out)
        comp.wait_stream(s_in)
        comp.wait_stream(s_out)
        end_ev.record(comp)

    def host_buffers(self):
        pin = lambda t: torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        h = {"W": pin(self.W[0]), "G": pin(self.G[0]),
             "X": {M: pin(self.X[M]) for M in self.Ms},
             "Wdq": pin(self.Wdq), "dW": pin(self.dW), "Wq": pin(self.Wq), "S": pin(self.S),
             "Y": {M: pin(self.Y[M]) for M in self.Ms}}
        h["W"].copy_(self.W[0])
        h["G"].copy_(self.G[0])
        for M in self.Ms:
            h["X"][M].copy_(self.X[M])
        h2d = h["W"].nbytes + h["G"].nbytes + sum(x.nbytes for x in h["X"].values())
        d2h = (h["Wdq"].nbytes + h["dW"].nbytes + h["Wq"].nbytes + h["S"].nbytes +
               sum(y.nbytes for y in h["Y"].values()))
        return h, h2d, d2h

    @property
    def step_bytes(self):
        return sum(self.bytes.values())

    @property
    def step_flops(self):
        return sum(self.flops.values())

    def config(self):
        return decode_config()


def decode_config():
    cfg = synth.Decode()
    return {"workload": "decode GEMV sweep: W[12288,4096] BF16 N(0,0.02^2) + 0.1% x20 "
                        "outliers, group 32, X[M,4096] N(0,1), M in {1,8,16,32}; step = "
                        "fake_quant + STE (separate buffer) + quantize_pack of W, then "
                        "the W4A16 GEMM for each M",
            "N": cfg.N, "K": cfg.K, "M": list(cfg.Ms), "group": 32,
            "l2": "inputs larger than L2: W and grads alternate over 2 copies (100 MB "
                  "each), the GEMMs rotate over 8 packed copies (28.3 MB each)"}


# ---------------------------------------------------------------------------
# CPU oracle arm (cpu_baseline and --impl reference)
# ---------------------------------------------------------------------------

def oracle_decode_step(state):
    import oracle
    oracle.fake_quant(state["W"])
    oracle.ste_backward(state["G"])
    Wq, S = oracle.quantize_pack(state["W"])
    for M, X in state["X"].items():
        oracle.w4a16_gemm(X, Wq, S, want_r=False)


def oracle_state(rows: int):
    """The decode workload restricted to the first `rows` rows of W (and of the
    gradient); the GEMMs then produce the first `rows` columns of Y."""
    cfg = synth.Decode()
    W = synth.bits(cfg.weight()[:rows])
    G = synth.bits(cfg.grads()[:rows])
    X = {M: synth.bits(cfg.activations(M)) for M in cfg.Ms}
    K = cfg.K
    nk = rows * K
    b = 4 * nk + 4 * nk + (2 * nk + nk // 2 + nk // 16)
    for M in cfg.Ms:
        b += nk // 2 + nk // 16 + 2 * M * K + 2 * M * rows
    return {"W": W, "G": G, "X": X}, b


def _cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def time_oracle(target_s: float = 15.0, rows: int = 1024, target_1t_s: float = 8.0):
    """The oracle on the host cores: all of them (the reported value) and one
    thread, on the same bounded sample of the decode workload."""
    import oracle
    st, nbytes = oracle_state(rows)

    def timed(budget_s):
        t0 = time.perf_counter()
        oracle_decode_step(st)
        one = time.perf_counter() - t0
        reps = max(1, int(budget_s / max(one, 1e-3)))
        t0 = time.perf_counter()
        for _ in range(reps):
            oracle_decode_step(st)
        return (time.perf_counter() - t0) / reps, reps

    cores = oracle.get_threads()
    dt, reps = timed(target_s)
    oracle.set_threads(1)
    try:
        dt1, reps1 = timed(target_1t_s)
    finally:
        oracle.set_threads(cores)
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": cores,
            "kind": "oracle",
            "sample": f"decode workload restricted to W rows 0..{rows - 1} of 12288 "
                      f"({rows / 12288:.1%} of each kernel's work), {reps} timed passes "
                      f"after one warm pass ({reps1} on one thread)",
            "sec_per_pass": dt,
            "value_1_thread": nbytes / dt1 / 1e9,
            "cpu_model": _cpu_model()}


def _timed_both(fn, budget_s, budget_1t_s):
    """Seconds per call of fn on all oracle threads and on one thread (each the
    mean over as many calls as fit the budget, after one warm call)."""
    import oracle

    def timed(budget):
        t0 = time.perf_counter()
        fn()
        one = time.perf_counter() - t0
        reps = max(1, int(budget / max(one, 1e-3)))
        t0 = time.perf_counter()
        for _ in range(reps):
            fn()
        return (time.perf_counter() - t0) / reps, reps

    cores = oracle.get_threads()
    dt, reps = timed(budget_s)
    oracle.set_threads(1)
    try:
        dt1, reps1 = timed(budget_1t_s)
    finally:
        oracle.set_threads(cores)
    return dt, reps, dt1, reps1, cores


def time_oracle_configs(budget_s: float = 3.0, budget_1t_s: float = 2.0, device="cpu"):
    """The CPU oracle on the other configs, bounded samples, all host cores and
    one thread (a reported baseline, not a target).  The large inputs are
    generated on `device` (the same bytes the GPU runs use) and copied to the
    host before any timing."""
    import oracle
    res = {}
    # tiny layer: the whole hot path on W[1024, 1024], X[4, 1024]
    cfg = synth.TinyLayer()
    W, X = synth.bits(cfg.weight()), synth.bits(cfg.activations())
    G = synth.bits(synth.normal_bf16((cfg.N, cfg.K), 1e-3, 0, 5))

    def tiny():
        oracle.fake_quant(W)
        oracle.ste_backward(G)
        Wq, S = oracle.quantize_pack(W)
        oracle.w4a16_gemm(X, Wq, S, want_r=False)
    nk = cfg.N * cfg.K
    nb = 4 * nk + 4 * nk + (2 * nk + nk // 2 + nk // 16) + (nk // 2 + nk // 16 + 2 * X.size +
                                                            2 * cfg.M * cfg.N)
    dt, reps, dt1, reps1, cores = _timed_both(tiny, budget_s, budget_1t_s)
    res["tiny_layer"] = {"value": nb / dt / 1e9, "value_1_thread": nb / dt1 / 1e9,
                         "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"the whole config: fake_quant + STE + quantize_pack + "
                                   f"GEMM (M={cfg.M}) on W[{cfg.N},{cfg.K}]; {reps} / {reps1} "
                                   "timed passes"}
    # prefill at M = 512: the GEMM on 4 rows of X spread over M (every weight
    # group enters every row), throughput extrapolated to the full M
    pcfg = synth.Prefill()
    Wp = synth.bits(pcfg.weight(device))
    Wq, S = oracle.quantize_pack(Wp)
    del Wp
    Xp = synth.bits(pcfg.activations(512, device))
    rows = np.linspace(0, 511, 4).astype(np.int64)
    Xs = np.ascontiguousarray(Xp[rows])
    dt, reps, dt1, reps1, cores = _timed_both(
        lambda: oracle.w4a16_gemm(Xs, Wq, S, want_r=False), budget_s, budget_1t_s)
    fl = 2.0 * len(rows) * pcfg.N * pcfg.K
    res["prefill_m512"] = {"value": fl / dt / 1e12, "value_1_thread": fl / dt1 / 1e12,
                           "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                           "extrapolated": True,
                           "sample": f"W4A16 GEMM of {len(rows)} of the 512 rows of X (evenly spaced) "
                                     f"with the full W[{pcfg.N},{pcfg.K}]; the rate holds "
                                     f"for all 512 rows (time scales linearly in M); "
                                     f"{reps} / {reps1} timed calls"}
    del Wq, S
    # MoE decode, block 16: moe_align + both grouped GEMMs for 4 of the 16 tokens
    # with the routing folded onto 8 of the 128 experts (the per-slot work, one
    # expert's weights per routed token, is the same)
    mcfg = synth.MoEDecode()
    E8, T = 8, 4
    ids, _ = mcfg.routing(16)
    ids = ids[:T]
    ids8 = (ids.numpy() % E8).astype(np.int32)
    hid, inter, topk = mcfg.hidden, mcfg.inter, mcfg.topk
    Wg = synth.normal_bf16((E8, 2 * inter, hid), 0.02, 0, 11, device).cpu()
    Wd = synth.normal_bf16((E8, hid, inter), 0.02, 0, 12, device).cpu()
    Wg_dq = np.stack([oracle.fake_quant(synth.bits(Wg[e]))[0] for e in range(E8)])
    Wd_dq = np.stack([oracle.fake_quant(synth.bits(Wd[e]))[0] for e in range(E8)])
    del Wg, Wd
    A = synth.bits(mcfg.tokens(T))
    Hs = synth.bits(synth.normal_bf16((T * topk, inter), 1.0, 0, 13))

    def moe():
        s_ids, e_ids, npp = oracle.moe_align(ids8, E8, 16)
        oracle.moe_gemm(A, topk, Wg_dq, s_ids, e_ids, npp, T * topk, 16, want_r=False)
        oracle.moe_gemm(Hs, 1, Wd_dq, s_ids, e_ids, npp, T * topk, 16, want_r=False)
    dt, reps, dt1, reps1, cores = _timed_both(moe, budget_s, budget_1t_s)
    nb = E8 * (2 * inter * hid + hid * inter) * 9 // 16 + A.nbytes + Hs.nbytes + \
        2 * T * topk * (2 * inter + hid)
    res["moe_t16"] = {"value": nb / dt / 1e9, "value_1_thread": nb / dt1 / 1e9,
                      "unit": "GB/s", "cores": cores, "kind": "oracle",
                      "sample": f"moe_align + gate_up + down for {T} of the T=16 tokens, "
                                f"top-{topk}, block 16, "
                                f"with the routing folded onto {E8} of the 128 experts "
                                f"(bytes: those experts' packed weights + activations); "
                                f"{reps} / {reps1} timed passes"}
    return res


def _clocked(local, fn):
    """fn() with the clocks sampled around it; returns (fn's result, clocks)."""
    smp = ClockSampler(local)
    smp.start()
    try:
        r = fn()
    finally:
        clocks = smp.stop()
    return r, clocks


def run_config_extras(w4, dev, local, peaks):
    """The other configs' headline figures, measured in the default run with
    their own clock records: prefill GEMM at M = 2048, one MoE decode layer at
    T = 64, the 48-layer QAT weight pass."""
    l2 = torch.zeros(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    flush = lambda: _flush_l2(l2)
    out = {}
    r, c = _clocked(local, lambda: bench_prefill(w4, dev, peaks, [2048], 20, flush))
    out["prefill"] = {**r[0], "clocks": c,
                      "l2": "256 MB buffer read before every timed launch; median of 20"}
    torch.cuda.empty_cache()
    r, c = _clocked(local, lambda: bench_moe_layer(w4, dev, peaks, [64], 20, flush))
    out["moe_layer"] = {**r[0], "clocks": c,
                        "l2": "256 MB buffer read before every timed layer; median of 20"}
    torch.cuda.empty_cache()
    r, c = _clocked(local, lambda: bench_qat_pass(w4, dev, peaks, 3, flush))
    out["qat_pass"] = {"kernels": {x["kernel"]: x for x in r}, "clocks": c,
                       "l2": "each pass reads 9.7 GB (inputs far larger than L2); median of 3"}
    torch.cuda.empty_cache()
    r, c = _clocked(local, lambda: bench_qat_gemm(w4, dev, peaks, [2048], 10, flush))
    out["qat_gemm"] = {**r[0], "clocks": c,
                       "l2": "256 MB buffer read before every timed launch; median of 10"}
    torch.cuda.empty_cache()
    r, c = _clocked(local, lambda: bench_fp4(w4, dev, peaks, 10, flush))
    out["fp4"] = {**r, "clocks": c,
                  "l2": "256 MB buffer read before every timed launch; median of 10"}
    torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------------------
# Main
# ---------------------------------------------------------------------------

def dist_setup(n_gpus: int):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return rank, world, local


def max_over_ranks(x: float, world: int) -> float:
    """Max of a scalar over the ranks (the only collective: timing plumbing)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard(n_items: int, rank: int, world: int) -> range:
    """Contiguous, balanced share of n independent items for this rank."""
    lo = n_items * rank // world
    hi = n_items * (rank + 1) // world
    return range(lo, hi)


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    st, nbytes = oracle_state(args.ref_rows)
    for _ in range(args.warmup if args.warmup < 3 else 1):
        oracle_decode_step(st)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_decode_step(st)
    dt = (time.perf_counter() - t0) / args.steps
    value = nbytes / dt / 1e9
    sample = (f"decode workload restricted to W rows 0..{args.ref_rows - 1} of 12288 per "
              f"step ({args.ref_rows / 12288:.1%} of each kernel's work)")
    line = {"impl": "reference", "metric": METRIC, "metric_detail": METRIC_DETAIL,
            "value": value, "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": decode_config(),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": oracle.get_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# Extra workloads (their own lines; not the default bench line)
# ---------------------------------------------------------------------------

def _flush_l2(buf):
    # Read (not write) a buffer larger than L2: the L2 ends up full of clean
    # lines, so the timed kernel neither hits on its inputs nor pays for writing
    # back a flush buffer's dirty lines.
    torch.sum(buf.view(torch.int32))


def _time_kernel(fn, reps, flush):
    """Median device time (ms) of fn over reps: fn is captured into a CUDA graph
    between two timing events (no host gap inside the window); the L2 is
    flushed before every replay."""
    a = torch.cuda.Event(enable_timing=True, external=True)
    b = torch.cuda.Event(enable_timing=True, external=True)
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        a.record()
        fn()
        b.record()
    ts = []
    for _ in range(reps):
        flush()
        g.replay()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    ts.sort()
    return ts[len(ts) // 2], ts[len(ts) // 10], ts[(9 * len(ts)) // 10]


def bench_prefill(w4, dev, peaks, Ms, reps, flush):
    """Prefill GEMM (W[18432, 7168] Laplace(0, 0.015), group 32) at each M."""
    cfg = synth.Prefill()
    W = cfg.weight(dev)
    Wq, S = w4.quantize_pack(W)
    del W
    res = []
    for M in Ms:
        X = cfg.activations(M, dev)
        Y = torch.empty((M, cfg.N), dtype=torch.bfloat16, device=dev)
        fn = lambda: w4.w4a16_gemm(X, Wq, S, Y)
        for _ in range(3):
            fn()
        med, p10, p90 = _time_kernel(fn, reps, flush)
        fl = 2.0 * M * cfg.N * cfg.K
        tf = fl / (med * 1e-3) / 1e12
        res.append({"M": M, "N": cfg.N, "K": cfg.K, "ms": med, "p10": p10,
                    "p90": p90, "TFLOP/s": tf,
                    "frac_bf16_burst": tf / peaks["bf16_tflops"],
                    "frac_bf16_sustained": tf / peaks["bf16_tflops_sustained"]})
        del X, Y
    return res


def bench_moe_layer(w4, dev, peaks, Ts, reps, flush):
    """One whole MoE decode layer on the GPU (128 experts, top-8, hidden 4096,
    intermediate 1536): gating -> moe_align -> gate_up -> SiLU * up -> down ->
    weighted combine, block size from the library's rule."""
    cfg = synth.MoEDecode()
    E, topk, hid, inter = cfg.E, cfg.topk, cfg.hidden, cfg.inter
    Wg = cfg.gate_up_weight(dev)
    Wd = cfg.down_weight(dev)
    Wq_g = torch.empty((E, 2 * inter, hid // 8), dtype=torch.int32, device=dev)
    S_g = torch.empty((E, 2 * inter, hid // 32), dtype=torch.bfloat16, device=dev)
    Wq_d = torch.empty((E, hid, inter // 8), dtype=torch.int32, device=dev)
    S_d = torch.empty((E, hid, inter // 32), dtype=torch.bfloat16, device=dev)
    for e in range(E):
        w4.w4_quantize_pack(Wg[e], Wq_g[e], S_g[e])
        w4.w4_quantize_pack(Wd[e], Wq_d[e], S_d[e])
    del Wg, Wd
    per_expert = (2 * inter * hid + hid * inter) * 9 // 16
    res = []
    for T in Ts:
        slots = T * topk
        block = w4.w4_moe_block_size(T, topk, E)
        logits = cfg.logits(T, dev)
        X = cfg.tokens(T, dev)
        ids = torch.empty((T, topk), dtype=torch.int32, device=dev)
        wts = torch.empty((T, topk), dtype=torch.float32, device=dev)
        cap = w4.w4_moe_capacity(T, topk, E, block)
        s_ids = torch.empty(cap, dtype=torch.int32, device=dev)
        e_ids = torch.empty(cap // block, dtype=torch.int32, device=dev)
        npp = torch.empty(4, dtype=torch.int32, device=dev)[:1]
        C1 = torch.empty((slots, 2 * inter), dtype=torch.bfloat16, device=dev)
        H = torch.empty((slots, inter), dtype=torch.bfloat16, device=dev)
        C2 = torch.empty((slots, hid), dtype=torch.bfloat16, device=dev)
        out_t = torch.empty((T, hid), dtype=torch.bfloat16, device=dev)
        steps = [
            ("gate_topk", lambda: w4.w4_moe_gate_topk(logits, topk, ids, wts)),
            ("moe_align", lambda: w4.w4_moe_align(ids, E, block, s_ids, e_ids, npp)),
            ("gate_up", lambda: w4.w4_moe_w4a16_gemm(X, topk, Wq_g, S_g, s_ids, e_ids, npp,
                                                     block, slots, C1)),
            ("silu_mul", lambda: w4.w4_silu_mul(C1, H)),
            ("down", lambda: w4.w4_moe_w4a16_gemm(H, 1, Wq_d, S_d, s_ids, e_ids, npp, block,
                                                  slots, C2)),
            ("combine", lambda: w4.w4_moe_combine(C2, wts, out_t)),
        ]
        fused = [steps[0], steps[1],
                 ("gate_up_silu", lambda: w4.w4_moe_w4a16_gemm_silu(
                     X, topk, Wq_g, S_g, s_ids, e_ids, npp, block, slots, H)),
                 steps[4], steps[5]]
        cnt = torch.zeros(w4.w4_moe_combine_counter_bytes(T, hid), dtype=torch.uint8, device=dev)
        down_comb = ("down_combine", lambda: w4.w4_moe_w4a16_gemm_combine(
            H, Wq_d, S_d, s_ids, e_ids, npp, block, wts, C2, cnt, out_t))
        combined = steps[:4] + [down_comb]
        layer = lambda: [f() for _, f in steps]
        layer_fused = lambda: [f() for _, f in fused]
        layer_comb = lambda: [f() for _, f in combined]
        layer()
        layer_fused()
        layer_comb()
        torch.cuda.synchronize()
        active = int(torch.unique(ids).numel())
        lmed, lp10, lp90 = _time_kernel(layer, reps, flush)
        fmed = _time_kernel(layer_fused, reps, flush)[0]
        cmed = _time_kernel(layer_comb, reps, flush)[0]
        per = {}
        for name, f in steps + [fused[2], down_comb]:
            per[name] = _time_kernel(f, max(5, reps // 2), flush)[0] * 1e3
        act_bytes = (2 * T * hid + 4 * T * E + 8 * slots + 2 * slots * 2 * inter * 2 +
                     2 * slots * inter * 2 + 2 * slots * hid * 2 + 2 * T * hid)
        nb = active * per_expert + act_bytes
        gbs = nb / (lmed * 1e-3) / 1e9
        nb_fused = nb - 2 * slots * 2 * inter * 2 - 2 * slots * inter     # no gate_up round trip
        res.append({"T": T, "block": block, "active_experts": active,
                    "layer_us": lmed * 1e3, "p10_us": lp10 * 1e3,
                    "p90_us": lp90 * 1e3, "algorithmic_bytes": nb,
                    "GB/s": gbs, "frac": gbs / peaks["hbm_gbs"],
                    "layer_fused_us": fmed * 1e3,
                    "fused_frac": nb_fused / (fmed * 1e-3) / 1e9 / peaks["hbm_gbs"],
                    "layer_combine_fused_us": cmed * 1e3,
                    "combine_fused_frac": nb / (cmed * 1e-3) / 1e9 / peaks["hbm_gbs"],
                    "per_kernel_us": per})
    return res


def bench_qat_pass(w4, dev, peaks, reps, flush):
    """The QAT weight pass over the 48-layer stack (96 matrices, 4.83 G
    elements): fake_quant, STE into a separate buffer, quantize_pack, each over
    all matrices back to back."""
    cfg = synth.QATStack()
    mats = []
    for layer in range(cfg.layers):
        for which in range(2):
            W = cfg.weight(layer, which, dev)
            G = cfg.grad(layer, which, dev)
            rows, K = W.shape
            mats.append((W, G, torch.empty_like(W), torch.empty_like(W),
                         torch.empty((rows, K // 8), dtype=torch.int32, device=dev),
                         torch.empty((rows, K // 32), dtype=torch.bfloat16, device=dev)))
    n = cfg.elements

    def fq():
        for (W, G, Wdq, dW, Wq, S) in mats:
            w4.w4_fake_quant(W, Wdq)

    def ste():
        for (W, G, Wdq, dW, Wq, S) in mats:
            w4.w4_ste_backward(G, dW)

    def qp():
        for (W, G, Wdq, dW, Wq, S) in mats:
            w4.w4_quantize_pack(W, Wq, S)

    res = []
    for name, f, bpe in (("fake_quant", fq, 4.0), ("ste_backward", ste, 4.0),
                         ("quantize_pack", qp, 2.5625)):
        f()
        med, p10, p90 = _time_kernel(f, reps, flush)
        gbs = n * bpe / (med * 1e-3) / 1e9
        res.append({"kernel": name, "elements": n, "ms": med, "GB/s": gbs,
                    "frac": gbs / peaks["hbm_gbs"]})
    del mats
    return res


def bench_qat_gemm(w4, dev, peaks, Ms, reps, flush):
    """QAT GEMMs on a layer of the QAT stack (W[12288, 4096]) with the fake
    quantization fused into the weight prologue -- forward Y = X . Wdq^T and
    input gradient dX = dY . Wdq -- beside the unfused chain (w4_fake_quant,
    then a cuBLAS BF16 GEMM on the materialized Wdq)."""
    cfg = synth.QATStack()
    N, K = cfg.shapes[0]
    W = cfg.weight(0, 0, dev)
    Wdq = torch.empty_like(W)
    res = []
    for M in Ms:
        X = synth.normal_bf16((M, K), 1.0, 0, 400 + M, dev)
        dY = synth.normal_bf16((M, N), 1.0, 0, 500 + M, dev)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
        runs = {
            "forward_fused": lambda: w4.w4_qat_gemm(X, W, Y),
            "forward_unfused": lambda: (w4.w4_fake_quant(W, Wdq), torch.matmul(X, Wdq.t(), out=Y)),
            "dx_fused": lambda: w4.w4_qat_gemm_dx(dY, W, dX),
            "dx_unfused": lambda: (w4.w4_fake_quant(W, Wdq), torch.matmul(dY, Wdq, out=dX)),
        }
        fl = 2.0 * M * N * K
        r = {"M": M, "N": N, "K": K,
             "unfused": "w4_fake_quant + torch.matmul (cuBLAS BF16) on the materialized Wdq"}
        for name, f in runs.items():
            for _ in range(3):
                f()
            med, p10, p90 = _time_kernel(f, reps, flush)
            tf = fl / (med * 1e-3) / 1e12
            r[name] = {"ms": med, "p10": p10, "p90": p90, "TFLOP/s": tf,
                       "frac_bf16_burst": tf / peaks["bf16_tflops"]}
        res.append(r)
        del X, dY, Y, dX
    return res


def bench_fp4(w4, dev, peaks, reps, flush):
    """Micro-scaled FP4 weights (MXFP4 and NVFP4) on the decode layer's shape
    W[12288, 4096]: the W4A16 GEMM at M = 1 and 16 (GB/s of packed codes +
    scales + activations + output) and M = 2048 (TFLOP/s), and the quantizers
    (GB/s of BF16 in + codes and scales out)."""
    cfg = synth.Decode()
    W = cfg.weight(dev)
    N, K = cfg.N, cfg.K
    mx = w4.quantize_pack_mxfp4(W)
    nv = w4.quantize_pack_nvfp4(W)
    g = float(nv[2].item())
    res = {}
    for fmt, Wq, sc, run in (
            ("mxfp4", mx[0], mx[1], lambda X, Y: w4.w4a16_gemm_mxfp4(X, mx[0], mx[1], Y)),
            ("nvfp4", nv[0], nv[1], lambda X, Y: w4.w4a16_gemm_nvfp4(X, nv[0], nv[1], g, Y))):
        r = {}
        for M in (1, 16, 2048):
            X = cfg.activations(M, dev) if M <= 64 else synth.normal_bf16((M, K), 1.0, 0, 600, dev)
            Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            f = lambda: run(X, Y)
            for _ in range(3):
                f()
            med, p10, p90 = _time_kernel(f, reps, flush)
            nb = Wq.nbytes + sc.nbytes + X.nbytes + Y.nbytes
            gbs = nb / (med * 1e-3) / 1e9
            tf = 2.0 * M * N * K / (med * 1e-3) / 1e12
            r[f"gemm_m{M}"] = {"us": med * 1e3, "p10_us": p10 * 1e3, "p90_us": p90 * 1e3,
                               "GB/s": gbs, "frac_hbm": gbs / peaks["hbm_gbs"], "TFLOP/s": tf,
                               "frac_bf16_burst": tf / peaks["bf16_tflops"]}
            del X, Y
        Wq2, sc2 = torch.empty_like(Wq), torch.empty_like(sc)
        gd = torch.empty(1, dtype=torch.float32, device=dev)
        if fmt == "mxfp4":
            qf = lambda: w4.w4_quantize_pack_mxfp4(W, Wq2, sc2)
        else:
            qf = lambda: (w4.w4_nvfp4_tensor_scale(W, gd), w4.w4_quantize_pack_nvfp4(W, gd, Wq2, sc2))
        for _ in range(3):
            qf()
        med, _, _ = _time_kernel(qf, reps, flush)
        nb = W.nbytes + Wq.nbytes + sc.nbytes + (W.nbytes if fmt == "nvfp4" else 0)
        r["quantize_pack"] = {"us": med * 1e3, "GB/s": nb / (med * 1e-3) / 1e9,
                              "frac_hbm": nb / (med * 1e-3) / 1e9 / peaks["hbm_gbs"],
                              "bytes": "BF16 W in, codes + scales out" +
                                       (" (+ W read once more for the tensor amax)"
                                        if fmt == "nvfp4" else "")}
        res[fmt] = r
    return res


def run_extra(args):
    import int4_w4a16_b200 as w4
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w4.lib()
    peaks = load_peaks()
    l2 = torch.zeros(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    flush = lambda: _flush_l2(l2)
    reps = max(5, args.steps)
    out = {"workload": args.workload, "peaks": peaks, "l2": "256 MB buffer read before "
           "every timed launch", "reps": reps, "results": []}
    if args.workload == "prefill":
        out["results"] += bench_prefill(w4, dev, peaks, [args.m] if args.m else synth.Prefill().Ms,
                                        reps, flush)
    elif args.workload == "moe":
        cfg = synth.MoEDecode()
        Wg = cfg.gate_up_weight(dev)
        Wd = cfg.down_weight(dev)
        E = cfg.E
        Wq_g = torch.empty((E, 2 * cfg.inter, cfg.hidden // 8), dtype=torch.int32, device=dev)
        S_g = torch.empty((E, 2 * cfg.inter, cfg.hidden // 32), dtype=torch.bfloat16, device=dev)
        Wq_d = torch.empty((E, cfg.hidden, cfg.inter // 8), dtype=torch.int32, device=dev)
        S_d = torch.empty((E, cfg.hidden, cfg.inter // 32), dtype=torch.bfloat16, device=dev)
        for e in range(E):
            w4.w4_quantize_pack(Wg[e], Wq_g[e], S_g[e])
            w4.w4_quantize_pack(Wd[e], Wq_d[e], S_d[e])
        del Wg, Wd
        per_gu = 2 * cfg.inter * cfg.hidden * 9 // 16
        per_dn = cfg.hidden * cfg.inter * 9 // 16
        for T in ([args.m] if args.m else cfg.Ts):
            ids, _ = cfg.routing(T, args.skew)
            ids_d = ids.to(dev)
            active = len(set(ids.view(-1).tolist()))
            hist = torch.bincount(ids.view(-1).long(), minlength=E)
            X = cfg.tokens(T, dev)
            H = synth.normal_bf16((T * cfg.topk, cfg.inter), 1.0, 0, 300 + T, dev)
            for block in ([args.block] if args.block else cfg.blocks):
                s_ids, e_ids, npp = w4.moe_align(ids_d, E, block)
                C1 = torch.empty((T * cfg.topk, 2 * cfg.inter), dtype=torch.bfloat16, device=dev)
                C2 = torch.empty((T * cfg.topk, cfg.hidden), dtype=torch.bfloat16, device=dev)
                f_align = lambda: w4.w4_moe_align(ids_d, E, block, s_ids, e_ids, npp)
                f_gu = lambda: w4.w4_moe_w4a16_gemm(X, cfg.topk, Wq_g, S_g, s_ids, e_ids, npp,
                                                    block, T * cfg.topk, C1)
                f_dn = lambda: w4.w4_moe_w4a16_gemm(H, 1, Wq_d, S_d, s_ids, e_ids, npp, block,
                                                    T * cfg.topk, C2)
                for f in (f_align, f_gu, f_dn):
                    f()
                t_al = _time_kernel(f_align, reps, flush)[0]
                t_gu = _time_kernel(f_gu, reps, flush)[0]
                t_dn = _time_kernel(f_dn, reps, flush)[0]
                npad = int(npp.item())
                b_gu = active * per_gu + X.nbytes + C1.nbytes
                b_dn = active * per_dn + H.nbytes + C2.nbytes
                out["results"].append({
                    "T": T, "block": block, "skew": args.skew, "active_experts": active,
                    "max_expert_slots": int(hist.max()), "padded_slots": npad,
                    "moe_align_us": t_al * 1e3,
                    "gate_up_us": t_gu * 1e3, "gate_up_GB/s": b_gu / (t_gu * 1e-3) / 1e9,
                    "gate_up_frac": b_gu / (t_gu * 1e-3) / 1e9 / peaks["hbm_gbs"],
                    "down_us": t_dn * 1e3, "down_GB/s": b_dn / (t_dn * 1e-3) / 1e9,
                    "down_frac": b_dn / (t_dn * 1e-3) / 1e9 / peaks["hbm_gbs"]})
    elif args.workload == "moe_layer":
        out["results"] += bench_moe_layer(w4, dev, peaks,
                                          [args.m] if args.m else synth.MoEDecode().Ts, reps, flush)
    elif args.workload == "zp":
        # asymmetric (zero-point) groups: quantizer on the decode sweep's weights
        # (W[12288, 4096]), then the GEMM on that shape at decode and prefill
        # token counts, the symmetric path beside it
        cfg = synth.Decode()
        W = cfg.weight(dev)
        n = W.numel()
        Wq = torch.empty((cfg.N, cfg.K // 8), dtype=torch.int32, device=dev)
        S = torch.empty((cfg.N, cfg.K // 32), dtype=torch.bfloat16, device=dev)
        Z = torch.empty((cfg.N, cfg.K // 32), dtype=torch.uint8, device=dev)
        fq = lambda: w4.w4_quantize_pack_zp(W, Wq, S, Z)
        for _ in range(3):
            fq()
        med, p10, p90 = _time_kernel(fq, reps, flush)
        bpe = 2.0 + 0.5 + 3.0 / 32          # W read; codes, scale and zero point written
        gbs = n * bpe / (med * 1e-3) / 1e9
        out["results"].append({"kernel": "quantize_pack_zp", "elements": n, "us": med * 1e3,
                               "GB/s": gbs, "frac": gbs / peaks["hbm_gbs"]})
        Wq_s, S_s = w4.quantize_pack(W)
        del W
        for M in ([args.m] if args.m else (1, 16, 512, 2048)):
            X = synth.normal_bf16((M, cfg.K), 1.0, 0, 500 + M, dev)
            Y = torch.empty((M, cfg.N), dtype=torch.bfloat16, device=dev)
            fz = lambda: w4.w4a16_gemm_zp(X, Wq, S, Z, Y)
            fs = lambda: w4.w4a16_gemm(X, Wq_s, S_s, Y)
            for f in (fz, fs):
                for _ in range(3):
                    f()
            med, p10, p90 = _time_kernel(fz, reps, flush)
            smed = _time_kernel(fs, reps, flush)[0]
            byts = cfg.N * cfg.K * (0.5 + 3.0 / 32) + 2.0 * M * (cfg.K + cfg.N)
            fl = 2.0 * M * cfg.N * cfg.K
            out["results"].append({"kernel": "w4a16_gemm_zp", "M": M, "N": cfg.N, "K": cfg.K,
                                   "us": med * 1e3, "GB/s": byts / (med * 1e-3) / 1e9,
                                   "frac_hbm": byts / (med * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                   "TFLOP/s": fl / (med * 1e-3) / 1e12,
                                   "frac_bf16_burst": fl / (med * 1e-3) / 1e12 / peaks["bf16_tflops"],
                                   "symmetric_us": smed * 1e3})
    elif args.workload == "qat_gemm":
        out["results"] += bench_qat_gemm(w4, dev, peaks, [args.m] if args.m else [2048, 8192],
                                         reps, flush)
    elif args.workload == "fp4":
        out["results"].append(bench_fp4(w4, dev, peaks, reps, flush))
    elif args.workload == "gemv":
        # the decode GEMM alone, one activation height at a time (--m picks one)
        cfg = synth.Decode()
        W = cfg.weight(dev)
        Wq, S = w4.quantize_pack(W)
        del W
        # 16 copies of the packed weight (453 MB, several times the L2) for the
        # rotation measurement below
        n_rot = 16
        rot = [(Wq.clone(), S.clone()) for _ in range(n_rot)]
        for M in ([args.m] if args.m else cfg.Ms):
            X = cfg.activations(M, dev)
            Y = torch.empty((M, cfg.N), dtype=torch.bfloat16, device=dev)
            fn = lambda: w4.w4a16_gemm(X, Wq, S, Y)
            for _ in range(3):
                fn()
            med, p10, p90 = _time_kernel(fn, reps, flush)
            nb = Wq.nbytes + S.nbytes + X.nbytes + Y.nbytes
            gbs = nb / (med * 1e-3) / 1e9
            # the same GEMM over the 16 copies in turn, one CUDA graph between one
            # event pair: every launch reads weights that are not in L2, and no
            # flush kernel or event sits between launches
            rot_fn = lambda: [w4.w4a16_gemm(X, q, s_, Y) for q, s_ in rot]
            rot_fn()
            rmed, _, _ = _time_kernel(rot_fn, max(5, reps // 4), lambda: None)
            rus = rmed * 1e3 / n_rot
            out["results"].append({"M": M, "N": cfg.N, "K": cfg.K, "us": med * 1e3,
                                   "p10_us": p10 * 1e3, "p90_us": p90 * 1e3,
                                   "algorithmic_bytes": nb, "GB/s": gbs,
                                   "frac": gbs / peaks["hbm_gbs"],
                                   "rotated_us_per_launch": rus,
                                   "rotated_frac": nb / (rus * 1e-6) / 1e9 / peaks["hbm_gbs"]})
    elif args.workload == "quant":
        # the decode-weight quantizers one at a time
        cfg = synth.Decode()
        W = cfg.weight(dev)
        G = synth.normal_bf16(W.shape, 1e-3, 0, 1, dev)
        Wdq, dW = torch.empty_like(W), torch.empty_like(W)
        Wq = torch.empty((cfg.N, cfg.K // 8), dtype=torch.int32, device=dev)
        S = torch.empty((cfg.N, cfg.K // 32), dtype=torch.bfloat16, device=dev)
        n = W.numel()
        for name, f, bpe in (("fake_quant", lambda: w4.w4_fake_quant(W, Wdq), 4.0),
                             ("ste_backward", lambda: w4.w4_ste_backward(G, dW), 4.0),
                             ("quantize_pack", lambda: w4.w4_quantize_pack(W, Wq, S), 2.5625)):
            for _ in range(3):
                f()
            med, p10, p90 = _time_kernel(f, reps, flush)
            gbs = n * bpe / (med * 1e-3) / 1e9
            out["results"].append({"kernel": name, "elements": n, "us": med * 1e3,
                                   "GB/s": gbs, "frac": gbs / peaks["hbm_gbs"]})
    elif args.workload == "qat":
        out["results"] += bench_qat_pass(w4, dev, peaks, max(3, reps // 10), flush)
    w4.w4_device_status()
    print(json.dumps(out), flush=True)
    return 0


METRIC = "W4A16 GEMM HBM GB/s & TFLOP/s vs roofline; quantize/pack GB/s (1×B200)"
# What `value` is under that metric: algorithmic bytes of one whole step of the
# hot path (fake-quant + STE + quantize_pack of the decode weight, then the
# decode GEMM at each activation height) divided by the step's device time.
METRIC_DETAIL = ("hot-path step throughput: algorithmic bytes of fake_quant + STE + "
                 "quantize_pack + W4A16 GEMM (M = 1, 8, 16, 32) on the decode weight / step time")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--m", type=int, default=0,
                    help="one size only: the activation height (--workload gemv, prefill) or "
                         "the token count T (--workload moe)")
    ap.add_argument("--block", type=int, default=0, help="--workload moe: one block size only")
    ap.add_argument("--skew", type=float, default=0.0,
                    help="--workload moe: Zipf-like routing skew (0 = uniform logits)")
    ap.add_argument("--workload", default="decode",
                    choices=["decode", "prefill", "moe", "moe_layer", "qat", "qat_gemm", "gemv",
                             "quant", "zp", "fp4"],
                    help="decode is the bench line; the others print their own lines")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other configs' blocks (prefill, MoE layer, QAT pass)")
    ap.add_argument("--ref-rows", type=int, default=512)
    ap.add_argument("--e2e-steps", type=int, default=8)
    args = ap.parse_args()

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        return run_reference(args, rank, 1)

    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}))
        return 1
    if args.workload != "decode":
        return run_extra(args)
    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    import int4_w4a16_b200 as w4
    w4.lib()
    wl = DecodeWorkload(dev)
    peaks = load_peaks()
    stream = torch.cuda.current_stream()

    for _ in range(max(3, args.warmup)):
        wl.step()                       # eager warm-up (also sizes the GEMM workspace)
    w4.w4_device_status()

    # The timed steps run as one CUDA graph of K steps with no event inside, so
    # neither host launch overhead nor event records are in `value` (the e2e
    # figure below goes through the eager public API instead).  Two more graphs
    # of the same K steps, replayed after it, give the breakdown: one with an
    # event pair around every launch (per-kernel times), one with a single
    # event pair around each step's decode GEMM launches (the GEMM family).
    def ev():
        return torch.cuda.Event(enable_timing=True, external=True)

    def capture(nsteps, mode):
        evs = None
        if mode == "kernel":
            evs = [{k: (ev(), ev()) for k in wl.kernels} for _ in range(nsteps)]
        elif mode == "gemm":
            evs = [(ev(), ev()) for _ in range(nsteps)]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(nsteps):
                if mode == "kernel":
                    wl.step(evs[i])
                elif mode == "gemm":
                    wl.step(None, evs[i])
                else:
                    wl.step()
        return g, evs

    roll, _ = capture(8, None)
    timed, _ = capture(args.steps, None)
    timed_k, evs = capture(args.steps, "kernel")
    timed_g, gevs = capture(args.steps, "gemm")
    for _ in range(max(3, args.warmup)):
        roll.replay()
    timed_k.replay()
    timed_g.replay()
    torch.cuda.synchronize()

    sampler = ClockSampler(local) if rank == 0 else None
    if sampler:
        sampler.start()
    # pre-roll so that the clock sampler sees the GPU under this load
    t_end = time.perf_counter() + 0.6
    while time.perf_counter() < t_end:
        roll.replay()
    torch.cuda.synchronize()

    barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    timed.replay()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    elapsed_ms = t0.elapsed_time(t1)
    # the breakdown graphs, under the same load
    timed_k.replay()
    timed_g.replay()
    torch.cuda.synchronize()
    # post-roll for the sampler
    t_end = time.perf_counter() + 0.4
    while time.perf_counter() < t_end:
        roll.replay()
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    w4.w4_device_status()

    elapsed_ms = max_over_ranks(elapsed_ms, world)
    ms_per_step = elapsed_ms / args.steps
    value = world * wl.step_bytes * args.steps / (elapsed_ms * 1e-3) / 1e9

    # per-kernel averages over the timed region
    per = {}
    for k in wl.kernels:
        ts = [e[k][0].elapsed_time(e[k][1]) for e in evs]
        per[k] = sum(ts) / len(ts)
    rooflines = {}
    for k in wl.kernels:
        us = per[k] * 1e3
        gbs = wl.bytes[k] / (per[k] * 1e-3) / 1e9
        r = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
             "frac": gbs / peaks["hbm_gbs"], "us": us, "algorithmic_bytes": wl.bytes[k],
             "traffic": _traffic(k, "decode")}
        if k in wl.flops:
            r["tflops"] = wl.flops[k] / (per[k] * 1e-3) / 1e12
        rooflines[k] = r
    gemm_us = sum(a.elapsed_time(b) for a, b in gevs) / len(gevs) * 1e3
    gemm_us_per_kernel_sum = sum(per[k] for k in wl.kernels if k.startswith("gemm")) * 1e3
    gemm_bytes = sum(wl.bytes[k] for k in wl.kernels if k.startswith("gemm"))
    # The dominant kernel is the one with the largest share of the step; the four
    # decode GEMM launches (one kernel at four activation heights) count together.
    shares = {k: per[k] for k in wl.kernels if not k.startswith("gemm")}
    shares["w4a16_gemm"] = gemm_us * 1e-3
    dominant = max(shares, key=lambda k: shares[k])
    if dominant == "w4a16_gemm":
        gbs = gemm_bytes / (gemm_us * 1e-6) / 1e9
        dom_roofline = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": gbs / peaks["hbm_gbs"],
                        "traffic": _traffic("gemm_m16", "decode"),
                        "note": "decode GEMM, launches at M = 1, 8, 16, 32 together: "
                                "algorithmic bytes summed over the four / the time between "
                                "one event pair around the four launches; traffic is the "
                                "M = 16 launch's"}
    else:
        dom_roofline = {k: v for k, v in rooflines[dominant].items()
                        if k in ("bound", "achieved", "peak", "unit", "frac", "traffic")}

    # end to end through the public API, from pinned host memory
    host, h2d, d2h = wl.host_buffers()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    wl.e2e_run(host, 2, e0, e1)                         # warm-up
    torch.cuda.synchronize()
    barrier(world)
    wl.e2e_run(host, args.e2e_steps, e0, e1)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / args.e2e_steps
    e2e_value = world * wl.step_bytes / (e2e_ms * 1e-3) / 1e9
    launches = wl.launches_per_step * args.steps
    config = wl.config()

    cpu = None
    cpu_configs = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = time_oracle()
        cpu_configs = time_oracle_configs(device=dev)

    extras = {}
    if world == 1 and not args.no_extras:
        del wl, roll, timed, timed_k, timed_g
        torch.cuda.empty_cache()
        extras = run_config_extras(w4, dev, local, peaks)
        w4.w4_device_status()

    if rank == 0:
        line = {
            "metric": METRIC, "metric_detail": METRIC_DETAIL, "value": value, "unit": "GB/s",
            "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic", "config": config,
            "roofline": {"kernel": dominant, **dom_roofline, "peak_source": peaks["source"]},
            "rooflines": rooflines,
            "decode_gemm": {"GB/s": gemm_bytes / (gemm_us * 1e-6) / 1e9,
                            "frac": gemm_bytes / (gemm_us * 1e-6) / 1e9 / peaks["hbm_gbs"],
                            "us_4M_one_event_pair": gemm_us,
                            "us_4M_sum_of_per_kernel_events": gemm_us_per_kernel_sum},
            "cpu_baseline": cpu,
            "cpu_baseline_configs": cpu_configs,
            **extras,
            "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                    "steps": args.e2e_steps,
                    "pipelining": "step i+1's host-to-device copies and step i-1's "
                                  "device-to-host copies on their own streams, overlapping "
                                  "step i's kernels (two device buffer sets)"},
            "gpu_launches": launches,
            "launch": "timed steps replayed as one CUDA graph with no events inside; per-kernel "
                      "and GEMM-family times from two more replays of the same steps with events",
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

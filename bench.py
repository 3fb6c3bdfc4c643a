#!/usr/bin/env python
"""Benchmark of the NF4 frozen-base LoRA linear layer on B200.

One step = the whole hot path on one batch: NF4-quantize the frozen 4096x4096
weight with double quantization, forward (Zc = c·X·A, Y = X·Ŵ + Zc·B) and
backward (dZ, dX = dY·Ŵᵀ + dZ·Aᵀ, dA, dB) for M = 4096 tokens, r = 16,
alpha = 32.  With N > 1 processes (torchrun, one per GPU) every rank runs its
own batch of 4096 tokens against the same frozen weight (data parallel, weak
scaling) and dA, dB are summed across ranks with an NCCL all-reduce.

metric : fwd+bwd TFLOP/s = (4MKN + 6Mr(K+N)) per step per rank, summed over
         ranks, divided by the step time (max over ranks).  The step time
         includes the per-step quantization.
Also reported: the live roofline of the dominant kernel (the fused NF4 GEMM),
the GEMV GB/s sweep (M in 1/4/16 on 4096x11008 and 11008x4096) and the
quantize GB/s of the 8192x22016 weight, the end-to-end number with host
buffers, and the CPU oracle on a bounded sample.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "QLoRA NF4 linear fwd+bwd TFLOP/s (M=4096), GEMV GB/s; % of B200 roofline"
WORKLOAD = "proj-4096x4096-m4096-r16-dq"
M, K, N, R, ALPHA = 4096, 4096, 4096, 16, 32.0
ROTATE = 3          # input sets cycled per step: 3 x 96 MB of bf16 inputs > 2 x 126 MB L2


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of the
# fused kernel at M = K = N = 4096, mean of its forward and dX launches in one
# ncu capture of the current kernel; None once the kernel changes.
FUSED_TRAFFIC_BYTES = 0.5 * ((42661632 + 2432768) + (44022528 + 4504320))


def flops_step(Mt=M, Kt=K, Nt=N, r=R):
    return 4.0 * Mt * Kt * Nt + 6.0 * Mt * r * (Kt + Nt)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"hbm": float(d["hbm_gbs"]), "bf16": float(d["bf16_tflops"]),
                "bf16_sus": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "src": "measured"}
    except Exception:
        return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sus": 1400.0, "src": "fallback"}


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """SM clock and clock-event (throttle) reasons of this process's GPU,
    sampled every 0.5 ms through NVML while the timed region runs (the GPU is
    found by its UUID, so CUDA_VISIBLE_DEVICES does not matter); falls back to
    `nvidia-smi -lms 20` when NVML is not available."""
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, torch_device):
        self.dev = torch_device
        self.samples = []
        self.stop_flag = False
        self.thread = None
        self.proc = None
        self.smax = None

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
        if not uuid.startswith("GPU-"):
            uuid = "GPU-" + uuid
        return pynvml, pynvml.nvmlDeviceGetHandleByUUID(uuid)

    def start(self):
        try:
            nv, h = self._nvml_handle()
            self.smax = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))

            def loop():
                while not self.stop_flag:
                    try:
                        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                        rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.samples.append((float(sm), int(rs)))
                    except Exception:
                        pass
                    time.sleep(0.0005)
            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            return
        except Exception:
            self.thread = None
        try:
            idx = int(os.environ.get("LOCAL_RANK", "0"))
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.lines = []
            self.thread = threading.Thread(target=lambda: [self.lines.append(ln.strip())
                                                           for ln in self.proc.stdout], daemon=True)
            self.thread.start()
            time.sleep(0.2)
        except Exception:
            self.proc = None

    def stop(self):
        self.stop_flag = True
        sm, reasons = [], set()
        if self.proc is not None:
            time.sleep(0.05)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            names = [n for n, _ in self.REASONS]
            for ln in self.lines:
                parts = [q.strip() for q in ln.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    self.smax = float(parts[2])
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(nm)
            src = "nvidia-smi"
        elif self.thread is not None:
            self.thread.join(timeout=1.0)
            for f, rs in self.samples:
                sm.append(f)
                for nm, bit in self.REASONS:
                    if rs & bit:
                        reasons.add(nm)
            src = "nvml"
        else:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock source"]}
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.smax,
                "reasons": sorted(reasons), "samples": len(sm), "source": src}


# ---------------------------------------------------------------------------
# CPU oracle on a bounded sample (baseline only)
# ---------------------------------------------------------------------------
# reference arm (--impl reference): a slice per step, so that hundreds of steps
# still end within a few minutes
ORACLE_KS, ORACLE_MS = 1024, 256   # rows of W quantized, tokens pushed through fwd+bwd
# cpu_baseline leg of the GPU arm: the whole M = K = N = 4096 step, repeated
CPU_BASELINE_REPS = 3


def oracle_sample_inputs(ks=None, ms=None):
    import numpy as np
    from inputs import synthetic as S
    ks = ORACLE_KS if ks is None else ks
    ms = ORACLE_MS if ms is None else ms
    lin = S.config2(M=ms).linears[0]
    return (np.ascontiguousarray(lin.W[:ks]), np.ascontiguousarray(lin.X[:, :ks]),
            np.ascontiguousarray(lin.A[:ks]), lin.B, lin.dY)


def oracle_step(inputs):
    from oracle import nf4
    from oracle.linear import lora_backward, lora_forward
    W, X, A, B, G = inputs
    codes, absmax = nf4.quantize_nf4(W.ravel())
    payload, n = nf4.pack_codes(codes)
    code8, s2, off = nf4.double_quantize(absmax)
    a = nf4.decode_scales(absmax.size, code8=code8, s2=s2, offset=off)
    w_hat = nf4.dequantize(payload, n, a).reshape(W.shape)
    c = ALPHA / R
    lora_forward(X, w_hat, A, B, c)
    lora_backward(G, X, w_hat, A, B, c)


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return len(os.sched_getaffinity(0))


def oracle_flops():
    return flops_step(ORACLE_MS, ORACLE_KS, N, R)


SAMPLE_DESC = (f"oracle (NumPy fp64) on a slice: quantize+double-quantize+dequantize "
               f"W[:{ORACLE_KS}, :{N}], then fwd+bwd for {ORACLE_MS} tokens over K={ORACLE_KS}; "
               f"TFLOP/s from that slice's 4MKN+6Mr(K+N)")


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    inputs = oracle_sample_inputs()
    for _ in range(args.warmup):
        oracle_step(inputs)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(inputs)
    dt = (time.perf_counter() - t0) / args.steps
    v = oracle_flops() / dt / 1e12
    cores = oracle_threads()
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample": SAMPLE_DESC},
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": SAMPLE_DESC},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def make_sets(torch, dev, nsets):
    import numpy as np
    from inputs import synthetic as S
    sets = []
    for s in range(nsets):
        lin = S.config2(seed=s).linears[0]
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(dev).to(torch.bfloat16)
        sets.append({"W": t(lin.W), "X": t(lin.X), "dY": t(lin.dY), "A": t(lin.A), "B": t(lin.B),
                     "host": lin if s == 0 else None})
    return sets


def prof_read(q, kind):
    import ctypes as C
    ms, n = C.c_double(0), C.c_int64(0)
    q.lib.qlora_profile_read(kind, C.byref(ms), C.byref(n))
    return ms.value, n.value


def gemv_sweep(torch, q, dev, peaks):
    """Forward GEMV GB/s for M in {1,4,16} on 4096x11008 and 11008x4096 (DQ,
    r=16), >= 12 rotated weight copies (> 2x L2), replayed from a CUDA graph."""
    out = []
    gen = torch.Generator(device=dev)
    for (Kg, Ng) in ((4096, 11008), (11008, 4096)):
        ncopy = 12
        ws = []
        for i in range(ncopy):
            gen.manual_seed(1000 + i)
            W = (torch.randn((Kg, Ng), generator=gen, device=dev) * 0.02).to(torch.bfloat16)
            ws.append(q.quantize(W, double_quant=True))
            del W
        gen.manual_seed(7)
        A = (torch.randn((Kg, 16), generator=gen, device=dev) * 0.01).to(torch.bfloat16)
        B = (torch.randn((16, Ng), generator=gen, device=dev) * 0.01).to(torch.bfloat16)
        for Mg in (1, 4, 16):
            X = torch.randn((Mg, Kg), generator=gen, device=dev).to(torch.bfloat16)
            Y = torch.empty((Mg, Ng), dtype=torch.bfloat16, device=dev)
            Zc = torch.empty((Mg, 16), dtype=torch.bfloat16, device=dev)
            for w in ws:                       # warm-up, workspace sizing
                q.linear_forward(X, w, A, B, 2.0, Y=Y, Zc=Zc)
            torch.cuda.synchronize()
            st = q.new_status(dev)
            s = torch.cuda.Stream(device=dev)
            s.wait_stream(torch.cuda.current_stream(dev))
            with torch.cuda.stream(s):         # warm-up on the capture stream (its workspace)
                for w in ws:
                    q.linear_forward(X, w, A, B, 2.0, Y=Y, Zc=Zc, status=st)
            s.synchronize()
            g = torch.cuda.CUDAGraph()
            reps = 4
            with torch.cuda.stream(s):
                with torch.cuda.graph(g, stream=s):
                    for _ in range(reps):
                        for w in ws:
                            q.linear_forward(X, w, A, B, 2.0, Y=Y, Zc=Zc, status=st)
            for _ in range(3):
                g.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            per = e0.elapsed_time(e1) / (reps * ncopy) * 1e-3
            n1 = Kg * Ng // 64
            n2 = (n1 + 255) // 256
            nbytes = Kg * Ng // 2 + n1 + 4 * n2 + 4 + 2 * Mg * Kg + 2 * 16 * (Kg + Ng) + 2 * Mg * Ng
            gbs = nbytes / per / 1e9
            out.append({"M": Mg, "K": Kg, "N": Ng, "us": per * 1e6, "GB/s": gbs,
                        "frac": gbs / peaks["hbm"]})
            del g
        del ws
    return out


def quantize_bench(torch, q, dev, peaks):
    """Quantize (with DQ) of the 8192x22016 bf16 weight: GB/s of 2P + P/2 + n1 + 4n2 + 4."""
    gen = torch.Generator(device=dev)
    gen.manual_seed(5)
    Kq, Nq = 8192, 22016
    W = (torch.randn((Kq, Nq), generator=gen, device=dev) * 0.015).to(torch.bfloat16)
    w = q.quantize(W, double_quant=True)
    st = q.new_status(dev)
    ws = torch.empty(int(q.lib.qlora_nf4_quantize_workspace_size(Kq * Nq, 1)), dtype=torch.uint8,
                     device=dev)
    for _ in range(3):
        q.quantize(W, double_quant=True, out=w, status=st, workspace=ws)
    torch.cuda.synchronize()
    # launches back to back, no per-launch events (they would keep each launch
    # from overlapping its predecessor's tail)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 10
    e0.record()
    for _ in range(reps):
        q.quantize(W, double_quant=True, out=w, status=st, workspace=ws)
    e1.record()
    torch.cuda.synchronize()
    code, _ = q.status_sync(st)
    if code != 0:
        raise SystemExit(f"device status {code} in the quantize sweep")
    per = e0.elapsed_time(e1) / reps * 1e-3
    P = Kq * Nq
    n1 = P // 64
    n2 = (n1 + 255) // 256
    nbytes = 2 * P + P // 2 + n1 + 4 * n2 + 4
    gbs = nbytes / per / 1e9
    del W
    return {"shape": [Kq, Nq], "us": per * 1e6, "GB/s": gbs, "frac": gbs / peaks["hbm"]}


def run_case(args):
    """One kernel workload, --reps launches, no timing: the command ncu captures.
    gemv: forward with M <= 16 tokens (DQ weight, r = 16, c = 2);
    quantize: NF4 + DQ quantization of a K x N bf16 weight;
    merge: the merged bf16 weight of a K x N DQ weight with r = 64."""
    import torch
    import bit_nf4_quantized_pack_b200 as q
    dev = torch.device("cuda", 0)
    gen = torch.Generator(device=dev)
    gen.manual_seed(11)
    st = q.new_status(dev)
    if args.case == "gemv":
        Mg, Kg, Ng = (int(v) for v in (args.shape or "1,4096,11008").split(","))
        # two weights, alternated, so no launch reads the previous one from L2
        ws = []
        for _ in range(2):
            W = (torch.randn((Kg, Ng), generator=gen, device=dev) * 0.02).to(torch.bfloat16)
            ws.append(q.quantize(W, double_quant=True, status=st))
            del W
        A = (torch.randn((Kg, 16), generator=gen, device=dev) * 0.01).to(torch.bfloat16)
        B = (torch.randn((16, Ng), generator=gen, device=dev) * 0.01).to(torch.bfloat16)
        X = torch.randn((Mg, Kg), generator=gen, device=dev).to(torch.bfloat16)
        for i in range(args.reps):
            q.linear_forward(X, ws[i % 2], A, B, 2.0, status=st)
    elif args.case == "quantize":
        Kq, Nq = (int(v) for v in (args.shape or "8192,22016").split(","))
        W = (torch.randn((Kq, Nq), generator=gen, device=dev) * 0.015).to(torch.bfloat16)
        w = q.quantize(W, double_quant=True, status=st)
        for _ in range(args.reps):
            q.quantize(W, double_quant=True, out=w, status=st)
    else:
        Kq, Nq = (int(v) for v in (args.shape or "8192,22016").split(","))
        W = (torch.randn((Kq, Nq), generator=gen, device=dev) * 0.015).to(torch.bfloat16)
        w = q.quantize(W, double_quant=True, status=st)
        A = (torch.randn((Kq, 64), generator=gen, device=dev) * 0.01).to(torch.bfloat16)
        B = (torch.randn((64, Nq), generator=gen, device=dev) * 0.01).to(torch.bfloat16)
        for _ in range(args.reps):
            q.merge(w, A, B, 0.25, out=W, status=st)
    torch.cuda.synchronize()
    code = q.status_sync(st)
    print(json.dumps({"case": args.case, "shape": args.shape, "reps": args.reps, "status": list(code)}))
    return 0 if code[0] == 0 else 1


def layers_bench(torch, q, dev, peaks):
    """Forward + backward of the larger workloads, weights quantized (DQ) ahead:
    the 7B decoder-layer linear set (q, k, v, o 4096x4096; gate, up 4096x11008;
    down 11008x4096) and the 65B MLP slice (8192x22016, 22016x8192), M = 4096,
    r = 64, alpha = 16.  TFLOP/s of sum 4MKN + 6Mr(K+N); seeded normal inputs
    drawn on the GPU."""
    from inputs import synthetic as S
    gen = torch.Generator(device=dev)
    out = {}
    for name, shapes, sigma in (("layer7b", [(k, n) for _, k, n in S.LAYER7B], 0.02),
                                ("mlp65b", [(8192, 22016), (22016, 8192)], 0.015)):
        Mb, rb, c = 4096, 64, 16.0 / 64
        gen.manual_seed(9)
        layers = []
        for (Kb, Nb) in shapes:
            W = (torch.randn((Kb, Nb), generator=gen, device=dev) * sigma).to(torch.bfloat16)
            w = q.quantize(W, double_quant=True)
            del W
            mk = lambda *sh, sc: (torch.randn(sh, generator=gen, device=dev) * sc).to(torch.bfloat16)
            layers.append(dict(w=w, A=mk(Kb, rb, sc=0.01), B=mk(rb, Nb, sc=0.01), X=mk(Mb, Kb, sc=1.0),
                               G=mk(Mb, Nb, sc=1.0), Y=torch.empty((Mb, Nb), dtype=torch.bfloat16, device=dev),
                               Zc=torch.empty((Mb, rb), dtype=torch.bfloat16, device=dev),
                               dX=torch.empty((Mb, Kb), dtype=torch.bfloat16, device=dev),
                               dA=torch.empty((Kb, rb), dtype=torch.float32, device=dev),
                               dB=torch.empty((rb, Nb), dtype=torch.float32, device=dev)))
        st = q.new_status(dev)

        def run():
            for L in layers:
                q.linear_forward(L["X"], L["w"], L["A"], L["B"], c, Y=L["Y"], Zc=L["Zc"], status=st)
            for L in reversed(layers):
                q.linear_backward(L["G"], L["X"], L["Zc"], L["w"], L["A"], L["B"], c, dX=L["dX"],
                                  dA=L["dA"], dB=L["dB"], status=st)
        for _ in range(2):
            run()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 5
        e0.record()
        for _ in range(reps):
            run()
        e1.record()
        torch.cuda.synchronize()
        code, mask = q.status_sync(st)
        if code != 0:
            raise SystemExit(f"device status {code} (mask {mask}) in {name}")
        ms = e0.elapsed_time(e1) / reps
        flops = sum(4.0 * Mb * Kb * Nb + 6.0 * Mb * rb * (Kb + Nb) for Kb, Nb in shapes)
        out[name] = {"ms": ms, "TFLOP/s": flops / (ms * 1e-3) / 1e12,
                     "frac": flops / (ms * 1e-3) / 1e12 / peaks["bf16"], "linears": len(shapes)}
        del layers
        torch.cuda.empty_cache()
    return out


def merge_bench(torch, q, dev, peaks):
    """Merge/export of the 8192x22016 weight with r = 64 (DQ state): GB/s of
    P/2 + n1 + 4n2 + 4 (state) + 2r(K+N) (adapter) + 2P (bf16 output)."""
    gen = torch.Generator(device=dev)
    gen.manual_seed(6)
    Kq, Nq, rq = 8192, 22016, 64
    W = (torch.randn((Kq, Nq), generator=gen, device=dev) * 0.015).to(torch.bfloat16)
    w = q.quantize(W, double_quant=True)
    del W
    A = (torch.randn((Kq, rq), generator=gen, device=dev) * 0.01).to(torch.bfloat16)
    B = (torch.randn((rq, Nq), generator=gen, device=dev) * 0.01).to(torch.bfloat16)
    out = torch.empty((Kq, Nq), dtype=torch.bfloat16, device=dev)
    st = q.new_status(dev)
    for _ in range(3):
        q.merge(w, A, B, 0.25, out=out, status=st)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 10
    e0.record()
    for _ in range(reps):
        q.merge(w, A, B, 0.25, out=out, status=st)
    e1.record()
    torch.cuda.synchronize()
    per = e0.elapsed_time(e1) / reps * 1e-3
    P = Kq * Nq
    n1 = P // 64
    n2 = (n1 + 255) // 256
    nbytes = P // 2 + n1 + 4 * n2 + 4 + 2 * rq * (Kq + Nq) + 2 * P
    gbs = nbytes / per / 1e9
    del out, w
    return {"shape": [Kq, Nq], "r": rq, "us": per * 1e6, "GB/s": gbs, "frac": gbs / peaks["hbm"]}


def run_sweeps(args):
    """The named sweeps alone on GPU 0 (one JSON line): for iterating on one
    kernel family without the training step."""
    import torch
    import bit_nf4_quantized_pack_b200 as q
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    fns = {"gemv": gemv_sweep, "quantize": quantize_bench, "merge": merge_bench,
           "layers": layers_bench}
    out = {"sweeps": {}}
    for name in args.sweep.split(","):
        out["sweeps"][name] = fns[name](torch, q, dev, peaks)
    print(json.dumps(out), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--no-extras", action="store_true", help="skip the GEMV and quantize sweeps")
    ap.add_argument("--kernels-only", action="store_true",
                    help="only the timed steps (no e2e, sweeps or CPU baseline): for profilers")
    ap.add_argument("--case", choices=["gemv", "quantize", "merge"],
                    help="run one kernel workload --reps times and exit (for profilers)")
    ap.add_argument("--shape", default="",
                    help="M,K,N for --case gemv (default 1,4096,11008); K,N for --case quantize")
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--sweep", default="",
                    help="only these sweeps (comma list of gemv, quantize, merge, layers), no step")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.case:
        return run_case(args)
    if args.sweep:
        return run_sweeps(args)

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    import bit_nf4_quantized_pack_b200 as q
    peaks = load_peaks()
    c = ALPHA / R
    sets = make_sets(torch, dev, ROTATE)
    wbuf = q.NF4Weight.empty((K, N), True, dev)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    Zc = torch.empty((M, R), dtype=torch.bfloat16, device=dev)
    dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    from bit_nf4_quantized_pack_b200.dp import GradBucket
    grads = GradBucket(K, N, R, dev)      # dA, dB as views of one all-reduce bucket
    dA, dB = grads.dA, grads.dB
    status = q.new_status(dev)

    def step(i):
        s = sets[i % ROTATE]
        q.quantize(s["W"], double_quant=True, out=wbuf, status=status)
        q.linear_forward(s["X"], wbuf, s["A"], s["B"], c, Y=Y, Zc=Zc, status=status)
        q.linear_backward(s["dY"], s["X"], Zc, wbuf, s["A"], s["B"], c, dX=dX, dA=dA, dB=dB,
                          status=status)
        if world > 1:
            grads.all_reduce()

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    code, mask = q.status_sync(status)
    if code != 0:
        raise SystemExit(f"device status {code} (mask {mask}) during warm-up")

    # ---------------- timed region (device time, max over ranks) ----------------
    sampler = ClockSampler(dev) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    # The step time: no event between launches (an event recorded between two
    # launches keeps the second from starting while the first drains, and the
    # rank-r kernels from running beside the fused GEMM: tens of microseconds
    # per step); the library only counts its launches.
    q.lib.qlora_profile_reset()
    q.lib.qlora_profile_select(0)
    q.lib.qlora_profile_enable(1)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.steps):
        step(i)
    e1.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    _, launches = prof_read(q, -1)
    # The dominant kernel's launch time: the same steps again at once, with a
    # pair of events on the launching stream around every fused-GEMM launch
    # (and nothing else), under the same clock sampling.
    q.lib.qlora_profile_reset()
    q.lib.qlora_profile_select(0x3)
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    r0.record()
    for i in range(args.steps):
        step(i)
    r1.record()
    torch.cuda.synchronize()
    q.lib.qlora_profile_enable(0)
    clocks = sampler.stop() if sampler else None
    ms_launch_events = r0.elapsed_time(r1) / args.steps
    if world > 1:
        t = torch.tensor([ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    fwd_ms, fwd_n = prof_read(q, 0)
    bwd_ms, bwd_n = prof_read(q, 1)
    # per-class launch time per step, from a separate pass with every launch
    # bracketed by events (outside the timed region)
    q.lib.qlora_profile_reset()
    q.lib.qlora_profile_select(0xFFFFFFFF)
    q.lib.qlora_profile_enable(1)
    nb = 10
    for i in range(nb):
        step(i)
    torch.cuda.synchronize()
    q.lib.qlora_profile_enable(0)
    breakdown = {nm: prof_read(q, kind)[0] / nb * 1e3
                 for kind, nm in ((0, "fused_fwd"), (1, "fused_dX"), (2, "rank_r"), (3, "quantize"))}
    code, mask = q.status_sync(status)
    if code != 0:
        raise SystemExit(f"device status {code} (mask {mask}) in the timed region")
    value = world * flops_step() / (ms * 1e-3) / 1e12

    # dominant kernel: the fused NF4 GEMM (forward and dX launches together)
    f_fwd = 2.0 * M * K * N + 2.0 * M * R * N
    f_bwd = 2.0 * M * K * N + 2.0 * M * R * K
    kern_ms = (fwd_ms + bwd_ms) / max(1, fwd_n + bwd_n)
    kern_flops = (f_fwd * fwd_n + f_bwd * bwd_n) / max(1, fwd_n + bwd_n)
    achieved = kern_flops / (kern_ms * 1e-3) / 1e12 if kern_ms > 0 else None
    roofline = {"bound": "tensor", "kernel": "fused_nf4_gemm_kernel (fwd + dX)",
                "achieved": achieved, "peak": peaks["bf16"], "unit": "TFLOP/s",
                "frac": (achieved / peaks["bf16"]) if achieved else None,
                "traffic": FUSED_TRAFFIC_BYTES, "traffic_unit": "bytes per launch (ncu)",
                "peak_src": f"{peaks['src']} bf16 burst",
                "avg_launch_ms": kern_ms, "flops_per_launch": kern_flops,
                "fwd_ms": fwd_ms / max(1, fwd_n), "bwd_ms": bwd_ms / max(1, bwd_n),
                "timing": ("CUDA events around each fused-GEMM launch on its stream, over a "
                           "second pass of the same steps right after the timed one"),
                "ms_per_step_with_launch_events": ms_launch_events}

    # ---------------- end to end through the public API with host buffers ----------------
    e2e = None
    if not args.kernels_only:
        h = sets[0]["host"]
        pin = lambda a: torch.from_numpy(a.astype("float32")).to(torch.bfloat16).pin_memory()
        hW, hX, hG = pin(h.W), pin(h.X), pin(h.dY)
        hdA = torch.empty((K, R), dtype=torch.float32).pin_memory()
        hdB = torch.empty((R, N), dtype=torch.float32).pin_memory()
        dW, dXin, dG = torch.empty_like(sets[0]["W"]), torch.empty_like(sets[0]["X"]), \
            torch.empty_like(sets[0]["dY"])
        A_, B_ = sets[0]["A"], sets[0]["B"]

        # Two device input sets: the next step's inputs are copied from pinned
        # host memory on a copy stream while this step computes; every step's
        # copies and its D2H read of dA, dB are inside the timed region.
        dbufs = [(dW, dXin, dG), (torch.empty_like(dW), torch.empty_like(dXin), torch.empty_like(dG))]
        cs = torch.cuda.Stream(device=dev)
        comp = torch.cuda.current_stream(dev)
        ev_copied = [torch.cuda.Event(), torch.cuda.Event()]
        ev_used = [torch.cuda.Event(), torch.cuda.Event()]

        def issue_copy(i):
            b = i % 2
            cs.wait_event(ev_used[b])            # the step that last read these buffers
            with torch.cuda.stream(cs):
                for dst, src in zip(dbufs[b], (hW, hX, hG)):
                    dst.copy_(src, non_blocking=True)
                ev_copied[b].record(cs)

        def e2e_run(n, start_ev=None):
            if start_ev is not None:
                start_ev.record(comp)
                cs.wait_event(start_ev)
            issue_copy(0)
            for i in range(n):
                b = i % 2
                comp.wait_event(ev_copied[b])
                w_, x_, g_ = dbufs[b]
                q.quantize(w_, double_quant=True, out=wbuf, status=status)
                q.linear_forward(x_, wbuf, A_, B_, c, Y=Y, Zc=Zc, status=status)
                q.linear_backward(g_, x_, Zc, wbuf, A_, B_, c, dX=dX, dA=dA, dB=dB, status=status)
                ev_used[b].record(comp)
                if i + 1 < n:
                    issue_copy(i + 1)
                if world > 1:
                    grads.all_reduce()
                hdA.copy_(dA, non_blocking=True)
                hdB.copy_(dB, non_blocking=True)

        e2e_run(2)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        n_e2e = max(3, min(args.steps, 20))
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2e_run(n_e2e, start_ev=a0)
        a1.record(comp)
        torch.cuda.synchronize()
        ems = a0.elapsed_time(a1) / n_e2e
        if world > 1:
            t = torch.tensor([ems], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ems = float(t.item())
        h2d = (hW.numel() + hX.numel() + hG.numel()) * 2
        d2h = (hdA.numel() + hdB.numel()) * 4
        e2e = {"value": world * flops_step() / (ems * 1e-3) / 1e12, "unit": "TFLOP/s",
               "ms_per_step": ems, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    extras = {}
    if rank == 0 and not args.no_extras and not args.kernels_only:
        extras["gemv"] = gemv_sweep(torch, q, dev, peaks)
        extras["quantize"] = quantize_bench(torch, q, dev, peaks)
        extras["merge"] = merge_bench(torch, q, dev, peaks)
        extras["layers"] = layers_bench(torch, q, dev, peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.kernels_only:
        inputs = oracle_sample_inputs(K, M)
        t0 = time.perf_counter()
        for _ in range(CPU_BASELINE_REPS):
            oracle_step(inputs)
        dt = (time.perf_counter() - t0) / CPU_BASELINE_REPS
        cpu = {"value": flops_step() / dt / 1e12, "unit": "TFLOP/s", "cores": oracle_threads(),
               "kind": "oracle",
               "sample": (f"oracle (NumPy fp64): the whole step (quantize + double-quantize + "
                          f"dequantize W {K}x{N}, fwd + bwd for {M} tokens, r={R}), one input set, "
                          f"{CPU_BASELINE_REPS} repetitions, mean time"),
               "seconds": dt * CPU_BASELINE_REPS}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic",
                "config": {"workload": WORKLOAD, "M": M, "K": K, "N": N, "r": R, "alpha": ALPHA,
                           "double_quant": True, "parallelism": f"dp{world}",
                           "step": "quantize(W) + fwd + bwd" + (" + allreduce(dA,dB)" if world > 1 else ""),
                           "l2": f"{ROTATE} rotated input sets (W, X, dY: 96 MB each) > L2"},
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": int(launches), "clocks": clocks,
                "breakdown_us_per_step": breakdown}
        line.update(extras)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

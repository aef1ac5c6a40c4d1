"""Benchmark of the NVFP4 MLP training-step hot path on B200.

One step = the quantize kernels and the three block-scaled NVFP4 GEMMs of one
MLP linear layer's training step (tokens 16384, hidden 8192, ffn 28672):
    X  [16384 x 8192]  bf16 activations  -> 1D RNE codes            (fprop A)
    W  [28672 x 8192]  bf16 weight       -> 2D RNE codes, rowwise    (fprop B)
                                            + columnwise W^T codes   (dgrad B)
    Y  = X . W^T       [16384 x 28672]   bf16                         (fprop)
    dY [16384 x 28672] bf16 gradient     -> 1D SR codes              (dgrad A)
    dX = dY . W        [16384 x 8192]    bf16                         (dgrad)
    dY^T, X^T          16-point RHT (shared signs), dY SR, X RNE     (wgrad A, B)
    dW = dY^T . X      [28672 x 8192]    bf16                         (wgrad)
Inputs are seeded synthetic tensors (bf16) resident in HBM; every input
tensor is larger than the 126 MB L2, so consecutive steps do not hit in L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints one JSON line (rank 0).  Under torchrun each rank runs an independent
step on its own GPU (weak scaling, no collective on the data path).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 quantize GB/s (% HBM peak); block-scaled GEMM TFLOPS (% FP4 peak)"
WORKLOAD = "mlp_step_t16384_h8192_f28672"
T, H, F = 16384, 8192, 28672
FP4_OVER_BF16 = 4.0            # nominal dense FP4 / BF16 tensor peak ratio (9 / 2.25 PFLOP/s)
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS = 6650.0, 1590.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-chain", action="store_true", help="skip the chained-layer measurement (amax from the GEMM)")
    ap.add_argument("--op", default=None,
                    choices=["gemm", "gemm_amax", "quantize_1d", "quantize_1d_sr", "quantize_2d", "rht_t_sr",
                             "rht_t_rne", "quantize_1d_from_amax", "quantize_2d_from_amax", "mx_quantize",
                             "mx_gemm", "quantize_dual", "quantize_dual_sr",
                             "dequantize", "rht_sr", "rht_rne", "mx_dequantize", "scales_to_mma"],
                    help="time one kernel family alone on --shape (profiling mode)")
    ap.add_argument("--shape", default=None, help="M,N,K for gemm; rows,cols otherwise")
    ap.add_argument("--sweep", action="store_true",
                    help="quantizer sweep: 2^20 .. 2^30 elements in rows of 4096, three distributions, "
                         "1D RNE, 2D, RHT + SR row-wise and transposed (one JSON line per case)")
    ap.add_argument("--rht-order", type=int, default=16, choices=[16, 32, 64, 128],
                    help="points of the Hadamard transform for the rht_* ops (rht_t_*: transposed)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained", d["bf16_tflops"]), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


# ------------------------------------------------------------------ clocks --
class ClockSampler:
    """SM clocks and clock-event (throttle) reasons sampled during the timed
    region: NVML read every 10 ms on a thread, the same counters nvidia-smi
    reports (read only; nothing is set).  Without NVML, nvidia-smi's loop
    mode.  Only samples taken inside the timed region are kept."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80))

    def __init__(self, gpu_index: int, device=None):
        self.gpu = gpu_index
        self.device = device
        self.proc = None
        self.lines = []
        self.samples = []          # (perf_counter, sm MHz, reason mask)
        self.nvml = None
        self.handle = None
        self.max_mhz = None
        self.running = False

    def _nvml_handle(self):
        import pynvml as nv
        nv.nvmlInit()
        self.nvml = nv
        if self.device is not None:
            import torch
            props = torch.cuda.get_device_properties(self.device)
            try:
                return nv.nvmlDeviceGetHandleByUUID("GPU-" + str(props.uuid))
            except Exception:
                pass
            try:
                bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
                return nv.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                pass
        return nv.nvmlDeviceGetHandleByIndex(self.gpu)

    def start(self):
        try:
            self.handle = self._nvml_handle()
            nv = self.nvml
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(self.handle, nv.NVML_CLOCK_SM))
            self.running = True
            self.t = threading.Thread(target=self._poll, daemon=True)
            self.t.start()
            return
        except Exception:
            self.nvml = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _poll(self):
        nv, h = self.nvml, self.handle
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while self.running:
            try:
                self.samples.append((time.perf_counter(), float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                     int(get_reasons(h))))
            except Exception:
                pass
            time.sleep(0.01)

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz, mx = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            self.max_mhz = mx
            mask = 0
            for (n, bit), v in zip(self.REASONS[:4], parts[5:9]):
                if v.lower().startswith("active"):
                    mask |= bit
            self.samples.append((time.perf_counter(), mhz, mask))

    def stop(self, t_begin: float, t_end: float):
        if self.nvml is not None:
            self.running = False
            self.t.join(timeout=2)
            src = "nvml"
        elif self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.t.join(timeout=2)
            src = "nvidia-smi"
        else:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"], "samples": 0}
        inside = [x for x in self.samples if t_begin <= x[0] <= t_end]
        sm = [x[1] for x in inside]
        mask = 0
        for x in inside:
            mask |= x[2]
        reasons = [n for n, bit in self.REASONS if mask & bit]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(sm), "source": src}


# ----------------------------------------------------------- native arm ----
class Step:
    """Device buffers of one MLP step and the launch sequence through the C ABI."""

    def __init__(self, torch, N, G, dev):
        self.torch, self.N = torch, N
        t, h, f = T, H, F
        seed, rht_seed, sr_seed = G.seeds("mlp_step")
        self.rht_seed, self.sr_seed = rht_seed, sr_seed
        bf = torch.bfloat16
        u8 = torch.uint8
        host = {
            "x": G.activation(t, h, seed),
            "w": G.weight(f, h, seed + 1),
            "dy": G.gradient(t, f, seed + 2),
        }
        self.host_np = host
        self.dev = dev
        mk = lambda a: torch.from_numpy(a.view(np.int16)).view(bf)
        self.x = mk(host["x"]).to(dev)
        self.w = mk(host["w"]).to(dev)
        self.dy = mk(host["dy"]).to(dev)
        self._alloc()

    def twin(self):
        """A second set of device buffers for the same step (same host data,
        inputs not yet on the device): lets one step compute while the next
        one's inputs and the previous one's results cross PCIe."""
        t = object.__new__(Step)
        t.torch, t.N, t.rht_seed, t.sr_seed, t.host_np, t.dev = (self.torch, self.N, self.rht_seed, self.sr_seed,
                                                                  self.host_np, self.dev)
        t.x, t.w, t.dy = (self.torch.empty_like(v) for v in (self.x, self.w, self.dy))
        t._alloc()
        return t

    def _alloc(self):
        torch, N, dev = self.torch, self.N, self.dev
        t, h, f = T, H, F
        bf, u8 = torch.bfloat16, torch.uint8
        e = lambda *s: torch.empty(*s, dtype=u8, device=dev)
        mb = N.nvfp4_mma_scale_bytes
        self.xq = (e(t, h // 2), e(mb(t, h)))                       # fprop A
        self.wq = (e(f, h // 2), e(mb(f, h)), e(h, f // 2), e(mb(h, f)))   # fprop B, dgrad B
        self.dyq = (e(t, f // 2), e(mb(t, f)))                      # dgrad A
        self.dytq = (e(f, t // 2), e(mb(f, t)))                     # wgrad A
        self.xtq = (e(h, t // 2), e(mb(h, t)))                      # wgrad B
        self.gs = torch.zeros(8, dtype=torch.float32, device=dev)
        self.ws = torch.empty(2 * N.nvfp4_workspace_size(0, 0), dtype=u8, device=dev)   # the dual calls need two sets
        self.y = torch.empty(t, f, dtype=bf, device=dev)
        self.dx = torch.empty(t, h, dtype=bf, device=dev)
        self.dw = torch.empty(f, h, dtype=bf, device=dev)
        g = self.gs
        self.gp = [g[i:i + 1] for i in range(5)]
        # (name, kind, compulsory bytes (quantize: bf16 read + codes + scales written) or flops,
        #  bytes the two-pass quantizer moves (amax pass re-reads the input), kernels launched)
        q1 = 2 + 0.5 + 1 / 16
        q2 = 2 + 0.5 + 0.5 + 2 / 16
        # dual: one shared amax read, then one read per encode pass; two code sets written
        qd = 2 + 2 * (0.5 + 1 / 16)
        self.ops = [
            ("quantize_dual X (rowwise RNE + RHT X^T RNE)", "quant", t * h * qd, t * h * (qd + 4), 3),
            ("quantize_2d W (row + col codes)", "quant", f * h * q2, f * h * (q2 + 2), 2),
            ("gemm fprop", "gemm", 2.0 * t * f * h, 0, 1),
            ("quantize_dual dY (rowwise SR + RHT dY^T SR)", "quant", t * f * qd, t * f * (qd + 4), 3),
            ("gemm dgrad", "gemm", 2.0 * t * h * f, 0, 1),
            ("gemm wgrad", "gemm", 2.0 * f * h * t, 0, 1),
        ]

    def launch(self, i, s):
        N, ws = self.N, self.ws
        t, h, f = T, H, F
        ldb = ws.numel()
        if i == 0:
            N.nvfp4_quantize_dual(self.x, t, h, h, N.NVFP4_RNE, 0, self.xq[0], None, self.xq[1], self.gp[0],
                                  self.rht_seed, 0, self.xtq[0], None, self.xtq[1], self.gp[4], ws, ldb, s)
        elif i == 1:
            N.nvfp4_quantize_2d(self.w, f, h, h, self.wq[0], self.wq[2], None, self.wq[1], self.wq[3], self.gp[1], ws,
                                ldb, s)
        elif i == 2:
            N.nvfp4_gemm(self.xq[0], self.xq[1], self.gp[0], self.wq[0], self.wq[1], self.gp[1], t, f, h,
                         N.NVFP4_OUT_BF16, self.y, f, s)
        elif i == 3:
            N.nvfp4_quantize_dual(self.dy, t, f, f, N.NVFP4_SR, self.sr_seed, self.dyq[0], None, self.dyq[1],
                                  self.gp[2], self.rht_seed, self.sr_seed + 1, self.dytq[0], None, self.dytq[1],
                                  self.gp[3], ws, ldb, s)
        elif i == 4:
            N.nvfp4_gemm(self.dyq[0], self.dyq[1], self.gp[2], self.wq[2], self.wq[3], self.gp[1], t, h, f,
                         N.NVFP4_OUT_BF16, self.dx, h, s)
        elif i == 5:
            N.nvfp4_gemm(self.dytq[0], self.dytq[1], self.gp[3], self.xtq[0], self.xtq[1], self.gp[4], f, h, t,
                         N.NVFP4_OUT_BF16, self.dw, h, s)

    def run(self, stream, events=None):
        """Enqueue one step on a torch stream (events, if given, bracket each op)."""
        s = stream.cuda_stream
        for i in range(len(self.ops)):
            if events is not None:
                events[i][0].record(stream)
            self.launch(i, s)
            if events is not None:
                events[i][1].record(stream)


def max_over_ranks(value: float, dist, device) -> float:
    """The largest of every rank's value (replica timing: the job is as slow
    as its slowest GPU).  One all-reduce(MAX) of a single float."""
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_step_per_rank: float, world: int, ms_step: float) -> float:
    """Whole-job throughput: every rank runs the same step on its own data
    (weak scaling), so the job does world x the per-rank flops per step."""
    return flops_per_step_per_rank * world / (ms_step * 1e-3) / 1e12


def native(args):
    import torch
    import torch.distributed as dist
    from nvfp4_bit_block_amax_b200 import inputs as G
    from nvfp4_bit_block_amax_b200 import nvfp4 as N

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=300))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    N.lib()
    step = Step(torch, N, G, dev)
    s = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()

    with torch.cuda.stream(s):
        for _ in range(args.warmup):
            step.run(s)
    torch.cuda.synchronize()
    assert N.nvfp4_get_error(s.cuda_stream) == 0

    ops = step.ops
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in ops]
          for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local, dev)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    launches0 = N.nvfp4_kernel_launches()
    wall0 = time.perf_counter()
    t0.record(s)
    for k in range(args.steps):
        step.run(s, ev[k])
    t1.record(s)
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    launches = N.nvfp4_kernel_launches() - launches0
    barrier()
    clk = clocks.stop(wall0, wall0 + wall)
    assert N.nvfp4_get_error(s.cuda_stream) == 0
    ms_total = t0.elapsed_time(t1)
    if world > 1:
        ms_total = max_over_ranks(ms_total, dist, dev)
    ms_step = ms_total / args.steps
    per_op_ms = [statistics.mean(ev[k][i][0].elapsed_time(ev[k][i][1]) for k in range(args.steps))
                 for i in range(len(ops))]
    gemm_flops = sum(o[2] for o in ops if o[1] == "gemm")
    value = job_tflops(gemm_flops, world, ms_step)

    hbm, bf16, bf16_sus, peak_src = peaks()
    long_region = ms_total > 2000.0
    fp4_peak = (bf16_sus if long_region else bf16) * FP4_OVER_BF16
    kernels = []
    for (name, kind, work, moved, nk), ms in zip(ops, per_op_ms):
        if kind == "gemm":
            ach = work / (ms * 1e-3) / 1e12
            kernels.append({"op": name, "ms": round(ms, 4), "tflops": round(ach, 1),
                            "frac_fp4_peak": round(ach / fp4_peak, 4)})
        else:
            ach = work / (ms * 1e-3) / 1e9
            mv = moved / (ms * 1e-3) / 1e9
            kernels.append({"op": name, "ms": round(ms, 4), "gbs_compulsory": round(ach, 1),
                            "frac_hbm_compulsory": round(ach / hbm, 4), "gbs_moved": round(mv, 1),
                            "frac_hbm_moved": round(mv / hbm, 4)})
    gemm_ms = sum(ms for o, ms in zip(ops, per_op_ms) if o[1] == "gemm")
    quant_ms = sum(ms for o, ms in zip(ops, per_op_ms) if o[1] == "quant")
    quant_bytes = sum(o[2] for o in ops if o[1] == "quant")
    quant_moved = sum(o[3] for o in ops if o[1] == "quant")
    gemm_ach = gemm_flops / (gemm_ms * 1e-3) / 1e12
    traffic = load_traffic()
    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e2m1/ue4m3 -> f32",
        "data": "synthetic (seeded PCG64: N(0,1) activations with 0.05% x100 outliers, N(0,0.015^2) weight, "
                "Laplace(0,1e-3) gradient with 0.1% x1000 outliers)",
        "config": {"workload": WORKLOAD, "tokens": T, "hidden": H, "ffn": F,
                   "step": "quantize X(1D RNE), W(2D RNE, row+col), dY(1D SR), RHT dY^T(SR), RHT X^T(RNE); "
                           "GEMMs fprop, dgrad, wgrad (bf16 out)",
                   "l2": "every input tensor > 126 MB L2 (no flush needed)", "parallelism": f"replicas x{world}"},
        "quantize_gbs_compulsory": round(quant_bytes / (quant_ms * 1e-3) / 1e9, 1),
        "quantize_frac_hbm_compulsory": round(quant_bytes / (quant_ms * 1e-3) / 1e9 / hbm, 4),
        "quantize_gbs_moved": round(quant_moved / (quant_ms * 1e-3) / 1e9, 1),
        "quantize_frac_hbm_moved": round(quant_moved / (quant_ms * 1e-3) / 1e9 / hbm, 4),
        "peaks": {"hbm_gbs": hbm, "fp4_tflops": round(fp4_peak, 1), "source": peak_src},
        "gemm_tflops": round(gemm_ach, 1),
        "gemm_frac_fp4_peak": round(gemm_ach / fp4_peak, 4),
        "kernels": kernels,
        "roofline": {"bound": "tensor", "achieved": round(gemm_ach, 1), "peak": round(fp4_peak, 1),
                     "unit": "TFLOP/s", "frac": round(gemm_ach / fp4_peak, 4), "traffic": traffic,
                     "kernel": "gemm_nvf4_pair_kernel (3 GEMMs, mean over launches)",
                     "peak_source": f"{peak_src} {'sustained' if long_region else 'burst'} bf16 x {FP4_OVER_BF16} "
                                    "(nominal FP4/BF16 dense ratio)"},
        "clocks": clk,
        "gpu_launches": int(launches),
        "wall_s_timed": round(wall, 3),
    }
    if not args.no_chain:
        result["chain"] = chain(torch, N, G, step, s, args)
    if not args.no_e2e:
        result["e2e"] = e2e(torch, N, step, s, args, dist if world > 1 else None, world, dev)
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        result["cpu_baseline"] = cpu_baseline(target_s=12.0)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def chain(torch, N, G, step, s, args):
    """Two chained layers with the amax handed over by its producer ("NVFP4
    Is a Scaling System", "Where speed and accuracy claims can fail":
    quantization and scale handling cost work): Y = X . W1^T by the GEMM that
    also writes max |Y| (nvfp4_gemm_amax), Y quantized in one read from that
    amax (nvfp4_quantize_1d_from_amax), then Z = Yq . W2^T, W2 [hidden x ffn]
    2D-quantized outside the timed region.  Beside it, the two-pass
    quantize of the same Y (amax pass + encode), for the comparison.  X and W1
    are the step's quantized operands."""
    t, h, f = T, H, F
    dev = step.dev
    cs = s.cuda_stream
    w2 = torch.from_numpy(G.weight(h, f, G.seeds("mlp_step")[0] + 3).view(np.int16)).view(torch.bfloat16).to(dev)
    e = lambda *sh: torch.empty(*sh, dtype=torch.uint8, device=dev)
    mb = N.nvfp4_mma_scale_bytes
    g = torch.zeros(8, dtype=torch.float32, device=dev)
    w2q = (e(h, f // 2), e(mb(h, f)))
    N.nvfp4_quantize_2d(w2, h, f, f, w2q[0], None, None, w2q[1], None, g[0:1], step.ws, step.ws.numel(), cs)
    del w2
    yq, yq2 = (e(t, f // 2), e(mb(t, f))), (e(t, f // 2), e(mb(t, f)))
    z = torch.empty(t, h, dtype=torch.bfloat16, device=dev)
    y, amax = step.y, g[1:2]
    ops = [
        lambda: N.nvfp4_gemm_amax(step.xq[0], step.xq[1], step.gp[0], step.wq[0], step.wq[1], step.gp[1], t, f, h,
                                  N.NVFP4_OUT_BF16, y, f, amax, cs),
        lambda: N.nvfp4_quantize_1d_from_amax(y, t, f, f, 0, N.NVFP4_RNE, 0, amax, yq[0], None, yq[1], g[2:3], cs),
        lambda: N.nvfp4_gemm(yq[0], yq[1], g[2:3], w2q[0], w2q[1], g[0:1], t, h, f, N.NVFP4_OUT_BF16, z, h, cs),
        lambda: N.nvfp4_quantize_1d(y, t, f, f, 0, N.NVFP4_RNE, 0, yq2[0], None, yq2[1], g[3:4], step.ws,
                                    step.ws.numel(), cs),
    ]
    names = ["gemm_amax up (Y = X W1^T, + max|Y|)", "quantize_1d_from_amax Y (one read)", "gemm down (Z = Yq W2^T)",
             "quantize_1d Y two-pass (comparison, not in the chain)"]
    for _ in range(max(args.warmup, 1)):
        for op in ops:
            op()
    torch.cuda.synchronize()
    n = max(args.steps, 3)
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in ops] for _ in range(n)]
    for k in range(n):
        for i, op in enumerate(ops):
            ev[k][i][0].record(s)
            op()
            ev[k][i][1].record(s)
    torch.cuda.synchronize()
    assert N.nvfp4_get_error(cs) == 0
    same = bool(torch.equal(yq[0], yq2[0]) and torch.equal(yq[1], yq2[1]) and torch.equal(g[2], g[3]))
    ms = [statistics.mean(ev[k][i][0].elapsed_time(ev[k][i][1]) for k in range(n)) for i in range(len(ops))]
    hbm = peaks()[0]
    elems = t * f
    comp = elems * (2 + 0.5 + 1 / 16)
    moved2 = elems * (2 + 2 + 0.5 + 1 / 16)
    chain_ms = ms[0] + ms[1] + ms[2]
    flops = 2 * 2.0 * t * f * h
    return {"workload": f"X [{t} x {h}] -> Y = X W1^T [{t} x {f}] bf16 -> Yq (1D RNE) -> Z = Yq W2^T [{t} x {h}] bf16",
            "steps": n, "ms_per_chain": round(chain_ms, 4), "tflops": round(flops / (chain_ms * 1e-3) / 1e12, 1),
            "ops": [{"op": nm, "ms": round(m, 4)} for nm, m in zip(names, ms)],
            "quantize_single_read": {"ms": round(ms[1], 4), "gbs": round(comp / (ms[1] * 1e-3) / 1e9, 1),
                                     "frac_hbm": round(comp / (ms[1] * 1e-3) / 1e9 / hbm, 4),
                                     "bytes_per_elem": 2.5625},
            "quantize_two_pass": {"ms": round(ms[3], 4), "gbs_moved": round(moved2 / (ms[3] * 1e-3) / 1e9, 1),
                                  "frac_hbm_moved": round(moved2 / (ms[3] * 1e-3) / 1e9 / hbm, 4),
                                  "gbs_compulsory": round(comp / (ms[3] * 1e-3) / 1e9, 1),
                                  "frac_hbm_compulsory": round(comp / (ms[3] * 1e-3) / 1e9 / hbm, 4),
                                  "bytes_per_elem_moved": 4.5625},
            "single_read_equals_two_pass": same}


def load_traffic():
    """DRAM bytes per GEMM launch from the committed ncu record, or None when
    the record is missing or was taken on a different gemm.cu (the counters
    then no longer describe the kernel that runs)."""
    p = os.path.join(ROOT, "profiles", "gemm_traffic.json")
    src = os.path.join(ROOT, "nvfp4_bit_block_amax_b200", "csrc", "gemm.cu")
    try:
        rec = json.load(open(p))
        data = open(src, "rb").read()
        sha = hashlib.sha1(b"blob %d\0" % len(data) + data).hexdigest()   # git's blob id
        return rec.get("bytes_per_launch") if rec.get("gemm_cu_sha1") == sha else None
    except (OSError, ValueError):
        return None


def e2e(torch, N, step, s, args, dist=None, world=1, dev=None):
    """The same step through the C ABI with host buffers: every step copies its
    inputs in from pinned host memory and its three bf16 results out.  Two
    sets of device buffers let step k compute while the inputs of step k+1
    and the results of step k-1 cross PCIe (one stream each way); the timed
    region runs from the first copy in to the last copy out.  With several
    ranks (one per GPU, each on its own host buffers) the time is the slowest
    rank's and the value and byte counts are the whole job's."""
    hx = torch.from_numpy(step.host_np["x"].view(np.int16)).view(torch.bfloat16).pin_memory()
    hw = torch.from_numpy(step.host_np["w"].view(np.int16)).view(torch.bfloat16).pin_memory()
    hdy = torch.from_numpy(step.host_np["dy"].view(np.int16)).view(torch.bfloat16).pin_memory()
    oy = torch.empty(step.y.shape, dtype=torch.bfloat16).pin_memory()
    odx = torch.empty(step.dx.shape, dtype=torch.bfloat16).pin_memory()
    odw = torch.empty(step.dw.shape, dtype=torch.bfloat16).pin_memory()
    h2d = sum(t.numel() * 2 for t in (hx, hw, hdy))
    d2h = sum(t.numel() * 2 for t in (oy, odx, odw))
    n = max(3, min(args.steps, 40))
    sets = [step, step.twin()]
    s_in, s_out = torch.cuda.Stream(device=step.dev), torch.cuda.Stream(device=step.dev)
    ev = lambda: torch.cuda.Event()
    computed = [None, None]     # last compute of each buffer set
    drained = [None, None]      # last copy-out of each buffer set

    # Per-tensor events: an op waits only for the input it reads (X, then W,
    # then dY arrive in that order) and each result leaves as soon as its GEMM
    # is done, so the first step starts computing before all of its inputs
    # have crossed and the last one's early results overlap its later work.
    need = {0: "x", 1: "w", 3: "dy"}              # op index -> the input it first reads
    done_by = {2: "y", 4: "dx", 5: "dw"}          # op index -> the result it completes
    names = [o[0] for o in step.ops]
    assert (names[0].startswith("quantize_dual X") and names[1].startswith("quantize_2d W")
            and names[2] == "gemm fprop" and names[3].startswith("quantize_dual dY")
            and names[4] == "gemm dgrad" and names[5] == "gemm wgrad"), names

    def one(k):
        b = sets[k % 2]
        landed = {}
        with torch.cuda.stream(s_in):
            if computed[k % 2] is not None:
                s_in.wait_event(computed[k % 2])        # inputs of set k%2 no longer read
            for name, src in (("x", hx), ("w", hw), ("dy", hdy)):
                getattr(b, name).copy_(src, non_blocking=True)
                landed[name] = ev()
                landed[name].record(s_in)
        ready = {}
        with torch.cuda.stream(s):
            if drained[k % 2] is not None:
                s.wait_event(drained[k % 2])            # results of set k%2 copied out
            for i in range(len(b.ops)):
                if i in need:
                    s.wait_event(landed[need[i]])
                b.launch(i, s.cuda_stream)
                if i in done_by:
                    ready[done_by[i]] = ev()
                    ready[done_by[i]].record(s)
            computed[k % 2] = ready["dw"]                # the last op of the step
        with torch.cuda.stream(s_out):
            for name, dst in (("y", oy), ("dx", odx), ("dw", odw)):
                s_out.wait_event(ready[name])
                dst.copy_(getattr(b, name), non_blocking=True)
            out = ev()
            out.record(s_out)
            drained[k % 2] = out

    for k in range(2):
        one(k)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    for k in range(n):
        one(k)
    z.record(s_out)
    torch.cuda.synchronize()
    ms = a.elapsed_time(z) / n
    if dist is not None:
        ms = max_over_ranks(ms, dist, dev)
    flops = sum(o[2] for o in step.ops if o[1] == "gemm")
    return {"value": round(job_tflops(flops, world, ms), 2), "unit": "TFLOP/s", "ms_per_step": round(ms, 3),
            "h2d_bytes_per_step": int(h2d) * world, "d2h_bytes_per_step": int(d2h) * world, "steps": n,
            "overlap": "step k computes while step k+1's inputs and step k-1's results cross PCIe; "
                       "each op waits only for its own input, each result leaves when its GEMM is done"}


# ------------------------------------------------------------- oracle arm ----
def oracle_step(t, h, f):
    """The whole step on a [t x h], [f x h], [t x f] sample, in the CPU oracle:
    quantize (1D RNE, 2D, 1D SR, RHT SR/RNE transposed), dequantize exactly,
    float64 GEMMs.  Returns (seconds, flops)."""
    from nvfp4_bit_block_amax_b200 import inputs as G
    from oracle import oracle as O
    seed, rs, ss = G.seeds("mlp_step")
    x = G.activation(t, h, seed)
    w = G.weight(f, h, seed + 1)
    dy = G.gradient(t, f, seed + 2)
    t0 = time.perf_counter()
    cx, sx, gx = O.quantize_1d(x)
    cw, ccw, sw, gw = O.quantize_2d(w)
    xh = O.dequantize_f64(cx, sx, 0, gx, t, h)
    wh = O.dequantize_f64(cw, sw, 1, gw, f, h)
    y = xh @ wh.T
    cd, sd, gd = O.quantize_1d(dy, rounding=1, sr_seed=ss)
    dyh = O.dequantize_f64(cd, sd, 0, gd, t, f)
    wth = O.dequantize_f64(ccw, np.ascontiguousarray(sw.T), 1, gw, h, f)
    dx = dyh @ wth.T
    ca, sa, ga = O.quantize_1d(dy, transpose=True, rht=True, rht_seed=rs, rounding=1, sr_seed=ss + 1)
    cb, sb, gb = O.quantize_1d(x, transpose=True, rht=True, rht_seed=rs, rounding=0)
    dw = O.dequantize_f64(ca, sa, 0, ga, f, t) @ O.dequantize_f64(cb, sb, 0, gb, h, t).T
    dt = time.perf_counter() - t0
    del y, dx, dw
    return dt, 3 * 2.0 * t * h * f


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_model():
    """The host CPU's model name (from /proc/cpuinfo), or the platform's."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or platform.machine()


SAMPLE = (512, 1024, 2048)   # tokens, hidden, ffn of the oracle's sample of the step
QSAMPLE = (1024, 8192)       # rows, cols of the quantizer oracle's sample (rows of the step's activation recipe)


_QX = {}


def _oracle_sample(rows, cols):
    from nvfp4_bit_block_amax_b200 import inputs as G
    if (rows, cols) not in _QX:
        _QX[(rows, cols)] = G.activation(rows, cols, G.seeds("mlp_step")[0])
    return _QX[(rows, cols)]


def _oracle_rows_worker(args):
    """One process of the multi-core quantizer oracle on Q rows [r0, r1) of
    the sample: the amax of those rows (sg is None), or their codes given the
    global scale sg (spawned, no GPU)."""
    r0, r1, rows, cols, sg = args
    from oracle import oracle as O
    x = _oracle_sample(rows, cols)
    if sg is None:
        return O.amax(x[r0:r1])
    O.quantize_1d_rows(x, sg, range(r0, r1))
    return 0.0


def quantizer_oracle_rates(procs=None):
    """The scalar C quantizer (1D RNE: amax pass, then encode) on a [1024 x
    8192] sample of the step's activation recipe: GB/s of compulsory bytes
    (2.5625 per element) on one thread, and with the rows split over a
    process pool on every host core (both passes; spawn start, so no fork
    after CUDA)."""
    import multiprocessing as mp
    from oracle import oracle as O
    rows, cols = QSAMPLE
    x = _oracle_sample(rows, cols)
    O.lib()
    t0 = time.perf_counter()
    sg = O.global_scale(O.amax(x))
    O.quantize_1d_rows(x, sg, range(rows))
    t1 = time.perf_counter() - t0
    nbytes = rows * cols * (2 + 0.5 + 1 / 16)
    procs = procs or os.cpu_count() or 1
    ctx = mp.get_context("spawn")
    step = (rows + procs - 1) // procs
    ranges = [(r, min(rows, r + step)) for r in range(0, rows, step)]
    with ctx.Pool(len(ranges)) as pool:
        pool.map(_oracle_rows_worker, [(a, b, rows, cols, None) for a, b in ranges])   # warm: imports, sample
        t0 = time.perf_counter()
        amax = max(pool.map(_oracle_rows_worker, [(a, b, rows, cols, None) for a, b in ranges]))
        sg_n = O.global_scale(amax)
        pool.map(_oracle_rows_worker, [(a, b, rows, cols, sg_n) for a, b in ranges])
        tn = time.perf_counter() - t0
    assert sg_n == sg
    return {"sample": f"1D RNE quantize of a [{rows} x {cols}] bf16 activation (amax pass + encode, "
                      f"{nbytes / 1e6:.1f} MB compulsory)",
            "gbs_1_thread": round(nbytes / t1 / 1e9, 4), "gbs_all_cores": round(nbytes / tn / 1e9, 4),
            "processes": len(ranges)}


def cpu_baseline(target_s=12.0):
    t, h, f = SAMPLE
    secs, flops, n = 0.0, 0.0, 0
    while secs < target_s and n < 8:
        dt, fl = oracle_step(t, h, f)
        secs += dt
        flops += fl
        n += 1
    blas = blas_threads()
    out = {"value": round(flops / secs / 1e12, 6), "unit": "TFLOP/s", "cores": blas, "kind": "oracle",
           "sample": f"{n} oracle passes of the step at tokens {t}, hidden {h}, ffn {f} (same recipes); scalar C "
                     "quantizers on 1 thread, float64 BLAS GEMMs", "seconds": round(secs, 2),
           "threads": {"quantizers": 1, "blas_gemm": blas}, "host_cores": os.cpu_count(), "cpu_model": cpu_model()}
    try:
        out["quantizer_oracle"] = quantizer_oracle_rates()
    except Exception as e:   # the pool is a report, not part of the contract
        out["quantizer_oracle"] = {"error": repr(e)[:200]}
    return out


REF_SAMPLE = (256, 512, 1024)   # tokens, hidden, ffn of each step of the reference arm


def reference(args):
    """The oracle as the reference arm: each step is the whole MLP step at
    tokens 256, hidden 512, ffn 1024 (a bounded sample of the bench's
    workload, same recipes), on the host cores.  The line names that sample;
    its value is the sample's throughput, not the full step's."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    t, h, f = REF_SAMPLE
    for _ in range(args.warmup):
        oracle_step(t, h, f)
    secs, flops = 0.0, 0.0
    for _ in range(args.steps):
        dt, fl = oracle_step(t, h, f)
        secs += dt
        flops += fl
    v = flops / secs / 1e12
    blas = blas_threads()
    sample = (f"each step: the whole MLP step (quantize X 1D RNE, W 2D, dY 1D SR, RHT dY^T SR / X^T RNE; three "
              f"float64 GEMMs) at tokens {t}, hidden {h}, ffn {f} -- a sample of {WORKLOAD}")
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32 quantizers, f64 GEMM",
            "data": "synthetic (same seeded recipes)",
            "config": {"workload": WORKLOAD, "sample_of_workload": True, "tokens": t, "hidden": h, "ffn": f,
                       "parallelism": "oracle on host"},
            "cpu_baseline": {"kind": "oracle", "cores": blas, "value": round(v, 6), "unit": "TFLOP/s",
                             "sample": sample, "threads": {"quantizers": 1, "blas_gemm": blas},
                             "host_cores": os.cpu_count(), "cpu_model": cpu_model()},
            "e2e": {"value": round(v, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def micro(args):
    """One kernel family alone, for profiling (device-resident random inputs).
    Prints {op, shape, ms, throughput}; not a bench line."""
    import torch
    from nvfp4_bit_block_amax_b200 import nvfp4 as N
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    N.lib()
    dims = [int(v) for v in args.shape.split(",")]
    g = torch.Generator(device=dev)
    g.manual_seed(1234)
    s = torch.cuda.Stream(device=dev)
    if args.op == "mx_gemm":
        M, Nn, K = dims
        a = torch.randint(0, 256, (M, K // 2), dtype=torch.uint8, device=dev, generator=g)
        b = torch.randint(0, 256, (Nn, K // 2), dtype=torch.uint8, device=dev, generator=g)
        sa = torch.randint(120, 130, (N.nvfp4_mma_scale_bytes(M, K),), dtype=torch.uint8, device=dev, generator=g)
        sb = torch.randint(120, 130, (N.nvfp4_mma_scale_bytes(Nn, K),), dtype=torch.uint8, device=dev, generator=g)
        c = torch.empty(M, Nn, dtype=torch.bfloat16, device=dev)
        fn = lambda: N.nvfp4_mxfp4_gemm(a, sa, b, sb, M, Nn, K, N.NVFP4_OUT_BF16, c, Nn, s)
        work, unit = 2.0 * M * Nn * K, "TFLOP/s"
    elif args.op in ("gemm", "gemm_amax"):
        M, Nn, K = dims
        a = torch.randint(0, 256, (M, K // 2), dtype=torch.uint8, device=dev, generator=g)
        b = torch.randint(0, 256, (Nn, K // 2), dtype=torch.uint8, device=dev, generator=g)
        sa = torch.randint(0x30, 0x40, (N.nvfp4_mma_scale_bytes(M, K),), dtype=torch.uint8, device=dev, generator=g)
        sb = torch.randint(0x30, 0x40, (N.nvfp4_mma_scale_bytes(Nn, K),), dtype=torch.uint8, device=dev, generator=g)
        gs = torch.ones(2, dtype=torch.float32, device=dev)
        c = torch.empty(M, Nn, dtype=torch.bfloat16, device=dev)
        if args.op == "gemm_amax":
            camax = torch.empty(1, dtype=torch.float32, device=dev)
            fn = lambda: N.nvfp4_gemm_amax(a, sa, gs[0:1], b, sb, gs[1:2], M, Nn, K, N.NVFP4_OUT_BF16, c, Nn,
                                           camax, s)
        else:
            fn = lambda: N.nvfp4_gemm(a, sa, gs[0:1], b, sb, gs[1:2], M, Nn, K, N.NVFP4_OUT_BF16, c, Nn, s)
        work, unit = 2.0 * M * Nn * K, "TFLOP/s"
    else:
        R, C = dims
        x = torch.randn(R, C, device=dev, generator=g).to(torch.bfloat16)
        ws = torch.empty(N.nvfp4_workspace_size(R, C), dtype=torch.uint8, device=dev)
        gs = torch.empty(1, dtype=torch.float32, device=dev)
        tr = args.op.startswith("rht_t")
        qr, qc = (C, R) if tr else (R, C)
        codes = torch.empty(qr, qc // 2, dtype=torch.uint8, device=dev)
        smma = torch.empty(N.nvfp4_mma_scale_bytes(qr, qc), dtype=torch.uint8, device=dev)
        unit = "GB/s"
        if args.op in ("quantize_1d", "quantize_1d_sr"):
            rnd = N.NVFP4_SR if args.op.endswith("sr") else N.NVFP4_RNE
            fn = lambda: N.nvfp4_quantize_1d(x, R, C, C, 0, rnd, 7, codes, None, smma, gs, ws, ws.numel(), s)
            work = R * C * (2 + 0.5 + 1 / 16)
        elif args.op == "quantize_1d_from_amax":
            amax = x.float().abs().max().reshape(1).contiguous()
            fn = lambda: N.nvfp4_quantize_1d_from_amax(x, R, C, C, 0, N.NVFP4_RNE, 7, amax, codes, None, smma, gs, s)
            work = R * C * (2 + 0.5 + 1 / 16)
        elif args.op == "quantize_2d_from_amax":
            amax = x.float().abs().max().reshape(1).contiguous()
            cc = torch.empty(C, R // 2, dtype=torch.uint8, device=dev)
            sm2 = torch.empty(N.nvfp4_mma_scale_bytes(C, R), dtype=torch.uint8, device=dev)
            fn = lambda: N.nvfp4_quantize_2d_from_amax(x, R, C, C, amax, codes, cc, None, smma, sm2, gs, s)
            work = R * C * (2 + 0.5 + 0.5 + 2 / 16)
        elif args.op in ("quantize_dual", "quantize_dual_sr"):
            rnd = N.NVFP4_SR if args.op.endswith("sr") else N.NVFP4_RNE
            ct = torch.empty(C, R // 2, dtype=torch.uint8, device=dev)
            smt = torch.empty(N.nvfp4_mma_scale_bytes(C, R), dtype=torch.uint8, device=dev)
            gt = torch.empty(1, dtype=torch.float32, device=dev)
            ws2 = torch.empty(2 * N.nvfp4_workspace_size(R, C), dtype=torch.uint8, device=dev)
            fn = lambda: N.nvfp4_quantize_dual(x, R, C, C, rnd, 7, codes, None, smma, gs, 5, 8, ct, None, smt, gt,
                                               ws2, ws2.numel(), s)
            work = R * C * (2 + 2 * (0.5 + 1 / 16))
        elif args.op == "mx_quantize":
            fn = lambda: N.nvfp4_mxfp4_quantize(x, R, C, C, codes, None, smma, s)
            work = R * C * (2 + 0.5 + 1 / 32)
        elif args.op == "quantize_2d":
            cc = torch.empty(C, R // 2, dtype=torch.uint8, device=dev)
            sm2 = torch.empty(N.nvfp4_mma_scale_bytes(C, R), dtype=torch.uint8, device=dev)
            fn = lambda: N.nvfp4_quantize_2d(x, R, C, C, codes, cc, None, smma, sm2, gs, ws, ws.numel(), s)
            work = R * C * (2 + 0.5 + 0.5 + 2 / 16)
        elif args.op == "mx_dequantize":
            sc = torch.randint(118, 136, (R, C // 32), dtype=torch.uint8, device=dev, generator=g)
            out = torch.empty(R, C, dtype=torch.bfloat16, device=dev)
            fn = lambda: N.nvfp4_mxfp4_dequantize(codes, sc, R, C, N.NVFP4_OUT_BF16, out, s)
            work = R * C * (0.5 + 1 / 32 + 2)
        elif args.op == "scales_to_mma":
            sc = torch.randint(0x30, 0x40, (R, C // 16), dtype=torch.uint8, device=dev, generator=g)
            fn = lambda: N.nvfp4_scales_to_mma(sc, 0, R, C, smma, s)
            work = R * (C // 16) + N.nvfp4_mma_scale_bytes(R, C)
        elif args.op == "dequantize":
            sc = torch.randint(0x30, 0x40, (R, C // 16), dtype=torch.uint8, device=dev, generator=g)
            out = torch.empty(R, C, dtype=torch.bfloat16, device=dev)
            gs.fill_(1.0)
            fn = lambda: N.nvfp4_dequantize(codes, sc, 0, gs, R, C, N.NVFP4_OUT_BF16, out, s)
            work = R * C * (0.5 + 1 / 16 + 2)
        else:
            rnd = N.NVFP4_SR if args.op.endswith("sr") else N.NVFP4_RNE
            n = args.rht_order
            fn = lambda: N.nvfp4_rht_quantize_n(x, R, C, C, int(tr), n, 5, rnd, 6, codes, None, smma, gs, ws,
                                                ws.numel(), s)
            work = R * C * (2 + 0.5 + 1 / 16)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(args.steps):
        fn()
    e1.record(s)
    torch.cuda.synchronize()
    assert N.nvfp4_get_error(s.cuda_stream) == 0
    ms = e0.elapsed_time(e1) / args.steps
    scale = 1e12 if unit == "TFLOP/s" else 1e9
    print(json.dumps({"op": args.op, "shape": dims, **({"rht_order": args.rht_order} if args.op.startswith("rht")
                                                         else {}), "ms": round(ms, 4), "throughput": round(work / (ms * 1e-3) / scale, 1),
                      "unit": unit, "note": "profiling mode (one op alone), not a bench line"}), flush=True)


def sweep(args):
    """Quantizer sweep on the device: [R x 4096] bf16 for R = 256, 4096, 65536,
    262144 (2^20 .. 2^30 elements); values N(0,1), sign * exp(N(0, 2)), or
    N(0,1) with 0.1% set to +-1e4 (drawn with torch on the device: timing only,
    not the seeded numpy streams the parity tests use).  Per case the CUDA-event
    time of each op (both passes), GB/s on the compulsory bytes (one read) and
    on the bytes moved (two reads), and whether the input fits in L2."""
    import torch
    from nvfp4_bit_block_amax_b200 import nvfp4 as N
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    N.lib()
    hbm = peaks()[0]
    g = torch.Generator(device=dev)
    g.manual_seed(4000)
    s = torch.cuda.Stream(device=dev)
    C = 4096
    for dist in ("normal", "lognormal", "outliers"):
        for R in (256, 4096, 65536, 262144):
            n = R * C
            f = torch.randn(R, C, device=dev, generator=g)
            if dist == "lognormal":
                sign = torch.where(torch.rand(R, C, device=dev, generator=g) < 0.5, -1.0, 1.0)
                f = sign * torch.exp(2.0 * f)
            elif dist == "outliers":
                k = max(1, round(0.001 * n))
                idx = torch.randint(0, n, (k,), device=dev, generator=g)
                f.view(-1)[idx] = torch.where(torch.rand(k, device=dev, generator=g) < 0.5, -1e4, 1e4)
            x = f.to(torch.bfloat16)
            del f
            ws = torch.empty(N.nvfp4_workspace_size(R, C), dtype=torch.uint8, device=dev)
            gs = torch.empty(1, dtype=torch.float32, device=dev)
            cr = torch.empty(R, C // 2, dtype=torch.uint8, device=dev)
            ct = torch.empty(C, R // 2, dtype=torch.uint8, device=dev)
            mr = torch.empty(N.nvfp4_mma_scale_bytes(R, C), dtype=torch.uint8, device=dev)
            mt = torch.empty(N.nvfp4_mma_scale_bytes(C, R), dtype=torch.uint8, device=dev)
            q1 = 2 + 0.5 + 1 / 16
            q2 = 2 + 0.5 + 0.5 + 2 / 16
            cases = [
                ("1d_rne", lambda: N.nvfp4_quantize_1d(x, R, C, C, 0, N.NVFP4_RNE, 0, cr, None, mr, gs, ws,
                                                       ws.numel(), s), q1),
                ("2d_rne", lambda: N.nvfp4_quantize_2d(x, R, C, C, cr, ct, None, mr, mt, gs, ws, ws.numel(), s), q2),
                ("rht_sr_rowwise", lambda: N.nvfp4_rht_quantize_sr(x, R, C, C, 0, 5, N.NVFP4_SR, 6, cr, None, mr, gs,
                                                                   ws, ws.numel(), s), q1),
                ("rht_sr_transposed", lambda: N.nvfp4_rht_quantize_sr(x, R, C, C, 1, 5, N.NVFP4_SR, 6, ct, None, mt,
                                                                      gs, ws, ws.numel(), s), q1),
            ]
            for name, fn, per in cases:
                steps = 20 if n >= (1 << 28) else 100
                for _ in range(3):
                    fn()
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(s)
                for _ in range(steps):
                    fn()
                e1.record(s)
                torch.cuda.synchronize()
                assert N.nvfp4_get_error(s.cuda_stream) == 0
                ms = e0.elapsed_time(e1) / steps
                comp = n * per / (ms * 1e-3) / 1e9
                moved = n * (per + 2) / (ms * 1e-3) / 1e9
                print(json.dumps({"sweep": name, "dist": dist, "rows": R, "cols": C, "elements": n,
                                  "ms": round(ms, 4), "gbs_compulsory": round(comp, 1),
                                  "gbs_moved": round(moved, 1), "frac_hbm_moved": round(moved / hbm, 3),
                                  "l2_resident": n * 2 < 126e6}), flush=True)
            del x, cr, ct, mr, mt
            torch.cuda.empty_cache()


if __name__ == "__main__":
    a = parse()
    if a.sweep:
        sweep(a)
    elif a.op:
        micro(a)
    elif a.impl == "reference":
        reference(a)
    else:
        native(a)

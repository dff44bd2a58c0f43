"""Benchmark: Flux single-stream block forward at S=4608, dim 3072, 24 x 128,
MLP 12288, bf16, on B200 through the C ABI (libdit.so).

One step = one block forward (adaLN modulation, LayerNorm+modulate, fused
QKV|MLP-in GEMM with GELU, QK RMSNorm+RoPE, flash attention, output GEMM
with the gated residual) over one synthetic batch-1 input already resident in
HBM.  The weights of one block (282 MB) and its activations exceed the 126 MB
L2, so every step streams them from HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torch.distributed.run, one independent replica per GPU (the
block is data-parallel over samples; there is no exchange step), and reports
the whole-job throughput (weak scaling).  --impl reference times the fp64 CPU
oracle on the host cores instead (rank 0 only).
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Flux single-stream block ms & TFLOP/s at S=4608 bf16; % of tensor/HBM roofline"
UNIT = "TFLOP/s"
WORKLOAD = "flux_single_block_S4608_D3072_H24_M12288_bf16"
S_TXT, GRID, D, H, M = 512, 64, 3072, 24, 12288
S = S_TXT + GRID * GRID
KERNELS = ["adaln_modulation", "modulate_norm", "gemm_qkv_mlp_gelu_qknorm_rope", "attention",
           "gemm_out_gated_residual"]


def block_flops(S_=S):
    gemm1 = 2.0 * S_ * D * (3 * D + M)
    attn = 4.0 * S_ * S_ * H * 128
    gemm2 = 2.0 * S_ * (D + M) * D
    mod = 2.0 * D * 3 * D
    return {"adaln_modulation": mod, "modulate_norm": 0.0, "gemm_qkv_mlp_gelu_qknorm_rope": gemm1,
            "attention": attn, "gemm_out_gated_residual": gemm2}


def block_bytes(S_=S):
    """Algorithmic HBM bytes per launch (read once + write once)."""
    return {
        "adaln_modulation": 3 * D * D * 2 + D * 2 + 3 * D * 4,
        "modulate_norm": 2 * S_ * D * 2,
        "gemm_qkv_mlp_gelu_qknorm_rope": S_ * D * 2 + (3 * D + M) * D * 2 + S_ * (3 * D + M) * 2 + S_ * 64 * 8,
        "attention": 4 * S_ * D * 2,
        "gemm_out_gated_residual": S_ * (D + M) * 2 + D * (D + M) * 2 + 2 * S_ * D * 2,
    }


KERNEL_BOUND = {"adaln_modulation": "hbm", "modulate_norm": "hbm", "gemm_qkv_mlp_gelu_qknorm_rope": "tensor",
                "attention": "tensor", "gemm_out_gated_residual": "tensor"}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": float(j["hbm_gbs"]), "bf16_tflops": float(j["bf16_tflops"]),
                "bf16_tflops_sustained": float(j.get("bf16_tflops_sustained", j["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------------------
# Clock sampling during the timed region
# ----------------------------------------------------------------------------

REASON_COLS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]


def _nvml_handle(torch, dev_index):
    """NVML handle of the CUDA device, matched by UUID (NVML numbers every GPU
    of the machine; CUDA only the visible ones)."""
    import pynvml
    pynvml.nvmlInit()
    props = torch.cuda.get_device_properties(dev_index)
    uuid = str(getattr(props, "uuid", ""))
    if uuid:
        try:
            return pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except pynvml.NVMLError:
            pass
    return pynvml.nvmlDeviceGetHandleByIndex(dev_index)


class ClockSampler:
    """Read-only sampling of the SM clock (every ~1 ms), power and clock-event
    reasons (every ~5 ms) through NVML on a background thread, so that even a
    20 ms timed region holds tens of samples.  Falls back to nvidia-smi at
    100 ms when NVML is not available.  Changes no GPU setting."""

    def __init__(self, index: int):
        self.index = index
        self.samples = []   # (time, sm_mhz)
        self.slow = []      # (time, power_w, reason bits)
        self.max_mhz = None
        self.mode = None
        self._stop = threading.Event()
        self.t = None
        self.proc = None

    def start(self):
        try:
            import pynvml
            import torch
            self.h = _nvml_handle(torch, self.index)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
            self.bits = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                         "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                         "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                         "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
            self.mode = "nvml"
            self.t = threading.Thread(target=self._nvml_loop, daemon=True)
            self.t.start()
            return
        except Exception:
            self.mode = None
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.mode = "nvidia-smi"
        self.t = threading.Thread(target=self._smi_loop, daemon=True)
        self.t.start()

    def _nvml_loop(self):
        import pynvml
        n = 0
        while not self._stop.is_set():
            t = time.time()
            try:
                self.samples.append((t, float(pynvml.nvmlDeviceGetClockInfo(self.h, pynvml.NVML_CLOCK_SM))))
                if n % 5 == 0:
                    pw = pynvml.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                    rb = pynvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    self.slow.append((t, pw, rb))
            except pynvml.NVMLError:
                pass
            n += 1
            time.sleep(0.001)

    def _smi_loop(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 7:
                t = time.time()
                try:
                    self.samples.append((t, float(parts[0])))
                    self.max_mhz = float(parts[1])
                except ValueError:
                    continue
                rb = sum(1 << i for i in range(4) if parts[3 + i].lower().startswith("active"))
                try:
                    pw = float(parts[2])
                except ValueError:
                    pw = None
                self.slow.append((t, pw, rb))

    def stop(self):
        self._stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.t is not None:
            self.t.join(timeout=5)

    def summary(self, t0, t1):
        """Median SM clock over the samples taken in [t0, t1] while the GPU
        was busy (above 500 MHz), the clock-event reasons seen there, and the
        largest power drawn."""
        win = [(t, v) for (t, v) in self.samples if t0 <= t <= t1]
        slow = [x for x in self.slow if t0 - 0.005 <= x[0] <= t1 + 0.005]
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0, "source": self.mode}
        sm = [v for (_, v) in win]
        busy = [v for v in sm if v > 500] or sm
        reasons = set()
        for (_, _, rb) in slow:
            for i, name in enumerate(REASON_COLS):
                bit = self.bits[name] if self.mode == "nvml" else (1 << i)
                if rb & bit:
                    reasons.add(name)
        pw = [p for (_, p, _) in slow if p is not None]
        return {"sm_mhz": statistics.median(busy), "sm_min_mhz": min(busy), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(win), "power_w_max": max(pw) if pw else None,
                "source": self.mode + (" 1 ms" if self.mode == "nvml" else " 100 ms")}


# ----------------------------------------------------------------------------
# Our arm
# ----------------------------------------------------------------------------


def make_block(torch, dev, seed):
    """Random-init weights of the block (N(0, 0.02) linears, zero biases, unit
    norm scales) and N(0, 1) inputs, drawn on the device from a seeded
    generator."""
    g = torch.Generator(device=dev)
    g.manual_seed(seed)

    def nrm(*shape, std=1.0):
        return (torch.randn(*shape, generator=g, device=dev, dtype=torch.float32) * std).to(torch.bfloat16)

    w = {"W_mod": nrm(3 * D, D, std=0.02), "b_mod": torch.zeros(3 * D, device=dev, dtype=torch.bfloat16),
         "W1": nrm(3 * D + M, D, std=0.02), "b1": torch.zeros(3 * D + M, device=dev, dtype=torch.bfloat16),
         "q_scale": torch.ones(128, device=dev, dtype=torch.bfloat16),
         "k_scale": torch.ones(128, device=dev, dtype=torch.bfloat16),
         "W2": nrm(D, D + M, std=0.02), "b2": torch.zeros(D, device=dev, dtype=torch.bfloat16)}
    x = nrm(S, D)
    vec = nrm(1, D)
    return w, x, vec


def max_over_ranks(value, world, device="cpu"):
    """Largest value over all ranks (the job's time is its slowest rank)."""
    if world <= 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_step, steps, world, elapsed_ms):
    """Whole-job throughput: every rank runs `steps` independent replica steps."""
    return world * flops_per_step * steps / (elapsed_ms * 1e-3) / 1e12


def run_ours(args, rank, world, local_rank):
    import torch
    import diffusion_transformer_block_flux_b200 as dit
    from diffusion_transformer_block_flux_b200 import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dit.lib()  # raises if the CUDA library is missing
    if args.l2_keep_weights_mb:
        dit.dit_set_weight_l2_persist(args.l2_keep_weights_mb << 20)
    w, x, vec = make_block(torch, dev, seed=1234 + rank)
    ids = torch.from_numpy(synth.flux_ids(S_TXT, GRID, GRID)).to(dev)
    rope = torch.empty((S, 64, 2), dtype=torch.float32, device=dev)
    dit.dit_rope_table(ids, (8, 28, 28), 10000.0, rope)
    cfg = dit.block_cfg(1, S, D, H, M)
    ws = torch.empty(dit.dit_single_block_workspace(cfg), dtype=torch.uint8, device=dev)
    out = torch.empty_like(x)
    cw = dit.single_weights(w)
    stream = torch.cuda.current_stream(dev)

    def step(evs=None):
        dit.dit_single_block_fwd(cfg, cw, x, vec, rope, out, ws, events=evs)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st, code = dit.dit_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error word {code:#x} after warm-up")

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(KERNELS) + 1)] for _ in range(K)]
    for row in evs:  # torch creates the CUDA event on first record
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    wall0 = time.time()
    # headline: K plain block forwards
    t_start.record(stream)
    for i in range(K):
        step()
    t_end.record(stream)
    torch.cuda.synchronize()
    wallh = time.time()
    # breakdown: K more forwards with an event before and after every kernel
    for i in range(K):
        step(evs[i])
    torch.cuda.synchronize()
    wall1 = time.time()
    if world > 1:
        torch.distributed.barrier()
    time.sleep(0.05)
    sampler.stop()
    clocks = sampler.summary(wall0, wallh)
    clocks_breakdown = sampler.summary(wallh, wall1)
    elapsed_ms = t_start.elapsed_time(t_end)
    per_kernel = {k: statistics.mean(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(K))
                  for j, k in enumerate(KERNELS)}
    elapsed_ms = max_over_ranks(elapsed_ms, world, dev)
    st, code = dit.dit_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error word {code:#x} in the timed region")

    # ---- end to end through the C ABI with host buffers ----
    # dit_single_block_fwd_host: every request's input is copied from page-locked
    # host memory and its output copied back, pipelined against the compute
    NH = 4  # host request buffers, reused round robin
    xs_h = [x.cpu().pin_memory() for _ in range(NH)]
    vecs_h = [vec.cpu().pin_memory() for _ in range(NH)]
    outs_h = [torch.empty((S, D), dtype=torch.bfloat16).pin_memory() for _ in range(NH)]
    hws = torch.empty(dit.dit_single_block_host_workspace(cfg), dtype=torch.uint8, device=dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    Ke = max(1, min(K, 200))

    def e2e(n):
        idx = [i % NH for i in range(n)]
        dit.dit_single_block_fwd_host(cfg, cw, [xs_h[i] for i in idx], [vecs_h[i] for i in idx],
                                      [outs_h[i] for i in idx], rope, hws)

    e2e(max(3, min(args.warmup, 10)))
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0.record(stream)
    e2e(Ke)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    st, code = dit.dit_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error word {code:#x} in the end-to-end run")

    flops = block_flops()
    total_flops = sum(flops.values())
    ms_per_step = elapsed_ms / K
    value = whole_job_tflops(total_flops, K, world, elapsed_ms)
    e2e_value = whole_job_tflops(total_flops, Ke, world, e2e_ms)

    pk = peaks()
    # a block timed inside a long run of blocks: the power-capped (sustained) tensor peak applies
    # when the clock record shows the power cap, the burst peak otherwise
    capped = "sw_power_cap" in clocks.get("reasons", [])
    bf16_peak = pk["bf16_tflops_sustained"] if capped else pk["bf16_tflops"]
    dom = max(per_kernel, key=per_kernel.get)
    nbytes = block_bytes()
    if KERNEL_BOUND[dom] == "tensor":
        achieved = flops[dom] / (per_kernel[dom] * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": bf16_peak, "unit": "TFLOP/s",
                "frac": round(achieved / bf16_peak, 4)}
    else:
        achieved = nbytes[dom] / (per_kernel[dom] * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / pk["hbm_gbs"], 4)}
    roof["kernel"] = dom
    roof["traffic"] = traffic_for(dom)
    roof["traffic_unit"] = "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)"
    if pk["source"] == "measured":
        roof["peak_source"] = ("measured sustained, power-capped" if capped and roof["bound"] == "tensor"
                               else "measured burst") + " (MEASURED_PEAKS.json)"
    else:
        roof["peak_source"] = "fallback"
    kernels = {}
    mhz = clocks_breakdown.get("sm_mhz")
    for k in KERNELS:
        ent = {"ms": round(per_kernel[k], 4), "share": round(per_kernel[k] / sum(per_kernel.values()), 4)}
        if mhz:  # time x median SM clock of the breakdown pass: clock-independent work in cycles
            ent["mcycles"] = round(per_kernel[k] * 1e-3 * mhz, 4)
        if KERNEL_BOUND[k] == "tensor":
            a = flops[k] / (per_kernel[k] * 1e-3) / 1e12
            ent.update({"tflops": round(a, 1), "frac_of_bf16_peak": round(a / bf16_peak, 4)})
        else:
            a = nbytes[k] / (per_kernel[k] * 1e-3) / 1e9
            ent.update({"gbs": round(a, 1), "frac_of_hbm_peak": round(a / pk["hbm_gbs"], 4)})
        kernels[k] = ent
    block_frac = (total_flops / (ms_per_step * 1e-3) / 1e12) / bf16_peak
    res = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "global_batch": world, "seq_len": S, "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2 (282 MB of block weights + 0.25 GB activations per step)"
                         + (f"; {args.l2_keep_weights_mb} MB persisting L2 set-aside for the output GEMM's weight"
                            if args.l2_keep_weights_mb else "")},
        "ms_per_block": round(ms_per_step, 4), "blocks_per_s": round(world * 1e3 / ms_per_step, 1),
        "block_frac_of_bf16_peak": round(block_frac, 4),
        "gpu_launches": len(KERNELS) * K,
        "e2e": {"value": round(e2e_value, 2), "unit": UNIT, "api": "dit_single_block_fwd_host, pinned host buffers",
                "h2d_bytes_per_step": S * D * 2 + D * 2,
                "d2h_bytes_per_step": S * D * 2, "steps": Ke},
        "roofline": roof, "kernels": kernels, "clocks": clocks, "clocks_breakdown_pass": clocks_breakdown,
    }
    return res


# DRAM bytes (read + write) per launch from one ncu capture of each kernel
# (profiles/*.ncu.md), with a hash of the kernel's sources at capture time.
# A kernel whose sources changed since reports traffic null.
NCU_TRAFFIC = {
    "gemm_qkv_mlp_gelu_qknorm_rope": (338256384, ("gemm.cuh", "common.cuh"), "2799a2b0fa42beec"),
    "gemm_out_gated_residual": (436618752, ("gemm.cuh", "common.cuh"), "2799a2b0fa42beec"),
    "attention": (94130688, ("attention.cuh", "common.cuh"), "38a153274e62a573"),
    "modulate_norm": (28391168, ("elementwise.cuh", "common.cuh"), "8fa8fb1c7db5f362"),
    "adaln_modulation": (56746752, ("elementwise.cuh", "common.cuh"), "8fa8fb1c7db5f362"),
}


def traffic_for(kernel):
    import hashlib
    ent = NCU_TRAFFIC.get(kernel)
    if ent is None:
        return None
    nbytes, files, digest = ent
    m = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "diffusion_transformer_block_flux_b200", "csrc", f), "rb") as fh:
            m.update(fh.read())
    return nbytes if m.hexdigest()[:16] == digest else None


# ----------------------------------------------------------------------------
# CPU oracle (reference arm and cpu_baseline leg)
# ----------------------------------------------------------------------------


def oracle_inputs(n_tokens):
    """Seeded cfg-2 weights and the first n_tokens tokens (text first, then
    image rows) of the cfg-2 input, widened to fp64."""
    from diffusion_transformer_block_flux_b200 import synth
    shape = synth.FLUX
    w = synth.to_f64(synth.single_block_weights(shape))
    a = synth.block_activations(shape)
    x = synth.bf16_bits_to_f64(a["x"][:n_tokens])
    vec = synth.bf16_bits_to_f64(a["vec"])
    return w, x, vec, a["ids"][:n_tokens]


def oracle_block_time(n_tokens, reps, w=None):
    from oracle import dit_oracle as O
    if w is None:
        w, x, vec, ids = oracle_inputs(n_tokens)
    else:
        w, x, vec, ids = w
    times = []
    for _ in range(reps):
        t0 = time.perf_counter()
        O.single_block(x, vec, ids, w, H)
        times.append(time.perf_counter() - t0)
    return times


def cores_used():
    for var in ("OPENBLAS_NUM_THREADS", "OMP_NUM_THREADS", "MKL_NUM_THREADS"):
        if os.environ.get(var):
            return int(os.environ[var])
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n and n[0]:
            return int(n[0])
    except Exception:
        pass
    return os.cpu_count()


def sub_flops(n):
    return sum(block_flops(n).values())


def cpu_baseline(n_tokens=1024, reps=2):
    inp = oracle_inputs(n_tokens)
    oracle_block_time(64, 1, (inp[0], inp[1][:64], inp[2], inp[3][:64]))  # warm BLAS threads
    times = oracle_block_time(n_tokens, reps, inp)
    t = statistics.mean(times)
    return {"value": round(sub_flops(n_tokens) / t / 1e12, 5), "unit": UNIT, "cores": cores_used(),
            "kind": "oracle",
            "sample": f"fp64 numpy oracle single-stream block on the first {n_tokens} of the 4608 tokens "
                      f"(full dim 3072, 24 heads, MLP 12288, same weights), mean of {reps} runs "
                      f"of {t:.2f} s; TFLOP/s = algorithmic FLOPs of that sub-block / time"}


def run_reference(args):
    """Reference arm: the fp64 oracle as it stands, on the host cores.  Each
    step runs the block on a leading token window sized so the whole
    --steps/--warmup run stays within about two minutes."""
    budget_s = 120.0
    calib_n = 128
    inp = oracle_inputs(S)
    full_w = inp[0]
    t_cal = min(oracle_block_time(calib_n, 2, (full_w, inp[1][:calib_n], inp[2], inp[3][:calib_n])))
    per_token = t_cal / calib_n
    per_step = budget_s / max(1, args.steps + args.warmup)
    n = int(max(64, min(S, (per_step / per_token) // 64 * 64)))
    sub = (full_w, inp[1][:n], inp[2], inp[3][:n])
    oracle_block_time(n, args.warmup, sub)
    times = oracle_block_time(n, args.steps, sub)
    total = sum(times)
    value = sub_flops(n) * args.steps / total / 1e12
    sample = (f"fp64 numpy oracle single-stream block on the first {n} of the 4608 tokens per step "
              f"(full dim 3072, 24 heads, MLP 12288); TFLOP/s = algorithmic FLOPs of that sub-block / time")
    return {
        "metric": METRIC, "value": round(value, 5), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "global_batch": 1, "seq_len": S, "parallelism": "none",
                   "tokens_per_step": n},
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 5), "unit": UNIT, "cores": cores_used(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 5), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------------------
# Further workloads (one GPU): the double-stream block, the video block, the
# whole 57-block x 50-step loop as one CUDA graph, and the HBM-bound kernels
# in isolation.  Each prints its own JSON line; the default workload above is
# the headline metric.
# ----------------------------------------------------------------------------


_LAST_CLOCKS = {}


def _event_time(torch, fn, K, W, stream):
    """Mean CUDA-event time of fn over K calls after W warm-up calls; the clock
    record of the timed calls is kept in _LAST_CLOCKS for the JSON line."""
    for _ in range(W):
        fn()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    time.sleep(0.05)
    t0 = time.time()
    e0.record(stream)
    for _ in range(K):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    sampler.stop()
    _LAST_CLOCKS.clear()
    _LAST_CLOCKS.update(sampler.summary(t0, t1))
    return e0.elapsed_time(e1) / K


def _rand(torch, g, dev, *shape, std=1.0):
    return (torch.randn(*shape, generator=g, device=dev, dtype=torch.float32) * std).to(torch.bfloat16)


def _extra_line(workload, ms, flops, K, W, extra=None):
    pk = peaks()
    tf = flops / (ms * 1e-3) / 1e12
    res = {"metric": f"{workload} ms & TFLOP/s (bf16)", "value": round(tf, 2), "unit": "TFLOP/s", "n_gpus": 1,
           "steps": K, "warmup": W, "ms_per_step": round(ms, 4), "higher_is_better": True, "dtype": "bf16",
           "data": "synthetic", "config": {"workload": workload},
           "frac_of_bf16_peak": round(tf / pk["bf16_tflops"], 4), "algorithmic_flops": flops,
           "clocks": dict(_LAST_CLOCKS)}
    if extra:
        res.update(extra)
    return res


def run_double(args):
    import torch
    import diffusion_transformer_block_flux_b200 as dit
    from diffusion_transformer_block_flux_b200 import synth
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    g.manual_seed(7)
    w = {}
    for st in ("txt", "img"):
        z = lambda n: torch.zeros(n, device=dev, dtype=torch.bfloat16)
        w[st] = {"W_mod": _rand(torch, g, dev, 6 * D, D, std=0.02), "b_mod": z(6 * D),
                 "W_qkv": _rand(torch, g, dev, 3 * D, D, std=0.02), "b_qkv": z(3 * D),
                 "q_scale": torch.ones(128, device=dev, dtype=torch.bfloat16),
                 "k_scale": torch.ones(128, device=dev, dtype=torch.bfloat16),
                 "W_proj": _rand(torch, g, dev, D, D, std=0.02), "b_proj": z(D),
                 "W_mlp1": _rand(torch, g, dev, M, D, std=0.02), "b_mlp1": z(M),
                 "W_mlp2": _rand(torch, g, dev, D, M, std=0.02), "b_mlp2": z(D)}
    img, txt = _rand(torch, g, dev, S - S_TXT, D), _rand(torch, g, dev, S_TXT, D)
    vec = _rand(torch, g, dev, 1, D)
    ids = torch.from_numpy(synth.flux_ids(S_TXT, GRID, GRID)).to(dev)
    rope = torch.empty((S, 64, 2), dtype=torch.float32, device=dev)
    dit.dit_rope_table(ids, (8, 28, 28), 10000.0, rope)
    cfg = dit.block_cfg(1, S, D, H, M, n_txt=S_TXT)
    ws = torch.empty(dit.dit_double_block_workspace(cfg), dtype=torch.uint8, device=dev)
    io, to = torch.empty_like(img), torch.empty_like(txt)
    cw = dit.double_weights(w)
    ms = _event_time(torch, lambda: dit.dit_double_block_fwd(cfg, cw, img, txt, vec, rope, io, to, ws),
                     args.steps, args.warmup, torch.cuda.current_stream())
    flops = 2.0 * S * D * (3 * D + D + 2 * M) + 4.0 * S * S * H * 128 + 2 * 2.0 * D * 6 * D
    return _extra_line("flux_double_block_T512_I4096_D3072_bf16", ms, flops, args.steps, args.warmup,
                       {"gpu_launches_per_step": 11})


def run_video(args):
    import torch
    import diffusion_transformer_block_flux_b200 as dit
    from diffusion_transformer_block_flux_b200 import synth
    vs = synth.VIDEO
    Dv, Mv, Sv, Hv, C = vs.D, vs.M, vs.S, vs.H, vs.n_ctx
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    g.manual_seed(9)
    shapes = {"W_mod": (6 * Dv, Dv), "W_qkv": (3 * Dv, Dv), "W_o": (Dv, Dv), "W_cq": (Dv, Dv),
              "W_ckv": (2 * Dv, Dv), "W_co": (Dv, Dv), "W_f1": (Mv, Dv), "W_f2": (Dv, Mv)}
    w = {}
    for nm, shp in shapes.items():
        w[nm] = _rand(torch, g, dev, *shp, std=0.02)
        w["b" + nm[1:]] = torch.zeros(shp[0], device=dev, dtype=torch.bfloat16)
    x, ctx, vec = _rand(torch, g, dev, Sv, Dv), _rand(torch, g, dev, C, Dv), _rand(torch, g, dev, 1, Dv)
    ids = torch.from_numpy(synth.video_ids(vs.frames, vs.grid_h, vs.grid_w)).to(dev)
    rope = torch.empty((Sv, 64, 2), dtype=torch.float32, device=dev)
    dit.dit_rope_table(ids, (22, 21, 21), 10000.0, rope)
    cfg = dit.block_cfg(1, Sv, Dv, Hv, Mv)
    ws = torch.empty(dit.dit_video_block_workspace(cfg, C), dtype=torch.uint8, device=dev)
    out = torch.empty_like(x)
    cw = dit.video_weights(w)
    K = max(3, args.steps // 10)
    ms = _event_time(torch, lambda: dit.dit_video_block_fwd(cfg, cw, x, ctx, C, vec, rope, out, ws),
                     K, args.warmup, torch.cuda.current_stream())
    flops = (2.0 * Sv * Dv * (3 * Dv + Dv + Dv + Dv + 2 * Mv) + 2.0 * C * Dv * 2 * Dv + 4.0 * Sv * Sv * Hv * 128
             + 4.0 * Sv * C * Hv * 128 + 2.0 * Dv * 6 * Dv)
    return _extra_line("video_block_S28350_D1536_H12_M8960_ctx512_bf16", ms, flops, K, args.warmup,
                       {"gpu_launches_per_step": 13})


def run_ring8(args):
    """One rank's compute in a CP=8 ring over the Flux sequence (4608 tokens
    = 8 x 576 per rank, 24 heads x 128), on one GPU: attention of the 576 local
    queries against the 8 key/value shards, each step after the first merged
    into the running result, captured as one CUDA graph (the transfers between
    ranks are not part of this single-GPU measurement).  G shards per attention
    step: G = 1 is the ring (8 steps), G = 8 gathers every shard first (1
    step).  splits = 1: one attention launch per step, merging in its epilogue
    (dit_attention / dit_attention_accumulate, 72 CTAs); splits = 2, the ring
    plan's default at this size: the step's keys are cut in two parts computed
    side by side (144 CTAs) and merged with the running result by
    log-sum-exp (dit_attention_split).  The headline is the ring (G = 1) as
    the plan runs it."""
    import torch
    import diffusion_transformer_block_flux_b200 as dit
    from diffusion_transformer_block_flux_b200.sequence_parallel import auto_key_splits
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    g.manual_seed(13)
    N, Sl = 8, S // 8
    NB = 4  # buffer sets, rotated so K/V shards are not all L2-resident from the last replay
    q = [_rand(torch, g, dev, Sl, D) for _ in range(NB)]
    kv = [_rand(torch, g, dev, 2, S, D) for _ in range(NB)]
    o = torch.empty((Sl, D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((1, H, Sl), dtype=torch.float32, device=dev)
    auto = auto_key_splits(Sl, H, dev)
    ws = torch.empty(max(1, dit.dit_attention_split_workspace(1, Sl, H, max(2, auto))), dtype=torch.uint8,
                     device=dev)
    K = max(5, args.steps // 4)
    flops = 4.0 * Sl * S * H * 128
    per_g = {}
    for splits in sorted({1, auto}):
        for G in (1, 2, 4, 8):
            def ring(i, G=G, splits=splits):
                k, v = kv[i][0], kv[i][1]
                for j in range(0, N, G):
                    ks, vs = k[j * Sl:(j + G) * Sl], v[j * Sl:(j + G) * Sl]
                    if splits > 1:
                        dit.dit_attention_split(q[i], ks, vs, o, 1, Sl, G * Sl, H, splits, ws, lse=lse,
                                                accumulate=j > 0)
                    elif j == 0:
                        dit.dit_attention(q[i], ks, vs, o, 1, Sl, G * Sl, H, lse=lse)
                    else:
                        dit.dit_attention_accumulate(q[i], ks, vs, o, lse, 1, Sl, G * Sl, H)

            for i in range(NB):
                ring(i)
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                for i in range(NB):
                    ring(i)
            ms = _event_time(torch, graph.replay, K, 3, torch.cuda.current_stream()) / NB
            del graph
            tf = flops / (ms * 1e-3) / 1e12
            per_g[f"G{G}_splits{splits}"] = {"ms": round(ms, 4), "tflops": round(tf, 1),
                                             "frac_of_bf16_peak": round(tf / peaks()["bf16_tflops"], 4),
                                             "launches": (N // G) * (2 if splits > 1 else 1)}
    st, code = dit.dit_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error word {code:#x}")
    head = per_g[f"G1_splits{auto}"]
    ms1 = head["ms"]
    return _extra_line("ring_cp8_rank_compute_S4608_576q_24x128", ms1, flops, K * NB, 3,
                       {"us_per_hop": round(ms1 * 1e3 / N, 2), "hops": N, "key_splits": auto,
                        "gpu_launches_per_step": head["launches"], "shards_per_step": per_g,
                        "context": "the compile_graph page, section 5: one attention segment of the 8-card ring "
                                   "took 0.073 ms on H20"})


def run_loop(args):
    """Flux.1-dev-shaped denoising loop at 1024^2: 19 double + 38 single blocks,
    50 flow-match Euler steps, captured once as one CUDA graph and replayed."""
    import torch
    import diffusion_transformer_block_flux_b200 as dit
    from diffusion_transformer_block_flux_b200 import synth
    ls = synth.FLUX_LOOP
    if args.loop_blocks or args.loop_steps:
        # a shorter or shallower loop of the same width (profiling captures on a few GB)
        nd, ns = (int(v) for v in args.loop_blocks.split(",")) if args.loop_blocks else (ls.n_double, ls.n_single)
        ls = synth.loop_shape(synth.FLUX, nd, ns, args.loop_steps or ls.steps, channels=ls.channels,
                              txt_in=ls.txt_in)
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    g.manual_seed(11)
    z = lambda n: torch.zeros(n, device=dev, dtype=torch.bfloat16)
    one = lambda n: torch.ones(n, device=dev, dtype=torch.bfloat16)
    r = lambda *shape: _rand(torch, g, dev, *shape, std=0.02)
    F = 4 * ls.channels
    mw = {"W_img_in": r(D, F), "b_img_in": z(D), "W_txt_in": r(D, ls.txt_in), "b_txt_in": z(D),
          "W_t1": r(D, ls.t_dim), "b_t1": z(D), "W_t2": r(D, D), "b_t2": z(D),
          "W_fmod": r(2 * D, D), "b_fmod": z(2 * D), "W_out": r(F, D), "b_out": z(F), "double": [], "single": []}
    for _ in range(ls.n_double):
        mw["double"].append({st: {"W_mod": r(6 * D, D), "b_mod": z(6 * D), "W_qkv": r(3 * D, D), "b_qkv": z(3 * D),
                                  "q_scale": one(128), "k_scale": one(128), "W_proj": r(D, D), "b_proj": z(D),
                                  "W_mlp1": r(M, D), "b_mlp1": z(M), "W_mlp2": r(D, M), "b_mlp2": z(D)}
                             for st in ("txt", "img")})
    for _ in range(ls.n_single):
        mw["single"].append({"W_mod": r(3 * D, D), "b_mod": z(3 * D), "W1": r(3 * D + M, D), "b1": z(3 * D + M),
                             "q_scale": one(128), "k_scale": one(128), "W2": r(D, D + M), "b2": z(D)})
    model = dit.Model(mw, D=D, H=H, M=M, channels=ls.channels, txt_dim=ls.txt_in, t_dim=ls.t_dim)
    lat = _rand(torch, g, dev, ls.channels, 2 * GRID, 2 * GRID, std=1.0)
    txt = _rand(torch, g, dev, S_TXT, ls.txt_in, std=1.0)
    ids = torch.from_numpy(synth.flux_ids(S_TXT, GRID, GRID)).to(dev)
    out = torch.empty((ls.channels, 2 * GRID, 2 * GRID), dtype=torch.float32, device=dev)
    fresh = dit.cached_schedule(ls.steps) if args.cache else None
    # classifier-free guidance as the SDXL guide runs it: on for the first 75% of the steps
    unc = _rand(torch, g, dev, S_TXT, ls.txt_in, std=1.0) if args.cfg else None
    cfg_steps = (3 * ls.steps) // 4
    io = dit.loop_io(S_TXT, GRID, GRID, ls.steps, lat, txt, ids, out, fresh=fresh, cache_order=1,
                     txt_uncond=unc, guidance=3.5, cfg_steps=cfg_steps)
    ws = torch.empty(dit.dit_forward_workspace(model, io), dtype=torch.uint8, device=dev)
    t0 = time.time()
    graph = dit.Graph(model, io, ws)
    t_build = time.time() - t0
    stream = torch.cuda.current_stream()
    K = max(1, min(3, args.steps))
    W = 3
    ms = _event_time(torch, lambda: graph.launch(stream.cuda_stream), K, W, stream)
    st, code = dit.dit_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error word {code:#x}")
    single = sum(block_flops().values())
    dbl = 2.0 * S * D * (3 * D + D + 2 * M) + 4.0 * S * S * H * 128 + 2 * 2.0 * D * 6 * D
    emb = 2.0 * (S_TXT * ls.txt_in * D + (S - S_TXT) * F * D + ls.t_dim * D + D * D) + 2.0 * D * 2 * D \
        + 2.0 * (S - S_TXT) * D * F
    fresh_steps = [i for i in range(ls.steps) if fresh is None or fresh[i]]
    n_fwd = len(fresh_steps) + (sum(1 for i in fresh_steps if i < cfg_steps) if args.cfg else 0)
    flops = n_fwd * (ls.n_double * dbl + ls.n_single * single + emb)
    n_nodes = graph.nodes()
    graph.destroy()
    name = (ls.name + ("_step_cache" if fresh is not None else "") + ("_cfg%dof%d" % (cfg_steps, ls.steps) if args.cfg
            else "") + "_%dforwards_one_cuda_graph" % n_fwd)
    return _extra_line(name, ms, flops, K, W,
                       {"s_per_image": round(ms / 1e3, 3), "graph_nodes": n_nodes, "model_forwards": n_fwd,
                        "graph_build_s": round(t_build, 2), "graph_launches_per_image": 1})


def run_kernels(args):
    """HBM-bound kernels alone at the Flux single-block shape.  Each iteration
    uses the next of 4 buffer sets (> L2 in total), so every launch reads HBM."""
    import torch
    import diffusion_transformer_block_flux_b200 as dit
    from diffusion_transformer_block_flux_b200 import synth
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    g.manual_seed(3)
    pk = peaks()
    NB = 4
    xs = [_rand(torch, g, dev, S, D) for _ in range(NB)]
    ys = [torch.empty_like(xs[0]) for _ in range(NB)]
    mods = [torch.randn(3 * D, generator=g, device=dev) for _ in range(NB)]
    qkvs = [_rand(torch, g, dev, S, 3 * D) for _ in range(NB)]
    Ws = [_rand(torch, g, dev, 3 * D, D, std=0.02) for _ in range(NB)]
    vec = _rand(torch, g, dev, 1, D)
    mout = torch.empty((1, 3 * D), dtype=torch.float32, device=dev)
    ones = torch.ones(128, device=dev, dtype=torch.bfloat16)
    ids = torch.from_numpy(synth.flux_ids(S_TXT, GRID, GRID)).to(dev)
    rope = torch.empty((S, 64, 2), dtype=torch.float32, device=dev)
    dit.dit_rope_table(ids, (8, 28, 28), 10000.0, rope)
    it = [0]

    def nxt():
        it[0] = (it[0] + 1) % NB
        return it[0]

    def ln():
        i = nxt()
        dit.dit_modulate_norm(xs[i], mods[i][:D], mods[i][D:2 * D], ys[i], 1, S)

    def qk():
        i = nxt()
        q = qkvs[i]
        dit.dit_qk_norm_rope(q[:, :D], q[:, D:2 * D], ones, ones, rope, q[:, :D], q[:, D:2 * D], 1, S, H)

    def ada():
        i = nxt()
        dit.dit_adaln_modulation(vec, Ws[i], None, mout)

    mo = [_rand(torch, g, dev, S, D) for _ in range(NB)]
    ml = [torch.randn((1, H, S), generator=g, device=dev) for _ in range(2 * NB)]

    def merge():  # one ring hop's merge: running result + new part, in place
        i = nxt()
        dit.dit_attention_merge([ys[i], mo[i]], [ml[2 * i], ml[2 * i + 1]], ys[i], ml[2 * i], 1, S, H)

    def copy():  # yardstick, not part of the path: a library copy of the LayerNorm's bytes
        i = nxt()
        ys[i].copy_(xs[i])

    # R launches per CUDA graph, so that host-side call overhead is not timed
    R = 4 * NB
    K = max(5, args.steps // R)
    stream = torch.cuda.current_stream()
    res = {}
    for name, fn, nbytes in (("modulate_norm", ln, 2 * S * D * 2),
                             ("qk_norm_rope", qk, 4 * S * D * 2 + S * 64 * 8),
                             ("adaln_modulation", ada, 3 * D * D * 2),
                             ("attention_merge_2parts", merge, 3 * S * D * 2 + 3 * H * S * 4),
                             ("torch_copy_same_bytes_as_modulate_norm", copy, 2 * S * D * 2)):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for _ in range(R):
                fn()
        ms = _event_time(torch, graph.replay, K, 3, torch.cuda.current_stream()) / R
        del graph
        gbs = nbytes / (ms * 1e-3) / 1e9
        res[name] = {"us": round(ms * 1e3, 2), "gbs": round(gbs, 1), "frac_of_hbm_peak": round(gbs / pk["hbm_gbs"], 4),
                     "bytes": nbytes}
    st, code = dit.dit_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error word {code:#x}")
    return {"metric": "HBM-bound kernels alone, Flux single-block shape (S=4608, D=3072)", "unit": "GB/s",
            "n_gpus": 1, "steps": K * R, "warmup": args.warmup, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "hbm_kernels_S4608_D3072", "l2": "4 rotating buffer sets, > L2 in total",
                       "timing": f"{R} launches per CUDA graph, {K} replays, CUDA events"},
            "hbm_peak_gbs": pk["hbm_gbs"], "kernels": res}


def run_cfg_batch(args):
    """Classifier-free guidance as one batch-2 pass or as two batch-1 passes:
    the single-stream block (S=4608) and the double-stream block (512 + 4096)
    at B = 2 against two B = 1 calls on the same two samples (the SDXL guide,
    section 3.3, runs the conditional and unconditional halves as one batch)."""
    import torch
    import diffusion_transformer_block_flux_b200 as dit
    from diffusion_transformer_block_flux_b200 import synth
    dev = torch.device("cuda", 0)
    w, x, vec = make_block(torch, dev, seed=21)
    x2 = torch.cat([x, torch.roll(x, 1, 0)])
    vec2 = torch.cat([vec, vec])
    ids = torch.from_numpy(synth.flux_ids(S_TXT, GRID, GRID)).to(dev)
    rope = torch.empty((S, 64, 2), dtype=torch.float32, device=dev)
    dit.dit_rope_table(ids, (8, 28, 28), 10000.0, rope)
    cw = dit.single_weights(w)
    c1, c2 = dit.block_cfg(1, S, D, H, M), dit.block_cfg(2, S, D, H, M)
    ws = torch.empty(dit.dit_single_block_workspace(c2), dtype=torch.uint8, device=dev)
    o2 = torch.empty_like(x2)
    K, W = args.steps, args.warmup
    st = torch.cuda.current_stream()
    t2 = _event_time(torch, lambda: dit.dit_single_block_fwd(c2, cw, x2, vec2, rope, o2, ws), K, W, st)
    clk2 = dict(_LAST_CLOCKS)

    def two():
        dit.dit_single_block_fwd(c1, cw, x2[:S], vec2[:1], rope, o2[:S], ws)
        dit.dit_single_block_fwd(c1, cw, x2[S:], vec2[1:], rope, o2[S:], ws)
    t1 = _event_time(torch, two, K, W, st)
    flops = 2 * block_flops_total()
    res = _extra_line("cfg_single_block_batch2_vs_2x_batch1_S4608_D3072", t2, flops, K, W,
                      {"ms_batch2": round(t2, 4), "ms_two_batch1": round(t1, 4),
                       "batch2_speedup": round(t1 / t2, 4), "clocks_batch2": clk2})
    return res


def block_flops_total(S_=S):
    return sum(block_flops(S_).values())


EXTRA = {"double": run_double, "video": run_video, "loop": run_loop, "kernels": run_kernels, "ring8": run_ring8,
         "cfg_batch": run_cfg_batch}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["single"] + sorted(EXTRA), default="single",
                    help="single = the headline Flux single-stream block (default)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cache", action="store_true",
                    help="loop workload: model-level step cache (26 model forwards for 50 steps)")
    ap.add_argument("--cfg", action="store_true",
                    help="loop workload: classifier-free guidance on the first 75%% of the steps")
    ap.add_argument("--loop-blocks", default="",
                    help="loop workload: 'double,single' block counts instead of 19,38 (same width)")
    ap.add_argument("--loop-steps", type=int, default=0,
                    help="loop workload: Euler steps instead of 50")
    ap.add_argument("--l2-keep-weights-mb", type=int, default=0,
                    help="persisting L2 set-aside (MB) for the output GEMMs' weights (dit_set_weight_l2_persist); 0 = off")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.workload != "single":
        import torch
        torch.cuda.set_device(0)
        print(json.dumps(EXTRA[args.workload](args)), flush=True)
        return 0
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args)), flush=True)
        return 0

    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE", file=sys.stderr)
    if world > 1:
        import datetime
        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        res = run_ours(args, rank, world, local_rank)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline()
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

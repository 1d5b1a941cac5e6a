#!/usr/bin/env python
"""Throughput of the LatentMoE layer forward through the C-ABI library.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one lmoe_forward over the README-scale "acc" layer (T=4096 tokens,
d=2048, l=512, m=1408, N'=256, K'=24, two shared SwiGLU experts of width 1408,
bf16 operands, fp32 accumulation) on synthetic seeded inputs resident in HBM.
Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA events
on the launch stream, with a 512 MiB write between steps to flush the 126 MB
L2; barrier + synchronize on both sides; the max over ranks is reported.
With N > 1 (torchrun) every rank runs an independent replica on its own
tokens (the layer forward has no exchange step on one GPU): weak scaling.

The JSON line also carries: the roofline of the dominant kernel (per-stage
CUDA events recorded inside the library during a second timed pass, so that
the first pass -- the `value` -- times plain forwards), the whole
layer's roofline, an end-to-end number through lmoe_forward_host_batches
(a stream of batches in host buffers, every batch's copies inside the timed
region; the single-call lmoe_forward_host rate beside it), the fp64 oracle
timed on a bounded
sample on the host cores, the launch count, and SM clocks sampled during the
timed region.  --impl reference times the oracle alone on the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "LatentMoE fwd tokens/s (1 B200) & % roofline, d2048 l512 N'256 K'24 bf16"
UNIT = "tokens/s"
FLUSH_BYTES = 512 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="readme_acc",
                    choices=["readme_acc", "readme_eff", "prefill", "decode", "relu2_95b",
                             "decode_fp8", "relu2_95b_fp8", "decode_nvfp4",
                             "relu2_95b_nvfp4"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--ep", type=int, default=0,
                    help="expert parallelism over this many ranks: under torchrun with as many "
                         "GPUs, one rank per GPU with NCCL all-to-alls; on one GPU, that many "
                         "ranks emulated in one process (copies for the exchange)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the workload's token count T (a smaller case of the same "
                         "layer, e.g. for a profiler capture); the line's config names it")
    ap.add_argument("--pass", dest="which", choices=["forward", "backward"], default="forward",
                    help="backward: time lmoe_backward (dx and every weight gradient, "
                         "forward activations recomputed) instead of the forward")
    return ap.parse_args()


def workload(name, tokens=None):
    from dataclasses import replace
    from latent_mixture_experts_top_b200 import configs
    cfg = {"readme_acc": configs.README_ACC, "readme_eff": configs.README_EFF,
           "prefill": configs.PREFILL, "decode": configs.DECODE,
           "relu2_95b": configs.RELU2_95B, "decode_fp8": configs.DECODE_FP8,
           "relu2_95b_fp8": configs.RELU2_95B_FP8, "decode_nvfp4": configs.DECODE_NVFP4,
           "relu2_95b_nvfp4": configs.RELU2_95B_NVFP4}[name]
    if tokens is not None and tokens != cfg.T:
        cfg = replace(cfg, name=f"{cfg.name}@T{tokens}", T=tokens)
    return cfg


def n_mats(cfg):
    """Weight matrices per expert: SwiGLU 3 (gate, up, out), squared ReLU 2."""
    return 2 if cfg.activation == "relu2" else 3


def config_json(cfg, n_gpus):
    return {"workload": cfg.name, "T": cfg.T, "d": cfg.d, "l": cfg.l, "m": cfg.m,
            "n_routed": cfg.n_routed, "k_active": cfg.k_active, "n_shared": cfg.n_shared,
            "m_shared": cfg.m_shared, "variant": cfg.variant, "activation": cfg.activation,
            "expert_weights": cfg.weights,
            "router_bias": cfg.has_router_bias, "global_batch": cfg.T * n_gpus,
            "seq_len": cfg.T, "parallelism": f"replicas x{n_gpus} (no exchange)",
            "l2": "flushed by a 512 MiB write between timed steps"}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- algorithmic work
def stage_work(cfg, touched=None):
    """(FLOPs, algorithmic bytes, intermediate bytes) of one launch of each
    profiled stage.

    FLOPs count 2 per multiply-add of the layer's definition (no padding, no
    masked rows); memory-only stages have 0.  Algorithmic bytes are the
    layer's own inputs and outputs that the stage must move once: the weights
    it multiplies by (for an expert GEMM, those of the ``touched`` distinct
    experts, all N' when not given), x into the first GEMM and y out of the
    last.  Intermediates (logits, ids, gates, dispatch indices, z, the
    permuted z, H, O, u and the shared hidden) are not algorithmic bytes:
    their traffic depends on how the path is cut into kernels, so it is
    reported apart, in the third entry.  The shared experts' gate/up GEMM
    overlaps stages 1-3 on a side stream and is not a stage of its own (see
    shared_gate_up_work).
    """
    T, d, l, m, N, K = cfg.T, cfg.d, cfg.l, cfg.m, cfg.n_routed, cfg.k_active
    ns, ms = cfg.n_shared, cfg.m_shared
    E = N if touched is None else touched
    TK = T * K
    gu = n_mats(cfg) - 1          # gate+up (2) or up (1) rows per hidden column
    ew = expert_weight_bytes(cfg)
    ky = l + ns * ms
    return {
        0: (2.0 * T * d * (N + l), 2.0 * T * d + 2.0 * d * (N + l), 4.0 * T * N + 2.0 * T * l),
        1: (0.0, 0.0, 4.0 * T * N + 8.0 * TK),
        2: (0.0, 0.0, 4.0 * TK * 5),
        3: (0.0, 0.0, 2.0 * TK * l * 2 + 4.0 * TK),
        4: (2.0 * TK * l * gu * m, ew * E * gu * m * l, 2.0 * TK * l + 2.0 * TK * m),
        5: (2.0 * TK * m * l, ew * E * l * m, 2.0 * TK * m + 2.0 * TK * l),
        6: (0.0, 0.0, 2.0 * TK * l + 8.0 * TK + 2.0 * T * l),
        7: (2.0 * T * ky * d, 2.0 * d * ky + 2.0 * T * d, 2.0 * T * ky),
    }


def shared_gate_up_work(cfg):
    """(FLOPs, algorithmic bytes, intermediate bytes) of the side-stream
    shared-expert gate/up GEMM: its weights are algorithmic; x is counted
    once, by stage 0; the shared hidden it writes is an intermediate."""
    gu = n_mats(cfg) - 1
    nsms = cfg.n_shared * cfg.m_shared
    return (2.0 * cfg.T * cfg.d * gu * nsms, 2.0 * cfg.d * gu * nsms, 2.0 * cfg.T * nsms)


def stage_bound(flops, nbytes, peaks):
    """'tensor' or 'hbm': whichever takes longer at the measured peaks (a
    stage with neither FLOPs nor algorithmic bytes is a memory-bound helper:
    'hbm')."""
    if flops <= 0.0 and nbytes <= 0.0:
        return "hbm"
    t_tensor = flops / (peaks["bf16_tflops"] * 1e12)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    return "tensor" if t_tensor >= t_hbm else "hbm"


def backward_flops(cfg):
    """Algorithmic FLOPs of one lmoe_backward call: the recomputed forward
    activations (x-GEMM, expert gate/up and down), the data gradients (dy W_y,
    DO W_o, dAB W_gu, dXcat W_x) and the weight gradients (dy^T [u|h_s],
    dXcat^T x, DO^T H, dAB^T zp), 2 flops per multiply-add."""
    T, d, l, m, N, K = cfg.T, cfg.d, cfg.l, cfg.m, cfg.n_routed, cfg.k_active
    gu = n_mats(cfg) - 1
    nsms = cfg.n_shared * cfg.m_shared
    TK = T * K
    xrows = N + l + gu * nsms        # router, W_down and shared gate/up rows
    ky = l + nsms
    fwd = 2.0 * T * d * xrows + 2.0 * TK * l * gu * m + 2.0 * TK * m * l
    data = 2.0 * T * d * ky + 2.0 * TK * l * m + 2.0 * TK * gu * m * l + 2.0 * T * xrows * d
    wgt = 2.0 * T * d * ky + 2.0 * T * xrows * d + 2.0 * TK * l * m + 2.0 * TK * gu * m * l
    return fwd + data + wgt


def layer_flops(cfg):
    T, d, l, m, N, K = cfg.T, cfg.d, cfg.l, cfg.m, cfg.n_routed, cfg.k_active
    nm = n_mats(cfg)
    return 2.0 * T * (d * N + 2 * d * l + nm * K * l * m + nm * cfg.n_shared * d * cfg.m_shared)


def expert_weight_bytes(cfg):
    """Bytes per routed-expert weight: 2 (bf16); 1 (E4M3); NVFP4 half a byte
    of E2M1 code plus one E4M3 block scale per 16 weights.  The f32 row
    scales (one per weight row of length >= 512, < 0.01 byte per weight) are
    left out."""
    return {"fp8": 1.0, "nvfp4": 0.5 + 1.0 / 16}.get(cfg.weights, 2.0)


def layer_bytes(cfg, ids=None):
    """Weights actually touched (router, projections, shared, the distinct
    experts hit) + x in + y out; bf16 except E4M3 routed experts."""
    d, l, m, N = cfg.d, cfg.l, cfg.m, cfg.n_routed
    touched = N if ids is None else len(set(ids.reshape(-1).tolist()))
    nm = n_mats(cfg)
    w = N * d + 2 * d * l + nm * cfg.n_shared * d * cfg.m_shared
    experts = touched * nm * l * m * expert_weight_bytes(cfg)
    return 2.0 * (w + 2 * cfg.T * d) + experts


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML (read-only)."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x10: "sync_boost"}

    def __init__(self, index, period=0.002):
        self.index, self.period = index, period
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            return self
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def _run(self):
        nv = self._nv
        get_r = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = get_r(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def stop(self):
        self._stop.set()
        if self._t:
            self._t.join()
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples), "source": "nvml" if self.ok else "unavailable"}


# ---------------------------------------------------------------- oracle timing
def oracle_rate(cfg, inp_np, budget_s, max_tokens=None):
    """Tokens/s of the fp64 oracle (full layer incl. router) on the host."""
    import numpy as np
    import oracle
    L = oracle.Layer(w_router=inp_np["w_router"],
                     b_router=None if inp_np["b_router"] is None else inp_np["b_router"].astype(np.float64),
                     w_down=inp_np["w_down"], w_up=inp_np["w_up"], w_gate=inp_np["w_gate"],
                     w_upx=inp_np["w_upx"], w_out=inp_np["w_out"], s_gate=inp_np["s_gate"],
                     s_up=inp_np["s_up"], s_out=inp_np["s_out"], k_active=cfg.k_active,
                     activation=cfg.activation, act_fp8=cfg.weights == "fp8",
                     act_fp4=cfg.weights == "nvfp4")
    x = inp_np["x"]
    cal = min(cfg.T, max(8, oracle.threads()))
    t0 = time.perf_counter()
    oracle.forward(L, x, tokens=np.arange(cal))
    per_tok = (time.perf_counter() - t0) / cal
    n = int(max(cal, min(cfg.T if max_tokens is None else max_tokens, budget_s / per_tok)))
    t0 = time.perf_counter()
    oracle.forward(L, x, tokens=np.arange(n))
    dt = time.perf_counter() - t0
    return n / dt, n, dt, oracle.threads(), L


def numpy_inputs(inp):
    from latent_mixture_experts_top_b200 import synth
    return {k: (None if v is None else synth.to_numpy(v)) for k, v in inp.items()}


# ---------------------------------------------------------------- reference arm
def run_reference(args):
    _, rank, _ = rank_env()
    if rank != 0:
        return 0      # the oracle runs once, on rank 0; other ranks do no work
    import numpy as np
    import torch
    import oracle
    from latent_mixture_experts_top_b200 import synth
    cfg = workload(args.workload, args.tokens)
    inp = synth.make_inputs(cfg, args.seed, "cpu")
    n = numpy_inputs(inp)
    rate_cal, _, _, cores, L = oracle_rate(cfg, n, budget_s=2.0, max_tokens=64)
    budget = 150.0 / max(1, args.steps + args.warmup)      # whole run within minutes
    per_step = int(max(1, min(cfg.T, budget * rate_cal)))
    toks = np.arange(per_step)
    for _ in range(args.warmup):
        oracle.forward(L, n["x"], tokens=toks)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.forward(L, n["x"], tokens=toks)
    dt = time.perf_counter() - t0
    value = per_step * args.steps / dt
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_json(cfg, 1),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"{per_step} tokens (0..{per_step - 1}) of the "
                                       f"T={cfg.T} workload per step, full layer incl. router"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- ranks
def rank_env():
    """(world size, rank, local rank) from the torchrun environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def reduce_max_over_ranks(v: float, world: int, device: str) -> float:
    """Max of a per-rank time over all ranks (the slowest rank sets the job's
    time); identity on one rank.  Needs an initialised process group."""
    if world == 1:
        return float(v)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, world: int, max_ms_per_step: float) -> float:
    """Whole-job tokens/s: every rank runs its own replica on its own tokens
    (no exchange), so the job moves world * tokens_per_rank per step, in the
    slowest rank's step time."""
    return tokens_per_rank * world / (max_ms_per_step / 1e3)


# ---------------------------------------------------------------- our arm
def traffic_from_profiles(kernel_key, workload_name, sha):
    """DRAM bytes per launch of ``kernel_key`` on this workload from a
    committed ncu summary, if it was taken on the current kernel source (else
    None).  Summary lines read
    ``traffic_bytes_per_launch[<kernel>@<workload>] = <bytes> source_sha256=<sha>``."""
    d = os.path.join(ROOT, "profiles")
    if not os.path.isdir(d):
        return None
    pat = re.compile(r"traffic_bytes_per_launch\[(\w+)@(\w+)\]\s*=\s*([0-9.eE+]+)"
                     r"\s+source_sha256=(\w+)")
    for fn in sorted(os.listdir(d)):
        if not fn.endswith((".md", ".txt")):
            continue
        with open(os.path.join(d, fn)) as f:
            for mt in pat.finditer(f.read()):
                if (mt.group(1) == kernel_key and mt.group(2) == workload_name
                        and mt.group(4) == sha):
                    return float(mt.group(3))
    return None


def kernel_source_sha():
    h = hashlib.sha256()
    for fn in ("tc_gemm.cu", "ptx_sm100.cuh", "common.cuh", "route_kernels.cu"):
        with open(os.path.join(ROOT, "latent_mixture_experts_top_b200", "csrc", fn), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist
    from latent_mixture_experts_top_b200 import lmoe, synth

    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    def allmax(v):
        return reduce_max_over_ranks(v, world, "cuda")

    cfg = workload(args.workload, args.tokens)
    inp = synth.make_inputs(cfg, args.seed, "cuda")
    layer = lmoe.LatentMoELayer(cfg, inp)
    x = inp["x"]
    y = torch.empty_like(x)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        flush.fill_(1)
        layer.forward(x, y)
    torch.cuda.synchronize()
    if lmoe.lmoe_device_status(layer.handle) != 0:
        raise RuntimeError("device status error during warm-up")

    K = args.steps

    def timed_steps(n):
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        barrier()
        torch.cuda.synchronize()
        for i in range(n):
            flush.fill_(1)                    # evict L2 outside the timed window
            starts[i].record(stream)
            lmoe.lmoe_forward(layer.handle, x, y, cfg.T, stream)
            ends[i].record(stream)
        torch.cuda.synchronize()
        barrier()
        return [a.elapsed_time(b) for a, b in zip(starts, ends)]

    # Timed region for `value`: K plain forwards (no in-library events).
    launches0 = lmoe.lmoe_launches(layer.handle)
    clocks = ClockSampler(local).start()
    step_ms = timed_steps(K)
    clk = clocks.stop()
    launches = lmoe.lmoe_launches(layer.handle) - launches0
    # Second timed pass for the per-kernel split: the library records CUDA
    # events between its stages on the launch stream.
    n_prof = min(K, 100)
    lmoe.lmoe_profile(layer.handle, n_prof)
    prof_step_ms = timed_steps(n_prof)
    stage_ms, n_prof, _ = lmoe.lmoe_stage_times(layer.handle)
    lmoe.lmoe_profile(layer.handle, 0)
    if lmoe.lmoe_device_status(layer.handle) != 0:
        raise RuntimeError("device status error during timing")
    total_ms = allmax(sum(step_ms))
    ms_per_step = total_ms / K
    value = job_throughput(cfg.T, world, ms_per_step)

    peaks, peak_src = load_peaks()
    ids = layer.route(x)[0].cpu().numpy()
    work = stage_work(cfg, touched=len(set(ids.reshape(-1).tolist())))
    avg_stage = [t / max(1, n_prof) for t in stage_ms]
    dom = max(range(len(avg_stage)), key=lambda i: avg_stage[i])
    flops, nbytes, inter = work[dom]
    kind = stage_bound(flops, nbytes, peaks)
    if kind == "tensor":
        amount, unit, peak = flops, "TFLOP/s", peaks["bf16_tflops"]
        achieved = amount / (avg_stage[dom] / 1e3) / 1e12
    else:
        amount, unit, peak = nbytes, "GB/s", peaks["hbm_gbs"]
        achieved = amount / (avg_stage[dom] / 1e3) / 1e9
    sha = kernel_source_sha()
    traffic = traffic_from_profiles(lmoe.STAGE_NAMES[dom], cfg.name, sha)
    roofline = {"bound": kind, "kernel": lmoe.STAGE_NAMES[dom], "achieved": achieved,
                "peak": peak, "unit": unit, "frac": achieved / peak, "traffic": traffic,
                "peak_source": f"{peak_src} (burst)" if kind == "tensor" else peak_src,
                "algorithmic_per_launch": amount, "algorithmic_flops": flops,
                "algorithmic_bytes": nbytes, "intermediate_bytes": inter,
                "bytes_ratio_with_intermediates": (nbytes + inter) / nbytes if nbytes else None,
                "avg_launch_ms": avg_stage[dom]}
    F, B = layer_flops(cfg), layer_bytes(cfg, ids)
    t_roof = max(F / (peaks["bf16_tflops"] * 1e12), B / (peaks["hbm_gbs"] * 1e9))
    layer_roof = {"flops": F, "bytes": B, "roofline_ms": 1e3 * t_roof,
                  "bound": "tensor" if F / (peaks["bf16_tflops"] * 1e12) >= B / (peaks["hbm_gbs"] * 1e9) else "hbm",
                  "frac": 1e3 * t_roof / ms_per_step,
                  "achieved_tflops": F / (ms_per_step / 1e3) / 1e12}

    # end to end through the public API with host buffers: a stream of
    # e2e_steps batches (two pinned host buffer pairs, alternating), each
    # batch copied in, computed and copied out inside the timed region
    e2e_steps = args.e2e_steps or max(3, min(K, 50))
    x_hs = [x.cpu().pin_memory() for _ in range(2)]
    y_hs = [torch.empty_like(x_hs[0]).pin_memory() for _ in range(2)]
    xs = [x_hs[i % 2] for i in range(e2e_steps)]
    ys = [y_hs[i % 2] for i in range(e2e_steps)]
    lmoe.lmoe_forward_host_batches(layer.handle, xs[:2], ys[:2], cfg.T)
    barrier()
    t0 = time.perf_counter()
    lmoe.lmoe_forward_host_batches(layer.handle, xs, ys, cfg.T)
    e2e_s = allmax(time.perf_counter() - t0)
    # one batch per call (copies overlap only within the call)
    barrier()
    t1 = time.perf_counter()
    for _ in range(3):
        lmoe.lmoe_forward_host(layer.handle, x_hs[0], y_hs[0], cfg.T)
    single_s = allmax(time.perf_counter() - t1)
    io_bytes = cfg.T * cfg.d * x.element_size()
    e2e = {"value": cfg.T * world * e2e_steps / e2e_s, "unit": UNIT,
           "h2d_bytes_per_step": io_bytes, "d2h_bytes_per_step": io_bytes,
           "steps": e2e_steps,
           "api": "lmoe_forward_host_batches (pinned host buffers, one call over the steps)",
           "single_call": {"value": cfg.T * world * 3 / single_s, "unit": UNIT,
                           "api": "lmoe_forward_host, one call per step", "steps": 3}}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, n_tok, dt, cores, _ = oracle_rate(cfg, numpy_inputs(inp), budget_s=12.0)
        cpu = {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{n_tok} tokens (0..{n_tok - 1}) of the T={cfg.T} workload, full "
                         f"layer incl. router, fp64, {dt:.1f} s"}

    layer.close()
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic: x~N(0,1), weights~N(0,0.02), seeded",
                "config": config_json(cfg, world), "roofline": roofline,
                "layer_roofline": layer_roof, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": launches, "clocks": clk,
                "stages_ms": {lmoe.STAGE_NAMES[i]: avg_stage[i] for i in range(len(avg_stage))},
                "stages_source": f"second timed pass of {n_prof} steps with in-library stage events "
                                 f"({statistics.mean(prof_step_ms):.4f} ms/step)",
                "step_ms_min": min(step_ms), "step_ms_median": statistics.median(step_ms)}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def oracle_backward_rate(cfg, inp_np, dy_np, budget_s):
    """Tokens/s of the fp64 oracle's backward (dx and every weight gradient)."""
    import numpy as np
    import oracle
    L = oracle.Layer(w_router=inp_np["w_router"],
                     b_router=None if inp_np["b_router"] is None else inp_np["b_router"].astype(np.float64),
                     w_down=inp_np["w_down"], w_up=inp_np["w_up"], w_gate=inp_np["w_gate"],
                     w_upx=inp_np["w_upx"], w_out=inp_np["w_out"], s_gate=inp_np["s_gate"],
                     s_up=inp_np["s_up"], s_out=inp_np["s_out"], k_active=cfg.k_active,
                     activation=cfg.activation)
    x = inp_np["x"]
    cal = min(cfg.T, max(8, oracle.threads()))
    t0 = time.perf_counter()
    oracle.backward(L, x, dy_np[:cal], tokens=np.arange(cal))
    per_tok = (time.perf_counter() - t0) / cal
    n = int(max(cal, min(cfg.T, budget_s / per_tok)))
    t0 = time.perf_counter()
    oracle.backward(L, x, dy_np[:n], tokens=np.arange(n))
    dt = time.perf_counter() - t0
    return n / dt, n, dt, oracle.threads()


def run_backward(args):
    """One step = one lmoe_backward over the workload (the forward
    activations it needs are recomputed inside the call)."""
    import numpy as np
    import torch
    import torch.distributed as dist
    from latent_mixture_experts_top_b200 import lmoe, synth

    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    cfg = workload(args.workload, args.tokens)
    inp = synth.make_inputs(cfg, args.seed, "cuda")
    dy = synth.make_cotangent(cfg, args.seed, "cuda")
    layer = lmoe.LatentMoELayer(cfg, inp, training=True)
    x = inp["x"]
    dx = torch.empty_like(x)
    grads = {k: torch.empty(v, dtype=torch.float32, device="cuda")
             for k, v in layer.grad_shapes().items()}
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        flush.fill_(1)
        lmoe.lmoe_backward(layer.handle, x, dy, dx, grads, cfg.T, stream)
    torch.cuda.synchronize()
    if lmoe.lmoe_device_status(layer.handle) != 0:
        raise RuntimeError("device status error during warm-up")
    K = args.steps
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    launches0 = lmoe.lmoe_launches(layer.handle)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local).start()
    for i in range(K):
        flush.fill_(1)
        starts[i].record(stream)
        lmoe.lmoe_backward(layer.handle, x, dy, dx, grads, cfg.T, stream)
        ends[i].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    launches = lmoe.lmoe_launches(layer.handle) - launches0
    if lmoe.lmoe_device_status(layer.handle) != 0:
        raise RuntimeError("device status error during timing")
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    ms_per_step = reduce_max_over_ranks(sum(step_ms), world, "cuda") / K
    value = job_throughput(cfg.T, world, ms_per_step)
    peaks, peak_src = load_peaks()
    F = backward_flops(cfg)
    achieved = F / (ms_per_step / 1e3) / 1e12
    roofline = {"bound": "tensor", "kernel": "lmoe_backward (every launch of the call)",
                "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"], "traffic": None,
                "peak_source": f"{peak_src} (burst)", "algorithmic_per_launch": F,
                "avg_launch_ms": ms_per_step}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        dy_np = dy.float().cpu().numpy().astype(np.float64)
        rate, n_tok, dt, cores = oracle_backward_rate(cfg, numpy_inputs(inp), dy_np, 12.0)
        cpu = {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{n_tok} tokens (0..{n_tok - 1}) of the T={cfg.T} workload, dx and "
                         f"every weight gradient, fp64, {dt:.1f} s"}
    layer.close()
    if rank == 0:
        line = {"metric": "LatentMoE layer backward tokens/s (1 B200), dx + all weight gradients",
                "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic: x~N(0,1), dy~N(0,1), weights~N(0,0.02), seeded",
                "config": dict(config_json(cfg, world), which="backward"),
                "roofline": roofline, "cpu_baseline": cpu,
                "e2e": {"value": None, "note": "no host-buffer backward call in the API"},
                "gpu_launches": launches, "clocks": clk,
                "step_ms_min": min(step_ms), "step_ms_median": statistics.median(step_ms)}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_ep(args):
    """One step = one expert-parallel forward of T tokens per rank (the
    phases of lmoe_ep_* with the two l-wide all-to-alls between them)."""
    import torch
    import torch.distributed as dist
    from latent_mixture_experts_top_b200 import ep, lmoe, synth

    W = args.ep
    if W < 2:
        raise SystemExit("--ep needs at least 2 ranks")
    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    emulated = world == 1
    if not emulated and world != W:
        raise SystemExit(f"--ep {W} needs {W} ranks (got {world}) or one (emulated)")
    if not emulated:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    cfg = workload(args.workload, args.tokens)
    inp = synth.make_inputs(cfg, args.seed, "cuda")       # same weights on every rank
    ranks = range(W) if emulated else [rank]
    layers = [lmoe.LatentMoELayer(cfg, inp, ep_rank=r, ep_world=W) for r in ranks]
    backends = [ep.CudaBackend(L) for L in layers]
    g = torch.Generator(device="cuda").manual_seed(1000 + rank)
    xs = [(torch.randn((cfg.T, cfg.d), generator=g, device="cuda")).to(inp["x"].dtype)
          for _ in ranks]
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        if emulated:
            return ep.forward_emulated(backends, xs)
        return [ep.forward(backends[0], xs[0], W)]

    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()
    K = args.steps
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    if not emulated:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local).start()
    for i in range(K):
        flush.fill_(1)
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    total = sum(step_ms)
    if not emulated:
        total = reduce_max_over_ranks(total, world, "cuda")
        dist.barrier()
    ms_per_step = total / K
    for L in layers:
        if lmoe.lmoe_device_status(L.handle) != 0:
            raise RuntimeError("device status error")
        L.close()
    if rank == 0:
        line = {"metric": f"LatentMoE expert-parallel fwd tokens/s, {W} ranks",
                "value": cfg.T * W / (ms_per_step / 1e3), "unit": UNIT, "n_gpus": world,
                "steps": K, "warmup": args.warmup, "ms_per_step": ms_per_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic: x~N(0,1) per rank, weights~N(0,0.02), seeded",
                "config": dict(config_json(cfg, W),
                               parallelism=f"expert-parallel x{W}" +
                               (" (emulated on one GPU: phases of every rank in turn, "
                                "exchange by device copies)" if emulated else " (NCCL)")),
                "gpu_launches": None, "clocks": clk,
                "step_ms_min": min(step_ms), "step_ms_median": statistics.median(step_ms)}
        print(json.dumps(line), flush=True)
    if not emulated:
        dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.ep:
        return run_ep(args)
    if args.which == "backward":
        return run_backward(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())

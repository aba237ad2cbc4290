#!/usr/bin/env python
"""Throughput of the bidirectional selective scan (S6) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                    [--conv] [--zoh] [--bwd]

One step is one pass of the whole scan -- softplus Delta, the forward and backward
recurrences, readout, D skip, the merge of the directions and the silu(z) gate --
over one batch of the workload, through the library's C ABI.  The default workload
is the 1024 px Vim-Tiny scan (batch 8, L = 4097, d_inner 384, d_state 16, bf16 I/O,
fp32 state).  Inputs are seeded synthetic tensors shaped like the pages' workloads.
--conv times the same scan with the pathways' kernel-3 convolution + SiLU fused in
front (the input tensor is then x, the convolutions' input); --zoh times it with the
exact zero-order-hold Bbar = (exp(Delta A) - 1) / A * B in place of Delta B; --bwd
times the derivative of the scan (every input's gradient from a seeded dout).

Multi-GPU (torchrun, one process per GPU): the batch items are independent, so every
rank runs the same workload on its own inputs with no collective on the data path
(weak scaling); NCCL is used only for the barrier and the max over ranks of the time.

--impl reference times the fp64 CPU oracle (the correctness reference, not tuned) on
the host cores, on a bounded sample of the same workload; under torchrun only rank 0
runs it.

Rank 0 prints one JSON line.
"""
import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_BYTES = 126 * 2**20
MEASURED = os.path.join(ROOT, "MEASURED_PEAKS.json")
# FP32 lanes per SM on B200 (an FMA counts as one lane-op); 148 SMs.
FP32_LANES_PER_SM = 128
SMS = 148


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="vim_tiny_1024px_bf16")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing leg")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="skip the forward timing of the other workloads (other_configs)")
    ap.add_argument("--conv", action="store_true",
                    help="Vim workloads: time the scan with the fused kernel-3 convolution + SiLU front")
    ap.add_argument("--zoh", action="store_true",
                    help="time the scan with the exact zero-order-hold Bbar instead of Delta B")
    ap.add_argument("--block", action="store_true",
                    help="Vim workloads: time vim_block_scan (x_proj + dt_proj + the convolution front + scan)")
    ap.add_argument("--bwd", action="store_true",
                    help="Vim workloads: time the scan's derivative (vim_scan_bidir_bwd) instead")
    ap.add_argument("--ckpt", action="store_true",
                    help="Vim workloads: the forward scan keeps the derivative's chunk states "
                         "(vim_scan_bidir_ckpt); with --bwd, time the derivative that takes them "
                         "(vim_scan_bidir_bwd_ckpt; the states are the forward pass's outputs, formed "
                         "before the timed region)")
    ap.add_argument("--e2e-slices", type=int, default=4,
                    help="pieces of the batch in the end-to-end figure's host-memory entry point")
    return ap.parse_args()


def peaks():
    try:
        with open(MEASURED) as f:
            m = json.load(f)
        return dict(hbm_gbs=float(m["hbm_gbs"]), sm_max_mhz=float(m.get("sm_max_mhz", 1965.0)),
                    source="measured")
    except Exception:
        return dict(hbm_gbs=6650.0, sm_max_mhz=1965.0, source="fallback")


def profiled_traffic(w, bwd=False, zoh=False, conv=False):
    """DRAM bytes per launch of the dominant kernel (pair_main, with the fused front or the
    exact hold or neither; bwd_main for the derivative, with or without the exact hold) from
    the committed ncu summary of this workload and mode, or None when there is none or the
    kernel source changed since it was captured."""
    import hashlib
    import re

    if bwd:
        name = f"ncu_bwd_main_zoh_{w.name}.md" if zoh else f"ncu_bwd_kernels_{w.name}.md"
        source, kernel = "bwd_kernels.cuh", "bwd_main"
    else:
        if conv and zoh:
            return None
        mode = "conv_" if conv else "zoh_" if zoh else ""
        name, source, kernel = f"ncu_scan_kernels_{mode}{w.name}.md", "scan_kernels.cuh", "pair_main"
    path = os.path.join(ROOT, "profiles", name)
    src = os.path.join(ROOT, "vision_mamba_selective_b200", "csrc", source)
    try:
        text = open(path).read()
        fp = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    except OSError:
        return None
    m = re.search(rf"traffic_bytes_per_launch {kernel}: (\d+)", text)
    f = re.search(rf"kernel source fingerprint \(sha256 of {re.escape(source)}, first 16 hex\): ([0-9a-f]+)", text)
    if not m or not f or f.group(1) != fp:
        return None
    return int(m.group(1))


def block_params(w, seed):
    """Weights of the block's projections, drawn as the block parity tests draw them:
    Wx ~ N(0, 1/d_inner) (bf16) [2, d_inner, 2N+1]; dt_proj weights ~ N(0, 0.5) and
    biases log(expm1(s)), s log-uniform in [1e-3, 1e-1]; the convolution front uniform
    in +-1/sqrt(3)."""
    import torch

    g = torch.Generator().manual_seed(seed)
    Di, N = w.channels, w.d_state
    Wx = (torch.randn((2, Di, 2 * N + 1), generator=g) / math.sqrt(Di)).to(torch.bfloat16).contiguous()
    Wdt = (torch.randn((2, Di), generator=g) * 0.5).contiguous()
    s = torch.exp(math.log(1e-3) + (math.log(1e-1) - math.log(1e-3)) * torch.rand((2, Di), generator=g,
                                                                                   dtype=torch.float64))
    dt_bias = torch.log(torch.expm1(s)).float().contiguous()
    k = 3 ** -0.5
    cw = ((torch.rand((2, Di, 3), generator=g) * 2 - 1) * k).contiguous()
    cb = ((torch.rand((2, Di), generator=g) * 2 - 1) * k).contiguous()
    return dict(Wx=Wx, Wdt=Wdt, dt_bias=dt_bias, conv_w=cw, conv_b=cb)


def algorithmic_bwd(w):
    """Algorithmic bytes and FP32 lane-ops of one derivative step (Vim with shared B/C,
    or the cross-scan with B/C per direction).

    Bytes: reads of u, delta_raw, z, dout and writes of du, d delta_raw, dz per
    token-channel; B, C read and dB, dC (fp32) written per token; parameters and
    their derivatives once.  Ops: 11 FP32 lane-ops per state per direction per
    token-channel -- the forward state update (decay multiply, Delta*B*u, FMA), the
    readout for dz, the dC term, and in the adjoint sweep the C*dy update, the decay
    multiply, the h_(t-1) product, the dA, A- and B-weighted sums and the dB term.
    """
    el = 4 if w.dtype == "f32" else 2
    n_bc_sets = 1 if w.kind == "vim" else w.directions
    bc = 2 * w.batch * w.tokens * w.d_state * (el + 4) * n_bc_sets
    params = 2 * w.directions * w.channels * (w.d_state + 2) * 4
    nbytes = 7 * w.tok_ch * el + bc + params
    ops = 11 * w.d_state * w.directions * w.tok_ch
    return nbytes, ops


def algorithmic(w, conv=False):
    """Algorithmic bytes and FP32 lane-ops of one step.

    Bytes: one read of u, delta_raw, z and one write of y per token-channel, one read
    of B and C per token (per direction when they are separate), the fp32 parameters
    once.  Ops: the recurrence core, 4 FP32 lane-ops per state per direction per
    token-channel (decay, Delta*B*u, the state update, the readout).
    """
    el = 4 if w.dtype == "f32" else 2
    n_bc_sets = 1 if w.kind == "vim" else w.directions
    bc = 2 * w.batch * w.tokens * w.d_state * el * n_bc_sets
    params = w.directions * w.channels * (w.d_state + 2 + (4 if conv else 0)) * 4
    nbytes = 4 * w.tok_ch * el + bc + params
    ops = 4 * w.d_state * w.directions * w.tok_ch
    return nbytes, ops


class ClockSampler:
    """NVML samples of the SM clock and the clock-event reasons, in a thread."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index, period=0.0005):
        self.ok = False
        try:
            import pynvml
            import torch

            pynvml.nvmlInit()
            self.nv = pynvml
            uuid = str(torch.cuda.get_device_properties(index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover
            self.err = repr(e)
        self.period = period
        self.samples, self.reasons = [], 0
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        med = statistics.median(self.samples) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


def conv_params(w, seed):
    """Depthwise kernel-3 weights [2, channels, 3] and biases [2, channels] of the two
    pathways' convolution front, uniform in +-1/sqrt(3) (a default Conv1d init)."""
    import torch

    g = torch.Generator().manual_seed(seed)
    k = 3 ** -0.5
    cw = (torch.rand((2, w.channels, 3), generator=g) * 2 - 1) * k
    cb = (torch.rand((2, w.channels), generator=g) * 2 - 1) * k
    return cw.contiguous(), cb.contiguous()


def run_oracle(w, x, threads, zoh=False):
    import oracle

    oracle.set_threads(threads)
    t = time.perf_counter()
    if "Wx" in x and "dout" in x:
        oracle.vim_block_scan_bwd(x["u"], x["Wx"], x["Wdt"], x["A"], x["D"], x["dt_bias"], x["z"], x["dout"],
                                  conv_w=x["conv_w"], conv_b=x["conv_b"])
    elif "Wx" in x:
        oracle.vim_block_scan(x["u"], x["Wx"], x["Wdt"], x["A"], x["D"], x["dt_bias"], x["z"],
                              conv_w=x["conv_w"], conv_b=x["conv_b"])
    elif "dout" in x and "conv_w" in x:
        oracle.vim_bidir_conv_bwd(x["u"], x["conv_w"], x["conv_b"], x["delta"], x["z"], x["B"], x["C"], x["A"],
                                  x["D"], x["delta_bias"], x["dout"], zoh=zoh)
    elif "dout" in x and w.kind == "vim":
        oracle.vim_bidir_bwd(x["u"], x["delta"], x["z"], x["B"], x["C"], x["A"], x["D"], x["delta_bias"], x["dout"],
                             zoh=zoh)
    elif "dout" in x:
        oracle.cross_scan4_bwd(x["u"], x["delta"], x["z"], x["B"], x["C"], x["A"], x["D"], x["delta_bias"], x["dout"],
                               zoh=zoh)
    elif "conv_w" in x:
        oracle.vim_bidir_conv(x["u"], x["conv_w"], x["conv_b"], x["delta"], x["z"], x["B"], x["C"], x["A"],
                              x["D"], x["delta_bias"], zoh=zoh)
    elif w.kind == "vim":
        oracle.vim_bidir(x["u"], x["delta"], x["z"], x["B"], x["C"], x["A"], x["D"], x["delta_bias"], zoh=zoh)
    else:
        oracle.cross_scan4(x["u"], x["delta"], x["z"], x["B"], x["C"], x["A"], x["D"], x["delta_bias"],
                           zoh=zoh)
    return time.perf_counter() - t


def bwd_dout(w, seed):
    """dout for the derivative runs: drawn like z, in the workload's dtype."""
    import torch

    g = torch.Generator().manual_seed(seed)
    return torch.randn((w.batch, w.tokens, w.channels), generator=g).to(w.torch_dtype()).contiguous()


CPU_SECONDS = 10.0   # host time the cpu_baseline leg spends on the oracle (about)


def oracle_sample(w, target_s, conv=False, bwd=False, block=False):
    """A bounded sample of the workload for the oracle: its first batch items and
    first channels at the full sequence length, sized for about ``target_s`` seconds
    of fp64 work on the host cores (calibrated on a small run)."""
    from vision_mamba_selective_b200 import workloads as wl

    cores = cpu_cores()
    full = wl.make_inputs(w)
    if bwd:
        full["dout"] = bwd_dout(w, w.seed + 2).reshape(full["u"].shape).contiguous()
    if block:
        full.update(block_params(w, w.seed + 3))
    if conv:
        full["conv_w"], full["conv_b"] = conv_params(w, w.seed + 1)
    step = 8

    def cut(b, c):
        x = {}
        for k, v in full.items():
            if k in ("u", "delta", "z", "dout"):
                x[k] = v[:b, ..., :c].contiguous()
            elif k in ("B", "C"):
                x[k] = (v[:b] if w.kind == "vim" else v[:, :b]).contiguous()
            elif k == "Wx":
                x[k] = v[:, :c, :].contiguous()
            else:
                x[k] = v[..., :c, :].contiguous() if k in ("A", "conv_w") else v[..., :c].contiguous()
        return w.scaled(batch=b, channels=c), x

    cal_c = min(w.channels, 64)
    s, x = cut(1, cal_c)
    t = max(run_oracle(s, x, cores), 1e-4)
    per = t / s.tok_ch
    want = max(1, int(target_s / per))                      # token-channels to process
    per_item = w.tokens * w.channels
    if want >= per_item:
        b, c = min(w.batch, want // per_item), w.channels
    else:
        b, c = 1, max(step, min(w.channels, (want // w.tokens) // step * step))
    return cut(b, c) + (cores,)


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def reference_arm(args, w):
    """The oracle, as it stands, on the host cores: K timed steps of a bounded sample."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    per_step = min(2.0, 150.0 / max(1, args.steps + args.warmup))
    s, x, cores = oracle_sample(w, per_step, conv=args.conv, bwd=args.bwd, block=args.block)
    for _ in range(args.warmup):
        run_oracle(s, x, cores, args.zoh)
    times = [run_oracle(s, x, cores, args.zoh) for _ in range(args.steps)]
    sec = sum(times) / len(times)
    value = s.tok_ch / sec
    sample = (f"{s.batch} of {w.batch} batch items x {s.channels} of {w.channels} channels at the full "
              f"{w.tokens} tokens ({s.tok_ch} token-channels) per step, fp64")
    line = {
        "impl": "reference", "metric": "bidirectional S6 scan token-channels/s at L=4097; achieved HBM GB/s vs peak",
        "value": value, "unit": "tok*ch/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_name(w, args), "batch_per_gpu": w.batch, "tokens": w.tokens,
                   "channels": w.channels, "d_state": w.d_state, "io_dtype": w.dtype},
        "cpu_baseline": {"value": value, "unit": "tok*ch/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tok*ch/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def time_forward(w, dev, steps, warmup=3):
    """Device time of the plain forward scan of workload ``w`` (its own seeded inputs,
    rotating copies larger than L2), with per-kernel times from the events entry
    point.  Returns the numbers one line of ``other_configs`` reports."""
    import torch

    from vision_mamba_selective_b200 import vimscan as vs
    from vision_mamba_selective_b200 import workloads as wl

    host = wl.make_inputs(w)
    keys = ["u", "delta", "z", "B", "C"]
    set_bytes = sum(host[k].numel() * host[k].element_size() for k in keys) + wl.output_bytes(w)
    nsets = max(2, math.ceil(2.2 * L2_BYTES / set_bytes))
    params = {k: host[k].to(dev) for k in ("A", "D", "delta_bias")}
    sets = []
    for _ in range(nsets):
        s = {k: host[k].to(dev) for k in keys}
        s["y"] = torch.empty_like(s["u"])
        sets.append(s)
    which = 0 if w.kind == "vim" else 1
    ws = torch.empty(max(1, vs.vim_scan_workspace_bytes(which, w.batch, w.L if w.kind == "vim" else w.H, w.W,
                                                          w.channels, w.d_state)), dtype=torch.uint8, device=dev)
    fn = vs.vim_scan_bidir if w.kind == "vim" else vs.vmamba_cross_scan4
    pairs = 1 if w.kind == "vim" else 2

    def step(i, events=None):
        s = sets[i % nsets]
        fn(s["u"], s["delta"], s["z"], s["B"], s["C"], params["A"], params["D"], params["delta_bias"], y=s["y"],
           workspace=ws, events=events)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(steps):
        step(i)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(1 + 3 * pairs)] for _ in range(steps)]
    for i in range(steps):
        step(i, evs[i])
    torch.cuda.synchronize()
    names = ["pair_carry", "pair_combine", "pair_main"]
    kernel_ms = {}
    for p in range(pairs):
        for k in range(3):
            a = 1 + 3 * p + k
            t = sum(evs[i][a - 1].elapsed_time(evs[i][a]) for i in range(steps)) / steps
            kernel_ms[f"{names[k]}[{p}]" if pairs > 1 else names[k]] = t
    nbytes, ops = algorithmic(w)
    pk = peaks()
    peak_ops = SMS * FP32_LANES_PER_SM * pk["sm_max_mhz"] * 1e6
    main_ms = sum(v for k, v in kernel_ms.items() if k.startswith("pair_main"))
    return {"ms_per_step": ms, "tok_ch_per_s": w.tok_ch / (ms * 1e-3),
            "hbm_frac_whole_step": nbytes / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
            "fp32_frac_pair_main": ops / (main_ms * 1e-3) / peak_ops,
            "fp32_frac_whole_step": ops / (ms * 1e-3) / peak_ops,
            "kernel_ms": kernel_ms, "steps": steps, "io_dtype": w.dtype,
            "shape": {"batch": w.batch, "tokens": w.tokens, "channels": w.channels, "d_state": w.d_state}}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def vs_ckpt_shape(w):
    """Shape of the forward pass's checkpoints for a workload."""
    from vision_mamba_selective_b200 import vimscan as vs

    if w.kind == "vim":
        return vs.ckpt_shape(w.batch, w.L, w.channels, w.d_state)
    return vs.cross_ckpt_shape(w.batch, w.H, w.W, w.channels, w.d_state)


def workload_name(w, args):
    return (w.name + ("+conv_front" if args.conv else "") + ("+zoh_exact" if args.zoh else "")
            + ("+derivative" if args.bwd else "") + ("+projections+conv_front" if args.block else "")
            + ("+checkpoints" if args.ckpt else ""))


def main():
    args = parse()
    from vision_mamba_selective_b200 import workloads as wl

    w = wl.BY_NAME[args.workload]
    if (args.conv or args.block) and w.kind != "vim":
        raise SystemExit("--conv and --block apply to the Vim workloads only")
    if args.block and (args.conv or args.zoh or w.dtype != "bf16"):
        raise SystemExit("--block runs alone (or with --bwd), on a bf16 workload")
    if args.bwd and args.conv and w.kind != "vim":
        raise SystemExit("--bwd --conv applies to the Vim workloads only")
    if args.ckpt and args.block:
        raise SystemExit("--ckpt applies to the scans (Vim with or without its front, the cross-scan), not the block")
    if args.impl == "reference":
        reference_arm(args, w)
        return

    import torch
    import torch.distributed as dist

    from vision_mamba_selective_b200 import replicas

    rank, local, world = replicas.env_rank_world()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        replicas.init("nccl", device=dev)

    from vision_mamba_selective_b200 import vimscan as vs

    # ---- inputs: rank-specific seed; enough rotating copies to exceed L2 ---------
    host = wl.make_inputs(w, seed=replicas.rank_seed(w.seed, rank))
    act_keys = ["u", "delta", "z", "B", "C"]
    el = 4 if w.dtype == "f32" else 2
    out_bytes = w.tok_ch * el
    if args.bwd:
        host["dout"] = bwd_dout(w, replicas.rank_seed(w.seed + 2, rank)).reshape(host["u"].shape).contiguous()
        act_keys.append("dout")
        out_bytes = 3 * w.tok_ch * el + 2 * w.batch * w.tokens * w.d_state * 4 * (1 if w.kind == "vim" else 4)
    ck_shape = vs_ckpt_shape(w) if args.ckpt else None
    set_bytes = sum(host[k].numel() * host[k].element_size() for k in act_keys) + out_bytes
    nsets = max(2, math.ceil(2.2 * L2_BYTES / set_bytes))
    params = {k: host[k].to(dev) for k in ("A", "D", "delta_bias")}
    sets = []
    for _ in range(nsets):
        s = {k: host[k].to(dev) for k in act_keys}
        s["y"] = torch.empty_like(s["u"])
        if args.ckpt:
            s["ck"] = torch.empty(ck_shape, dtype=torch.float32, device=dev)
        if args.bwd:
            f32 = lambda *shape: torch.empty(shape, dtype=torch.float32, device=dev)
            s["out"] = dict(du=torch.empty_like(s["u"]), ddelta=torch.empty_like(s["u"]), dz=torch.empty_like(s["u"]),
                            dB=f32(*s["B"].shape), dC=f32(*s["C"].shape), dA=f32(w.directions, w.channels, w.d_state),
                            dD=f32(w.directions, w.channels), ddelta_bias=f32(w.directions, w.channels))
            if args.conv:   # x's derivative in place of u's, and the fronts' parameters
                s["out"]["dx"] = s["out"].pop("du")
                s["out"]["dconv_w"] = f32(2, w.channels, 3)
                s["out"]["dconv_b"] = f32(2, w.channels)
            if args.block:  # the block's parameters: projections, fronts, A, D
                s["out"] = dict(dx=torch.empty_like(s["u"]), dz=torch.empty_like(s["u"]),
                                dWx=f32(2, w.channels, 2 * w.d_state + 1), dWdt=f32(2, w.channels),
                                ddt_bias=f32(2, w.channels), dA=f32(2, w.channels, w.d_state), dD=f32(2, w.channels),
                                dconv_w=f32(2, w.channels, 3), dconv_b=f32(2, w.channels))
        sets.append(s)
    if w.kind == "vim":
        ws_bytes = vs.vim_scan_workspace_bytes(0, w.batch, w.L, 0, w.channels, w.d_state)
    else:
        ws_bytes = vs.vim_scan_workspace_bytes(1, w.batch, w.H, w.W, w.channels, w.d_state)
    if args.bwd and w.kind == "vim":
        ws_bytes = vs.vim_scan_bwd_workspace_bytes(w.batch, w.L, w.channels, w.d_state, False)
        if args.conv:
            ws_bytes = vs.vim_scan_conv_bwd_workspace_bytes(w.batch, w.L, w.channels, w.d_state,
                                                            vs.VIM_F32 if w.dtype == "f32" else vs.VIM_BF16, False)
    elif args.bwd:
        ws_bytes = int(vs.lib.vmamba_cross_scan4_bwd_workspace_bytes(w.batch, w.H, w.W, w.channels, w.d_state))
    if args.block:
        ws_bytes = vs.vim_block_workspace_bytes(w.batch, w.L, w.channels, w.d_state)
        if args.bwd:
            ws_bytes = vs.vim_block_bwd_workspace_bytes(w.batch, w.L, w.channels, w.d_state)
        blk = block_params(w, w.seed + 3)
        params.update({k: v.to(dev) for k, v in blk.items()})
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    fn = vs.vim_scan_bidir if w.kind == "vim" else vs.vmamba_cross_scan4
    if args.conv:
        cw, cb = conv_params(w, w.seed + 1)
        params["conv_w"], params["conv_b"] = cw.to(dev), cb.to(dev)

    def step(i, events=None):
        s = sets[i % nsets]
        if args.block and args.bwd:
            vs.vim_block_scan_bwd(s["u"], params["Wx"], params["Wdt"], params["dt_bias"], params["A"], params["D"],
                                  s["z"], s["dout"], conv_w=params["conv_w"], conv_b=params["conv_b"], workspace=ws,
                                  out=s["out"])
            return
        if args.block:
            # u holds x, the block's input; B, C and delta come from the projections
            vs.vim_block_scan(s["u"], params["Wx"], params["Wdt"], params["dt_bias"], params["A"], params["D"],
                              s["z"], conv_w=params["conv_w"], conv_b=params["conv_b"], y=s["y"], workspace=ws,
                              events=events)
            return
        if args.bwd and args.conv:
            # u holds x; the derivative through the pathways' convolution fronts
            vs.vim_scan_bidir_conv_bwd(s["u"], params["conv_w"], params["conv_b"], s["delta"], s["z"], s["B"], s["C"],
                                       params["A"], params["D"], params["delta_bias"], s["dout"], workspace=ws,
                                       out=s["out"], zoh=args.zoh, ckpt=s["ck"] if args.ckpt else None)
            return
        if args.bwd and w.kind == "vim":
            vs.vim_scan_bidir_bwd(s["u"], s["delta"], s["z"], s["B"], s["C"], params["A"], params["D"],
                                  params["delta_bias"], s["dout"], workspace=ws, out=s["out"], events=events,
                                  zoh=args.zoh, ckpt=s["ck"] if args.ckpt else None)
            return
        if args.bwd:
            vs.vmamba_cross_scan4_bwd(s["u"], s["delta"], s["z"], s["B"], s["C"], params["A"], params["D"],
                                      params["delta_bias"], s["dout"], workspace=ws, out=s["out"], zoh=args.zoh,
                                      ckpt=s["ck"] if args.ckpt else None)
            return
        if args.conv:
            # u holds x, the pathways' common input in front of the convolutions
            vs.vim_scan_bidir_conv(s["u"], params["conv_w"], params["conv_b"], s["delta"], s["z"], s["B"],
                                   s["C"], params["A"], params["D"], params["delta_bias"], y=s["y"],
                                   workspace=fws if args.ckpt else ws, events=events, zoh=args.zoh,
                                   ckpt=s["ck"] if args.ckpt else None)
            return
        if args.ckpt:
            fn(s["u"], s["delta"], s["z"], s["B"], s["C"], params["A"], params["D"], params["delta_bias"],
               y=s["y"], workspace=fws, events=events, zoh=args.zoh, ckpt=s["ck"])
            return
        fn(s["u"], s["delta"], s["z"], s["B"], s["C"], params["A"], params["D"], params["delta_bias"],
           y=s["y"], workspace=ws, events=events, zoh=args.zoh)

    if args.ckpt:
        # the forward scan's workspace, and with --bwd the states each input set's forward
        # pass leaves (inputs of the derivative, formed before any timing)
        fws_bytes = (vs.vim_scan_workspace_bytes(0, w.batch, w.L, 0, w.channels, w.d_state) if w.kind == "vim"
                     else vs.vim_scan_workspace_bytes(1, w.batch, w.H, w.W, w.channels, w.d_state))
        fws = torch.empty(max(fws_bytes, 1), dtype=torch.uint8, device=dev)
        if args.bwd:
            for s in sets:
                if args.conv:
                    vs.vim_scan_bidir_conv(s["u"], params["conv_w"], params["conv_b"], s["delta"], s["z"], s["B"],
                                           s["C"], params["A"], params["D"], params["delta_bias"], y=s["y"],
                                           workspace=fws, zoh=args.zoh, ckpt=s["ck"])
                else:
                    fn(s["u"], s["delta"], s["z"], s["B"], s["C"], params["A"], params["D"], params["delta_bias"],
                       y=s["y"], workspace=fws, zoh=args.zoh, ckpt=s["ck"])
            torch.cuda.synchronize()

    barrier = replicas.barrier

    def max_over_ranks(v):
        return replicas.max_over_ranks(v, device=dev)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    # ---- timed region -----------------------------------------------------------
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start.record()
        for i in range(args.steps):
            step(i)
        end.record()
        torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(start.elapsed_time(end))
    ms_step = ms / args.steps
    value = world * w.tok_ch * args.steps / (ms * 1e-3)

    # ---- per-kernel times (same launches plus event records), after the timed region
    kernels_per_pair = 3
    pairs = 1 if w.kind == "vim" else 2
    nev = 4 if args.bwd else (5 if args.block else 1 + kernels_per_pair * pairs)
    whole_call = args.bwd and (w.kind != "vim" or args.conv or args.block)
    if whole_call:
        nev = 2       # the cross-scan's and the front's derivatives have no per-phase events:
                      # the whole call is timed
    prof_steps = min(args.steps, 200)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(prof_steps)]
    for i in range(prof_steps):
        step(i, events=evs[i])
    torch.cuda.synchronize()
    per_kernel = {}
    if args.block and not args.bwd:
        for a, name in enumerate(["xproj", "pair_carry", "pair_combine", "pair_main"], start=1):
            t = [evs[i][a - 1].elapsed_time(evs[i][a]) for i in range(prof_steps)]
            per_kernel[name] = sum(t) / len(t)
        launches_per_step = 1 + (3 if w.tokens > 256 else 1)
    elif whole_call:
        t = []
        for i in range(prof_steps):
            e0, e1 = evs[i]
            e0.record()
            step(i)
            e1.record()
        torch.cuda.synchronize()
        t = [evs[i][0].elapsed_time(evs[i][1]) for i in range(prof_steps)]
        if args.block:
            per_kernel["vim_block_scan_bwd"] = sum(t) / len(t)
            # the projection, the fronts, pair_carry, pair_combine, adj_carry, pair_combine,
            # bwd_main, four dB/dC reductions, two column sums for the parameters; dl/ds,
            # two for dWdt, dl/du and dWx partials, two for dWx; the fronts' derivative and
            # two column sums
            launches_per_step = 2 + (4 if w.tokens > 32 else 0) + 1 + 4 + 2 + 1 + 2 + 1 + 2 + 1 + 2
        elif args.conv:
            per_kernel["vim_scan_bidir_conv_bwd"] = sum(t) / len(t)
            # the fronts' forward kernel, pair_carry, pair_combine, adj_carry, pair_combine,
            # bwd_main, two dB/dC reductions, two column sums for the parameters, the
            # fronts' derivative and two column sums for their taps and biases
            launches_per_step = 1 + ((2 if args.ckpt else 4) if w.tokens > 32 else 0) + 1 + 2 + 2 + 1 + 2
        else:
            per_kernel["vmamba_cross_scan4_bwd"] = sum(t) / len(t)
            # per pair: pair_carry, pair_combine, adj_carry, pair_combine, bwd_main, four
            # dB/dC reductions, one two-pass column sum
            launches_per_step = 2 * (((2 if args.ckpt else 4) if w.tokens > 32 else 0) + 1 + 4 + 2)
    elif args.bwd:
        for a, name in enumerate(["summaries", "bwd_main", "reductions"], start=1):
            t = [evs[i][a - 1].elapsed_time(evs[i][a]) for i in range(prof_steps)]
            per_kernel[name] = sum(t) / len(t)
        # pair_carry, pair_combine (not with the forward's checkpoints), adj_carry,
        # pair_combine (more than one chunk of 32 tokens), bwd_main, two dB/dC reductions,
        # one two-pass column sum
        launches_per_step = ((2 if args.ckpt else 4) if w.tokens > 32 else 0) + 1 + 2 + 2
    else:
        names = ["pair_carry", "pair_combine", "pair_main"]
        for p in range(pairs):
            for k in range(kernels_per_pair):
                a = 1 + 3 * p + k
                t = [evs[i][a - 1].elapsed_time(evs[i][a]) for i in range(prof_steps)]
                per_kernel[f"{names[k]}[{p}]" if pairs > 1 else names[k]] = sum(t) / len(t)
        # sequences longer than one chunk (256 tokens) take carry, combine and main
        launches_per_step = pairs * (3 if w.tokens > 256 else 1)

    # ---- end to end: pinned host inputs -> device -> scan -> host result ---------
    if args.ckpt and args.bwd:
        host["ck"] = sets[0]["ck"].cpu()
        act_keys.append("ck")
    pinned = {k: host[k].pin_memory() for k in act_keys}
    if args.bwd:
        keys = ("dx", "dz", "dWx") if args.block else ("dx" if args.conv else "du", "ddelta", "dz", "dB", "dC")
        res_dev = [sets[0]["out"][k] for k in keys]
    else:
        res_dev = [sets[0]["y"]]
    res_host = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in res_dev]
    h2d = sum(pinned[k].numel() * pinned[k].element_size() for k in act_keys)
    d2h = sum(t.numel() * t.element_size() for t in res_host)

    def fetch():
        for hst, dv in zip(res_host, res_dev):
            hst.copy_(dv, non_blocking=True)

    # the Vim forward scan has a host-memory entry point, which pipelines the copies of
    # batch pieces with their scans; the other modes copy everything, run, copy back
    host_entry = w.kind == "vim" and not (args.bwd or args.block or args.conv or args.ckpt)
    if host_entry:
        slices = max(1, min(args.e2e_slices, w.batch))
        hws = torch.empty(max(vs.vim_scan_host_workspace_bytes(w.batch, w.L, w.channels, w.d_state,
                                                              vs.VIM_F32 if w.dtype == "f32" else vs.VIM_BF16,
                                                              slices, False), 1), dtype=torch.uint8, device=dev)
        e2e_method = (f"vim_scan_bidir_host: host inputs and output, the batch in {slices} pieces whose "
                      "uploads, scans and downloads overlap on three streams")

        def e2e_step():
            vs.vim_scan_bidir_host(pinned["u"], pinned["delta"], pinned["z"], pinned["B"], pinned["C"],
                                   params["A"], params["D"], params["delta_bias"], y=res_host[0], slices=slices,
                                   workspace=hws, zoh=args.zoh)
    else:
        e2e_method = "pinned inputs copied in, the step, the result copied out, on one stream"

        def e2e_step():
            for k in act_keys:
                sets[0][k].copy_(pinned[k], non_blocking=True)
            step(0)
            fetch()
    e2e_steps = min(args.steps, 50)
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(e2e_steps):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1))
    e2e_value = world * w.tok_ch * e2e_steps / (e2e_ms * 1e-3)

    # ---- roofline of the dominant kernel -----------------------------------------
    pk = peaks()
    nbytes, ops = algorithmic_bwd(w) if args.bwd else algorithmic(w, args.conv)
    if args.ckpt:   # the checkpoints: written by the forward pass, read by the derivative
        nbytes += math.prod(vs_ckpt_shape(w)) * 4
    main_name = "bwd_main" if args.bwd else "pair_main"
    if whole_call:
        main_name = ("vim_block_scan_bwd" if args.block else "vim_scan_bidir_conv_bwd" if args.conv
                     else "vmamba_cross_scan4_bwd")   # the whole call
    main_ms = sum(v for k, v in per_kernel.items() if k.startswith(main_name))
    clocks = clk.summary()
    peak_ops = SMS * FP32_LANES_PER_SM * pk["sm_max_mhz"] * 1e6 / 1e12
    achieved_ops = ops / (main_ms * 1e-3) / 1e12
    if whole_call or args.block:
        traffic = None
    elif args.bwd:
        traffic = profiled_traffic(w, bwd=True, zoh=args.zoh)
    elif args.ckpt:
        traffic = None   # no capture of the forward kernel writing checkpoints
    else:
        traffic = profiled_traffic(w, zoh=args.zoh, conv=args.conv)
    roofline = {
        "bound": "alu", "kernel": main_name, "achieved": achieved_ops, "peak": peak_ops,
        "unit": "Tops/s", "frac": achieved_ops / peak_ops,
        "traffic": traffic,
        "traffic_source": ("ncu capture committed under profiles/ (same kernel source fingerprint), not "
                           "measured in this run" if traffic is not None else None),
        "algorithmic_bytes": nbytes,
        "ops_per_launch": ops, "ms_per_launch": main_ms,
        "peak_basis": f"{SMS} SMs x {FP32_LANES_PER_SM} FP32 lanes x {pk['sm_max_mhz']:.0f} MHz",
        "hbm_gbs_whole_step": nbytes / (ms_step * 1e-3) / 1e9,
        "hbm_frac_whole_step": nbytes / (ms_step * 1e-3) / 1e9 / pk["hbm_gbs"],
        "hbm_peak_gbs": pk["hbm_gbs"], "peak_source": pk["source"],
    }

    projection = None
    if args.block and not args.bwd:
        # x_proj: x read once; B and C (bf16), the step input (fp32) and u (bf16, for the
        # scan) written per pathway
        M = w.batch * w.tokens
        pb = (M * w.channels * 2 + 2 * (2 * M * w.d_state * 2 + M * 4 + M * w.channels * 2)
              + 2 * w.channels * (2 * w.d_state + 1) * 2)
        pms = per_kernel["xproj"]
        projection = {"kernel": "xproj_kernel", "bound": "hbm", "ms_per_launch": pms, "algorithmic_bytes": pb,
                      "achieved_gbs": pb / (pms * 1e-3) / 1e9, "peak_gbs": pk["hbm_gbs"],
                      "frac": pb / (pms * 1e-3) / 1e9 / pk["hbm_gbs"]}

    # ---- the other workloads of the target (forward scan only), timed the same way ---
    others = None
    if not (args.no_other_configs or args.bwd or args.conv or args.zoh or args.block):
        others = {}
        for ow in wl.WORKLOADS:
            if ow.name == w.name:
                continue
            others[ow.name] = time_forward(ow, dev, steps=max(10, min(args.steps, 50)))
            torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        s, x, cores = oracle_sample(w, CPU_SECONDS, conv=args.conv, bwd=args.bwd, block=args.block)
        # a sample that is the whole workload may finish in well under the target: run it
        # again until the target is reached, and report the mean rate
        sec, runs = 0.0, 0
        while runs == 0 or sec < CPU_SECONDS:
            sec += run_oracle(s, x, cores, args.zoh)
            runs += 1
        # the same oracle on one host thread, on a sample of about a quarter of the time
        s1, x1, _ = oracle_sample(w, CPU_SECONDS / 4 / max(1, cores) * 1.0, conv=args.conv, bwd=args.bwd,
                                  block=args.block)
        sec1, runs1 = 0.0, 0
        while runs1 == 0 or sec1 < CPU_SECONDS / 4:
            sec1 += run_oracle(s1, x1, 1, args.zoh)
            runs1 += 1
        cpu = {"value": runs * s.tok_ch / sec, "unit": "tok*ch/s", "cores": cores, "kind": "oracle",
               "cpu_model": cpu_model(),
               "sample": f"{s.batch} of {w.batch} batch items x {s.channels} of {w.channels} channels "
                         f"at the full {w.tokens} tokens ({s.tok_ch} token-channels), {runs} run(s), "
                         f"fp64, {sec:.2f} s",
               "single_thread": {"value": runs1 * s1.tok_ch / sec1, "unit": "tok*ch/s", "cores": 1,
                                 "sample": f"{s1.batch} batch items x {s1.channels} channels at the full "
                                           f"{w.tokens} tokens, {runs1} run(s), fp64, {sec1:.2f} s"}}

    if rank == 0:
        line = {
            "metric": "bidirectional S6 scan token-channels/s at L=4097; achieved HBM GB/s vs peak",
            "value": value, "unit": "tok*ch/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded, shaped like the pages' workloads)",
            "config": {"workload": workload_name(w, args), "batch_per_gpu": w.batch, "tokens": w.tokens,
                       "channels": w.channels, "d_state": w.d_state, "io_dtype": w.dtype,
                       "parallelism": f"replicas x{world} (batch shards, no collective)",
                       "l2": f"{nsets} rotating input sets of {set_bytes / 1e6:.0f} MB each, "
                             f"{nsets * set_bytes / 1e6:.0f} MB in all (L2: {L2_BYTES / 1e6:.0f} MB): each step "
                             f"reads a set written {nsets - 1} steps earlier"},
            "hbm_gbs": roofline["hbm_gbs_whole_step"], "hbm_frac": roofline["hbm_frac_whole_step"],
            "kernel_ms": per_kernel,
            "roofline": roofline,
            "projection": projection,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "tok*ch/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps, "method": e2e_method},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
            "other_configs": others,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

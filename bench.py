#!/usr/bin/env python
"""Throughput benchmark of RIB window attention on B200.

One step = the whole hot path over one batch of the 96x96-window training
workload (B=4, 192x192 map, 6 heads, d=32, rank 16, shift 48, MLP
64->128->96): position tokens -> forward -> backward with position-MLP
gradients (+ an all-reduce of those gradients across ranks when N > 1).
Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl rib|reference]

--gpus N runs N ranks, one per GPU: under an outer torchrun launch WORLD_SIZE
must equal N; without one, N > 1 re-launches this script under
torch.distributed.run with N processes on this node.

--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload on this host's cores (rank 0 only).

Roofline fractions divide by the measured burst bf16 peak: the timed loops
are a fraction of a second long and the sampled SM clock stays at its
maximum, so the seconds-long, power-capped sustained figure does not apply.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "RIB window-attention TFLOP/s and tokens/s (fwd, fwd+bwd) at 96×96 windows"
D_QK, D_V = 48, 32


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="rib", choices=["rib", "reference"])
    ap.add_argument("--workload", default="w96train")
    ap.add_argument("--bwd-kernel", default="auto", choices=["auto", "per_item", "persistent"],
                    help="form of the attention backward kernel (default: by window size)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the table of every workload definition")
    ap.add_argument("--step-only", action="store_true",
                    help="run only warm-up + timed training steps (for profiler launch lists)")
    ap.add_argument("--cla-only", action="store_true",
                    help="run only the convolutional local attention gate and the gated "
                         "forward, warm-up + timed (for profiler captures)")
    return ap.parse_args()


def world_plan(gpus: int, env=None):
    """What to do with --gpus N given the launcher's environment.

    Returns "run" (the ranks are in place), "relaunch" (no outer launcher and
    N > 1: start N ranks under torch.distributed.run) or raises ValueError
    when an outer launcher started a different number of ranks than N."""
    env = os.environ if env is None else env
    if gpus < 1:
        raise ValueError(f"--gpus must be >= 1, got {gpus}")
    ws = env.get("WORLD_SIZE")
    if ws is None:
        return "relaunch" if gpus > 1 else "run"
    if int(ws) != gpus:
        raise ValueError(f"--gpus {gpus} but the launcher started WORLD_SIZE={ws} ranks")
    return "run"


def relaunch_cmd(gpus: int, argv, port: int):
    """torch.distributed.run command that starts `gpus` ranks of this script
    on this node (rendezvous on 127.0.0.1)."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={gpus}", "--master-addr", "127.0.0.1",
            "--master-port", str(port), os.path.abspath(__file__)] + list(argv)


def free_port() -> int:
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def max_over_ranks(value: float, device) -> float:
    """The largest of every rank's value (all ranks must call it)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def bench_config(w, world: int):
    """The `config` object of the bench line, the same for both arms."""
    return {"workload": workload_desc(w), "global_batch": w.batch * world,
            "map": [w.height, w.width], "window": w.windows[0], "shift": w.shifts[0],
            "heads": w.heads, "head_dim": w.head_dim, "rank": w.rank,
            "parallelism": f"dp{world}",
            "l2": "inputs larger than L2 (qkv 170 MB + dout 57 MB per rank)"
                  if w.name == "w96train" else "per-step inputs as generated"}


def roofline_entry(kernel, flop_per_launch, avg_ms, pk, traffic=None):
    """Achieved algorithmic TFLOP/s of one launch against the measured burst
    bf16 peak."""
    ach = flop_per_launch / (avg_ms * 1e-3) / 1e12
    return {"kernel": kernel, "bound": "tensor", "achieved": ach, "peak": pk["bf16_tflops"],
            "unit": "TFLOP/s", "frac": ach / pk["bf16_tflops"], "traffic": traffic,
            "flop_per_launch": flop_per_launch, "avg_ms": avg_ms,
            "frac_of_sustained": ach / pk["bf16_tflops_sustained"],
            "peak_source": f"{pk['source']} bf16_tflops (burst)"}


def flops(w, layer=0):
    """Algorithmic FLOPs of one layer: fwd 2N^2(d_qk+d_v), bwd 2N^2(3d_qk+2d_v)
    per (batch, window, head) unit (the backward counts the score recompute)."""
    M = w.windows[layer]
    N = M * M
    units = w.units(layer)
    return units * 2.0 * N * N * (D_QK + D_V), units * 2.0 * N * N * (3 * D_QK + 2 * D_V)


def workload_desc(w):
    return (f"{w.name}: B={w.batch} {w.height}x{w.width} map, {w.windows[0]}x{w.windows[0]} windows, "
            f"shift {w.shifts[0]}, {w.heads} heads, d={w.head_dim}, rank {w.rank}, "
            f"MLP {4 * w.n_freq}->{w.hidden}->{w.heads * w.rank}, fwd+bwd with MLP grads")


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons every 200 ms."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_id: str):
        self.device_id = device_id
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.device_id, f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons, pw = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                mx.append(float(f[1]))
                pw.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "power_w_max": max(pw) if pw else None, "reasons": sorted(reasons)}


# ---------------------------------------------------------------- peaks

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# The source files a kernel is built from: its own header, the headers it
# includes and the host file that launches it (grid, shared memory, tensor
# maps).  A kernel not listed depends on every source.
KERNEL_SOURCES = {
    "attn_fwd_kernel": ("attn_fwd.cuh", "geom.cuh", "ptx.cuh", "rib.cu"),
    "attn_bwd_kernel": ("attn_bwd.cuh", "geom.cuh", "ptx.cuh", "rib.cu"),
    "cla_gate_kernel": ("cla.cuh", "ptx.cuh", "rib.cu"),
}


def kernel_source_hash(kernel=None):
    """Hash of the sources of `kernel` (all kernel sources when it is None or
    not listed), to tell whether stored ncu counters still describe the
    kernel being timed."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "windowed_attention_implicit_b200", "csrc")
    names = KERNEL_SOURCES.get(kernel)
    if names is None:
        names = [f for f in os.listdir(csrc) if f.endswith((".cu", ".cuh"))]
    for f in sorted(names):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def stored_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if it still
    matches the current sources of the kernel; else None."""
    p = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("source_hash") != kernel_source_hash(kernel):
        return None
    return d.get("dram_bytes_per_launch")


def config_sweep(I, R, dev, rank, world, timed, steps, warmup, peak, pk):
    """Every workload definition through the public API: the forward of all
    its layers (position tokens cached per geometry) and, for the training
    ones, the training step (position tokens, forward, backward with the MLP
    gradients, per layer).  Algorithmic FLOPs: 160 N^2 (fwd) and 416 N^2 (bwd)
    per unit; tokens = B*H*W per layer."""
    import torch
    from windowed_attention_implicit_b200.schedule import LayerSpec, RIBLayerStack
    res = {}
    for name in ("tiny", "w32", "cyclic", "w96train", "w96infer"):
        w0 = I.get_workload(name)
        w = I.get_workload(name, seed=w0.seed + 7919 * rank)
        layers = []
        for l in range(w.layers):
            inp = I.make_layer_inputs(w, l, with_dout=w.backward)
            mlp = R.PositionMLP.from_params(inp["freqs"], inp["mlp_q"], inp["mlp_k"], w.heads,
                                            w.rank, device=dev)
            layers.append((inp["qkv"].to(dev), inp["dout"].to(dev) if w.backward else None, mlp))
        if w.shared_mlp:
            layers = [(q, g, layers[0][2]) for q, g, _ in layers]
        specs = [LayerSpec(w.windows[l], w.shifts[l], layers[l][2]) for l in range(w.layers)]
        stack = RIBLayerStack(specs)
        qkvs = [q for q, _, _ in layers]
        f_fwd = sum(160.0 * (w.windows[l] ** 2) ** 2 * w.units(l) for l in range(w.layers))
        f_bwd = sum(416.0 * (w.windows[l] ** 2) ** 2 * w.units(l) for l in range(w.layers))
        tok = w.layers * w.tokens()

        def fwd_pass():
            stack.forward(qkvs)

        for _ in range(warmup):
            fwd_pass()
        ms_f, kern_f, _ = timed(fwd_pass, steps, trace=True)
        ms_f /= steps
        line = {"layers": w.layers, "windows": list(w.windows), "shifts": list(w.shifts),
                "map": [w.batch, w.height, w.width], "heads": w.heads,
                "fwd_ms": ms_f, "fwd_tflops": world * f_fwd / (ms_f * 1e-3) / 1e12,
                "fwd_tokens_per_s": world * tok / (ms_f * 1e-3),
                "fwd_frac": f_fwd / (ms_f * 1e-3) / 1e12 / peak}
        if w.backward:
            ws = {}

            def train_step():
                for l, (qkv, dout, mlp) in enumerate(layers):
                    M, sh = w.windows[l], w.shifts[l]
                    _, _, q16, k16 = R.rib_pos_tokens(mlp, M)
                    out, lse = R.rib_window_attn_fwd(qkv, M, sh, q16, k16)
                    if l not in ws:
                        ws[l] = torch.empty(max(R.rib_window_attn_bwd_workspace(
                            w.batch, w.height, w.width, w.heads, w.head_dim, M, w.rank,
                            mlp if w.mlp_grads else None), 256), device=dev, dtype=torch.uint8)
                    R.rib_window_attn_bwd(qkv, out, dout, lse, M, sh, q16, k16,
                                          mlp=mlp if w.mlp_grads else None, workspace=ws[l])

            for _ in range(warmup):
                train_step()
            ms_t, _, _ = timed(train_step, steps)
            ms_t /= steps
            line.update({"step_ms": ms_t,
                         "step_tflops": world * (f_fwd + f_bwd) / (ms_t * 1e-3) / 1e12,
                         "step_tokens_per_s": world * tok / (ms_t * 1e-3),
                         "step_frac": (f_fwd + f_bwd) / (ms_t * 1e-3) / 1e12 / peak})
            # the same step captured once in a CUDA graph and replayed: the
            # entry points only enqueue on the current stream, so the whole
            # step (every layer's position tokens, forward and backward) is
            # one graph launch, without the per-call host and launch costs
            try:
                side = torch.cuda.Stream()
                side.wait_stream(torch.cuda.current_stream())
                with torch.cuda.stream(side):
                    train_step()
                torch.cuda.current_stream().wait_stream(side)
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph):
                    train_step()
            except RuntimeError as e:   # reported, never fatal to the bench line
                line["step_graph_error"] = str(e).splitlines()[0][:200]
            else:
                for _ in range(warmup):
                    graph.replay()
                ms_g, _, _ = timed(graph.replay, steps)
                ms_g /= steps
                line.update({"step_graph_ms": ms_g,
                             "step_graph_tflops": world * (f_fwd + f_bwd) / (ms_g * 1e-3) / 1e12})
                del graph
        # bytes of one forward (qkv read, out written, lse written) against HBM
        byt = w.layers * w.tokens() * w.heads * (3 * 64 + 64 + 4)
        line["fwd_gbs"] = byt / (ms_f * 1e-3) / 1e9
        line["fwd_frac_hbm"] = line["fwd_gbs"] / pk["hbm_gbs"]
        res[name] = line
        del layers, qkvs, stack
        torch.cuda.empty_cache()
    # the tiny workload as stated, in fp32: its forward on the tf32 path
    w = I.get_workload("tiny", seed=I.get_workload("tiny").seed + 7919 * rank)
    inp = I.make_layer_inputs(w, 0, qkv_dtype=torch.float32)
    mlp = R.PositionMLP.from_params(inp["freqs"], inp["mlp_q"], inp["mlp_k"], w.heads, w.rank,
                                    device=dev)
    M, sh = w.windows[0], w.shifts[0]
    qkv32 = inp["qkv"].to(dev)
    qp32, kp32, _, _ = R.rib_pos_tokens(mlp, M)
    out32 = torch.empty((w.batch, w.height, w.width, w.heads, w.head_dim), device=dev)
    lse32 = torch.empty((w.batch, w.heads, w.height, w.width), device=dev)

    def fwd32():
        R.rib_window_attn_fwd_tf32(qkv32, M, sh, qp32, kp32, out=out32, lse=lse32)

    for _ in range(warmup):
        fwd32()
    ms32, kern32, _ = timed(fwd32, steps, trace=True)
    ms32 /= steps
    f32 = 160.0 * (M * M) ** 2 * w.units(0)
    k32 = kern32.get("attn_fwd_tf32_kernel", (1, ms32 * steps))
    res["tiny_fp32"] = {"layers": 1, "windows": [M], "shifts": [sh],
                        "map": [w.batch, w.height, w.width], "heads": w.heads,
                        "precision": "fp32 inputs, tf32 tensor cores (kind::tf32), fp32 out",
                        "fwd_ms": ms32, "fwd_tflops": world * f32 / (ms32 * 1e-3) / 1e12,
                        "fwd_tokens_per_s": world * w.tokens() / (ms32 * 1e-3),
                        "fwd_kernel_ms": k32[1] / k32[0]}
    return res


def infer_line(wi, ms_pass, kern, steps, world, peak):
    """The 12-layer forward pass of the large-image inference workload."""
    M = wi.windows[0]
    N = M * M
    units = wi.batch * (wi.height // M) * (wi.width // M) * wi.heads
    f_layer = 160.0 * N * N * units
    fwd = kern.get("attn_fwd_kernel", (1, 0.0))
    k_ms = fwd[1] / max(fwd[0], 1)
    return {"workload": f"{wi.name}: B={wi.batch} {wi.height}x{wi.width} map, {M}x{M} windows, "
                        f"{wi.layers} layers, shifts {'/'.join(str(x) for x in wi.shifts[:2])}, "
                        "forward only, Qp/Kp computed once and reused",
            "ms_per_pass": ms_pass,
            "tflops": world * wi.layers * f_layer / (ms_pass * 1e-3) / 1e12,
            "tokens_per_s": world * wi.layers * wi.batch * wi.height * wi.width / (ms_pass * 1e-3),
            "fwd_kernel_ms": k_ms,
            "fwd_kernel_frac": f_layer / (k_ms * 1e-3) / 1e12 / peak if k_ms else None,
            "pos_tokens_launches_per_pass": kern.get("pos_tokens_kernel", (0, 0.0))[0] / steps}


def copy_line(kern_ga, kern_sc, x_map, pk):
    """rib_window_gather / rib_window_scatter of the qkv map: each call reads
    and writes the whole map once (bf16), against the measured HBM copy."""
    byt = 2 * x_map.numel() * x_map.element_size()
    ga = kern_ga["window_copy_kernel"]
    sc = kern_sc["window_copy_kernel"]
    g_ms, s_ms = ga[1] / ga[0], sc[1] / sc[0]
    return {"kernel": "window_copy_kernel", "bound": "hbm", "bytes_per_call": byt,
            "gather_ms": g_ms, "scatter_ms": s_ms,
            "gather_gbs": byt / (g_ms * 1e-3) / 1e9, "scatter_gbs": byt / (s_ms * 1e-3) / 1e9,
            "gather_frac_hbm": byt / (g_ms * 1e-3) / 1e9 / pk["hbm_gbs"],
            "scatter_frac_hbm": byt / (s_ms * 1e-3) / 1e9 / pk["hbm_gbs"],
            "map": list(x_map.shape)}


def pos_line(w, per_kernel, pk):
    """The position-token kernel inside the step: both MLPs over the M*M
    window tokens.  FMA-bound: FLOPs of the two Linear layers per token and
    MLP, against the fp32 FMA rate of 148 SMs x 128 lanes x 2 at the measured
    clock; bytes written (Qp, Kp in fp32 and bf16) as its HBM figure."""
    k = per_kernel.get("pos_tokens_kernel")
    if k is None:
        return None
    N = w.windows[0] ** 2
    din, out = 4 * w.n_freq, w.heads * w.rank
    flops = 2 * N * 2 * (din * w.hidden + w.hidden * out)
    byt = 2 * N * out * (4 + 2)
    t = k["avg_ms"] * 1e-3
    fma_peak = 148 * 128 * 2 * 1.965e9 / 1e12
    return {"kernel_ms": k["avg_ms"], "bound": "fma", "flops": flops,
            "tflops_fp32": flops / t / 1e12, "fma_peak_tflops": fma_peak,
            "frac_fma": flops / t / 1e12 / fma_peak, "bytes_written": byt,
            "gbs": byt / t / 1e9}


def mask_line(w, ms_step, kern, f_fwd, f_bwd, peak):
    """The training step with the shifted-window region mask (an optional
    variant): its time and the two attention kernels' rates, counted with the
    unmasked step's FLOPs (masked pairs still pass through the MMAs)."""
    per = {k: v[1] / v[0] for k, v in kern.items()}
    line = {"training_step_ms": ms_step, "kernels_ms": per,
            "workload": f"{w.name} with the mask of shift {w.shifts[0]}"}
    for k, f in (("attn_fwd_kernel", f_fwd), ("attn_bwd_kernel", f_bwd),
                 ("attn_bwd_persistent_kernel", f_bwd)):
        if k in per:
            line[k.replace("attn_", "").replace("_kernel", "") + "_frac"] = (
                f / (per[k] * 1e-3) / 1e12 / peak)
    return line


def cla_line(w, kern_g, ms_gate_total, ms_fwd_cla_total, ms_fwd, pk, ms_cla_step_total,
             kern_cs, ms_step):
    """Convolutional local attention (measured beside the hot path, not part
    of its step): the gate kernel against the HBM roofline (x read + G
    written, 2 bytes each per pixel and channel) and the extra cost of
    applying the gate in the forward epilogue."""
    steps = kern_g["cla_gate_kernel"][0]
    ms_g = kern_g["cla_gate_kernel"][1] / steps
    C = w.heads * w.head_dim
    byt = 2 * w.batch * w.height * w.width * C * 2
    gbs = byt / (ms_g * 1e-3) / 1e9
    fwd_cla = ms_fwd_cla_total / steps
    step = ms_cla_step_total / steps
    bwd_k = {k: v[1] / v[0] for k, v in kern_cs.items() if k.startswith("cla_bwd")}
    return {"gate_kernel_ms": ms_g, "gate_bytes": byt, "gate_gbs": gbs,
            "gate_frac_hbm": gbs / pk["hbm_gbs"], "fwd_cla_ms": fwd_cla,
            "fwd_cla_extra_ms": fwd_cla - ms_fwd, "bound": "hbm",
            "training_step_with_cla_ms": step, "cla_extra_ms_per_step": step - ms_step,
            "cla_bwd_kernels_ms": bwd_k,
            "workload": f"x, G bf16 [{w.batch}][{w.height}][{w.width}][{C}]"}


# ---------------------------------------------------------------- oracle leg

def oracle_sample(w, inputs, rows, unit=(0, 0, 0)):
    """fp64 oracle fwd+bwd of `rows` query rows of one unit; returns
    (seconds, algorithmic FLOPs of the sample)."""
    import numpy as np
    import oracle as O
    M, s = w.windows[0], w.shifts[0]
    b, win, h = unit
    qp, kp = O.pos_tokens(inputs["freqs"], inputs["mlp_q"], inputs["mlp_k"], M, w.heads, w.rank)
    qc, kc, v, qpf, kpf = O.gather_unit(inputs["qkv"][b:b + 1], qp, kp, M, s, 0, win, h)
    dout = O.window_partition(inputs["dout"][b:b + 1].float().numpy(), M, s)[0, win, :, h]
    sl = slice(0, rows)
    tau = O.default_scale(w.head_dim, w.rank)
    t0 = time.perf_counter()
    O.attention_unit_rows(qc, kc, v, qpf, kpf, tau, rows=sl)
    g = O.attention_unit_backward(qc[sl], kc, v, qpf[sl], kpf, tau, dout[sl])
    dt = time.perf_counter() - t0
    del g
    N = M * M
    return dt, 2.0 * rows * N * (D_QK + D_V) + 2.0 * rows * N * (3 * D_QK + 2 * D_V)


def oracle_cores():
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def run_reference(args, w):
    """The oracle on this host's cores; under N ranks only rank 0 works and
    prints, the others exit 0 at once."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import rib_inputs as I
    inputs = I.make_layer_inputs(w, 0)
    N = w.windows[0] ** 2
    # size the per-step sample so the whole run stays within a few minutes
    t256, _ = oracle_sample(w, inputs, 256)
    budget = 150.0 / max(1, args.steps + args.warmup)
    rows = int(max(256, min(N, 256 * int(budget / max(t256, 1e-3)))))
    units = [(b, win, h) for b in range(w.batch) for win in range((w.height // w.windows[0]) *
                                                                   (w.width // w.windows[0]))
             for h in range(w.heads)]
    for i in range(args.warmup):
        oracle_sample(w, inputs, rows, units[i % len(units)])
    tot_t = tot_f = 0.0
    for i in range(args.steps):
        dt, f = oracle_sample(w, inputs, rows, units[(args.warmup + i) % len(units)])
        tot_t += dt
        tot_f += f
    value = tot_f / tot_t / 1e12
    cores = oracle_cores()
    sample = f"{rows} of {N} query rows of one unit per step (fwd+bwd), fp64 numpy oracle"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- GPU leg

def run_rib(args, w):
    import torch
    import torch.distributed as dist
    import rib_inputs as I
    import windowed_attention_implicit_b200 as R

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        if torch.cuda.device_count() < world:
            raise SystemExit(f"{world} ranks but only {torch.cuda.device_count()} GPUs visible")
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    R.library()
    from windowed_attention_implicit_b200 import _abi
    R.rib_set_bwd_kernel({"auto": _abi.RIB_BWD_AUTO, "per_item": _abi.RIB_BWD_PER_ITEM,
                          "persistent": _abi.RIB_BWD_PERSISTENT}[args.bwd_kernel])

    M, s = w.windows[0], w.shifts[0]
    # each rank trains on its own batch: seeds differ per rank (weak scaling)
    wr = I.get_workload(w.name, seed=w.seed + 7919 * rank)
    host = I.make_layer_inputs(wr, 0)
    mlp = R.PositionMLP.from_params(host["freqs"], host["mlp_q"], host["mlp_k"], w.heads, w.rank,
                                    device=dev)
    qkv = host["qkv"].to(dev)
    dout = host["dout"].to(dev)
    B, H, W, heads, d = w.batch, w.height, w.width, w.heads, w.head_dim
    pshape = (heads, M, M, w.rank)
    qp = torch.empty(pshape, device=dev)
    kp = torch.empty(pshape, device=dev)
    q16 = torch.empty(pshape, device=dev, dtype=torch.bfloat16)
    k16 = torch.empty(pshape, device=dev, dtype=torch.bfloat16)
    out = torch.empty((B, H, W, heads, d), device=dev, dtype=torch.bfloat16)
    lse = torch.empty((B, heads, H, W), device=dev)
    dqkv = torch.empty_like(qkv)
    dqp = torch.empty(pshape, device=dev)
    dkp = torch.empty(pshape, device=dev)
    shapes = [t.shape for t in (mlp.q_w1, mlp.q_b1, mlp.q_w2, mlp.q_b2,
                                mlp.k_w1, mlp.k_b1, mlp.k_w2, mlp.k_b2)]
    flat = torch.empty(sum(int(torch.Size(sh).numel()) for sh in shapes), device=dev)
    views, off = [], 0
    for sh in shapes:
        n = int(torch.Size(sh).numel())
        views.append(flat[off:off + n].view(sh))
        off += n
    dmlp = R.PositionMLPGrad(*views)
    ws = torch.empty(R.rib_window_attn_bwd_workspace(B, H, W, heads, d, M, w.rank, mlp),
                     device=dev, dtype=torch.uint8)

    def step():
        R.rib_pos_tokens(mlp, M, qp, kp, q16, k16)
        R.rib_window_attn_fwd(qkv, M, s, q16, k16, out=out, lse=lse)
        R.rib_window_attn_bwd(qkv, out, dout, lse, M, s, q16, k16, mlp=mlp, dqkv=dqkv,
                              dqp=dqp, dkp=dkp, dmlp=dmlp, workspace=ws)
        if world > 1:
            dist.all_reduce(flat)

    def fwd_only():
        R.rib_window_attn_fwd(qkv, M, s, q16, k16, out=out, lse=lse)

    # convolutional local attention gate on this workload's feature map
    # (C = heads * d channels) and the forward with the gate applied
    cla_p = I.make_cla(heads * d, w.seed)
    cla = R.ClaGate.from_params(cla_p.w_dw, cla_p.b_dw, cla_p.w_pw, cla_p.b_pw, device=dev)
    feat = I.make_features(B, H, W, heads * d, w.seed).to(dev)
    gate = torch.empty_like(feat)
    out_g = torch.empty_like(out)

    def cla_gate_only():
        R.rib_cla_gate(feat, cla, gate=gate)

    # a training step with the gate: the upstream gradient is that of O' = O * G
    d_att = torch.empty_like(dout)
    dfeat = torch.empty_like(feat)
    cla_ws = torch.empty(R.rib_cla_bwd_workspace(B, H, W, heads * d), device=dev,
                         dtype=torch.uint8)

    def cla_step():
        R.rib_pos_tokens(mlp, M, qp, kp, q16, k16)
        R.rib_cla_gate(feat, cla, gate=gate)
        R.rib_window_attn_fwd_cla(qkv, M, s, gate, q16, k16, out=out, out_gated=out_g, lse=lse)
        R.rib_cla_bwd(feat, cla, gate, out, dout, dout=d_att, dx=dfeat, workspace=cla_ws)
        R.rib_window_attn_bwd(qkv, out, d_att, lse, M, s, q16, k16, mlp=mlp, dqkv=dqkv,
                              dqp=dqp, dkp=dkp, dmlp=dmlp, workspace=ws)

    def fwd_cla():
        R.rib_window_attn_fwd_cla(qkv, M, s, gate, q16, k16, out=out, out_gated=out_g, lse=lse)

    # the same training step with the shifted-window region mask
    def masked_step():
        R.rib_pos_tokens(mlp, M, qp, kp, q16, k16)
        R.rib_window_attn_fwd(qkv, M, s, q16, k16, out=out, lse=lse, region_mask=True)
        R.rib_window_attn_bwd(qkv, out, dout, lse, M, s, q16, k16, mlp=mlp, dqkv=dqkv,
                              dqp=dqp, dkp=dkp, dmlp=dmlp, workspace=ws, region_mask=True)

    def timed(fn, steps, trace=False):
        stream = torch.cuda.current_stream()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        if trace:
            R.rib_trace_enable(True)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        kern = R.rib_trace_collect() if trace else None
        if trace:
            R.rib_trace_enable(False)
        ms = a.elapsed_time(b)
        if world > 1:
            dist.barrier()
            ms = max_over_ranks(ms, dev)
        return ms, kern, None

    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler("GPU-" + str(props.uuid)) if rank == 0 else None
    if sampler:
        sampler.start()       # samples cover warm-up and every timed loop below
    if args.cla_only:
        def cla_bwd_only():
            R.rib_cla_bwd(feat, cla, gate, out, dout, dout=d_att, dx=dfeat, workspace=cla_ws)

        for _ in range(args.warmup):
            cla_gate_only()
            fwd_cla()
            cla_bwd_only()
        ms_g, _, _ = timed(cla_gate_only, args.steps)
        ms_c, _, _ = timed(fwd_cla, args.steps)
        ms_b, kern_b, _ = timed(cla_bwd_only, args.steps, trace=True)
        if sampler:
            sampler.stop()
        if world > 1:
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps({"cla_only": True, "cla_gate_ms": ms_g / args.steps,
                              "fwd_cla_ms": ms_c / args.steps,
                              "cla_bwd_ms": ms_b / args.steps,
                              "cla_bwd_kernels_ms": {k: v[1] / v[0] for k, v in kern_b.items()}}))
        return 0
    for _ in range(args.warmup):
        step()
    code, site = R.rib_last_status()
    if code != 0:
        raise RuntimeError(f"kernel status {R.rib_status_string(code)} at site {site}")
    ms, kern, _ = timed(step, args.steps, trace=True)
    ms_step = ms / args.steps
    f_fwd, f_bwd = flops(w)
    value = world * (f_fwd + f_bwd) / (ms_step * 1e-3) / 1e12
    tokens_s = world * w.tokens() / (ms_step * 1e-3)

    if args.step_only:
        if sampler:
            sampler.stop()
        if world > 1:
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps({"step_only": True, "ms_per_step": ms_step, "kernels": kern}))
        return 0
    for _ in range(args.warmup):
        fwd_only()
    ms_f, kern_f, _ = timed(fwd_only, args.steps, trace=True)
    ms_fwd = ms_f / args.steps
    code, site = R.rib_last_status()
    if code != 0:
        raise RuntimeError(f"kernel status {R.rib_status_string(code)} at site {site}")

    for _ in range(args.warmup):
        cla_gate_only()
        fwd_cla()
    ms_g, kern_g, _ = timed(cla_gate_only, args.steps, trace=True)
    ms_c, _, _ = timed(fwd_cla, args.steps)
    for _ in range(args.warmup):
        cla_step()
    ms_cs, kern_cs, _ = timed(cla_step, args.steps, trace=True)
    for _ in range(args.warmup):
        masked_step()
    ms_m, kern_m, _ = timed(masked_step, args.steps, trace=True)

    # the window gather / scatter of the workload's qkv map (the partition
    # with cyclic shift as a standalone TMA copy), against the HBM roofline
    C3 = 3 * heads * d
    x_map = qkv.view(B, H, W, C3)
    xw = torch.empty((B, (H // M) * (W // M), M * M, C3), device=dev, dtype=torch.bfloat16)
    x_back = torch.empty_like(x_map)

    def gather_only():
        R.rib_window_gather(x_map, M, s, out=xw)

    def scatter_only():
        R.rib_window_scatter(xw, H, W, M, s, out=x_back)

    for _ in range(args.warmup):
        gather_only()
        scatter_only()
    _, kern_ga, _ = timed(gather_only, args.steps, trace=True)
    _, kern_sc, _ = timed(scatter_only, args.steps, trace=True)
    del xw, x_back

    # large-image inference: 12 forward layers (shifts alternating 0 / M/2)
    # over a 576 x 384 map, Qp/Kp computed once and reused by every window
    # and layer (the stack's geometry cache)
    from windowed_attention_implicit_b200.schedule import LayerSpec, RIBLayerStack
    wi = I.get_workload("w96infer", seed=I.get_workload("w96infer").seed + 7919 * rank)
    inp0 = I.make_layer_inputs(wi, 0, with_dout=False)
    mlp_i = R.PositionMLP.from_params(inp0["freqs"], inp0["mlp_q"], inp0["mlp_k"], wi.heads,
                                      wi.rank, device=dev)
    stack = RIBLayerStack([LayerSpec(wi.windows[l], wi.shifts[l], mlp_i)
                           for l in range(wi.layers)])
    qkvs = [inp0["qkv"].to(dev)] + [I.make_layer_inputs(wi, l, with_dout=False)["qkv"].to(dev)
                                    for l in range(1, wi.layers)]

    def infer_pass():
        stack.forward(qkvs)

    for _ in range(args.warmup):
        infer_pass()
    ms_inf, kern_inf, _ = timed(infer_pass, args.steps, trace=True)
    del qkvs, stack
    pk_s = peaks()
    sweep = config_sweep(I, R, dev, rank, world, timed, min(args.steps, 10), args.warmup,
                         pk_s["bf16_tflops"], pk_s) if not args.no_sweep else None
    code, site = R.rib_last_status()
    if code != 0:
        raise RuntimeError(f"kernel status {R.rib_status_string(code)} at site {site}")

    pk = peaks()
    peak = pk["bf16_tflops"]
    launches = sum(n for n, _ in kern.values())
    per_kernel = {k: {"launches": n, "total_ms": t, "avg_ms": t / n,
                      "share": t / sum(x for _, x in kern.values())} for k, (n, t) in kern.items()}
    top = max(per_kernel, key=lambda k: per_kernel[k]["total_ms"])
    kflops = {"attn_bwd_kernel": f_bwd, "attn_bwd_persistent_kernel": f_bwd,
              "attn_fwd_kernel": f_fwd}
    both = {k: roofline_entry(k, f, per_kernel[k]["avg_ms"], pk, stored_traffic(k, w.name))
            for k, f in kflops.items() if k in per_kernel}
    roof = None
    if top in both:
        roof = dict(both[top])
        roof["kernels"] = both
    fwd_k = kern_f.get("attn_fwd_kernel", (1, ms_f))
    fwd_ach = f_fwd / (fwd_k[1] / fwd_k[0] * 1e-3) / 1e12

    e2e = None
    if not args.no_e2e:
        # the same step with the inputs copied from pinned host memory and the
        # results read back, every step, all inside the timed region
        h_qkv = host["qkv"].pin_memory()
        h_dout = host["dout"].pin_memory()
        nb = lambda t: t.numel() * t.element_size()

        # (1) serialised: upload, step, read-back on one stream
        h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h_dqkv = torch.empty(dqkv.shape, dtype=dqkv.dtype).pin_memory()
        h_flat = torch.empty(flat.shape, dtype=flat.dtype).pin_memory()

        def e2e_step():
            qkv.copy_(h_qkv, non_blocking=True)
            dout.copy_(h_dout, non_blocking=True)
            step()
            h_out.copy_(out, non_blocking=True)
            h_dqkv.copy_(dqkv, non_blocking=True)
            h_flat.copy_(flat, non_blocking=True)

        for _ in range(max(3, args.warmup // 2)):
            e2e_step()
        ms_serial, _, _ = timed(e2e_step, args.steps)

        # (2) pipelined: uploads and read-backs on copy streams of their own,
        # device tensors double-buffered, so step i+1's upload and step i-1's
        # read-back overlap step i's kernels
        b_qkv, b_dout = [qkv, torch.empty_like(qkv)], [dout, torch.empty_like(dout)]
        b_out, b_dqkv = [out, torch.empty_like(out)], [dqkv, torch.empty_like(dqkv)]
        b_flat = [flat, torch.empty_like(flat)]
        b_dmlp = [dmlp]
        views2, off2 = [], 0
        for sh in shapes:
            n = int(torch.Size(sh).numel())
            views2.append(b_flat[1][off2:off2 + n].view(sh))
            off2 += n
        b_dmlp.append(R.PositionMLPGrad(*views2))
        hb_out = [h_out, torch.empty(out.shape, dtype=out.dtype).pin_memory()]
        hb_dqkv = [h_dqkv, torch.empty(dqkv.shape, dtype=dqkv.dtype).pin_memory()]
        hb_flat = [h_flat, torch.empty(flat.shape, dtype=flat.dtype).pin_memory()]
        s_up, s_down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        comp = torch.cuda.current_stream()
        ev = {k: [torch.cuda.Event(), torch.cuda.Event()] for k in ("up", "comp", "down")}
        used = {k: [False, False] for k in ev}

        def piped_step(i):
            bi = i % 2
            with torch.cuda.stream(s_up):
                if used["comp"][bi]:
                    s_up.wait_event(ev["comp"][bi])   # step i-2 has read buffer bi
                b_qkv[bi].copy_(h_qkv, non_blocking=True)
                b_dout[bi].copy_(h_dout, non_blocking=True)
                ev["up"][bi].record(s_up)
            comp.wait_event(ev["up"][bi])
            if used["down"][bi]:
                comp.wait_event(ev["down"][bi])       # step i-2's results are read
            R.rib_pos_tokens(mlp, M, qp, kp, q16, k16)
            R.rib_window_attn_fwd(b_qkv[bi], M, s, q16, k16, out=b_out[bi], lse=lse)
            R.rib_window_attn_bwd(b_qkv[bi], b_out[bi], b_dout[bi], lse, M, s, q16, k16,
                                  mlp=mlp, dqkv=b_dqkv[bi], dqp=dqp, dkp=dkp,
                                  dmlp=b_dmlp[bi], workspace=ws)
            if world > 1:
                dist.all_reduce(b_flat[bi])
            ev["comp"][bi].record(comp)
            used["comp"][bi] = True
            with torch.cuda.stream(s_down):
                s_down.wait_event(ev["comp"][bi])
                hb_out[bi].copy_(b_out[bi], non_blocking=True)
                hb_dqkv[bi].copy_(b_dqkv[bi], non_blocking=True)
                hb_flat[bi].copy_(b_flat[bi], non_blocking=True)
                ev["down"][bi].record(s_down)
            used["down"][bi] = True

        def piped(steps):
            for k in used:
                used[k] = [False, False]
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(comp)
            for i in range(steps):
                piped_step(i)
            comp.wait_event(ev["down"][(steps - 1) % 2])   # the last read-back is in
            b.record(comp)
            torch.cuda.synchronize()
            t = a.elapsed_time(b)
            if world > 1:
                dist.barrier()
                t = max_over_ranks(t, dev)
            return t

        piped(max(3, args.warmup // 2))
        ms_e = piped(args.steps)
        e_step = ms_e / args.steps
        e2e = {"value": world * (f_fwd + f_bwd) / (e_step * 1e-3) / 1e12, "unit": "TFLOP/s",
               "ms_per_step": e_step,
               "tokens_per_s": world * w.tokens() / (e_step * 1e-3),
               "h2d_bytes_per_step": nb(h_qkv) + nb(h_dout),
               "d2h_bytes_per_step": nb(h_out) + nb(h_dqkv) + nb(h_flat),
               "pipelined": "uploads and read-backs on two copy streams, device tensors "
                            "double-buffered; every step copies its inputs in and its "
                            "results out",
               "serial_ms_per_step": ms_serial / args.steps}

    clocks = sampler.stop() if sampler else None
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        N = M * M
        dt, f = oracle_sample(w, host, N)
        cpu = {"value": f / dt / 1e12, "unit": "TFLOP/s", "cores": oracle_cores(),
               "kind": "oracle", "seconds": dt,
               "sample": f"1 of {w.units()} units (batch 0, window 0, head 0), all {N} rows, "
                         "fwd+bwd, fp64 numpy oracle"}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) features and upstream grads, N(0,0.02) MLP weights)",
        "config": bench_config(w, world),
        "tokens_per_s": tokens_s,
        "fwd": {"tflops": world * f_fwd / (ms_fwd * 1e-3) / 1e12, "ms": ms_fwd,
                "tokens_per_s": world * w.tokens() / (ms_fwd * 1e-3),
                "kernel_tflops": fwd_ach, "kernel_frac": fwd_ach / peak,
                "kernel_frac_of": "measured burst bf16 peak"},
        "roofline": roof,
        "cla": cla_line(w, kern_g, ms_g, ms_c, ms_fwd, pk, ms_cs, kern_cs, ms_step),
        "region_mask": mask_line(w, ms_m / args.steps, kern_m, f_fwd, f_bwd, peak),
        "gather": copy_line(kern_ga, kern_sc, x_map, pk),
        "inference": infer_line(wi, ms_inf / args.steps, kern_inf, args.steps, world, peak),
        "configs": sweep,
        "pos_tokens": pos_line(w, per_kernel, pk),
        "kernels": per_kernel,
        "gpu_launches": launches,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "clocks": clocks,
        "peaks": pk,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    try:
        plan = world_plan(args.gpus)
    except ValueError as e:
        print(f"bench.py: {e}", file=sys.stderr)
        return 2
    if plan == "relaunch":
        return subprocess.call(relaunch_cmd(args.gpus, sys.argv[1:], free_port()))
    import rib_inputs as I
    w = I.get_workload(args.workload)
    if args.impl == "reference":
        return run_reference(args, w)
    return run_rib(args, w)


if __name__ == "__main__":
    sys.exit(main())

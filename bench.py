#!/usr/bin/env python
"""FusedBitLinear benchmark on B200: tokens/s for the HGRNBit projection hot path.

One step = every FusedBitLinear projection of the workload's layers applied to one batch of T
tokens: per layer i/f/g_proj (input x_attn), o_proj (x_o), gate_proj with the SiLU-GLU
epilogue (x_mlp) and down_proj fed by gate_proj's GLU output h.  The default data flow
("path") chains only what this path itself links, gate_proj's GLU output into down_proj; the
layer's other inputs come from the recurrence, the residual stream and the norms, which are
outside the path, so they are seeded synthetic activations, one set per layer.  "--dataflow
chained" instead feeds every projection from an earlier one (o from g, gate from o, the next
layer from down), the dependency depth of a real layer-by-layer decode.  Each projection is the
full forward: RMSNorm + int8 activation quantisation, then the tcgen05 ternary contraction with
the dequantisation epilogue; projections that read the same input (i/f/g) share its
quantisation.  Weights are quantised and packed once before timing (the offline step of the
method); packed weights rotate over enough distinct copies that every step streams them from
HBM, not L2.

The headline line times the largest single-GPU workload (the 1.3B-shaped prefill, tensor-bound)
and, in a "decode" object beside it, the HBM-bound decode workloads (1.3B at 1/8/64 tokens,
2.7B at 8 tokens), each with its own step time, weight GB/s, roofline fraction and clocks.
An "mlgru" object times the MLGRU recurrence with its swish gate norm (the step after
i/f/g_proj), alone and fused with o_proj's activation quantisation, on the 1.3B prefill
shape, and at one decode token; its roofline is the special-function unit, which binds it,
with HBM beside it.  A "backward" object times the straight-through backward of one 1.3B
layer's six projections at the prefill length (input- and weight-gradient calls, fp16
tensor-core contractions) against the measured bf16 dense peak.

Arms:
  default            the CUDA library through its C ABI; the timed region replays CUDA
                     graphs of whole steps with inputs resident in HBM.
  --impl reference   the oracle (scalar C, host cores) on a bounded sample of the same step.

Launch: python bench.py [--gpus N --steps K --warmup W] [--workload NAME]; for N > 1 under
torch.distributed.run, one replica per GPU (the projection shards by tokens with no
exchange), timing = max over ranks.  Rank 0 prints one JSON line.
"""
import argparse
import concurrent.futures
import hashlib
import json
import math
import os
import platform
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "FusedBitLinear tokens/s; weight GB/s (decode), int8 TOPS (prefill) vs roofline"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
NOMINAL_INT8_TOPS = 4500.0          # B200 dense int8, datasheet
INT8_PER_BF16 = 2.0                 # nominal dense int8 / bf16 throughput ratio
GRAPH_SAMPLES = 8                   # distinct step graphs carrying per-launch timing events
# The straight-through backward leg: one 1.3B layer's six projections (hidden 2048, MLP 5632)
# at the prefill length: i/f/g/o 2048 -> 2048, gate 2048 -> 11264 (the GLU's 2I rows), down
# 5632 -> 2048.
BACKWARD_SHAPE = ("hgrn1p3b_layer_backward_t32768", 32768, 2048, 5632)


# ----------------------------------------------------------------------------- helpers
def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["mmf", "reference"], default="mmf")
    ap.add_argument("--workload", default=synth.workloads.DEFAULT,
                    choices=sorted(synth.WORKLOADS))
    ap.add_argument("--decode", default=",".join(synth.workloads.DECODE_SUITE),
                    help="comma-separated decode workloads reported beside the headline "
                         "('' for none)")
    ap.add_argument("--decode-seconds", type=float, default=0.5,
                    help="least timed GPU time of each decode entry")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the straight-through backward leg")
    ap.add_argument("--backward-tokens", type=int, default=BACKWARD_SHAPE[1],
                    help="tokens of the backward leg (smaller for a profiler capture)")
    ap.add_argument("--no-mlgru", action="store_true",
                    help="skip the MLGRU recurrence + gate norm entry")
    ap.add_argument("--cpu-seconds", type=float, default=8.0,
                    help="target host time of each CPU-baseline leg")
    ap.add_argument("--path", choices=["auto", "program", "launches"], default="auto",
                    help="one program launch per step (decode, T <= 64) or per-projection launches")
    ap.add_argument("--dataflow", choices=sorted(DATAFLOWS), default="path",
                    help="which projections feed which (see the module docstring)")
    return ap.parse_args(argv)


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def reduce_max(value, world, device=None):
    """Max of a float over ranks (identity when world == 1)."""
    if world == 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(tokens_per_step, steps, world, max_seconds):
    """Whole-job tokens/s: every rank runs its own replica on its own tokens."""
    return tokens_per_step * steps * world / max_seconds


def measured_peaks():
    """(hbm GB/s, bf16 TFLOP/s burst, bf16 TFLOP/s sustained, source)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return (float(d["hbm_gbs"]), float(d["bf16_tflops"]),
                float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured")
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS, "fallback"


def tensor_peak(clocks, bf16_burst, bf16_sustained):
    """int8 peak of the contraction: the measured bf16 dense burst rate times the nominal
    int8/bf16 ratio (the conservative denominator), and beside it the same scaled by the SM
    clock seen during the run (the tensor rate follows the clock) and the sustained figure."""
    burst = INT8_PER_BF16 * bf16_burst
    sm, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    scale = min(1.0, sm / mx) if sm and mx else 1.0
    return burst, burst * scale, INT8_PER_BF16 * bf16_sustained


# the sources each profiled kernel is built from (its own file plus the shared device headers)
KERNEL_SOURCES = {
    "program_kernel": ["program.cu"],
    "ternary_gemm": ["ternary_gemm.cu", "prefill_ss.cu", "backward.cuh"],
    "act_quant": ["act_quant.cu"],
    "mlgru": ["mlgru.cu"],
    "backward": ["backward.cu", "backward.cuh", "prefill_ss.cu"],
}


def kernel_source_sha(kernel):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "ternary_weight_lm_b200", "csrc")
    for name in sorted(set(KERNEL_SOURCES[kernel] + ["kernels.cuh", "ptx.cuh"])):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel, workload):
    """dram bytes per launch recorded from an ncu capture in profiles/, if the kernel's sources
    are unchanged since (the summary names the hash of those sources it was taken at)."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path, encoding="utf-8").read()
    m_sha = re.search(r"source_sha:\s*([0-9a-f]+)", text)
    m_b = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if kernel not in KERNEL_SOURCES or not m_sha or not m_b or \
            m_sha.group(1) != kernel_source_sha(kernel):
        return None
    return float(m_b.group(1))


class ClockSampler:
    """nvidia-smi clock/throttle samples every 200 ms while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.thread.join(timeout=5)

    def summary(self):
        return summarise_clock_lines(self.lines)


def summarise_clock_lines(lines):
    """Median SM clock, the maximum, and every throttle reason seen active, from nvidia-smi
    csv lines (index, sm, max sm, power, active mask, four reason flags)."""
    sm, mx, reasons = [], None, set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for ln in lines:
        parts = [p.strip() for p in ln.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm.append(float(parts[1]))
            mx = float(parts[2])
        except ValueError:
            continue
        for name, flag in zip(names, parts[5:9]):
            if flag.lower() == "active":
                reasons.add(name)
    if not sm:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
    return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
            "samples": len(sm)}


# ----------------------------------------------------------------------------- workload
def projection_bytes(p, T):
    """Algorithmic HBM bytes of one contraction launch: the packed weights (N*K/4), the int8
    activation codes it reads (T*K), gamma and the code sums (8T) and its fp16 output."""
    n_out = p.N // 2 if p.glu else p.N
    return p.N * p.K // 4 + T * p.K + 8 * T + 2 * T * n_out


def quant_bytes(K, T, in_bytes=2):
    """Algorithmic bytes of one RMSNorm + quantisation launch: x in, codes + gamma + sums out."""
    return in_bytes * T * K + T * K + 8 * T


def step_bytes(wl):
    """Algorithmic HBM bytes of one step run as one program launch: every projection's packed
    weights, each distinct input read once (fp16) and each output written once; the int8 codes
    are an on-chip/L2 intermediate.  Both data flows have, per layer, three distinct inputs of
    width H (shared by i/f/g, then o's, then gate's) and the GLU output of width I (down's)."""
    T, tot = wl.T, 0
    widths = {}
    for p in wl.projections:
        n_out = p.N // 2 if p.glu else p.N
        tot += p.N * p.K // 4 + 2 * T * n_out
        widths.setdefault(SOURCE_OF.get(p.name, p.name), p.K)
    tot += sum(2 * T * k for k in widths.values())
    return tot * wl.layers


# Which input each projection reads, and the dependency level it runs at, per data flow.
# "path": i/f/g/o/gate read the layer's synthetic inputs (level 0), down reads the GLU output
# (level 1).  "chained": i/f/g read the layer input, o reads g's output, gate reads o's
# output, down reads the GLU output, the next layer reads down's output (4 levels per layer).
SOURCE_OF = {"i_proj": "x_attn", "f_proj": "x_attn", "g_proj": "x_attn", "proj": "x_attn",
             "o_proj": "x_o", "gate_proj": "x_mlp", "down_proj": "h"}
DATAFLOWS = {
    "path": {"i_proj": 0, "f_proj": 0, "g_proj": 0, "o_proj": 0, "gate_proj": 0,
             "down_proj": 1, "proj": 0},
    "chained": {"i_proj": 0, "f_proj": 0, "g_proj": 0, "o_proj": 1, "gate_proj": 2,
                "down_proj": 3, "proj": 0},
}
LEVELS_PER_LAYER = {"path": 2, "chained": 4}   # "path": the layers are independent, so a
# whole step has 2 levels; "chained": 4 per layer, one after another
DATAFLOW_TEXT = {
    "path": ("per layer: i/f/g read x_attn, o reads x_o, gate reads x_mlp (seeded synthetic "
             "activations, one set per layer: their producers are outside this path); down "
             "reads gate's GLU output"),
    "chained": ("per layer: i/f/g read the layer input, o reads g's output, gate reads o's "
                "output, down reads the GLU output, the next layer reads down's"),
}


class GpuWorkload:
    """Device buffers for one replica: packed weight copies, the step inputs, the step outputs,
    and either one planned program per weight copy (T <= 64) or per-projection launches."""

    def __init__(self, wl, device, path="auto", dataflow="path"):
        import torch
        import ternary_weight_lm_b200 as mmf
        self.torch, self.mmf = torch, mmf
        self.wl, self.dev = wl, device
        self.dataflow = dataflow
        self.level_of = DATAFLOWS[dataflow]
        T = wl.T
        H = wl.projections[0].K
        need = 2 * L2_BYTES
        self.copies = max(1, -(-need // (wl.packed_bytes_per_layer * wl.layers)))
        xdt = np.float32 if wl.x_dtype == "f32" else np.float16
        self.ydt = torch.float32 if wl.y_dtype == "f32" else torch.float16
        # one seeded layer quantised by the library; every other layer and copy is a byte copy at
        # a distinct address (identical bytes stream exactly like distinct ones)
        self.Wp, self.beta = {}, {}
        nz = 0
        for p in wl.projections:
            W = torch.from_numpy(synth.weights(0, p.name, p.N, p.K)).to(device)
            Wp0, b0 = mmf.quantize_weights(W)
            del W
            # nonzero codes of this projection (2-bit fields holding e = c + 1 != 1), counted
            # on the side for the report; the step itself never looks at this
            nz += sum(int(((Wp0 >> s) & 3).ne(1).sum()) for s in (0, 2, 4, 6))
            n = self.copies * wl.layers
            self.Wp[p.name] = [Wp0] + [Wp0.clone() for _ in range(n - 1)]
            self.beta[p.name] = [b0] + [b0.clone() for _ in range(n - 1)]
        self.nonzero_frac = nz / wl.weights_per_layer
        # step inputs: "path" has one set of synthetic activations per layer and source,
        # "chained" only the first layer's input.  All of a step's outside inputs are views of
        # one contiguous device buffer, and all of its outputs views of another, so that the
        # end-to-end measurement moves each with one copy per step.
        srcs = sorted({SOURCE_OF.get(p.name, "x_attn") for p in wl.projections} - {"h"})
        nl = wl.layers if dataflow == "path" else 1
        srcs_l = srcs if dataflow == "path" else ["x_attn"]
        self.xin_buf = torch.empty((nl * len(srcs_l), T, H),
                                   dtype=torch.float32 if xdt == np.float32 else torch.float16,
                                   device=device)
        self.xin = []
        for l in range(nl):
            d = {}
            for j, src in enumerate(srcs_l):
                v = self.xin_buf[l * len(srcs_l) + j]
                v.copy_(torch.from_numpy(synth.activations(
                    0, src if l == 0 else f"{src}/layer{l}", T, H, dtype=xdt,
                    outlier_frac=wl.outlier_frac, outlier_scale=wl.outlier_scale)))
                d[src] = v
            self.xin.append(d)
        self.x = self.xin[0]["x_attn"]
        widths = [p.N // 2 if p.glu else p.N for p in wl.projections]
        self.yout_buf = torch.empty(wl.layers * T * sum(widths), dtype=self.ydt, device=device)
        self.y, off = [], 0
        for _ in range(wl.layers):
            d = {}
            for p, w in zip(wl.projections, widths):
                d[p.name] = self.yout_buf[off:off + T * w].view(T, w)
                off += T * w
            self.y.append(d)
        self.use_program = (path == "program") or (path == "auto" and T <= 64)
        self.programs = []
        if self.use_program:
            for c in range(self.copies):
                self.programs.append(mmf.Program(self.projection_list(c), T))
        else:
            kmax = max(p.K for p in wl.projections)
            self.qws = mmf.workspace(max(mmf.mmf_quantized_workspace_bytes(T, p.K, p.N)
                                         for p in wl.projections), device)
            self.A = torch.empty((T, kmax), dtype=torch.int8, device=device)
            self.gamma = torch.empty(T, dtype=torch.float32, device=device)
            self.rowsum = torch.empty(T, dtype=torch.int32, device=device)

    def input_of(self, l, p):
        ys = self.y[l]
        if p.name == "down_proj":
            return ys["gate_proj"]                  # the GLU output, in both data flows
        if self.dataflow == "path":
            return self.xin[l][SOURCE_OF.get(p.name, "x_attn")]
        if p.name in ("i_proj", "f_proj", "g_proj", "proj"):
            return self.x if l == 0 else self.y[l - 1]["down_proj"]
        if p.name == "o_proj":
            return ys["g_proj"]
        return ys["o_proj"]                         # gate_proj

    @property
    def step_inputs(self):
        """The device tensor a step reads from outside (copied in from the host in e2e)."""
        return self.xin_buf

    @property
    def step_outputs(self):
        """The device tensor holding every output of a step (copied back in e2e)."""
        return self.yout_buf

    def projection_list(self, c):
        out = []
        for l in range(self.wl.layers):
            li = c * self.wl.layers + l
            for p in self.wl.projections:
                out.append(dict(x=self.input_of(l, p), Wp=self.Wp[p.name][li],
                                beta=self.beta[p.name][li], y=self.y[l][p.name], glu=p.glu,
                                level=self.level_of[p.name] if self.dataflow == "path" else
                                LEVELS_PER_LAYER["chained"] * l + self.level_of[p.name]))
        return out

    def launch_groups(self, l):
        """The launches of layer l in dependency order: each distinct input is quantised once,
        then every projection reading it runs its contraction."""
        groups = []
        for p in sorted(self.wl.projections, key=lambda q: self.level_of[q.name]):
            x = self.input_of(l, p)
            for gx, members in groups:
                if gx is x:
                    members.append(p)
                    break
            else:
                groups.append((x, [p]))
        return groups

    def run_step(self, step_index, mark=None):
        """One step through the public entry points: one program launch, or per layer one
        RMSNorm + quantisation launch per distinct input and one contraction launch per
        projection.  `mark(kind, nbytes, nops)` is called after every launch (timing events)."""
        c = step_index % self.copies
        if self.use_program:
            self.programs[c].run()
            if mark:
                mark("program_kernel", step_bytes(self.wl), self.ops_per_step)
            return
        mmf, T = self.mmf, self.wl.T
        in_bytes = 4 if self.wl.x_dtype == "f32" else 2
        for l in range(self.wl.layers):
            li = c * self.wl.layers + l
            for x, members in self.launch_groups(l):
                K = x.shape[1]
                A = self.A.view(-1)[:T * K].view(T, K)
                mmf.mmf_quantize_activations(x, None, 1e-8, A, self.gamma, self.rowsum)
                if mark:
                    mark("act_quant", quant_bytes(K, T, in_bytes), 0)
                for p in members:
                    mmf.mmf_bitlinear_forward_quantized(A, self.gamma, self.rowsum,
                                                        self.Wp[p.name][li],
                                                        self.beta[p.name][li], p.N, p.glu,
                                                        self.y[l][p.name], self.qws)
                    if mark:
                        mark("ternary_gemm", projection_bytes(p, T), 2 * T * p.N * p.K)

    @property
    def launches_per_step(self):
        if self.use_program:
            return 1
        return sum(1 + len(m) for m_l in range(self.wl.layers)
                   for _, m in self.launch_groups(m_l))

    @property
    def packed_bytes_per_step(self):
        return self.wl.packed_bytes_per_layer * self.wl.layers

    @property
    def ops_per_step(self):
        return 2 * self.wl.T * self.wl.weights_per_layer * self.wl.layers


# ----------------------------------------------------------------------------- GPU arm
def gpu_index(local_rank):
    if "CUDA_VISIBLE_DEVICES" in os.environ:
        return os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank]
    return local_rank


def time_workload(wl, args, dev, stream, world, local_rank, steps, warmup, with_e2e):
    """Times `steps` steps of CUDA-graph replays of workload `wl`, inputs resident.  Per-kernel
    durations come from timing events captured inside the same graphs (the launches path) or
    are the step itself (the program path: one launch per step)."""
    import torch
    import ternary_weight_lm_b200 as mmf
    g = GpuWorkload(wl, dev, args.path, args.dataflow)
    T = wl.T
    with torch.cuda.stream(stream):
        for i in range(max(warmup, 3)):
            g.run_step(i)
    torch.cuda.synchronize()
    if mmf.mmf_get_device_status() != 0:
        raise RuntimeError("device status reported a timeout during warm-up")

    # ---- graphs.  Program path: one graph runs `chunk` consecutive steps (rotating the weight
    # copies).  Launches path: GRAPH_SAMPLES graphs of one step each, with a timing event
    # after every launch; the timed region replays them in turn.
    records = []    # per sample graph: [(kind, nbytes, nops, ev_start, ev_end), ...]

    def capture_program(n_steps):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            for i in range(n_steps):
                g.run_step(i)
        return gr

    def capture_timed(j):
        gr = torch.cuda.CUDAGraph()
        rec = []
        with torch.cuda.graph(gr, stream=stream):
            prev = torch.cuda.Event(enable_timing=True, external=True)
            prev.record(stream)

            def mark(kind, nbytes, nops):
                nonlocal prev
                e = torch.cuda.Event(enable_timing=True, external=True)
                e.record(stream)
                rec.append((kind, nbytes, nops, prev, e))
                prev = e
            g.run_step(j, mark)
        records.append(rec)
        return gr

    if g.use_program:
        chunk = max(1, min(g.copies, steps))
        g_main = capture_program(chunk)
        rem = steps % chunk
        g_rem = capture_program(rem) if rem else None
        graphs = None
    else:
        # one graph per weight copy (at least GRAPH_SAMPLES), so that the replays rotate over
        # every copy
        graphs = [capture_timed(j) for j in range(min(steps, max(GRAPH_SAMPLES, g.copies)))]
    torch.cuda.synchronize()

    def replay_steps(n):
        if g.use_program:
            for _ in range(n // chunk):
                g_main.replay()
            if n % chunk:
                g_rem.replay()
        else:
            for i in range(n):
                graphs[i % len(graphs)].replay()

    with torch.cuda.stream(stream):
        replay_steps(chunk if g.use_program else len(graphs))
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    # ---- timed region: `steps` steps of graph replays
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_index(local_rank)) as clk:
        barrier()
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            start.record()
            replay_steps(steps)
            end.record()
        torch.cuda.synchronize()
        barrier()
    elapsed_s = reduce_max(start.elapsed_time(end) / 1e3, world, dev)
    clocks = clk.summary()
    if mmf.mmf_get_device_status() != 0:
        raise RuntimeError("device status reported a timeout in the timed region")
    ms_per_step = elapsed_s * 1e3 / steps

    # ---- per-kernel durations inside the same replays
    per_kernel = {}
    if g.use_program:
        per_kernel["program_kernel"] = [ms_per_step * steps, steps,
                                        step_bytes(wl) * steps, g.ops_per_step * steps]
        kernel_timing = ("one launch per step: the kernel's average is the step time of the "
                         "timed graph replays")
    else:
        for rec in records:          # each sample graph's last replay inside the timed region
            for kind, nbytes, nops, e0, e1 in rec:
                acc = per_kernel.setdefault(kind, [0.0, 0, 0.0, 0.0])
                acc[0] += e0.elapsed_time(e1)
                acc[1] += 1
                acc[2] += nbytes
                acc[3] += nops
        kernel_timing = (f"timing events captured between the launches of {len(graphs)} step "
                         f"graphs, read after their last replay inside the timed region")
    total_ms = sum(v[0] for v in per_kernel.values())
    kernels = {k: {"launches": v[1], "avg_us": round(1e3 * v[0] / max(1, v[1]), 3),
                   "share": round(v[0] / total_ms, 4) if total_ms else None,
                   "achieved_gbs": round(v[2] / (v[0] / 1e3) / 1e9, 1) if v[0] else None,
                   "achieved_tops": round(v[3] / (v[0] / 1e3) / 1e12, 1) if v[0] and v[3]
                   else None}
               for k, v in per_kernel.items()}
    dominant = max(per_kernel, key=lambda k: per_kernel[k][0])
    hbm_peak, bf16_burst, bf16_sust, peak_kind = measured_peaks()
    dom = per_kernel[dominant]
    dom_s = dom[0] / 1e3
    if not g.use_program and dom[3] > 0 and T > 64:
        # prefill: the contraction is bound by the int8 tensor pipe
        achieved = dom[3] / dom_s / 1e12
        peak, peak_clk, peak_sust = tensor_peak(clocks, bf16_burst, bf16_sust)
        step_tops = g.ops_per_step / (ms_per_step / 1e3) / 1e12
        roofline = {"bound": "tensor", "kernel": dominant, "achieved": round(achieved, 1),
                    "peak": round(peak, 1), "unit": "TOPS", "frac": round(achieved / peak, 4),
                    "peak_source": f"{peak_kind} bf16 dense burst x {INT8_PER_BF16:g}, the nominal "
                                   f"int8/bf16 ratio (no measured int8 entry)",
                    "frac_of_clock_scaled_peak": round(achieved / peak_clk, 4),
                    "frac_of_sustained_proxy": round(achieved / peak_sust, 4),
                    "frac_of_nominal_4p5_pops": round(achieved / NOMINAL_INT8_TOPS, 4),
                    "step_tops": round(step_tops, 1),
                    "step_frac": round(step_tops / peak, 4),
                    "ops_per_launch": dom[3] / dom[1],
                    "nonzero_frac_of_weights": round(g.nonzero_frac, 4),
                    "frac_counting_nonzero_adds_only": round(achieved * g.nonzero_frac / peak, 4),
                    "traffic": profiled_traffic(dominant, wl.name)}
    else:
        achieved = dom[2] / dom_s / 1e9
        roofline = {"bound": "hbm", "kernel": dominant, "achieved": round(achieved, 1),
                    "peak": hbm_peak, "unit": "GB/s", "frac": round(achieved / hbm_peak, 4),
                    "peak_source": peak_kind + " copy bandwidth",
                    "bytes_per_launch": dom[2] / dom[1],
                    "traffic": profiled_traffic(dominant, wl.name)}

    # ---- e2e: the public API with host buffers, copies inside the timed region
    e2e = None
    if with_e2e:
        hx = g.step_inputs.cpu().pin_memory()
        hy = torch.empty_like(g.step_outputs, device="cpu").pin_memory()
        h2d = hx.numel() * hx.element_size()
        d2h = hy.numel() * hy.element_size()
        e2e_steps = max(3, min(steps, int(2.0 / max(1e-6, ms_per_step / 1e3 +
                                                   (h2d + d2h) / 20e9))))
        with torch.cuda.stream(stream):
            for i in range(3):
                g.run_step(i)
        torch.cuda.synchronize()
        barrier()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            s0.record()
            for i in range(e2e_steps):
                g.step_inputs.copy_(hx, non_blocking=True)
                g.run_step(i)
                hy.copy_(g.step_outputs, non_blocking=True)
            s1.record()
        torch.cuda.synchronize()
        barrier()
        e2e_s = reduce_max(s0.elapsed_time(s1) / 1e3, world, dev)
        e2e = {"value": round(aggregate_throughput(T, e2e_steps, world, e2e_s), 1),
               "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "steps": e2e_steps,
               "path": ("mmf_program_run (one launch per step)" if g.use_program else
                        "mmf_quantize_activations once per distinct input + "
                        "mmf_bitlinear_forward_quantized per projection") +
                       ", every step input from pinned host memory in one copy, every step "
                       "output back to pinned host memory in one copy"}

    res = {
        "workload": wl.name, "value": aggregate_throughput(T, steps, world, elapsed_s),
        "ms_per_step": ms_per_step, "steps": steps, "clocks": clocks, "roofline": roofline,
        "kernels": kernels, "kernel_timing": kernel_timing, "e2e": e2e,
        "launches": g.launches_per_step * steps,
        "weight_gbs": g.packed_bytes_per_step * steps * world / elapsed_s / 1e9,
        "int8_tops": g.ops_per_step * steps * world / elapsed_s / 1e12,
        "copies": g.copies, "path": "program" if g.use_program else "launches",
    }
    del g
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


def run_gpu(args, rank, world, local_rank):
    import torch
    from ternary_weight_lm_b200 import build as lib_build

    if rank == 0:
        lib_build.build()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.set_device(local_rank)
    dev = torch.device(f"cuda:{local_rank}")
    stream = torch.cuda.Stream(device=dev)
    wl = synth.WORKLOADS[args.workload]
    head = time_workload(wl, args, dev, stream, world, local_rank, args.steps, args.warmup,
                         not args.no_e2e)
    decode = {}
    for name in [n for n in args.decode.split(",") if n and n != args.workload]:
        dwl = synth.WORKLOADS[name]
        # each entry runs for at least --decode-seconds of GPU time (step times from 0.03 to
        # 0.25 ms), so that the clock samples cover it
        est_ms = max(0.02, dwl.packed_bytes_per_layer * dwl.layers / 3e12 * 1e3)
        n_steps = max(args.steps, int(math.ceil(args.decode_seconds * 1e3 / est_ms)))
        r = time_workload(dwl, args, dev, stream, world, local_rank, n_steps, args.warmup, False)
        decode[name] = {k: r[k] for k in ("value", "ms_per_step", "steps", "clocks", "roofline",
                                          "weight_gbs", "path", "launches", "copies")}
        decode[name]["unit"] = "tokens/s"
        decode[name]["tokens_per_step"] = dwl.T
        decode[name]["layers_per_step"] = dwl.layers
    head["decode"] = decode
    if not args.no_mlgru:
        head["mlgru"] = time_mlgru(args, dev, stream, world, local_rank)
    if not args.no_backward:
        head["backward"] = time_backward(args, dev, stream, world, local_rank)
    return head


# ----------------------------------------------------------------------------- MLGRU
# The recurrence and gate norm that follow i/f/g_proj, on the 1.3B prefill shape (T tokens of
# hidden size H) and at one decode token.
MLGRU_SHAPE = ("hgrn1p3b_mlgru_t32768", 32768, 2048)


def mlgru_bytes(T, H, quantized=False, in_bytes=2):
    """Algorithmic HBM bytes of one MLGRU call: I, F and G read once and o written once (fp16),
    or, fused, o_proj's int8 codes, gamma and code sums written instead of o."""
    out = T * H + 8 * T if quantized else in_bytes * T * H
    return 3 * in_bytes * T * H + out


# The MLGRU's gate arithmetic runs on the SM's special-function unit (exp2 and reciprocal):
# per element three such operations in the chunk-map pass (two exponentials and one
# reciprocal for both gates) and five in the output pass (the gates again, then the SiLU's
# exponential and reciprocal).  One call of a single chunk (T <= 32) runs the output pass
# alone.  The unit issues 16 operations per clock per SM (sm_100, CUDA's arithmetic throughput
# table); 148 SMs at the 1965 MHz maximum clock give the peak below.
XU_OPS_PER_CLOCK_PER_SM = 16
B200_SMS = 148
B200_MAX_SM_MHZ = 1965.0


def xu_peak_ops(sm_mhz=B200_MAX_SM_MHZ):
    return XU_OPS_PER_CLOCK_PER_SM * B200_SMS * sm_mhz * 1e6


def mlgru_xu_ops(T, H):
    """Special-function-unit operations of one MLGRU call over T tokens of H channels."""
    per_elem = 5 if T <= 32 else 8
    return per_elem * T * H


def mlgru_roofline(T, H, quantized, ms, hbm_peak, clocks):
    """Both bounds of one MLGRU call: HBM bytes over the copy peak and special-function-unit
    operations over that unit's peak.  The binding one (the longer time at peak) is reported
    as the roofline; the other stays beside it."""
    nbytes = mlgru_bytes(T, H, quantized)
    xu = mlgru_xu_ops(T, H)
    s = ms * 1e-3
    hbm_ach = nbytes / s / 1e9
    xu_peak = xu_peak_ops()
    sm = clocks.get("sm_mhz") if clocks else None
    hbm = {"bound": "hbm", "achieved": round(hbm_ach, 1), "peak": round(hbm_peak, 1),
           "unit": "GB/s", "frac": round(hbm_ach / hbm_peak, 4), "bytes_per_call": nbytes,
           "peak_source": "measured copy bandwidth"}
    alu = {"bound": "alu", "achieved": round(xu / s / 1e12, 3), "peak": round(xu_peak / 1e12, 3),
           "unit": "T special-function ops/s", "frac": round(xu / s / xu_peak, 4),
           "ops_per_call": xu,
           "peak_source": "16 exp2/reciprocal per clock per SM x 148 SMs x 1965 MHz",
           "frac_of_clock_scaled_peak": round(xu / s / xu_peak_ops(sm), 4) if sm else None}
    xu_bound = xu / xu_peak > nbytes / (hbm_peak * 1e9)
    main, other = (alu, hbm) if xu_bound else (hbm, alu)
    return dict(main, other_bound=other)


def time_mlgru(args, dev, stream, world, local_rank):
    """Times mmf_mlgru_forward and mmf_mlgru_forward_quantized (inputs resident in HBM, larger
    than L2) and one decode token's call."""
    import torch
    import ternary_weight_lm_b200 as mmf

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    name, T, H = MLGRU_SHAPE
    gen = torch.Generator(device=dev)
    gen.manual_seed(0)

    def rnd(t):
        return (torch.randn((t, H), generator=gen, device=dev) * 1.5).half()

    I, F, G = rnd(T), rnd(T), rnd(T)
    o = torch.empty((T, H), dtype=torch.float16, device=dev)
    A = torch.empty((T, H), dtype=torch.int8, device=dev)
    gam = torch.empty(T, dtype=torch.float32, device=dev)
    rs = torch.empty(T, dtype=torch.int32, device=dev)
    hT = torch.empty(H, dtype=torch.float32, device=dev)
    ws = mmf.workspace(mmf.mmf_mlgru_workspace_bytes(T, H), dev)
    I1, F1, G1 = rnd(1), rnd(1), rnd(1)
    o1 = torch.empty((1, H), dtype=torch.float16, device=dev)
    h1 = torch.zeros(H, dtype=torch.float32, device=dev)

    def plain():
        mmf.mmf_mlgru_forward(I, F, G, None, None, 1e-8, o, hT, ws, stream)

    def fused():
        mmf.mmf_mlgru_forward_quantized(I, F, G, None, None, 1e-8, None, 1e-8, A, gam, rs, hT,
                                        ws, stream)

    def decode():
        mmf.mmf_mlgru_forward(I1, F1, G1, h1, None, 1e-8, o1, h1, None, stream)

    hbm = measured_peaks()[0]
    out = {"workload": name, "T": T, "H": H, "dtype": "f16 in, f16 out (fused: int8 codes out)",
           "inputs": "seeded N(0, 1.5^2) on the device, 3 x %d MB resident, larger than L2"
                     % (T * H * 2 // 2 ** 20)}
    for label, fn, q, n, tokens in (("plain", plain, False, 50, T),
                                    ("fused_oproj_quant", fused, True, 50, T),
                                    ("decode_t1", decode, False, 2000, 1)):
        with torch.cuda.stream(stream):
            for _ in range(max(3, args.warmup)):
                fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(gpu_index(local_rank)) as clk:
            barrier()
            torch.cuda.synchronize()
            with torch.cuda.stream(stream):
                e0.record()
                for _ in range(n):
                    fn()
                e1.record()
            torch.cuda.synchronize()
            barrier()
        ms = reduce_max(e0.elapsed_time(e1) / n, world, dev)
        if mmf.mmf_get_device_status() != 0:
            raise RuntimeError("device status reported a timeout in the MLGRU leg")
        clocks = clk.summary()
        roof = mlgru_roofline(tokens, H, q, ms, hbm, clocks)
        roof["kernel"] = "mlgru call (chunk maps, carries, outputs)"
        roof["traffic"] = profiled_traffic("mlgru", name) if tokens == T else None
        out[label] = {
            "ms_per_call": round(ms, 4), "tokens_per_s": round(tokens * world / (ms * 1e-3), 1),
            "launches_per_call": 1 if tokens <= 32 else 3, "calls": n,
            "roofline": roof, "clocks": clocks}
    del I, F, G, o, A, ws
    torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------------------- backward
def time_backward(args, dev, stream, world, local_rank):
    """Times, per projection, the input-gradient call (dx: codes transposed, fp16 contraction
    over N, norm step) and the weight-gradient call (dW: gradient and codes transposed, fp16
    contraction over the tokens), with the forward's inputs, codes and the output gradients
    resident in HBM.  Events between the calls split a step into its two halves."""
    import torch
    import ternary_weight_lm_b200 as mmf

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    name, T, H, I = BACKWARD_SHAPE
    if args.backward_tokens != T:
        T = args.backward_tokens
        name = f"hgrn1p3b_layer_backward_t{T}"
    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    projs = [("i", "attn", H, H), ("f", "attn", H, H), ("g", "attn", H, H), ("o", "o", H, H),
             ("gate", "mlp", H, 2 * I), ("down", "h", I, H)]
    xs, codes = {}, {}
    for src, K in (("attn", H), ("o", H), ("mlp", H), ("h", I)):
        x = torch.randn((T, K), generator=gen, device=dev).half()
        A = torch.empty((T, K), dtype=torch.int8, device=dev)
        gam = torch.empty(T, dtype=torch.float32, device=dev)
        torch.cuda.synchronize()     # x was written on the current stream
        mmf.mmf_quantize_activations(x, None, 1e-8, A, gam, None, stream)
        xs[src], codes[src] = x, (A, gam)
    ps = []
    for pname, src, K, N in projs:
        W = torch.randn((N, K), generator=gen, device=dev) * 0.02
        Wp, beta = mmf.quantize_weights(W, stream)
        torch.cuda.synchronize()
        del W
        dy = torch.randn((T, N), generator=gen, device=dev).half()
        dx = torch.empty((T, K), dtype=torch.float16, device=dev)
        dW = torch.empty((N, K), dtype=torch.float32, device=dev)
        ps.append((pname, src, K, N, Wp, beta, dy, dx, dW))
    ws = mmf.workspace(max(mmf.mmf_backward_workspace_bytes(T, K, N) for _, _, K, N in projs),
                       dev)
    torch.cuda.synchronize()

    def step(marks=None):
        for pname, src, K, N, Wp, beta, dy, dx, dW in ps:
            A, gam = codes[src]
            mmf.mmf_bitlinear_backward(xs[src], None, 1e-8, A, gam, Wp, beta, N, dy, dx, None,
                                       None, ws, stream)
            if marks is not None:
                marks.append(("dgrad", 2.0 * T * N * K, torch.cuda.Event(enable_timing=True)))
                marks[-1][2].record(stream)
            mmf.mmf_bitlinear_backward(xs[src], None, 1e-8, A, gam, Wp, beta, N, dy, None, dW,
                                       None, ws, stream)
            if marks is not None:
                marks.append(("wgrad", 2.0 * T * N * K, torch.cuda.Event(enable_timing=True)))
                marks[-1][2].record(stream)

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            step()
    torch.cuda.synchronize()
    n = 8
    marks = []
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_index(local_rank)) as clk:
        barrier()
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            e0.record()
            for _ in range(n):
                step(marks)
            e1.record()
        torch.cuda.synchronize()
        barrier()
    ms = reduce_max(e0.elapsed_time(e1) / n, world, dev)
    if mmf.mmf_get_device_status() != 0:
        raise RuntimeError("device status reported a timeout in the backward leg")
    # each call's time runs from the previous mark (the timed region's start for the first)
    halves = {"dgrad": [0.0, 0.0], "wgrad": [0.0, 0.0]}
    prev = e0
    for kind, flops, ev in marks:
        halves[kind][0] += prev.elapsed_time(ev)
        halves[kind][1] += flops
        prev = ev
    flops_step = sum(4.0 * T * N * K for _, _, K, N, *_ in ps)
    _, bf16_burst, bf16_sust, peak_kind = measured_peaks()
    step_tflops = flops_step / (ms * 1e-3) / 1e12
    out = {"workload": name, "T": T, "hidden": H, "mlp": I,
           "projections": {p[0]: {"K": p[2], "N": p[3]} for p in ps},
           "dtype": "fp16 operands, fp32 accumulators (dx fp16, dW fp32)",
           "inputs": "seeded N(0,1) inputs and output gradients and the forward's codes, "
                     "resident in HBM",
           "ms_per_step": round(ms, 4), "tokens_per_s": round(T * world / (ms * 1e-3), 1),
           "steps": n, "calls_per_step": 2 * len(ps), "step_tflops": round(step_tflops, 1),
           "roofline": {"bound": "tensor", "kernel": "whole backward step",
                        "achieved": round(step_tflops, 1), "peak": round(bf16_burst, 1),
                        "unit": "TFLOP/s", "frac": round(step_tflops / bf16_burst, 4),
                        "peak_source": f"{peak_kind} bf16 dense burst (fp16 runs at the same "
                                       f"nominal rate)"},
           "clocks": clk.summary()}
    for kind, (t_ms, fl) in halves.items():
        achieved = fl / (t_ms * 1e-3) / 1e12
        out[kind] = {
            "ms_per_step": round(t_ms / n, 4),
            "roofline": {"bound": "tensor",
                         "kernel": kind + " calls: the fp16 pair GEMM (kind::f16) with the "
                                          "transpose and norm launches around it",
                         "achieved": round(achieved, 1), "peak": round(bf16_burst, 1),
                         "unit": "TFLOP/s", "frac": round(achieved / bf16_burst, 4),
                         "frac_of_sustained": round(achieved / bf16_sust, 4),
                         "flops_per_step": fl / n}}
    del ps, xs, codes, ws
    torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------------------- oracle arm
def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def oracle_sample(wl, n_tokens, dataflow="path"):
    """Inputs of a bounded sample of one step for the oracle: the first n_tokens tokens of the
    first layer's step inputs (the same seeded activations as the GPU arm's) and one layer's
    weights, quantised by the oracle itself."""
    import oracle
    H = wl.projections[0].K
    xdt = np.float32 if wl.x_dtype == "f32" else np.float16
    srcs = sorted({SOURCE_OF.get(p.name, "x_attn") for p in wl.projections} - {"h"})
    xs = {}
    for src in (srcs if dataflow == "path" else ["x_attn"]):
        x = synth.activations(0, src, wl.T, H, dtype=xdt, outlier_frac=wl.outlier_frac,
                              outlier_scale=wl.outlier_scale)
        xs[src] = np.ascontiguousarray(x[:n_tokens])
        del x
    weights = {}
    for p in wl.projections:
        W = synth.weights(0, p.name, p.N, p.K)
        beta = oracle.absmean_beta(W)
        weights[p.name] = (oracle.ternary_codes(W, beta), beta)
    return xs, weights


def oracle_step(wl, xs, weights, dataflow="path", pool=None, nthreads=1):
    """One layer of the step in the same data flow as the GPU arm, outputs rounded to the output
    dtype where they feed the next projection.  With a thread pool, each projection's output
    rows (weight rows) are split over `nthreads` threads, each running the oracle's own
    accumulation on its rows (the oracle's C code runs without the interpreter lock)."""
    import oracle
    ydt = np.float32 if wl.y_dtype == "f32" else np.float16
    level_of = DATAFLOWS[dataflow]
    outs, quant = {}, {}
    for p in sorted(wl.projections, key=lambda q: level_of[q.name]):
        if p.name == "down_proj":
            xin = outs["gate_proj"]
        elif dataflow == "path":
            xin = xs[SOURCE_OF.get(p.name, "x_attn")]
        elif p.name in ("i_proj", "f_proj", "g_proj", "proj"):
            xin = xs["x_attn"]
        elif p.name == "o_proj":
            xin = outs["g_proj"]
        else:
            xin = outs["o_proj"]
        c, beta = weights[p.name]
        key = id(xin)
        if key not in quant:
            quant[key] = oracle.rmsnorm_actquant(xin)
        q, gamma, _ = quant[key]
        if pool is None or nthreads <= 1:
            acc = oracle.ternary_accumulate(q, c)
        else:
            bounds = np.linspace(0, c.shape[0], nthreads + 1).astype(int)
            parts = list(pool.map(lambda ab: oracle.ternary_accumulate(q, c[ab[0]:ab[1]]),
                                  [(bounds[i], bounds[i + 1]) for i in range(nthreads)
                                   if bounds[i + 1] > bounds[i]]))
            acc = np.concatenate(parts, axis=1)
        y = oracle.dequant(acc, gamma, beta)
        if p.glu:
            y = oracle.silu_glu(y)
        outs[p.name] = y.astype(ydt)
    return outs


def _time_oracle(wl, xs, weights, n_tokens, seconds, dataflow, nthreads):
    xs = {k: np.ascontiguousarray(v[:n_tokens]) for k, v in xs.items()}
    pool = concurrent.futures.ThreadPoolExecutor(nthreads) if nthreads > 1 else None
    try:
        oracle_step(wl, xs, weights, dataflow, pool, nthreads)       # warm
        reps, t0 = 0, time.perf_counter()
        while True:
            oracle_step(wl, xs, weights, dataflow, pool, nthreads)
            reps += 1
            el = time.perf_counter() - t0
            if el >= seconds:
                break
    finally:
        if pool is not None:
            pool.shutdown()
    # one sample step covers one layer; a full step streams wl.layers layers
    return n_tokens * reps / el / wl.layers, reps, el


def oracle_tokens_per_s(wl, seconds, dataflow="path", threads=None):
    """The oracle on bounded samples of the step: one host thread, and all host cores with the
    output rows of each projection split over threads.  Token counts are sized so that each
    leg runs about `seconds`; prefill-sized steps use a slice of their tokens (at most 256),
    marked as extrapolated."""
    threads = threads or max(1, min(os.cpu_count() or 1, 64))
    xs, weights = oracle_sample(wl, min(wl.T, 256), dataflow)
    # the cost of one token through one layer, single-threaded
    t1, _, _ = _time_oracle(wl, xs, weights, 1, 0.0, dataflow, 1)
    per_tok = 1.0 / max(t1 * wl.layers, 1e-9)
    n_single = int(max(1, min(wl.T, 256, seconds / per_tok / 2)))
    n_thr = int(max(1, min(wl.T, 256, seconds * threads / per_tok / 2)))
    v1, r1, el1 = _time_oracle(wl, xs, weights, n_single, seconds, dataflow, 1)
    vt, rt, elt = _time_oracle(wl, xs, weights, n_thr, seconds, dataflow, threads)

    def leg(v, n, reps, el, th):
        return {"value": round(v, 3), "unit": "tokens/s", "threads": th,
                "sample": f"first {n} of {wl.T} tokens through all {len(wl.projections)} "
                          f"projections of one layer ({dataflow} data flow), repeated {reps} "
                          f"times ({el:.1f} s); tokens/s scaled by 1/{wl.layers} layers",
                "extrapolated": n < wl.T}
    single = leg(v1, n_single, r1, el1, 1)
    threaded = leg(vt, n_thr, rt, elt, threads)
    return vt, {"kind": "oracle", "value": round(vt, 3), "unit": "tokens/s", "cores": threads,
                "sample": threaded["sample"] + (" (extrapolated from the slice)"
                                                if threaded["extrapolated"] else ""),
                "single": single, "threaded": threaded,
                "hardware_concurrency": os.cpu_count(), "cpu_model": cpu_model()}


def run_reference(args, rank, world):
    wl = synth.WORKLOADS[args.workload]
    if rank != 0:
        return None
    # size each step so that warm-up + K steps stay within about two minutes
    df = args.dataflow
    threads = max(1, min(os.cpu_count() or 1, 64))
    pool = concurrent.futures.ThreadPoolExecutor(threads) if threads > 1 else None
    try:
        xs, weights = oracle_sample(wl, 1, df)
        t0 = time.perf_counter()
        oracle_step(wl, xs, weights, df, pool, threads)
        per_token_layer = time.perf_counter() - t0
        n_tok = int(max(1, min(wl.T, 256,
                               120.0 / max(1, args.steps + args.warmup) / per_token_layer)))
        xs, weights = oracle_sample(wl, n_tok, df)
        for _ in range(args.warmup):
            oracle_step(wl, xs, weights, df, pool, threads)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            oracle_step(wl, xs, weights, df, pool, threads)
        el = time.perf_counter() - t0
    finally:
        if pool is not None:
            pool.shutdown()
    tps = n_tok * args.steps / el / wl.layers
    cpu = {"kind": "oracle", "cores": threads, "value": round(tps, 3), "unit": "tokens/s",
           "sample": f"each step: first {n_tok} of {wl.T} tokens through every projection of "
                     f"one layer, output rows split over {threads} threads; tokens/s scaled by "
                     f"1/{wl.layers} layers" + (" (extrapolated)" if n_tok < wl.T else ""),
           "hardware_concurrency": os.cpu_count(), "cpu_model": cpu_model()}
    return {"impl": "reference", "metric": METRIC, "value": round(tps, 3), "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": config_of(wl, df), "cpu_baseline": cpu,
            "e2e": {"value": round(tps, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def config_of(wl, dataflow="path"):
    return {"workload": wl.name, "tokens_per_step": wl.T, "layers_per_step": wl.layers,
            "projections": ",".join(p.name + ("(glu)" if p.glu else "") for p in wl.projections),
            "x_dtype": wl.x_dtype, "y_dtype": wl.y_dtype, "parallelism": "replicas",
            "dataflow": DATAFLOW_TEXT[dataflow]}


def timing_setup(wl, res):
    return {"weight_copies": res["copies"],
            "l2": ("packed weights rotate over %d distinct copies (%.0f MB > 2x L2); "
                   "activations as a layer-by-layer step leaves them"
                   % (res["copies"], res["copies"] * wl.packed_bytes_per_layer * wl.layers / 1e6)),
            "timing": "CUDA graph replays of whole steps, CUDA events on the launch stream",
            "kernel_timing": res["kernel_timing"]}


# ----------------------------------------------------------------------------- main
def main(argv=None):
    args = parse_args(argv)
    rank, world, local_rank = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "gloo" if args.impl == "reference" else "nccl"
        if backend == "nccl":
            import torch
            torch.cuda.set_device(local_rank)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    try:
        if args.impl == "reference":
            line = run_reference(args, rank, world)
        else:
            res = run_gpu(args, rank, world, local_rank)
            wl = synth.WORKLOADS[args.workload]
            line = None
            if rank == 0:
                line = {
                    "metric": METRIC, "value": round(res["value"], 1), "unit": "tokens/s",
                    "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                    "ms_per_step": round(res["ms_per_step"], 6), "higher_is_better": True,
                    "scaling": "weak", "vs_baseline": None, "dtype": "int8",
                    "data": "synthetic", "config": config_of(wl, args.dataflow),
                    "timing_setup": timing_setup(wl, res),
                    "weight_gbs": round(res["weight_gbs"], 1),
                    "int8_tops": round(res["int8_tops"], 2),
                    "path": res["path"],
                    "roofline": res["roofline"], "kernels": res["kernels"],
                    "clocks": res["clocks"], "e2e": res["e2e"],
                    "gpu_launches": res["launches"],
                    "decode": res["decode"],
                }
                for k in ("mlgru", "backward"):
                    if k in res:
                        line[k] = res[k]
                if not args.no_cpu_baseline and world == 1:
                    _, cpu = oracle_tokens_per_s(wl, args.cpu_seconds, dataflow=args.dataflow)
                    line["cpu_baseline"] = cpu
                else:
                    line["cpu_baseline"] = None
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

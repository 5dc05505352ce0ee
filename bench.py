#!/usr/bin/env python
"""Benchmark of the blockwise-FP8 training-linear hot path on B200.

One step = the whole hot path over the linear stack of one 28-layer
Qwen3-1.7B-shaped training step at M = 16384 tokens (4 x 4096): for every
layer and each of its four linears (QKV 2048->4096, O 2048->2048, gate/up
2048->12288, down 6144->2048):
  1. 128x128 block quantisation of W (codes + transposed codes + scales;
     the four weights of a layer in one launch)
  2. row-wise + column-wise 1x128 / 128x1 quantisation of X (one pass)
  3. fprop  Y  = X W^T
  4. row-wise + column-wise quantisation of dY (one pass)
  5. dgrad  dX = dY W
  6. wgrad  dW = dY^T X
= 588 kernel launches (28 x (1 + 4 x 5)), 138.5 TFLOP of GEMM work per step.

Inputs are seeded synthetic tensors (synthetic/): X ~ N(0,1) with 0.1% x50
outliers, W ~ N(0,0.02), dY ~ N(0,1e-3) with 0.1% x100 outliers. Every layer
reuses its linear's input buffers; between two uses of a buffer the step
streams more than 1 GB through HBM (8x the 126 MB L2), so every launch reads
cold data ("inputs larger than L2").

Metric: GEMM TFLOP/s of the whole step (quantiser time included in the step
time). The JSON line also carries per-kernel achieved TFLOP/s or GB/s (CUDA
events around every launch of the timed region), the roofline of the
dominant kernel, the clocks seen during the timed region, an end-to-end
number with host<->device copies in the timed region, and the CPU oracle on
a bounded sample of the same workload.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

WORKLOAD = "stack28_m16384"
LAYERS = 28
KINDS = ("qkv", "o", "gate_up", "down")
TOKENS = 16384
METRIC = ("blockwise-FP8 GEMM TFLOP/s (fwd/dgrad/wgrad) & % FP8 peak; "
          "quantize GB/s % HBM")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0,
                  "bf16_tflops_sustained": 1400.0}
FP8_OVER_BF16 = 2.0   # nominal dense FP8 / BF16 tensor throughput (4.5 / 2.25)

# DRAM bytes (read + write) per launch of each kernel kind, from one ncu
# capture (gpu__time_duration.sum, dram__bytes_read.sum, dram__bytes_write.sum)
# of a one-layer step: its 18 launches are those every layer of the full step
# repeats at the same sizes, so their per-kind average is the full step's
# (profiles/dram_layer_m16384.md). Valid only for the kernel sources they were
# taken on: KERNEL_FINGERPRINT is kernel_fingerprint() of the sources at that
# time, and the numbers are reported as null once the code differs.
NCU_TRAFFIC_PER_LAUNCH = {
    "gemm_block_scaled": 184835040,
    "gemm_vector_scaled": 1189339648,
    "quant_rowcol": 217172992,
    "quant_weight_block": 147285760,
}
KERNEL_FINGERPRINT = "37a8d0789a95e96b"


def kernel_fingerprint():
    """sha256 (first 16 hex digits) of csrc/*.cu[h] in name order, each with
    its comments removed and whitespace collapsed: it changes with the code,
    not with its comments."""
    import hashlib
    import re
    h = hashlib.sha256()
    d = os.path.join(ROOT, "blockwise_fp8_linear_fp8bw_b200", "csrc")
    for f in sorted(os.listdir(d)):
        if f.endswith((".cu", ".cuh")):
            with open(os.path.join(d, f)) as fh:
                src = fh.read()
            src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
            src = re.sub(r"//[^\n]*", " ", src)
            h.update(" ".join(src.split()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel):
    if kernel_fingerprint() != KERNEL_FINGERPRINT:
        return None
    return NCU_TRAFFIC_PER_LAUNCH.get(kernel)


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-next-rows", action="store_true",
                   help="skip the timing of the rows beyond the step")
    p.add_argument("--layers", type=int, default=28,
                   help="layers per step (profiling runs use fewer)")
    p.add_argument("--linears", default="qkv,o,gate_up,down",
                   help="comma list of the linears in a layer")
    args = p.parse_args(argv)
    global LAYERS, KINDS
    LAYERS = args.layers
    KINDS = tuple(args.linears.split(","))
    return args


def kinds():
    from synthetic import LINEARS
    return [(kind, LINEARS[kind][0], LINEARS[kind][1]) for kind in KINDS]


def step_gemm_flops():
    return LAYERS * 3 * sum(2 * TOKENS * n * k for _, k, n in kinds())


def dist_env():
    """(world size, rank, local rank) as set by torchrun (1, 0, 0 otherwise)."""
    return (int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def free_port():
    import socket
    with socket.socket() as sock:
        sock.bind(("127.0.0.1", 0))
        return sock.getsockname()[1]


def launch_ranks(n, argv, script=None, timeout_s=3600):
    """Start `n` ranks of `script` (this file by default) with the arguments
    `argv`, one process per GPU on this node, under torch.distributed.run
    with a 127.0.0.1 rendezvous; returns the launcher's exit status. The
    launcher runs in its own process group, ended as a whole if it outlives
    `timeout_s`."""
    import signal
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           "--nproc-per-node", str(n), "--master-addr", "127.0.0.1",
           "--master-port", str(free_port()),
           script or os.path.abspath(__file__)] + list(argv)
    proc = subprocess.Popen(cmd, start_new_session=True)
    try:
        return proc.wait(timeout=timeout_s)
    except subprocess.TimeoutExpired:
        os.killpg(proc.pid, signal.SIGTERM)
        try:
            proc.wait(timeout=60)
        except subprocess.TimeoutExpired:
            os.killpg(proc.pid, signal.SIGKILL)
            proc.wait()
        return 124


def check_launch(gpus):
    """None when this process should run the benchmark itself; else the exit
    status to return: `--gpus N` (N > 1) outside a torchrun launch starts N
    ranks (launch_ranks) and reports their status; inside one, WORLD_SIZE
    must equal N."""
    if "WORLD_SIZE" not in os.environ:
        if gpus > 1:
            return launch_ranks(gpus, sys.argv[1:])
        return None
    world = int(os.environ["WORLD_SIZE"])
    if world != gpus:
        sys.stderr.write("bench.py: --gpus %d but WORLD_SIZE=%d (torchrun "
                         "--nproc-per-node must equal --gpus)\n"
                         % (gpus, world))
        return 2
    return None


def max_over_ranks(value, world, device):
    """The largest `value` over all ranks (an all-reduce MAX); the step time
    of a multi-GPU run is the slowest rank's."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(world, work_per_rank, seconds):
    """Whole-job throughput: every rank processes `work_per_rank` units in
    the (max-over-ranks) time `seconds`."""
    return world * work_per_rank / seconds


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
        return {"hbm_gbs": float(d["hbm_gbs"]),
                "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d["bf16_tflops_sustained"]),
                "source": "measured"}
    except Exception:
        d = dict(FALLBACK_PEAKS)
        d["source"] = "fallback"
        return d


# --------------------------------------------------------------------------
# CPU oracle on a bounded sample (the reference arm, and the cpu_baseline)
# --------------------------------------------------------------------------

class OracleSample:
    """The four linears of one layer at a reduced token count M' (instead of
    16384), plus quantisation of the same fraction of each weight; every GEMM
    and quantiser of the step scales linearly with M', so the sample's
    throughput stands for the step's."""

    def __init__(self, tokens):
        import oracle
        import synthetic as S
        self.oracle = oracle
        self.tokens = tokens
        self.threads = oracle.default_threads()
        self.items = []
        for kind, k, n in kinds():
            lin = S.Linear(kind, tokens, k, n, ("fprop", "dgrad", "wgrad"))
            w = S.draw_w(lin)
            qw, sw, _ = oracle.quantize_weight_block(w, want_transposed=False)
            wrows = max(16, (n * tokens // TOKENS) // 16 * 16)
            self.items.append(dict(x=S.draw_x(lin), dy=S.draw_dy(lin),
                                   w_slab=np.ascontiguousarray(w[:wrows]),
                                   qw=qw, sw=sw, m=tokens, n=n, k=k))
        self.flops = sum(3 * 2 * it["m"] * it["n"] * it["k"]
                         for it in self.items)

    def run(self):
        o = self.oracle
        nt = self.threads
        for it in self.items:
            o.quantize_weight_block(it["w_slab"], want_transposed=True)
            qx, sx = o.quantize_rowwise(it["x"])
            qx_t, sx_t = o.quantize_colwise(it["x"])
            o.gemm_fprop(qx, sx, it["qw"], it["sw"], nthreads=nt)
            qdy, sdy = o.quantize_rowwise(it["dy"])
            qdy_t, sdy_t = o.quantize_colwise(it["dy"])
            o.gemm_dgrad(qdy, sdy, it["qw"], it["sw"], nthreads=nt)
            o.gemm_wgrad(qdy_t, sdy_t, qx_t, sx_t, nthreads=nt)

    def describe(self):
        return ("the 4 linears of one layer (QKV, O, gate/up, down) at %d "
                "tokens instead of %d (1/%d of every GEMM and activation "
                "quantisation) plus 1/%d of each weight's block quantisation; "
                "fp64 oracle GEMMs on %d threads"
                % (self.tokens, TOKENS, TOKENS // self.tokens,
                   TOKENS // self.tokens, self.threads))


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:          # the CPU oracle runs once, on rank 0
        return 0
    sample = OracleSample(tokens=64)
    for _ in range(args.warmup):
        sample.run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        sample.run()
    dt = (time.perf_counter() - t0) / args.steps
    value = sample.flops / dt / 1e12
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": dt * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "layers": LAYERS, "tokens": TOKENS,
                   "sample_tokens": sample.tokens},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s",
                         "cores": sample.threads, "kind": "oracle",
                         "sample": sample.describe()},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# --------------------------------------------------------------------------
# GPU arm
# --------------------------------------------------------------------------

class LinearBuffers:
    """Device buffers of one linear kind (inputs + every intermediate)."""

    def __init__(self, kind, k, n, device):
        import torch
        import synthetic as S
        self.kind, self.k, self.n = kind, k, n
        m = TOKENS
        lin = S.Linear(kind, m, k, n, ("fprop", "dgrad", "wgrad"))
        self.host_x = S.draw_x(lin)
        self.host_w = S.draw_w(lin)
        self.host_dy = S.draw_dy(lin)

        def dev_bf16(a):
            t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
            return t.to(device)

        def e(shape, dt):
            return torch.empty(shape, dtype=dt, device=device)

        u8, f32, bf = torch.uint8, torch.float32, torch.bfloat16
        self.x, self.w, self.dy = (dev_bf16(self.host_x),
                                   dev_bf16(self.host_w),
                                   dev_bf16(self.host_dy))
        cd = lambda a: (a + 127) // 128  # noqa: E731
        self.qw, self.sw, self.qw_t = e((n, k), u8), e((cd(n), cd(k)), f32), \
            e((k, n), u8)
        self.qx, self.sx = e((m, k), u8), e((cd(k), m), f32)
        self.qx_t, self.sx_t = e((k, m), u8), e((cd(m), k), f32)
        self.qdy, self.sdy = e((m, n), u8), e((cd(n), m), f32)
        self.qdy_t, self.sdy_t = e((n, m), u8), e((cd(m), n), f32)
        self.y, self.dx, self.dw = e((m, n), bf), e((m, k), bf), e((n, k), bf)

    def weight_bytes(self):
        """Algorithmic bytes of this weight's block quantisation (bf16 in,
        codes, transposed codes, scales)."""
        n, k = self.n, self.k
        cd = lambda a: (a + 127) // 128  # noqa: E731
        return n * k * 2 + 2 * n * k + 4 * cd(n) * cd(k)

    def ops(self, o, stream, pow2=False):
        """[(kernel kind, algorithmic units, callable)] of this linear after
        its weight is quantised and before its weight gradient (layer_ops
        quantises a layer's weights in one launch and computes its weight
        gradients in another); pow2 selects the power-of-two-scale quantisers
        and GEMMs."""
        m, k, n = TOKENS, self.k, self.n
        cd = lambda a: (a + 127) // 128  # noqa: E731
        xq_bytes = m * k * 2 + 2 * m * k + 4 * (m * cd(k) + cd(m) * k)
        dyq_bytes = m * n * 2 + 2 * m * n + 4 * (m * cd(n) + cd(m) * n)
        f = 2 * m * n * k
        p2 = pow2
        return [
            ("quant_rowcol", xq_bytes,
             lambda: o.fp8bw_quantize_colwise(self.x, self.qx_t, self.sx_t,
                                              self.qx, self.sx, stream,
                                              pow2=p2)),
            ("gemm_block_scaled", f,
             lambda: o.fp8bw_gemm_fprop(self.qx, self.sx, self.qw, self.sw,
                                        self.y, stream, pow2=p2)),
            ("quant_rowcol", dyq_bytes,
             lambda: o.fp8bw_quantize_colwise(self.dy, self.qdy_t,
                                              self.sdy_t, self.qdy,
                                              self.sdy, stream, pow2=p2)),
            ("gemm_block_scaled", f,
             lambda: o.fp8bw_gemm_dgrad(self.qdy, self.sdy, self.qw_t, 1,
                                        self.sw, self.dx, stream, pow2=p2)),
        ]

    def wgrad_job(self):
        """(qdy_t, sdy_t, qx_t, sx_t, dw) of this linear's weight gradient."""
        return (self.qdy_t, self.sdy_t, self.qx_t, self.sx_t, self.dw)


def layer_ops(bufs, o, stream, pow2=False):
    """The ops of one layer: its weights' 128x128 block quantisation in one
    launch (all weights are quantised once per step, before they are used),
    then each linear's quantisers, fprop and dgrad, then the weight gradients
    of all its linears in one launch (they contract over the same tokens; a
    backward pass can defer them until the layer's dY are all known)."""
    ws = [b.w for b in bufs]
    qs, ss, qts = [b.qw for b in bufs], [b.sw for b in bufs], [b.qw_t for b in bufs]
    out = [("quant_weight_block", sum(b.weight_bytes() for b in bufs),
            lambda: o.fp8bw_quantize_weight_block_batch(ws, qs, ss, qts, stream,
                                                        pow2=pow2))]
    for b in bufs:
        out.extend(b.ops(o, stream, pow2=pow2))
    out.append(("gemm_vector_scaled", sum(2 * TOKENS * b.n * b.k for b in bufs),
                lambda: o.fp8bw_gemm_wgrad_batch([b.wgrad_job() for b in bufs],
                                                 stream, pow2=pow2)))
    return out


def linear_names(kinds):
    """'QKV, O, gate/up and down' for the linear kinds given, in order."""
    label = {"qkv": "QKV", "o": "O", "gate_up": "gate/up", "down": "down"}
    names = [label.get(k, k) for k in kinds]
    if len(names) < 2:
        return "".join(names)
    return ", ".join(names[:-1]) + " and " + names[-1]


def time_next_rows(o, bufs, stream, warmup, rounds):
    """Rows beyond the step, timed after it on the same buffers (not part of
    `value`): wgrad with an fp32 dW added into an fp32 main-grad buffer, the
    four linears of a layer in one launch (their operands together exceed
    L2)."""
    import torch
    dev = bufs[0].qx_t.device
    names = linear_names([b.kind for b in bufs])
    grads = [torch.zeros((b.n, b.k), dtype=torch.float32, device=dev)
             for b in bufs]
    jobs = [b.wgrad_job()[:4] + (g,) for b, g in zip(bufs, grads)]
    calls = [(sum(2 * TOKENS * b.n * b.k for b in bufs),
              lambda: o.fp8bw_gemm_wgrad_f32_batch(jobs, True, stream))]
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            for _, fn in calls:
                fn()
    torch.cuda.synchronize()
    ev = [[(torch.cuda.Event(enable_timing=True),
            torch.cuda.Event(enable_timing=True)) for _ in calls]
          for _ in range(rounds)]
    with torch.cuda.stream(stream):
        for r in range(rounds):
            for (_, fn), (e0, e1) in zip(calls, ev[r]):
                e0.record(stream)
                fn()
                e1.record(stream)
    torch.cuda.synchronize()
    o.fp8bw_check_device_error(stream)
    ms = sum(e0.elapsed_time(e1) for r in ev for e0, e1 in r)
    flop = rounds * sum(f for f, _ in calls)
    out = {"wgrad_f32_accumulate": {
        "achieved": flop / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
        "launches": rounds * len(calls), "avg_launch_ms": ms / (rounds * len(calls)),
        "what": "dW (fp32) += dY^T X for the %s linears at M=%d, one "
                "launch for all; timed after the step" % (names, TOKENS)}}

    # fprop and dgrad that also quantise their own bf16 output row-wise,
    # against the same GEMMs followed by the row-wise quantiser.
    def seq_time(seq, rounds=3):
        with torch.cuda.stream(stream):
            for _ in range(warmup):
                for fn in seq:
                    fn()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b_ = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record(stream)
            for _ in range(rounds):
                for fn in seq:
                    fn()
            b_.record(stream)
        torch.cuda.synchronize()
        o.fp8bw_check_device_error(stream)
        return a.elapsed_time(b_) / rounds

    fused, unfused = [], []
    for b in bufs:
        m = TOKENS
        u8, f32 = torch.uint8, torch.float32
        qy = torch.empty((m, b.n), dtype=u8, device=dev)
        sy = torch.empty(((b.n + 127) // 128, m), dtype=f32, device=dev)
        qdx = torch.empty((m, b.k), dtype=u8, device=dev)
        sdx = torch.empty(((b.k + 127) // 128, m), dtype=f32, device=dev)
        fused += [
            (lambda b=b, qy=qy, sy=sy: o.fp8bw_gemm_fprop_quant(
                b.qx, b.sx, b.qw, b.sw, b.y, qy, sy, stream)),
            (lambda b=b, qdx=qdx, sdx=sdx: o.fp8bw_gemm_dgrad_quant(
                b.qdy, b.sdy, b.qw_t, 1, b.sw, b.dx, qdx, sdx, stream))]
        unfused += [
            (lambda b=b: o.fp8bw_gemm_fprop(b.qx, b.sx, b.qw, b.sw, b.y,
                                            stream)),
            (lambda b=b, qy=qy, sy=sy: o.fp8bw_quantize_rowwise(b.y, qy, sy,
                                                                stream)),
            (lambda b=b: o.fp8bw_gemm_dgrad(b.qdy, b.sdy, b.qw_t, 1, b.sw,
                                            b.dx, stream)),
            (lambda b=b, qdx=qdx, sdx=sdx: o.fp8bw_quantize_rowwise(
                b.dx, qdx, sdx, stream))]
    t_f = seq_time(fused)
    t_u = seq_time(unfused)
    gfl = 2 * sum(2 * TOKENS * b.n * b.k for b in bufs)
    out["gemm_fused_rowwise_quant"] = {
        "achieved": gfl / (t_f * 1e-3) / 1e12, "unit": "TFLOP/s",
        "ms_fused": t_f, "ms_gemm_then_quantiser": t_u,
        "saved_frac": 1.0 - t_f / t_u,
        "what": "fprop and dgrad of the %s linears (M=%d) writing bf16 "
                "plus the row-wise E4M3 codes and scales of that output, "
                "against the same GEMMs followed by the row-wise quantiser; "
                "timed after the step" % (names, TOKENS)}
    del qy, sy, qdx, sdx

    # ... and writing both the row-wise and the transposed column-wise codes
    # (all a consumer linear needs), against the GEMMs followed by the
    # one-pass row + column quantiser.
    fused, unfused = [], []
    for b in bufs:
        m = TOKENS
        u8, f32 = torch.uint8, torch.float32
        cd = lambda a: (a + 127) // 128  # noqa: E731
        qy, sy = (torch.empty((m, b.n), dtype=u8, device=dev),
                  torch.empty((cd(b.n), m), dtype=f32, device=dev))
        qy_t, sy_t = (torch.empty((b.n, m), dtype=u8, device=dev),
                      torch.empty((cd(m), b.n), dtype=f32, device=dev))
        qdx, sdx = (torch.empty((m, b.k), dtype=u8, device=dev),
                    torch.empty((cd(b.k), m), dtype=f32, device=dev))
        qdx_t, sdx_t = (torch.empty((b.k, m), dtype=u8, device=dev),
                        torch.empty((cd(m), b.k), dtype=f32, device=dev))
        fused += [
            (lambda b=b, o4=(qy, sy, qy_t, sy_t): o.fp8bw_gemm_fprop_quant_rowcol(
                b.qx, b.sx, b.qw, b.sw, b.y, *o4, stream)),
            (lambda b=b, o4=(qdx, sdx, qdx_t, sdx_t): o.fp8bw_gemm_dgrad_quant_rowcol(
                b.qdy, b.sdy, b.qw_t, 1, b.sw, b.dx, *o4, stream))]
        unfused += [
            (lambda b=b: o.fp8bw_gemm_fprop(b.qx, b.sx, b.qw, b.sw, b.y,
                                            stream)),
            (lambda b=b, o4=(qy_t, sy_t, qy, sy): o.fp8bw_quantize_colwise(
                b.y, *o4, stream)),
            (lambda b=b: o.fp8bw_gemm_dgrad(b.qdy, b.sdy, b.qw_t, 1, b.sw,
                                            b.dx, stream)),
            (lambda b=b, o4=(qdx_t, sdx_t, qdx, sdx): o.fp8bw_quantize_colwise(
                b.dx, *o4, stream))]
    t_f = seq_time(fused)
    t_u = seq_time(unfused)
    out["gemm_fused_rowcol_quant"] = {
        "achieved": gfl / (t_f * 1e-3) / 1e12, "unit": "TFLOP/s",
        "ms_fused": t_f, "ms_gemm_then_quantiser": t_u,
        "saved_frac": 1.0 - t_f / t_u,
        "what": "fprop and dgrad of the %s linears (M=%d) writing bf16 "
                "plus the row-wise and the transposed column-wise E4M3 codes "
                "and scales of that output, against the same GEMMs followed "
                "by the one-pass row + column quantiser; timed after the "
                "step" % (names, TOKENS)}
    del fused, unfused

    # The whole step again with power-of-two scales (quantisers and GEMMs on
    # the tensor cores' UE8M0 block scaling), same buffers and order.
    step = []
    for _layer in range(LAYERS):
        step.extend(layer_ops(bufs, o, stream, pow2=True))
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            for _, _, fn in step:
                fn()
    torch.cuda.synchronize()
    steps = 3
    evs = [[(torch.cuda.Event(enable_timing=True),
             torch.cuda.Event(enable_timing=True)) for _ in step]
           for _ in range(steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record(stream)
        for s in range(steps):
            for (_, _, fn), (e0, e1) in zip(step, evs[s]):
                e0.record(stream)
                fn()
                e1.record(stream)
        t1.record(stream)
    torch.cuda.synchronize()
    o.fp8bw_check_device_error(stream)
    step_ms = t0.elapsed_time(t1) / steps
    kinds_ = {}
    for s in range(steps):
        for (kk, units, _), (e0, e1) in zip(step, evs[s]):
            d = kinds_.setdefault(kk, [0.0, 0])
            d[0] += e0.elapsed_time(e1)
            d[1] += units
    gflop = sum(u for kk, u, _ in step if kk.startswith("gemm"))
    out["pow2_step"] = {
        "achieved": gflop / (step_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
        "ms_per_step": step_ms, "steps": steps,
        "breakdown": {kk: (u / (ms_ * 1e-3) / 1e12 if kk.startswith("gemm")
                           else u / (ms_ * 1e-3) / 1e9)
                      for kk, (ms_, u) in kinds_.items()},
        "breakdown_units": "gemm_*: TFLOP/s, quant_*: GB/s",
        "what": "the same %d-layer step with power-of-two scales (s = 2^E, "
                "the smallest E with 448*2^E >= amax) applied by the tensor "
                "cores' UE8M0 block scaling; timed after the step" % LAYERS}
    out["configs"] = time_configs(o, bufs, stream)
    return out


def time_configs(o, bufs, stream, rounds=5):
    """The single-linear workloads of the parity configurations, one kernel
    at a time, each launch timed by CUDA events after an L2 flush (256 MB
    written): the QKV fprop at 8192 tokens, the MLP fprop (gate/up, down) and
    the MLP backward (dgrad and wgrad of down and gate/up) at 16384 tokens,
    with the quantisers of their inputs. Operands are the step's buffers
    (codes quantised during the step) where the shapes match."""
    import torch
    dev = bufs[0].x.device
    by = {b.kind: b for b in bufs}
    flush = torch.empty((256 << 20) if dev.type == "cuda" else 1024, dtype=torch.uint8,
                        device=dev)
    cd = lambda a: (a + 127) // 128  # noqa: E731

    def timed(fn):
        with torch.cuda.stream(stream):
            fn()
            fn()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(rounds)]
        with torch.cuda.stream(stream):
            for e0, e1 in evs:
                flush.zero_()
                e0.record(stream)
                fn()
                e1.record(stream)
        torch.cuda.synchronize()
        o.fp8bw_check_device_error(stream)
        return sum(e0.elapsed_time(e1) for e0, e1 in evs) / rounds

    rows = {}

    def gemm_row(name, m, n, k, fn):
        ms = timed(fn)
        rows[name] = {"achieved": 2 * m * n * k / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                      "us": ms * 1e3, "shape": [m, n, k]}

    def quant_row(name, nbytes, fn):
        ms = timed(fn)
        rows[name] = {"achieved": nbytes / (ms * 1e-3) / 1e9, "unit": "GB/s",
                      "us": ms * 1e3, "bytes": nbytes}

    if "qkv" in by:
        b, m = by["qkv"], TOKENS // 2
        x = b.x[:m]
        qx = torch.empty((m, b.k), dtype=torch.uint8, device=dev)
        sx = torch.empty((cd(b.k), m), dtype=torch.float32, device=dev)
        y = torch.empty((m, b.n), dtype=torch.bfloat16, device=dev)
        quant_row("qkv_m8192_quant_x_rowwise", m * b.k * 2 + m * b.k + 4 * m * cd(b.k),
                  lambda: o.fp8bw_quantize_rowwise(x, qx, sx, stream))
        gemm_row("qkv_m8192_fprop", m, b.n, b.k,
                 lambda: o.fp8bw_gemm_fprop(qx, sx, b.qw, b.sw, y, stream))
    m = TOKENS
    for kind in ("gate_up", "down"):
        if kind not in by:
            continue
        b = by[kind]
        xq = m * b.k * 2 + 2 * m * b.k + 4 * (m * cd(b.k) + cd(m) * b.k)
        dyq = m * b.n * 2 + 2 * m * b.n + 4 * (m * cd(b.n) + cd(m) * b.n)
        quant_row(kind + "_quant_x_rowcol", xq,
                  lambda b=b: o.fp8bw_quantize_colwise(b.x, b.qx_t, b.sx_t, b.qx, b.sx, stream))
        gemm_row(kind + "_fprop", m, b.n, b.k,
                 lambda b=b: o.fp8bw_gemm_fprop(b.qx, b.sx, b.qw, b.sw, b.y, stream))
        quant_row(kind + "_quant_dy_rowcol", dyq,
                  lambda b=b: o.fp8bw_quantize_colwise(b.dy, b.qdy_t, b.sdy_t, b.qdy, b.sdy,
                                                       stream))
        gemm_row(kind + "_dgrad", m, b.k, b.n,
                 lambda b=b: o.fp8bw_gemm_dgrad(b.qdy, b.sdy, b.qw_t, 1, b.sw, b.dx, stream))
        gemm_row(kind + "_wgrad", b.n, b.k, m,
                 lambda b=b: o.fp8bw_gemm_wgrad(b.qdy_t, b.sdy_t, b.qx_t, b.sx_t, b.dw,
                                                stream))
    del flush
    return {"rows": rows,
            "what": "the parity configurations' linears one kernel at a time, L2 "
                    "flushed before each launch (QKV fprop at M=%d; MLP fprop and "
                    "backward at M=%d); shape = [rows, cols, contraction]; timed "
                    "after the step" % (TOKENS // 2, TOKENS)}


class ClockSampler:
    """nvidia-smi samples every 200 ms; stop() summarises those taken inside
    the timed window (all of them if none fell inside)."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200", "-i",
                 gpu_id], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
        except Exception:
            self.proc = None

    def stop(self, window=None):
        """window: (start, end) in time.time() seconds of the timed region."""
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        return self.summarise(out, window)

    @staticmethod
    def summarise(out, window=None):
        import datetime
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        rows = []
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(
                    parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                ts = None
            try:
                rows.append((ts, float(parts[2]), float(parts[3]),
                             [n for n, v in zip(names, parts[6:10])
                              if v.lower().startswith("active")]))
            except ValueError:
                continue
        if window is not None:
            inside = [r for r in rows
                      if r[0] is not None and window[0] <= r[0] <= window[1]]
            rows = inside or rows
        if not rows:
            return None
        return {"sm_mhz": statistics.median(r[1] for r in rows),
                "sm_max_mhz": max(r[2] for r in rows),
                "reasons": sorted({n for r in rows for n in r[3]}),
                "samples": len(rows)}


def gpu_uuid(torch, dev):
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(dev)


def measure_replica(args, world, local):
    """Everything one rank (one GPU) measures: the timed steps, the
    per-kernel events, the rows beyond the step and the end-to-end step.
    Every collective here (barriers, the max over ranks) is taken by every
    rank in the same order. Returns the values the JSON line is made of; the
    step and e2e times are already the max over ranks."""
    import torch
    import torch.distributed as dist

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from blockwise_fp8_linear_fp8bw_b200 import ops as o

    stream = torch.cuda.Stream(device=dev)
    bufs = [LinearBuffers(kind, k, n, dev) for kind, k, n in kinds()]
    step_ops = []
    for _layer in range(LAYERS):
        step_ops.extend(layer_ops(bufs, o, stream))
    flops = step_gemm_flops()
    assert flops == sum(u for kk, u, _ in step_ops if kk.startswith("gemm"))

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    def run_step(events=None):
        if events is None:
            for _, _, fn in step_ops:
                fn()
        else:
            for (_, _, fn), (e0, e1) in zip(step_ops, events):
                e0.record(stream)
                fn()
                e1.record(stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            run_step()
    torch.cuda.synchronize()
    o.fp8bw_check_device_error(stream)

    # CUDA events around every launch of the last timed step (events on
    # every step would add ~2% to the step time they measure)
    events = [(torch.cuda.Event(enable_timing=True),
               torch.cuda.Event(enable_timing=True)) for _ in step_ops]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(gpu_uuid(torch, dev))
    time.sleep(0.6)
    barrier()
    torch.cuda.synchronize()
    wall0 = time.time()
    with torch.cuda.stream(stream):
        t_start.record(stream)
        for s in range(args.steps):
            run_step(events if s == args.steps - 1 else None)
        t_end.record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    barrier()
    clk = clocks.stop((wall0, wall1))
    o.fp8bw_check_device_error(stream)
    ms = max_over_ranks(t_start.elapsed_time(t_end) / args.steps, world, dev)

    # per-kernel durations inside the timed region
    per_kind = {}
    for (kk, units, _), (e0, e1) in zip(step_ops, events):
        d = per_kind.setdefault(kk, {"ms": 0.0, "units": 0, "launches": 0})
        d["ms"] += e0.elapsed_time(e1)
        d["units"] += units
        d["launches"] += 1

    next_rows = None
    if not args.no_next_rows:
        next_rows = time_next_rows(o, bufs, stream, args.warmup, 5)

    # ---------------------------------------------------------- end to end
    e2e = None
    if not args.no_e2e:
        pinned = []
        for b in bufs:
            hx = torch.from_numpy(b.host_x.view(np.int16)).view(
                torch.bfloat16).pin_memory()
            hw = torch.from_numpy(b.host_w.view(np.int16)).view(
                torch.bfloat16).pin_memory()
            hdy = torch.from_numpy(b.host_dy.view(np.int16)).view(
                torch.bfloat16).pin_memory()
            hdw = torch.empty(b.dw.shape, dtype=torch.bfloat16).pin_memory()
            pinned.append((hx, hw, hdy, hdw))
        h2d = LAYERS * sum(p[0].numel() * 2 + p[1].numel() * 2 +
                           p[2].numel() * 2 for p in pinned)
        d2h = LAYERS * sum(p[3].numel() * 2 for p in pinned)

        # Uploads of the next layer's X, W, dY run on a copy stream while the
        # current layer computes (two device input sets per linear, used in
        # turn); each layer's dW goes back to the host on a third stream
        # (two device dW buffers per linear). Events order every reuse.
        slots = []
        for b in bufs:
            spare = (torch.empty_like(b.x), torch.empty_like(b.w),
                     torch.empty_like(b.dy), torch.empty_like(b.dw))
            slots.append([(b.x, b.w, b.dy, b.dw), spare])
        up = torch.cuda.Stream(device=dev)
        down = torch.cuda.Stream(device=dev)
        ev = lambda: torch.cuda.Event()  # noqa: E731
        copied = [[ev() for _ in bufs] for _ in range(2)]
        computed = [[ev() for _ in bufs] for _ in range(2)]
        fetched = [[ev() for _ in bufs] for _ in range(2)]
        used = [[False] * len(bufs) for _ in range(2)]

        def e2e_step():
            for layer in range(LAYERS):
                sl = layer % 2
                for i, (b, (hx, hw, hdy, hdw)) in enumerate(zip(bufs, pinned)):
                    dx_, dw_, ddy, ddw = slots[i][sl]
                    with torch.cuda.stream(up):
                        if used[sl][i]:
                            up.wait_event(computed[sl][i])
                        dx_.copy_(hx, non_blocking=True)
                        dw_.copy_(hw, non_blocking=True)
                        ddy.copy_(hdy, non_blocking=True)
                        copied[sl][i].record(up)
                    stream.wait_event(copied[sl][i])
                    if used[sl][i]:
                        stream.wait_event(fetched[sl][i])
                    b.x, b.w, b.dy, b.dw = dx_, dw_, ddy, ddw
                for _, _, fn in layer_ops(bufs, o, stream):
                    fn()
                for i, (b, (hx, hw, hdy, hdw)) in enumerate(zip(bufs, pinned)):
                    computed[sl][i].record(stream)
                    with torch.cuda.stream(down):
                        down.wait_event(computed[sl][i])
                        hdw.copy_(b.dw, non_blocking=True)
                        fetched[sl][i].record(down)
                    used[sl][i] = True

        def join():
            # the compute stream waits for every outstanding copy
            for sl in range(2):
                for i in range(len(bufs)):
                    if used[sl][i]:
                        stream.wait_event(fetched[sl][i])

        start_ev = torch.cuda.Event()
        with torch.cuda.stream(stream):
            for _ in range(args.warmup):
                e2e_step()
            join()
        torch.cuda.synchronize()
        e_s = torch.cuda.Event(enable_timing=True)
        e_e = torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            e_s.record(stream)
            start_ev.record(stream)
            up.wait_event(start_ev)
            down.wait_event(start_ev)
            for _ in range(args.steps):
                e2e_step()
            join()
            e_e.record(stream)
        torch.cuda.synchronize()
        barrier()
        o.fp8bw_check_device_error(stream)
        for b, sl in zip(bufs, slots):     # back to the first input set
            b.x, b.w, b.dy, b.dw = sl[0]
        e2e_ms = max_over_ranks(e_s.elapsed_time(e_e) / args.steps, world,
                                dev)
        e2e = {"value": weak_scaling_value(world, flops, e2e_ms * 1e-3) / 1e12,
               "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "copies": "per layer, X/W/dY of its linears uploaded from pinned "
                         "host memory on a copy stream while the previous layer "
                         "computes; dW downloaded on another stream"}

    return {"ms": ms, "flops": flops, "per_kind": per_kind,
            "next_rows": next_rows, "clocks": clk, "e2e": e2e,
            "launches_per_step": len(step_ops)}


def run_gpu(args, measure=measure_replica):
    """One rank of the GPU arm: joins the process group (NCCL, one process
    per GPU) when there are several ranks, runs `measure`, and on rank 0
    prints the JSON line."""
    import datetime

    import torch
    import torch.distributed as dist

    world, rank, local = dist_env()
    if world > 1:
        kw = {}
        backend = "gloo"
        if torch.cuda.is_available():
            backend = "nccl"
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300),
                                **kw)
    try:
        res = measure(args, world, local)
    finally:
        if world > 1:
            dist.destroy_process_group()
    if rank != 0:
        return 0
    line = result_line(args, world, res)
    print(json.dumps(line))
    return 0


def result_line(args, world, res):
    """The JSON line of the GPU arm from what measure_replica returned."""
    ms, flops, per_kind = res["ms"], res["flops"], res["per_kind"]
    next_rows, clk, e2e = res["next_rows"], res["clocks"], res["e2e"]
    peaks = load_peaks()
    fp8_sustained = peaks["bf16_tflops_sustained"] * FP8_OVER_BF16
    fp8_burst = peaks["bf16_tflops"] * FP8_OVER_BF16
    breakdown = {}
    for kk, d in sorted(per_kind.items()):
        avg_ms = d["ms"] / d["launches"]
        if kk.startswith("gemm"):
            ach = d["units"] / (d["ms"] * 1e-3) / 1e12
            breakdown[kk] = {"achieved": ach, "unit": "TFLOP/s",
                             "frac_of_fp8_peak": ach / fp8_sustained,
                             "frac_of_fp8_peak_burst": ach / fp8_burst,
                             "flop_per_launch": d["units"] / d["launches"],
                             "dram_bytes_per_launch_ncu": ncu_traffic(kk),
                             "share": d["ms"] / ms,
                             "launches_per_step": d["launches"],
                             "avg_launch_ms": avg_ms}
        else:
            ach = d["units"] / (d["ms"] * 1e-3) / 1e9
            breakdown[kk] = {"achieved": ach, "unit": "GB/s",
                             "frac_of_hbm": ach / peaks["hbm_gbs"],
                             "bytes_per_launch": d["units"] / d["launches"],
                             "dram_bytes_per_launch_ncu": ncu_traffic(kk),
                             "share": d["ms"] / ms,
                             "launches_per_step": d["launches"],
                             "avg_launch_ms": avg_ms}
    dom = max(per_kind.items(), key=lambda kv: kv[1]["ms"])
    dk, dd = dom
    if dk.startswith("gemm"):
        ach = dd["units"] / (dd["ms"] * 1e-3) / 1e12
        roofline = {"kernel": dk, "bound": "tensor", "achieved": ach,
                    "peak": fp8_sustained, "unit": "TFLOP/s",
                    "frac": ach / fp8_sustained, "traffic": ncu_traffic(dk),
                    "frac_of_burst": ach / fp8_burst,
                    "peak_note": "%s sustained bf16 x %.0f (nominal FP8/BF16)"
                    % (peaks["source"], FP8_OVER_BF16)}
    else:
        ach = dd["units"] / (dd["ms"] * 1e-3) / 1e9
        roofline = {"kernel": dk, "bound": "hbm", "achieved": ach,
                    "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": ach / peaks["hbm_gbs"], "traffic": ncu_traffic(dk),
                    "peak_note": "%s copy bandwidth" % peaks["source"]}

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        sample = OracleSample(tokens=1024)
        t0 = time.perf_counter()
        sample.run()
        dt = time.perf_counter() - t0
        cpu = {"value": sample.flops / dt / 1e12, "unit": "TFLOP/s",
               "cores": sample.threads, "kind": "oracle",
               "sample": sample.describe(), "seconds": dt}

    if next_rows is not None:
        entries = list(next_rows.values())
        entries += list(next_rows.get("configs", {}).get("rows", {}).values())
        for d in entries:
            if d.get("unit") == "TFLOP/s":
                d["frac_of_fp8_peak"] = d["achieved"] / fp8_sustained
                d["frac_of_fp8_peak_burst"] = d["achieved"] / fp8_burst
            elif d.get("unit") == "GB/s":
                d["frac_of_hbm"] = d["achieved"] / peaks["hbm_gbs"]
    value = weak_scaling_value(world, flops, ms * 1e-3) / 1e12
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3",
        "data": "synthetic",
        "config": {"workload": WORKLOAD if (LAYERS, KINDS) == (28, (
                       "qkv", "o", "gate_up", "down")) else "partial",
                   "layers": LAYERS, "tokens": TOKENS,
                   "linears": {kd: [k, n] for kd, k, n in kinds()},
                   "gemm_tflop_per_step": flops / 1e12,
                   "l2": "inputs larger than L2 (>1 GB streamed between "
                         "reuses of any buffer)",
                   "per_launch_events": "CUDA events around every launch of "
                                        "the last timed step",
                   "parallelism": "replicas" if world > 1 else "single"},
        "gpu_launches": res["launches_per_step"] * args.steps,
        "roofline": roofline,
        "breakdown": breakdown,
        "next_rows": next_rows,
        "clocks": clk,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "peaks": {"hbm_gbs": peaks["hbm_gbs"],
                  "fp8_tflops_sustained": fp8_sustained,
                  "fp8_tflops_burst": fp8_burst,
                  "source": peaks["source"]},
    }
    return line


def main(argv=None, measure=measure_replica):
    args = parse_args(argv)
    status = check_launch(args.gpus)
    if status is not None:
        return status
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args, measure)


if __name__ == "__main__":
    sys.exit(main())

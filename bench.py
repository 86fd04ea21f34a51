"""Benchmark of the rotate-then-quantize hot path on B200 (one JSON line).

Workload: the attention-projection layer shape of the image DiTs in the
OrbitQuant write-up (hotelren.com/news/3376620, §3): d_in = d_out = 3072,
4608 tokens (a 64 x 64 latent patch grid + 512 text tokens), W4A4, RPBH h = 64.
Synthetic seeded data: Student-t(3) activations with 1% of channels x30,
N(0, 0.02^2) weights, both BF16.

One step = one pass of the whole path over one batch:
  rotate_quantize_act (x' = Pi x, norm, Lloyd-Max codes)  [HBM-bound]
  quantize_weights    (the same fused kernel on W's rows)  [HBM-bound]
  qlinear             (codes -> fp16 tiles -> tcgen05 MMA)  [tensor-bound]
Each kernel is bracketed by CUDA events on the launching stream.  Inputs
rotate over enough buffer sets that every step reads from HBM, not L2.

`value` is rotate_quantize_act throughput in GB/s of algorithmic bytes
(2d bytes in + d*b/8 + 4 bytes out per token); the qlinear TFLOP/s, the
roofline of the dominant kernel and the CPU oracle's own throughput ride
along.  --impl reference times the fp64 CPU oracle on the same workload.
"""

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

D, T, BITS_A, BITS_W, SEED = 3072, 4608, 4, 4, 0

# DRAM bytes (read + write) per launch from one ncu capture of each kernel as
# it stands (profiles/rotate_quantize_act_d3072_T32768_A4.md), or None once
# the kernel has changed since its counters were taken.  qlinear: the last
# capture of both launches of one call (code expansion + GEMM, caches flushed
# before each) gave (11_848_704 + 453_120) + (47_240_448 + 3_493_632) bytes;
# the GEMM's output stores changed after it, so no figure is reported.  The
# rotate-quantize capture ran 32768 tokens; its bytes are scaled to this
# workload's 4608 by the token count (its traffic grows with the tokens).
QLINEAR_DRAM_BYTES = None
ROTQ_DRAM_BYTES = round((201_406_720 + 28_677_376) * 4608 / 32768)
METRIC = "rotate_quantize GB/s (% HBM peak); qlinear TFLOP/s (% BF16 TC peak)"
WORKLOAD = "attn_proj d=3072 T=4608 W4A4 h=64 (Student-t(3) acts, 1% channels x30; N(0,0.02^2) weights)"


def qlinear_algorithmic_bytes(M=T, N=D, K=D, bits_a=BITS_A, bits_w=BITS_W):
    """Operand and result bytes of one qlinear call: activation codes, weight
    codes, s (fp32), r' (BF16) and Y (BF16).  The fp16 workspaces the call
    writes and reads back (weights N*K*2 and activations M*K*2, each way) are
    extra, reported beside it."""
    return M * K * bits_a // 8 + N * K * bits_w // 8 + 4 * M + 2 * N + 2 * M * N


def act_bytes_per_token(d=D, bits=BITS_A):
    return 2 * d + d * bits // 8 + 4


def weight_bytes_per_row(d=D, bits=BITS_W):
    return 2 * d + d * bits // 8 + 2


def to_bf16_tensor(x, dev):
    """BF16-valued fp32 numpy array -> torch.bfloat16 tensor on `dev`."""
    import torch
    return torch.from_numpy(synth.bf16_bits(x).view(np.int16)).view(torch.bfloat16).to(dev)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
            0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
            0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx),
                 "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.active",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 3:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
                mask = int(parts[2], 16)
            except ValueError:
                continue
            for bit, name in _REASONS.items():
                if mask & bit and name != "gpu_idle":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# multi-rank plumbing (replicas: each rank quantises its own token shard; no
# data-path collective, only the barrier and the timing reduction)
# ---------------------------------------------------------------------------

def rank_seed(rank):
    """Each rank draws its own token batch (a different shard of the job);
    the rotation and codebook are shared."""
    return SEED + rank


def reduce_job(times_ms, units, group=None, device=None):
    """Whole-job view of per-rank measurements: the max over ranks of every
    timing and the sum over ranks of the units processed."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(times_ms), dtype=torch.float64, device=device)
    u = torch.tensor([float(units)], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
        dist.all_reduce(u, op=dist.ReduceOp.SUM, group=group)
    return t.tolist(), u.item()


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args, rank, world):
    import torch
    import rotation_bit_ptq_b200 as rbq

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    pk = peaks()

    data = synth.attn_proj(seed=rank_seed(rank))
    X_host = data["X"]
    W_host = data["W"]
    r = rbq.RPBH(D, SEED)

    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    per_set = X_host.nbytes // 2 + W_host.nbytes // 2
    nsets = max(2, int(np.ceil(3 * l2 / per_set)))
    Xs = [to_bf16_tensor(X_host, dev) for _ in range(nsets)]
    Ws = [to_bf16_tensor(W_host, dev) for _ in range(nsets)]
    a_codes = [torch.empty((T, D * BITS_A // 8), dtype=torch.uint8, device=dev) for _ in range(nsets)]
    norms = [torch.empty((T,), dtype=torch.float32, device=dev) for _ in range(nsets)]
    w_codes = [torch.empty((D, D * BITS_W // 8), dtype=torch.uint8, device=dev) for _ in range(nsets)]
    rnorm = [torch.empty((D,), dtype=torch.bfloat16, device=dev) for _ in range(nsets)]
    Y = torch.empty((T, D), dtype=torch.bfloat16, device=dev)

    def step(i, ev=None):
        k = i % nsets
        if ev:
            ev[0].record(stream)
        rbq.rotate_quantize_act(r, Xs[k], BITS_A, a_codes[k], norms[k], stream=stream)
        if ev:
            ev[1].record(stream)
        rbq.quantize_weights(r, Ws[k], BITS_W, "lloydmax", w_codes[k], rnorm[k], stream=stream)
        if ev:
            ev[2].record(stream)
        rbq.qlinear(a_codes[k], norms[k], BITS_A, w_codes[k], rnorm[k], BITS_W, D, Y, stream=stream)
        if ev:
            ev[3].record(stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    assert rbq.device_error() == 0

    # Per-kernel launch durations: each kernel call over all buffer sets is
    # captured once into a CUDA graph (tables and codebooks were uploaded by
    # the warm-up calls), and the graph is replayed in the timed region, so
    # the durations are device time without the Python wrappers' launch
    # latency.  The whole-path step time below comes from direct API calls.
    calls = (
        lambda cs, k: rbq.rotate_quantize_act(r, Xs[k], BITS_A, a_codes[k], norms[k], stream=cs),
        lambda cs, k: rbq.quantize_weights(r, Ws[k], BITS_W, "lloydmax", w_codes[k], rnorm[k], stream=cs),
        lambda cs, k: rbq.qlinear(a_codes[k], norms[k], BITS_A, w_codes[k], rnorm[k], BITS_W, D, Y, stream=cs),
    )
    kernel_graphs = []
    if not args.no_graphs:
        try:
            for fn in calls:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, capture_error_mode="thread_local"):
                    cs = torch.cuda.current_stream()
                    for k in range(nsets):
                        fn(cs, k)
                kernel_graphs.append(g)
            for g in kernel_graphs:
                g.replay()
            torch.cuda.synchronize()
            assert rbq.device_error() == 0
        except Exception as exc:   # capture unsupported here: time direct calls
            print(f"bench: CUDA graph capture failed ({exc}); timing direct calls", file=sys.stderr)
            kernel_graphs = []
            torch.cuda.synchronize()
    kernel_reps = 3

    def kernel_pass(j, ev):
        ev[0].record(stream)
        for _ in range(kernel_reps):
            if kernel_graphs:
                kernel_graphs[j].replay()
            else:
                for k in range(nsets):
                    calls[j](stream, k)
        ev[1].record(stream)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step(args.warmup + i, evs[i])
    t_end.record(stream)
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(3)]
    for j in range(3):
        kernel_pass(j, kev[j])
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop()
    total_ms = t_start.elapsed_time(t_end)
    # per-kernel: average launch duration over kernel_reps x nsets launches,
    # expressed per `steps` launches so the formulas below stay per step
    nk = kernel_reps * nsets
    k1, k1w, k2 = [kev[j][0].elapsed_time(kev[j][1]) / nk * args.steps for j in range(3)]
    (total_ms, k1_ms, k1w_ms, k2_ms), job_tokens = reduce_job([total_ms, k1, k1w, k2],
                                                              T * args.steps, device=dev)

    act_bytes = act_bytes_per_token() * T
    flops = 2.0 * T * D * D
    gbs = act_bytes_per_token() * job_tokens / (k1_ms * 1e-3) / 1e9
    k1_avg_s = k1_ms / args.steps * 1e-3
    k2_avg_s = k2_ms / args.steps * 1e-3
    tflops = flops * args.steps * world / (k2_ms * 1e-3) / 1e12
    wgbs = weight_bytes_per_row() * D * args.steps * world / (k1w_ms * 1e-3) / 1e9

    # end to end through the public API with host buffers (every rank, its own
    # shard): the whole layer -- host X -> rotate_quantize_act -> qlinear (on
    # the resident weight codes, quantised offline) -> host Y -- and, as a
    # sub-key, the activation quantiser alone (host X -> codes and norms)
    e2e_ms, h2d, d2h = run_e2e_layer(r, X_host, w_codes[0], rnorm[0], dev, stream, args)
    act_ms, act_h2d, act_d2h = run_e2e(r, X_host, dev, stream, args)
    (e2e_ms, act_ms), e2e_tokens = reduce_job([e2e_ms, act_ms], T * args.steps, device=dev)
    e2e = {"value": round(act_bytes_per_token() * e2e_tokens / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "what": "whole layer through the C ABI: host X (pinned) -> rotate_quantize_act -> qlinear -> host Y "
                   "(BF16), every step's copies inside the timed region; value = activation bytes (2d + d*b/8 + 4 "
                   "per token) per second, the headline metric's unit",
           "tokens_per_s": round(e2e_tokens / (e2e_ms * 1e-3), 1),
           "layer_TFLOP/s": round(2.0 * D * D * e2e_tokens / (e2e_ms * 1e-3) / 1e12, 2),
           "rotate_quantize_only": {
               "value": round(act_bytes_per_token() * e2e_tokens / (act_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
               "h2d_bytes_per_step": act_h2d, "d2h_bytes_per_step": act_d2h,
               "what": "host X -> rotate_quantize_act -> host codes and norms"}}

    res = {
        "metric": METRIC, "value": round(gbs, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; BF16 Student-t(3) activations with 1% outlier channels x30, N(0,0.02^2) weights)",
        "config": {"workload": WORKLOAD, "tokens_per_gpu": T, "d_in": D, "d_out": D, "bits_a": BITS_A,
                   "bits_w": BITS_W, "parallelism": f"replicas x{world} (tokens sharded, no collective)",
                   "arithmetic": "rotate_quantize: BF16 in, fp32 transform and code search; qlinear: operand "
                                 "tiles are fp16 levels x sqrt(d) expanded from the codes, fp32 accumulation, "
                                 "BF16 out",
                   "l2": f"{nsets} rotating input sets ({nsets * per_set / 2**20:.0f} MiB > L2 {l2 / 2**20:.0f} MiB)"},
        "rotate_quantize": {"GB/s": round(gbs, 2), "frac_hbm": round(gbs / pk["hbm_gbs"], 4),
                            "avg_us": round(k1_avg_s * 1e6, 3)},
        "quantize_weights": {"GB/s": round(wgbs, 2), "frac_hbm": round(wgbs / pk["hbm_gbs"], 4),
                             "avg_us": round(k1w_ms / args.steps * 1e3, 3)},
        "qlinear": {"TFLOP/s": round(tflops, 2), "frac_bf16": round(tflops / pk["bf16_tflops"], 4),
                    "avg_us": round(k2_avg_s * 1e6, 3)},
        "roofline": {"kernel": "qlinear", "bound": "tensor", "achieved": round(flops / k2_avg_s / 1e12, 2),
                     "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(flops / k2_avg_s / 1e12 / pk["bf16_tflops"], 4), "traffic": QLINEAR_DRAM_BYTES,
                     "peak_source": pk["source"] + " bf16 burst",
                     "note": "achieved includes the per-call code expansion launch (weights and activations); "
                             "traffic (the ncu DRAM read + write of the two launches of one call) is null: "
                             "the GEMM's epilogue changed after the last capture",
                     "algorithmic_bytes": qlinear_algorithmic_bytes(),
                     "workspace_round_trip_bytes": 2 * 2 * (D * D + T * D)},
        "roofline_rotate_quantize": {"kernel": "rotate_quantize_act", "bound": "hbm",
                                     "achieved": round(act_bytes / k1_avg_s / 1e9, 2), "peak": pk["hbm_gbs"],
                                     "unit": "GB/s", "frac": round(act_bytes / k1_avg_s / 1e9 / pk["hbm_gbs"], 4),
                                     "traffic": ROTQ_DRAM_BYTES, "algorithmic_bytes": act_bytes,
                                     "peak_source": pk["source"]},
        # steps: rotate-quantize, weights, code expansion (weights and activations, one launch), GEMM;
        # kernel passes likewise x nsets x reps
        "gpu_launches": 4 * args.steps + 4 * kernel_reps * nsets,
        "timing": ("per-kernel: CUDA graphs of %d launches over the rotating sets, replayed %d times; "
                   "ms_per_step: direct API calls" % (nsets, kernel_reps)) if kernel_graphs else
                  "per-kernel and ms_per_step: direct API calls",
        "clocks": clk,
        "e2e": e2e,
    }
    return res


E2E_SLOTS = 3


def run_e2e(r, X_host, dev, stream, args):
    """rotate_quantize_act through the public API from pinned host memory:
    every step copies its input X host -> device, runs the kernel and copies
    the codes and norms back.  Three buffer sets and separate copy streams let
    step i+1's upload overlap step i's kernel and step i-1's download (PCIe
    moves both directions at once): an upload waits only for the kernel that
    last read its input buffer, a kernel only for its upload and for the
    download that last read its output buffers.  Every step's copies stay
    inside the timed region.  Returns (ms for args.steps steps, H2D bytes per
    step, D2H bytes per step)."""
    import torch
    import rotation_bit_ptq_b200 as rbq
    S = E2E_SLOTS
    xh = torch.from_numpy(synth.bf16_bits(X_host).view(np.int16)).view(torch.bfloat16).pin_memory()
    xd = [torch.empty_like(xh, device=dev) for _ in range(S)]
    cd = [torch.empty((T, D * BITS_A // 8), dtype=torch.uint8, device=dev) for _ in range(S)]
    nd = [torch.empty((T,), dtype=torch.float32, device=dev) for _ in range(S)]
    ch = [torch.empty((T, D * BITS_A // 8), dtype=torch.uint8).pin_memory() for _ in range(S)]
    nh = [torch.empty((T,), dtype=torch.float32).pin_memory() for _ in range(S)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    uploaded = [torch.cuda.Event() for _ in range(S)]
    computed = [torch.cuda.Event() for _ in range(S)]
    downloaded = [torch.cuda.Event() for _ in range(S)]
    for k in range(S):
        computed[k].record(stream)
        downloaded[k].record(s_out)

    def one(i):
        k = i % S
        s_in.wait_event(computed[k])                # the slot's input buffer is no longer read
        with torch.cuda.stream(s_in):
            xd[k].copy_(xh, non_blocking=True)
        uploaded[k].record(s_in)
        stream.wait_event(uploaded[k])
        stream.wait_event(downloaded[k])            # the slot's previous results are out
        rbq.rotate_quantize_act(r, xd[k], BITS_A, cd[k], nd[k], stream=stream)
        computed[k].record(stream)
        s_out.wait_event(computed[k])
        with torch.cuda.stream(s_out):
            ch[k].copy_(cd[k], non_blocking=True)
            nh[k].copy_(nd[k], non_blocking=True)
        downloaded[k].record(s_out)

    for i in range(max(3, args.warmup)):
        one(i)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    s_in.wait_event(a)
    s_out.wait_event(a)
    for i in range(args.steps):
        one(i)
    stream.wait_stream(s_in)
    stream.wait_stream(s_out)
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b), int(xh.numel() * 2), int(ch[0].numel() + nh[0].numel() * 4)


def run_e2e_layer(r, X_host, w_codes, rnorm, dev, stream, args):
    """The whole quantised layer through the public API from pinned host
    memory: every step copies its input X host -> device, quantises it
    (rotate_quantize_act), runs qlinear against the resident weight codes and
    copies Y (BF16) back.  Three buffer sets and separate copy streams overlap
    step i+1's upload and step i-1's download with step i's kernels (the same
    dependencies as run_e2e); every step's copies stay inside the timed
    region.  Returns (ms for args.steps steps, H2D bytes per step, D2H bytes
    per step)."""
    import torch
    import rotation_bit_ptq_b200 as rbq
    S = E2E_SLOTS
    xh = torch.from_numpy(synth.bf16_bits(X_host).view(np.int16)).view(torch.bfloat16).pin_memory()
    xd = [torch.empty_like(xh, device=dev) for _ in range(S)]
    cd = [torch.empty((T, D * BITS_A // 8), dtype=torch.uint8, device=dev) for _ in range(S)]
    nd = [torch.empty((T,), dtype=torch.float32, device=dev) for _ in range(S)]
    yd = [torch.empty((T, D), dtype=torch.bfloat16, device=dev) for _ in range(S)]
    yh = [torch.empty((T, D), dtype=torch.bfloat16).pin_memory() for _ in range(S)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    uploaded = [torch.cuda.Event() for _ in range(S)]
    computed = [torch.cuda.Event() for _ in range(S)]
    downloaded = [torch.cuda.Event() for _ in range(S)]
    for k in range(S):
        computed[k].record(stream)
        downloaded[k].record(s_out)

    def one(i):
        k = i % S
        s_in.wait_event(computed[k])                # the slot's input buffer is no longer read
        with torch.cuda.stream(s_in):
            xd[k].copy_(xh, non_blocking=True)
        uploaded[k].record(s_in)
        stream.wait_event(uploaded[k])
        stream.wait_event(downloaded[k])            # the slot's previous Y is out
        rbq.rotate_quantize_act(r, xd[k], BITS_A, cd[k], nd[k], stream=stream)
        rbq.qlinear(cd[k], nd[k], BITS_A, w_codes, rnorm, BITS_W, D, yd[k], stream=stream)
        computed[k].record(stream)
        s_out.wait_event(computed[k])
        with torch.cuda.stream(s_out):
            yh[k].copy_(yd[k], non_blocking=True)
        downloaded[k].record(s_out)

    for i in range(max(3, args.warmup)):
        one(i)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    s_in.wait_event(a)
    s_out.wait_event(a)
    for i in range(args.steps):
        one(i)
    stream.wait_stream(s_in)
    stream.wait_stream(s_out)
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b), int(xh.numel() * 2), int(yh[0].numel() * 2)


# ---------------------------------------------------------------------------
# the other workloads of the pages (kernel timings; inputs reused across
# iterations -- every case except the INT8 4096-wide ones exceeds L2)
# ---------------------------------------------------------------------------

def _time_us(fn, stream, warmup=3, iters=10):
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(iters):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / iters * 1e3


def _tile_rows(X, T):
    reps = -(-T // X.shape[0])
    return np.ascontiguousarray(np.tile(X, (reps, 1))[:T])


def run_suite(dev, stream, pk):
    """Every kernel of the path on the MLP pair (W2A4, W3A3), the INT8 W8A16
    single-stream DiT block and the video-DiT layers (W4A6)."""
    import torch
    import rotation_bit_ptq_b200 as rbq

    hbm, tc = pk["hbm_gbs"], pk["bf16_tflops"]
    out = {}

    def rotq_entry(us, T, d, bits):
        gbs = T * (2 * d + d * bits // 8 + 4) / (us * 1e-6) / 1e9
        return {"us": round(us, 2), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4)}

    def gemm_entry(us, M, N, K):
        tf = 2.0 * M * N * K / (us * 1e-6) / 1e12
        return {"us": round(us, 2), "TFLOP/s": round(tf, 1), "frac_bf16": round(tf / tc, 4)}

    def i8_entry(us, M, N, K, us_fp16, y8, y16, fp8=False):
        # int8 / fp8 dense peak: the measured bf16 peak times the nominal
        # 8-bit:bf16 ratio (4.5 / 2.25)
        ops = 2.0 * M * N * K / (us * 1e-6) / 1e12
        dev_ = float(torch.linalg.norm((y8.float() - y16.float())) / torch.linalg.norm(y16.float()))
        return {"us": round(us, 2), ("TFLOP/s" if fp8 else "TOPS"): round(ops, 1),
                ("frac_fp8" if fp8 else "frac_int8"): round(ops / (2 * tc), 4),
                "speedup_vs_fp16_levels": round(us_fp16 / us, 3), "rel_dev_from_exact_levels": round(dev_, 5)}

    # MLP pair: up 3072 -> 12288, down 12288 -> 3072, 4608 tokens
    m = synth.mlp()
    T = 4608
    Xu, Xd = to_bf16_tensor(m["X_up"], dev), to_bf16_tensor(m["X_dn"], dev)
    Wu, Wd = to_bf16_tensor(m["W_up"], dev), to_bf16_tensor(m["W_dn"], dev)
    ru, rd = rbq.RPBH(3072, 11), rbq.RPBH(12288, 12)
    mlp = {}
    for ba, bw in ((4, 2), (3, 3)):
        e = {}
        au, su = rbq.rotate_quantize_act(ru, Xu, ba)
        ad, sd = rbq.rotate_quantize_act(rd, Xd, ba)
        e["rotate_quantize d=3072"] = rotq_entry(_time_us(lambda: rbq.rotate_quantize_act(ru, Xu, ba, au, su, stream=stream), stream), T, 3072, ba)
        e["rotate_quantize d=12288"] = rotq_entry(_time_us(lambda: rbq.rotate_quantize_act(rd, Xd, ba, ad, sd, stream=stream), stream), T, 12288, ba)
        wu, nu = rbq.quantize_weights(ru, Wu, bw)
        wd, nd = rbq.quantize_weights(rd, Wd, bw)
        yu = torch.empty((T, 12288), dtype=torch.bfloat16, device=dev)
        yd = torch.empty((T, 3072), dtype=torch.bfloat16, device=dev)
        e["qlinear up 4608x12288x3072"] = gemm_entry(
            _time_us(lambda: rbq.qlinear(au, su, ba, wu, nu, bw, 3072, yu, stream=stream), stream), T, 12288, 3072)
        e["qlinear down 4608x3072x12288"] = gemm_entry(
            _time_us(lambda: rbq.qlinear(ad, sd, ba, wd, nd, bw, 12288, yd, stream=stream), stream), T, 3072, 12288)
        # the same layers with 8-bit integer levels on the INT8 tensor cores
        yu8 = rbq.qlinear_int8_levels(au, su, ba, wu, nu, bw, 3072)
        yd8 = rbq.qlinear_int8_levels(ad, sd, ba, wd, nd, bw, 12288)
        rbq.qlinear(au, su, ba, wu, nu, bw, 3072, yu)
        rbq.qlinear(ad, sd, ba, wd, nd, bw, 12288, yd)
        e["qlinear_int8_levels up"] = i8_entry(
            _time_us(lambda: rbq.qlinear_int8_levels(au, su, ba, wu, nu, bw, 3072, yu8, stream=stream), stream),
            T, 12288, 3072, e["qlinear up 4608x12288x3072"]["us"], yu8, yu)
        e["qlinear_int8_levels down"] = i8_entry(
            _time_us(lambda: rbq.qlinear_int8_levels(ad, sd, ba, wd, nd, bw, 12288, yd8, stream=stream), stream),
            T, 3072, 12288, e["qlinear down 4608x3072x12288"]["us"], yd8, yd)
        del yu8, yd8
        yu8 = rbq.qlinear_fp8_levels(au, su, ba, wu, nu, bw, 3072)
        yd8 = rbq.qlinear_fp8_levels(ad, sd, ba, wd, nd, bw, 12288)
        e["qlinear_fp8_levels up"] = i8_entry(
            _time_us(lambda: rbq.qlinear_fp8_levels(au, su, ba, wu, nu, bw, 3072, yu8, stream=stream), stream),
            T, 12288, 3072, e["qlinear up 4608x12288x3072"]["us"], yu8, yu, fp8=True)
        e["qlinear_fp8_levels down"] = i8_entry(
            _time_us(lambda: rbq.qlinear_fp8_levels(ad, sd, ba, wd, nd, bw, 12288, yd8, stream=stream), stream),
            T, 3072, 12288, e["qlinear down 4608x3072x12288"]["us"], yd8, yd, fp8=True)
        del yu8, yd8
        mlp[f"W{bw}A{ba}"] = e
    out["mlp_pair"] = mlp
    ru.close()
    rd.close()
    del Xu, Xd, Wu, Wd, yu, yd

    # INT8 rotate-then-quantize, W8A16, 4096 tokens; one block of the
    # 32-block single-stream DiT (the per-block work is the same in every block)
    int8 = {}
    params = sum(o * i for _, o, i in synth.INT8_DIT_SHAPES)
    rows = sum(o for _, o, _ in synth.INT8_DIT_SHAPES)
    block_quant_us = 0.0
    for name, n_out, d_in in synth.INT8_DIT_SHAPES:
        if name in ("k", "v", "o"):          # same shape as q: the weight pass is timed, the layer is not repeated
            W = to_bf16_tensor(synth.int8_dit_weight(0, name), dev)
            r = rbq.RPBH(d_in, 100 + d_in)
            q, sc = rbq.quantize_weights(r, W, 8, mode="int8")
            us = _time_us(lambda: rbq.quantize_weights(r, W, 8, "int8", q, sc, stream=stream), stream)
            block_quant_us += us
            int8[f"{name} {d_in}->{n_out}"] = {"quantize_weights_int8": {"us": round(us, 2)}}
            r.close()
            del W, q, sc
            continue
        W = to_bf16_tensor(synth.int8_dit_weight(0, name), dev)
        X = to_bf16_tensor(synth.int8_dit_act(d_in), dev)
        r = rbq.RPBH(d_in, 100 + d_in)
        q, sc = rbq.quantize_weights(r, W, 8, mode="int8")
        xr = rbq.rotate_act(r, X)
        y = torch.empty((4096, n_out), dtype=torch.bfloat16, device=dev)
        e = {}
        us = _time_us(lambda: rbq.quantize_weights(r, W, 8, "int8", q, sc, stream=stream), stream)
        block_quant_us += us
        gbs = n_out * (3 * d_in + 4) / (us * 1e-6) / 1e9
        e["quantize_weights_int8"] = {"us": round(us, 2), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4)}
        us = _time_us(lambda: rbq.rotate_act(r, X, xr, stream=stream), stream)
        gbs = 4096 * 4 * d_in / (us * 1e-6) / 1e9
        e["rotate_only"] = {"us": round(us, 2), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4)}
        e["qlinear_int8"] = gemm_entry(_time_us(lambda: rbq.qlinear_int8(xr, q, sc, y, stream=stream), stream),
                                       4096, n_out, d_in)
        # output error on 64 tokens, against the dense layer (fp32 reference
        # matmul, a report only): rotated INT8 vs naive per-channel INT8
        with torch.no_grad():
            xs, Wf = X[:64].float(), W.float()
            dense = xs @ Wf.t()
            scale_n = Wf.abs().amax(dim=1, keepdim=True) / 127.0
            Wn = torch.clamp(torch.round(Wf / torch.where(scale_n > 0, scale_n, torch.ones_like(scale_n))), -127, 127) * scale_n
            naive = xs @ Wn.t()
            err_rot = (y[:64].float() - dense).norm() / dense.norm()
            err_naive = (naive - dense).norm() / dense.norm()
        e["rel_error_rotated_int8"] = round(err_rot.item(), 5)
        e["rel_error_naive_int8"] = round(err_naive.item(), 5)
        # one scale for the whole tensor (two passes over W), same layer kernel
        qt, st_ = rbq.quantize_weights(r, W, 8, "int8_tensor")
        us = _time_us(lambda: rbq.quantize_weights(r, W, 8, "int8_tensor", qt, st_, stream=stream), stream)
        e["quantize_weights_int8_per_tensor"] = {"us": round(us, 2)}
        yt = rbq.qlinear_int8(xr[:64].contiguous(), qt, st_)
        with torch.no_grad():
            e["rel_error_rotated_int8_per_tensor"] = round(((yt.float() - dense).norm() / dense.norm()).item(), 5)
        del qt, st_, yt
        # zero point per channel (asymmetric), same layer GEMM on (q - z)
        qa, sa, za = rbq.quantize_weights_int8_asym(r, W)
        us = _time_us(lambda: rbq.quantize_weights_int8_asym(r, W, qa, sa, za, stream=stream), stream)
        e["quantize_weights_int8_asym"] = {"us": round(us, 2)}
        e["qlinear_int8_asym"] = gemm_entry(_time_us(lambda: rbq.qlinear_int8_asym(xr, qa, sa, za, y, stream=stream),
                                                     stream), 4096, n_out, d_in)
        ya = rbq.qlinear_int8_asym(xr[:64].contiguous(), qa, sa, za)
        with torch.no_grad():
            e["rel_error_rotated_int8_asym"] = round(((ya.float() - dense).norm() / dense.norm()).item(), 5)
        del qa, sa, za, ya
        int8[f"{name} {d_in}->{n_out}"] = e
        r.close()
        del W, X, q, sc, xr, y
    int8["model"] = {
        "blocks": 32, "params": 32 * params,
        "bf16_bytes": 2 * 32 * params, "int8_bytes": 32 * params + 4 * 32 * rows,
        "ratio": round((32 * params + 4 * 32 * rows) / (2 * 32 * params), 4),
        "pages_ratio": round(6.76 / 13.25, 4),
        "quantize_weights_int8_ms_one_block": round(block_quant_us * 1e-3, 3),
        "quantize_weights_int8_ms_all_blocks_derived": round(32 * block_quant_us * 1e-3, 3),
        "derived": "all 32 blocks = 32 x the measured block (every block has the same six shapes)",
    }
    out["int8_dit"] = int8

    # The rotation fused into the producing matmul (OrbitQuant §6.2): the DiT
    # block's MLP up-projection (4096 tokens, 4096 -> 16384, W8A16) whose GELU
    # output is the down-projection's input, rotated at d = 16384.  Unfused:
    # qlinear_int8 (BF16 y) -> GELU (a torch elementwise kernel, fp32 math on
    # the BF16 tensor) -> rotate_act.  Fused: one qlinear_int8_rotate_next on
    # the weight rows reordered (once, offline) by the next layer's permutation.
    W = to_bf16_tensor(synth.int8_dit_weight(0, "up"), dev)
    X = to_bf16_tensor(synth.int8_dit_act(4096), dev)
    r, nxt = rbq.RPBH(4096, 100 + 4096), rbq.RPBH(16384, 200 + 16384)
    xr = rbq.rotate_act(r, X)
    q, sc = rbq.quantize_weights(r, W, 8, mode="int8")
    qn, scn = rbq.rows_in_next_order(nxt, q), rbq.rows_in_next_order(nxt, sc)
    y = torch.empty((4096, 16384), dtype=torch.bfloat16, device=dev)
    g = torch.empty_like(y)
    xn = torch.empty_like(y)

    def unfused():
        rbq.qlinear_int8(xr, q, sc, y, stream=stream)
        torch.nn.functional.gelu(y, out=g)
        rbq.rotate_act(nxt, g, xn, stream=stream)

    us_un = _time_us(unfused, stream)
    us_gemm = _time_us(lambda: rbq.qlinear_int8(xr, q, sc, y, stream=stream), stream)
    us_rot = _time_us(lambda: rbq.rotate_act(nxt, g, xn, stream=stream), stream)
    us_fused = _time_us(lambda: rbq.qlinear_int8_rotate_next(xr, qn, scn, nxt, "gelu", xn, stream=stream), stream)
    out["fused_rotation_dit_mlp_up_into_down"] = {
        "unfused_us": round(us_un, 2), "unfused_parts_us": {"qlinear_int8": round(us_gemm, 2),
                                                            "gelu (torch)": round(us_un - us_gemm - us_rot, 2),
                                                            "rotate_act d=16384": round(us_rot, 2)},
        "fused_us": round(us_fused, 2), "speedup": round(us_un / us_fused, 3),
        "fused_TFLOP/s": round(2.0 * 4096 * 16384 * 4096 / (us_fused * 1e-6) / 1e12, 1)}
    r.close()
    nxt.close()
    del W, X, xr, q, sc, qn, scn, y, g, xn

    # The same fusion on the code layer (OrbitQuant §2.2): the MLP pair's
    # up-projection (4608 tokens, 3072 -> 12288, W2A4) whose GELU output is the
    # down-projection's input, quantised at d = 12288 with 4-bit codes.
    # Unfused: qlinear (BF16 y) -> GELU (torch) -> rotate_quantize_act.
    # Fused: qlinear_rotate_next (the rotation in the epilogue, BF16 x') ->
    # quantize_rotated (norm and codes only).
    m = synth.mlp()
    Xu, Wu = to_bf16_tensor(m["X_up"], dev), to_bf16_tensor(m["W_up"], dev)
    ru, nxt = rbq.RPBH(3072, 11), rbq.RPBH(12288, 12)
    au, su = rbq.rotate_quantize_act(ru, Xu, 4)
    wu, nu = rbq.quantize_weights(ru, Wu, 2)
    wn, nn_ = rbq.rows_in_next_order(nxt, wu), rbq.rows_in_next_order(nxt, nu)
    y = torch.empty((4608, 12288), dtype=torch.bfloat16, device=dev)
    g = torch.empty_like(y)
    xn = torch.empty_like(y)
    cn = torch.empty((4608, 12288 * 4 // 8), dtype=torch.uint8, device=dev)
    sn = torch.empty((4608,), dtype=torch.float32, device=dev)

    def unfused_codes():
        rbq.qlinear(au, su, 4, wu, nu, 2, 3072, y, stream=stream)
        torch.nn.functional.gelu(y, out=g)
        rbq.rotate_quantize_act(nxt, g, 4, cn, sn, stream=stream)

    def fused_codes():
        rbq.qlinear_rotate_next(au, su, 4, wn, nn_, 2, 3072, nxt, "gelu", xn, stream=stream)
        rbq.quantize_rotated(xn, 4, cn, sn, stream=stream)

    us_un = _time_us(unfused_codes, stream)
    us_gemm = _time_us(lambda: rbq.qlinear(au, su, 4, wu, nu, 2, 3072, y, stream=stream), stream)
    us_rq = _time_us(lambda: rbq.rotate_quantize_act(nxt, g, 4, cn, sn, stream=stream), stream)
    us_fused = _time_us(fused_codes, stream)
    us_fgemm = _time_us(lambda: rbq.qlinear_rotate_next(au, su, 4, wn, nn_, 2, 3072, nxt, "gelu", xn,
                                                        stream=stream), stream)
    us_qr = _time_us(lambda: rbq.quantize_rotated(xn, 4, cn, sn, stream=stream), stream)
    out["fused_rotation_mlp_w2a4_up_into_down_a4"] = {
        "unfused_us": round(us_un, 2),
        "unfused_parts_us": {"qlinear": round(us_gemm, 2), "gelu (torch)": round(us_un - us_gemm - us_rq, 2),
                             "rotate_quantize_act d=12288": round(us_rq, 2)},
        "fused_us": round(us_fused, 2),
        "fused_parts_us": {"qlinear_rotate_next": round(us_fgemm, 2), "quantize_rotated d=12288": round(us_qr, 2)},
        "speedup": round(us_un / us_fused, 3),
        "quantize_rotated": rotq_entry(us_qr, 4608, 12288, 4)}
    ru.close()
    nxt.close()
    del m, Xu, Wu, au, su, wu, nu, wn, nn_, y, g, xn, cn, sn

    # video DiT W4A6: 32760 tokens (21 frames x 1560), hidden 1536, MLP 8960
    T = 32760
    vid = {}
    acts = {}
    for d in (1536, 8960):
        X = to_bf16_tensor(_tile_rows(synth.video_act(d, 0, frames=[0, 1, 2, 3]), T), dev)
        r = rbq.RPBH(d, 1000 + d)
        a, sv = rbq.rotate_quantize_act(r, X, 6)
        vid[f"rotate_quantize d={d} A6"] = rotq_entry(
            _time_us(lambda: rbq.rotate_quantize_act(r, X, 6, a, sv, stream=stream), stream), T, d, 6)
        acts[d] = (a, sv, r)
        del X
    for n_out, d_in in ((1536, 1536), (8960, 1536), (1536, 8960)):
        a, sv, r = acts[d_in]
        W = to_bf16_tensor(synth.video_weight(n_out, d_in, 0), dev)
        wc, wn = rbq.quantize_weights(r, W, 4)
        y = torch.empty((T, n_out), dtype=torch.bfloat16, device=dev)
        vid[f"qlinear {T}x{n_out}x{d_in} W4A6"] = gemm_entry(
            _time_us(lambda: rbq.qlinear(a, sv, 6, wc, wn, 4, d_in, y, stream=stream), stream), T, n_out, d_in)
        del W, wc, wn, y
    for a, sv, r in acts.values():
        r.close()
    out["video_w4a6"] = vid

    # Transform ablation (OrbitQuant §2.3 and §3.3): RPBH against the block
    # Hadamard transform without the permutation (the same kernels with
    # pi = identity) and against a dense d x d rotation, which is a plain GEMM
    # x' = X R^T -- timed here as a cuBLAS BF16 matmul (the comparator only;
    # the pages report structured transforms > 25x faster than dense ones).
    # 4608 tokens of the attention-projection recipe, d = 3072 and 12288.
    abl = {}
    for d in (3072, 12288):
        T = 4608
        X = to_bf16_tensor(_tile_rows(synth.student_t_act(512, d, seed=31)[0], T), dev)
        e = {}
        xr = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
        codes = torch.empty((T, d // 2), dtype=torch.uint8, device=dev)
        norms = torch.empty((T,), dtype=torch.float32, device=dev)
        for label, r in (("RPBH", rbq.RPBH(d, 41)), ("block Hadamard (no permutation)", rbq.RPBH(d, 41, permute=False))):
            rbq.rotate_act(r, X, xr)
            rbq.rotate_quantize_act(r, X, 4, codes, norms)
            us = _time_us(lambda: rbq.rotate_act(r, X, xr, stream=stream), stream)
            e[f"rotate_only {label}"] = {"us": round(us, 2), "GB/s": round(T * 4 * d / (us * 1e-6) / 1e9, 1)}
            e[f"rotate_quantize A4 {label}"] = rotq_entry(
                _time_us(lambda: rbq.rotate_quantize_act(r, X, 4, codes, norms, stream=stream), stream), T, d, 4)
            r.close()
        R = (torch.randn((d, d), device=dev) / d ** 0.5).to(torch.bfloat16)
        with torch.no_grad():
            us = _time_us(lambda: torch.matmul(X, R.t(), out=xr), stream)
        e["dense rotation (cuBLAS BF16 GEMM)"] = {"us": round(us, 2), "TFLOP/s": round(2.0 * T * d * d / (us * 1e-6) / 1e12, 1)}
        e["dense / RPBH rotate_only time"] = round(us / e["rotate_only RPBH"]["us"], 2)
        e["RPBH / block Hadamard rotate_only time"] = round(
            e["rotate_only RPBH"]["us"] / e["rotate_only block Hadamard (no permutation)"]["us"], 3)
        abl[f"d={d}, {T} tokens"] = e
        del X, xr, codes, norms, R
    out["transform_ablation"] = abl

    # Bit-width sweep (per-layer widths, OrbitQuant §4.2-§4.4): the
    # attention projection (4608 x 3072 x 3072) at every activation width
    # with 4-bit weights and every weight width with 4-bit activations.
    data = synth.attn_proj(seed=5)
    X = to_bf16_tensor(data["X"], dev)
    W = to_bf16_tensor(data["W"], dev)
    r = rbq.RPBH(3072, 77)
    y = torch.empty((4608, 3072), dtype=torch.bfloat16, device=dev)
    sweep = {}
    wc4, wn4 = rbq.quantize_weights(r, W, 4)
    a4, s4 = rbq.rotate_quantize_act(r, X, 4)
    for b in (2, 3, 4, 5, 6, 8):
        a, sa = rbq.rotate_quantize_act(r, X, b)
        wc, wn = rbq.quantize_weights(r, W, b)
        sweep[f"A{b}"] = {
            "rotate_quantize": rotq_entry(
                _time_us(lambda: rbq.rotate_quantize_act(r, X, b, a, sa, stream=stream), stream), 4608, 3072, b),
            "qlinear W4A%d" % b: gemm_entry(
                _time_us(lambda: rbq.qlinear(a, sa, b, wc4, wn4, 4, 3072, y, stream=stream), stream), 4608, 3072, 3072),
            "qlinear W%dA4" % b: gemm_entry(
                _time_us(lambda: rbq.qlinear(a4, s4, 4, wc, wn, b, 3072, y, stream=stream), stream), 4608, 3072, 3072),
        }
        del a, sa, wc, wn
    out["bit_width_sweep_attn_proj"] = sweep
    # the attention projection with 8-bit integer levels (INT8 tensor cores)
    y16 = rbq.qlinear(a4, s4, 4, wc4, wn4, 4, 3072)
    y8 = rbq.qlinear_int8_levels(a4, s4, 4, wc4, wn4, 4, 3072)
    us16 = _time_us(lambda: rbq.qlinear(a4, s4, 4, wc4, wn4, 4, 3072, y, stream=stream), stream)
    out["int8_levels_attn_proj_W4A4"] = i8_entry(
        _time_us(lambda: rbq.qlinear_int8_levels(a4, s4, 4, wc4, wn4, 4, 3072, y8, stream=stream), stream),
        4608, 3072, 3072, us16, y8, y16)
    yf = rbq.qlinear_fp8_levels(a4, s4, 4, wc4, wn4, 4, 3072)
    out["fp8_levels_attn_proj_W4A4"] = i8_entry(
        _time_us(lambda: rbq.qlinear_fp8_levels(a4, s4, 4, wc4, wn4, 4, 3072, yf, stream=stream), stream),
        4608, 3072, 3072, us16, yf, y16, fp8=True)
    del y8, y16, yf
    r.close()
    del X, W, y, wc4, wn4, a4, s4
    torch.cuda.synchronize()
    assert rbq.device_error() == 0
    return out

# ---------------------------------------------------------------------------
# oracle (CPU) timings
# ---------------------------------------------------------------------------

def oracle_rotq_gbs(tokens, min_seconds, rank_seed=0):
    """The fp64 oracle's rotate-then-quantize on `tokens` tokens of the workload,
    repeated until `min_seconds` passed.  Returns (GB/s, seconds, reps)."""
    import oracle
    data = synth.attn_proj(seed=rank_seed)
    X = data["X"][:tokens].astype(np.float64)
    perm, signs = oracle.rpbh_draw(D, SEED)
    Pi = oracle.rpbh_matrix(perm, signs)
    _, bounds = oracle.lloydmax_table(D, BITS_A)
    reps, t0 = 0, time.perf_counter()
    while True:
        out = oracle.quantize_act(X, Pi, bounds)
        oracle.pack_codes(out["codes"], BITS_A)
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    return act_bytes_per_token() * tokens * reps / el / 1e9, el, reps


def oracle_rotq_gbs_single_thread(tokens, min_seconds):
    """oracle_rotq_gbs with the BLAS thread pools limited to one thread."""
    import threadpoolctl
    with threadpoolctl.threadpool_limits(limits=1):
        return oracle_rotq_gbs(tokens, min_seconds)


def cpu_cores():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max((i.get("num_threads", 1) for i in info), default=os.cpu_count())
    except Exception:
        return os.cpu_count()


def run_reference(args):
    """The oracle, as it stands, timed per step on a bounded token sample."""
    tokens = 512
    for _ in range(args.warmup):
        oracle_rotq_gbs(tokens, 0.0)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_rotq_gbs(tokens, 0.0)
    el = time.perf_counter() - t0
    gbs = act_bytes_per_token() * tokens * args.steps / el / 1e9
    cores = cpu_cores()
    return {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)", "config": {"workload": WORKLOAD, "tokens_per_step": tokens},
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"{tokens} of {T} tokens per step, dense fp64 Pi (numpy)"},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_kernel_only(args):
    """One kernel on a profiling-sized case (for ncu): a few launches, no
    timing.  rotate_quantize: 32768 tokens x 3072 (201 MB of BF16 input,
    larger than L2); qlinear (and its integer-level variant): the
    attention-projection GEMM 4608x3072x3072; qlinear_int8 and
    quantize_weights_int8: the DiT block's q projection, 4096 x 4096 x 4096."""
    import torch
    import rotation_bit_ptq_b200 as rbq
    dev = torch.device("cuda", 0)
    r = rbq.RPBH(D, SEED)
    if args.kernel_only in ("rotate_quantize", "rotate_only"):
        d = args.dim or D
        tokens = args.tokens or 32768
        if d != D:
            r.close()
            r = rbq.RPBH(d, SEED)
        X = to_bf16_tensor(synth.student_t_act(tokens, d, seed=SEED)[0], dev)
        for _ in range(args.launches):
            if args.kernel_only == "rotate_quantize":
                rbq.rotate_quantize_act(r, X, BITS_A)
            else:
                rbq.rotate_act(r, X)
    elif args.kernel_only == "quantize_weights":
        W = to_bf16_tensor(synth.attn_proj(seed=SEED)["W"], dev)
        for _ in range(args.launches):
            rbq.quantize_weights(r, W, BITS_W)
    elif args.kernel_only in ("qlinear_int8", "quantize_weights_int8"):
        # the single-stream DiT block's q projection: 4096 tokens, 4096 -> 4096
        r4 = rbq.RPBH(4096, 100 + 4096)
        W = to_bf16_tensor(synth.int8_dit_weight(0, "q"), dev)
        q, sc = rbq.quantize_weights(r4, W, 8, mode="int8")
        if args.kernel_only == "quantize_weights_int8":
            for _ in range(args.launches):
                rbq.quantize_weights(r4, W, 8, "int8", q, sc)
        else:
            xr = rbq.rotate_act(r4, to_bf16_tensor(synth.int8_dit_act(4096), dev))
            for _ in range(args.launches):
                rbq.qlinear_int8(xr, q, sc)
    else:
        data = synth.attn_proj(seed=SEED)
        a_codes, s = rbq.rotate_quantize_act(r, to_bf16_tensor(data["X"], dev), BITS_A)
        w_codes, rn = rbq.quantize_weights(r, to_bf16_tensor(data["W"], dev), BITS_W)
        fn = rbq.qlinear_int8_levels if args.kernel_only == "qlinear_int8_levels" else rbq.qlinear
        for _ in range(args.launches):
            fn(a_codes, s, BITS_A, w_codes, rn, BITS_W, D)
    torch.cuda.synchronize()
    assert rbq.device_error() == 0
    print(json.dumps({"kernel_only": args.kernel_only, "launches": args.launches, "ok": True}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-suite", action="store_true", help="skip the other workloads' kernel timings")
    ap.add_argument("--no-graphs", action="store_true", help="time direct API calls instead of graph replays")
    ap.add_argument("--kernel-only", choices=["rotate_quantize", "rotate_only", "quantize_weights", "qlinear",
                                                   "qlinear_int8_levels", "qlinear_int8", "quantize_weights_int8"],
                    help="run one kernel on a profiling-sized case (for ncu) instead of the benchmark")
    ap.add_argument("--tokens", type=int, default=0)
    ap.add_argument("--dim", type=int, default=0, help="--kernel-only rotate_*: input width (default 3072)")
    ap.add_argument("--launches", type=int, default=3)
    args = ap.parse_args()
    if args.kernel_only:
        run_kernel_only(args)
        return
    args.warmup = max(3, args.warmup)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)))
        return

    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    res = run_ours(args, rank, world)
    # The other workloads' kernel timings and the CPU baseline run at N = 1
    # only: at N > 1 they would hold every rank's GPU at the closing barrier.
    if world == 1 and not args.no_suite:
        import torch
        res["suite"] = run_suite(torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0))),
                                 torch.cuda.current_stream(), peaks())
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            gbs, el, reps = oracle_rotq_gbs(T, 10.0)
            res["cpu_baseline"] = {"value": round(gbs, 4), "unit": "GB/s", "cores": cpu_cores(), "kind": "oracle",
                                   "sample": f"all {T} tokens x {reps} reps ({el:.1f} s), dense fp64 Pi (numpy)"}
            gbs1, el1, reps1 = oracle_rotq_gbs_single_thread(512, 3.0)
            res["cpu_baseline"]["single_thread"] = {
                "value": round(gbs1, 4), "unit": "GB/s", "cores": 1,
                "sample": f"512 of {T} tokens x {reps1} reps ({el1:.1f} s), BLAS limited to one thread"}
        print(json.dumps(res))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

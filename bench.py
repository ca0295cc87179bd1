"""Benchmark of the block-sparse video attention forward pass on B200.

One step = the whole hot path on one batch: block selection (pool, coarse
scores, top-k) and the fine pass with its fused cube gather/scatter (plus the
linear-branch state for workloads that have one), all through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...      # the CPU oracle, timed on host cores

Prints one JSON line (rank 0).  `value` is the effective fine-pass TFLOP/s of
the whole step, 4 * N_valid * k * 64 * d * heads * B FLOPs per step (selected
blocks only), summed over ranks; every rank runs its own copy of the workload
(weak scaling, no data-path collective).
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_attention_30_b200 import HEADLINE, WORKLOADS, synth  # noqa: E402

METRIC = "fine-attn effective TFLOP/s & ms/call (selected blocks), % of B200 BF16 peak"
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
L2_FLUSH_BYTES = 256 << 20


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# Sources of the fine kernel the headline step runs (bf16, d = 128, k = 46:
# the one-cube-per-CTA kernel); a DRAM-traffic figure is reported only while
# they hash to the value recorded beside it.
FINE_SOURCES = ["fine_attn.cu", "softmax_step.cuh", "sm100.cuh", "common.cuh"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def fine_sources_hash():
    import hashlib
    csrc = os.path.join(ROOT, "block_sparse_attention_30_b200", "csrc")
    h = hashlib.sha256(b"".join(open(os.path.join(csrc, f), "rb").read() for f in FINE_SOURCES))
    return h.hexdigest()[:16]


def profiled_traffic(workload, path=TRAFFIC_FILE):
    """DRAM bytes (ncu dram__bytes_read.sum + dram__bytes_write.sum) per fine
    launch from the committed capture data, or None when the data lacks this
    workload or the kernel sources changed since the capture."""
    if not os.path.exists(path):
        return None
    data = json.load(open(path, encoding="utf-8"))
    if data.get("sources_sha256") != fine_sources_hash():
        return None
    val = data.get("bytes_per_launch", {}).get(workload)
    return int(val) if val is not None else None


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(
        os.environ.get("WORLD_SIZE", 1))


def rank_seed(workload_seed, rank):
    """Each rank works on its own batch: the workload's stream shifted by rank."""
    return workload_seed + 1000 * rank


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks (timings: the job
    is as slow as its slowest rank).  Single-process: returned unchanged."""
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def aggregate(world, flops_per_step, steps, total_ms, e2e_ms, fine_total_ms):
    """Whole-job figures from max-over-ranks times: every rank processed one
    workload per step, so the job did world * flops_per_step per step."""
    ms_per_step = total_ms / steps
    return {
        "ms_per_step": ms_per_step,
        "value": world * flops_per_step / (ms_per_step * 1e-3) / 1e12,
        "e2e": world * flops_per_step / (e2e_ms * 1e-3) / 1e12,
        "fine_ms": fine_total_ms / steps,
    }


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples taken during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.device_index = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.device_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, ValueError):
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
        self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


PAIR_MAX_TOPK = 24        # launch_fine: short rows run the persistent two-cube kernel


def fine_kernel_name(w):
    """The fine kernel vsa_sparse_attn_fwd launches for this workload."""
    if w.head_dim == 128 and not w.linear and w.topk <= PAIR_MAX_TOPK:
        return "fine_pair_kernel<128>"
    return "fine_attn_kernel<%d, %s>" % (w.head_dim, "LIN" if w.linear else "-")


def gpu_step_fn(w, q, k, v, out, attn, fine_events):
    """One hot-path pass on the current stream; fine_events brackets the fine kernel."""
    from block_sparse_attention_30_b200 import ops

    def step(record_fine=False):
        ops.vsa_select_blocks(q, k, w.T, w.H, w.W, w.topk, attn.block_idx, attn.workspace, w.tile)
        if w.linear:
            ops.vsa_linear_branch_fwd(k, v, attn.lin_S, attn.lin_z, w.T, w.H, w.W, attn.workspace)
        if record_fine:
            fine_events[0].record()
        ops.vsa_sparse_attn_fwd(q, k, v, attn.block_idx, out, w.T, w.H, w.W, w.topk,
                                attn.workspace, attn.lin_S, attn.lin_z, w.tile)
        if record_fine:
            fine_events[1].record()
    return step


def run_gpu(args):
    rank, local_rank, world = dist_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    from block_sparse_attention_30_b200 import build, ops
    build.build()
    w = WORKLOADS[args.workload]
    seed = rank_seed(list(WORKLOADS).index(w.name), rank)
    q_h, k_h, v_h = synth.make_workload_inputs(w, seed=seed)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    out = torch.empty_like(q)
    attn = ops.BlockSparseVideoAttention(w.B, w.heads, w.head_dim, w.T, w.H, w.W, w.topk, w.tile,
                                         linear=w.linear, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    fine_ev = [torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)]
    step = gpu_step_fn(w, q, k, v, out, attn, fine_ev)

    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()
    if attn.status() != 0:
        raise RuntimeError("device status not OK after warm-up")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    fine_ms = []
    clocks = ClockSampler(local_rank)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)                          # let the sampler take its first reading
    wall0 = time.perf_counter()
    for i in range(args.steps):
        flush.fill_(i & 255)                 # evict L2 between steps (outside the events)
        starts[i].record()
        step(record_fine=True)
        ends[i].record()
        ends[i].synchronize()
        fine_ms.append(fine_ev[0].elapsed_time(fine_ev[1]))
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = sum(step_ms)
    status = attn.status()

    # end to end through the public API (ops.HostPipeline): every step copies
    # its inputs from pinned host memory and its output back; consecutive
    # steps overlap (H2D of step i+1 and D2H of step i-1 under the kernels of
    # step i), as a batch stream through the library runs
    e2e_steps = max(2, min(args.steps, 8))
    qp, kp, vp = (x.pin_memory() for x in (q_h, k_h, v_h))
    outs_h = [torch.empty(q_h.shape, dtype=q_h.dtype).pin_memory() for _ in range(2)]
    pipe = ops.HostPipeline(attn, q_h.shape, q_h.dtype, dev)
    pipe.run([(qp, kp, vp, outs_h[0])])                       # warm-up (buffers, streams)
    pipe.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e0.record(pipe.s_in)
    e1 = pipe.run([(qp, kp, vp, outs_h[i % 2]) for i in range(e2e_steps)])
    pipe.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    h2d = 3 * q_h.numel() * q_h.element_size()
    d2h = outs_h[0].numel() * outs_h[0].element_size()

    total_ms, e2e_ms, fine_total = max_over_ranks([total_ms, e2e_ms, sum(fine_ms)], device=dev)

    if rank == 0:
        flops = w.fine_flops()
        agg = aggregate(world, flops, args.steps, total_ms, e2e_ms, fine_total)
        ms_per_step, value, fine_avg_ms = agg["ms_per_step"], agg["value"], agg["fine_ms"]
        fine_tflops = flops / (fine_avg_ms * 1e-3) / 1e12
        peaks, src = load_peaks()
        peak = peaks["bf16_tflops"]
        # pool, coarse, top-k, fine; + linear state and the (S, z) operand pack
        launches_per_step = 4 + (2 if w.linear else 0)
        result = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) noise + per-cube N(0,1) offsets, Wan latent shapes)",
            "config": {
                "workload": w.name, "B": w.B, "heads": w.heads, "head_dim": w.head_dim,
                "grid": [w.T, w.H, w.W], "tile": list(w.tile), "num_tiles": w.num_tiles,
                "topk": w.topk, "sparsity": round(w.sparsity, 4), "linear_branch": w.linear,
                "fine_flops_per_step": flops,
                "l2": "256 MiB write between steps (outside the timed events); inputs 3x%.0f MB exceed L2"
                      % (q_h.numel() * 2 / 1e6),
                "parallelism": f"independent batch per GPU x{world} (no data-path collective)",
            },
            "fine_kernel": {"ms_per_call": round(fine_avg_ms, 4), "tflops": round(fine_tflops, 2),
                            "pct_of_bf16_peak": round(100 * fine_tflops / peak, 2),
                            "pct_of_bf16_sustained": round(100 * fine_tflops / peaks["bf16_tflops_sustained"], 2)},
            "pct_of_bf16_peak": round(100 * (value / world) / peak, 2),
            "roofline": {
                "bound": "tensor", "kernel": fine_kernel_name(w),
                "achieved": round(fine_tflops, 2), "peak": peak, "unit": "TFLOP/s",
                "frac": round(fine_tflops / peak, 4),
                "peak_source": f"{src} bf16_tflops (burst)",
                "traffic": args.traffic if args.traffic is not None else profiled_traffic(w.name),
                "traffic_unit": "bytes per launch (ncu dram read+write)",
                "algorithmic_bytes": 4 * w.B * w.N * w.heads * w.head_dim * 2,
            },
            "e2e": {"value": round(agg["e2e"], 2), "unit": "TFLOP/s",
                    "ms_per_step": round(e2e_ms, 3), "steps": e2e_steps,
                    "pipelined": "ops.HostPipeline: H2D of step i+1 and D2H of step i-1 overlap the kernels of step i",
                    "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk,
            "device_status": status,
            "wall_s": round(wall, 3),
        }
        if world == 1 and not args.no_cpu_baseline:
            result["cpu_baseline"] = cpu_baseline(w, q_h, k_h, v_h, args.cpu_heads)
        print(json.dumps(result), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def run_sharded(args):
    """Sequence-sharded forward over N GPUs (strong scaling): every rank holds
    tokens [r*N/P, (r+1)*N/P) of q, k, v of ONE workload; a step is the
    seq -> heads all-to-all, select + fine on this rank's heads, and the
    heads -> seq all-to-all (block_sparse_attention_30_b200.sharded)."""
    import datetime
    import torch.distributed as dist
    rank, local_rank, world = dist_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    from block_sparse_attention_30_b200 import build, sharded
    build.build()
    w = WORKLOADS[args.workload]
    q_h, k_h, v_h = synth.make_workload_inputs(w, seed=list(WORKLOADS).index(w.name))
    Nl = w.N // world
    sl = slice(rank * Nl, (rank + 1) * Nl)
    qs, ks, vs = (x[:, sl].contiguous().to(dev) for x in (q_h, k_h, v_h))
    attn = sharded.SequenceShardedAttention(w.B, w.heads, w.head_dim, w.T, w.H, w.W, w.topk, w.tile,
                                            linear=w.linear, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        flush.fill_(1)
        attn(qs, ks, vs)
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clocks = ClockSampler(local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    for i in range(args.steps):
        flush.fill_(i & 255)
        starts[i].record()
        attn(qs, ks, vs)
        ends[i].record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    total_ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    # end to end: this rank's shard from pinned host memory and its output back
    qp, kp, vp = (x[:, sl].contiguous().pin_memory() for x in (q_h, k_h, v_h))
    out_h = torch.empty(qp.shape, dtype=qp.dtype).pin_memory()
    bufs = [torch.empty_like(qs) for _ in range(3)]
    e2e_steps = max(2, min(args.steps, 8))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    e0.record()
    for _ in range(e2e_steps):
        for b, hsrc in zip(bufs, (qp, kp, vp)):
            b.copy_(hsrc, non_blocking=True)
        out_h.copy_(attn(*bufs), non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], device=dev)
    status = attn.attn.status()
    if rank == 0:
        flops = w.fine_flops()
        ms = total_ms / args.steps
        peaks, src = load_peaks()
        print(json.dumps({
            "metric": METRIC, "value": round(flops / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) noise + per-cube N(0,1) offsets, Wan latent shapes)",
            "config": {"workload": w.name, "B": w.B, "heads": w.heads, "head_dim": w.head_dim,
                       "grid": [w.T, w.H, w.W], "topk": w.topk, "linear_branch": w.linear,
                       "fine_flops_per_step": flops,
                       "l2": "256 MiB write between steps (outside the timed events)",
                       "parallelism": f"sequence-sharded inputs, heads exchanged by all-to-all over {world} GPU(s)"},
            "comm": {"all_to_all_bytes_sent_per_rank_per_step": sharded.exchange_bytes(
                w.B, w.N, w.heads, w.head_dim, world), "collectives_per_step": 4 if world > 1 else 0},
            "pct_of_bf16_peak": round(100 * flops / (ms * 1e-3) / 1e12 / world / peaks["bf16_tflops"], 2),
            "e2e": {"value": round(flops / (e2e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                    "ms_per_step": round(e2e_ms, 3), "steps": e2e_steps,
                    "h2d_bytes_per_step": 3 * qp.numel() * qp.element_size() * world,
                    "d2h_bytes_per_step": out_h.numel() * out_h.element_size() * world},
            "gpu_launches": (4 + (2 if w.linear else 0)) * args.steps,
            "clocks": clk, "device_status": status,
        }), flush=True)
    if world > 1:
        dist.destroy_process_group()


# ------------------------------------------------------------ per-kernel lines

def run_kernels(args):
    """One JSON line per hot-path kernel on one workload: its time (CUDA
    events, median of `steps` calls, L2 flushed before each) against its own
    roofline -- HBM GB/s for the copies, pooling and the linear state, tensor
    TFLOP/s for the fine pass."""
    from block_sparse_attention_30_b200 import build, ops
    build.build()
    dev = torch.device("cuda", 0)
    w = WORKLOADS[args.workload]
    q_h, k_h, v_h = synth.make_workload_inputs(w)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    attn = ops.BlockSparseVideoAttention(w.B, w.heads, w.head_dim, w.T, w.H, w.W, w.topk, w.tile,
                                         linear=True, device=dev)
    out = torch.empty_like(q)
    nt = w.num_tiles
    tiles = torch.empty((w.B, w.heads, nt, 64, w.head_dim), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    peaks, src = load_peaks()
    elem = w.B * w.N * w.heads * w.head_dim * 2            # bytes of one [B][N][heads][d] tensor
    tile_bytes = tiles.numel() * 2

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        ts = []
        for i in range(max(args.steps, 3)):
            flush.fill_(i & 255)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return sorted(ts)[len(ts) // 2]

    rows = [
        ("gather_tiles (cube gather)", lambda: ops.vsa_gather_tiles(q, tiles, w.T, w.H, w.W, w.tile),
         "hbm", elem + tile_bytes),
        ("scatter_tiles (cube scatter)", lambda: ops.vsa_scatter_tiles(tiles, out, w.T, w.H, w.W, w.tile),
         "hbm", 2 * elem),
        ("select_blocks (pool, coarse scores, top-k)", lambda: ops.vsa_select_blocks(q, k, w.T, w.H, w.W, w.topk,
                                                                  attn.block_idx, attn.workspace, w.tile),
         "hbm", 2 * elem + w.B * w.heads * nt * w.topk * 4),
        ("linear_branch_fwd (linear state)", lambda: ops.vsa_linear_branch_fwd(k, v, attn.lin_S, attn.lin_z, w.T, w.H, w.W,
                                                                           attn.workspace),
         "hbm", 2 * elem),
        ("sparse_attn_fwd (fine pass, gather and scatter fused)", lambda: ops.vsa_sparse_attn_fwd(q, k, v, attn.block_idx, out, w.T, w.H, w.W,
                                                                            w.topk, attn.workspace, tile=w.tile),
         "tensor", w.fine_flops()),
        ("sparse_attn_fwd + linear apply", lambda: ops.vsa_sparse_attn_fwd(
            q, k, v, attn.block_idx, out, w.T, w.H, w.W, w.topk, attn.workspace, attn.lin_S, attn.lin_z, w.tile),
         "tensor", w.fine_flops()),
    ]
    # backward pass (trainable sparse branch): the training forward (with the
    # per-row lse) and the backward; algorithmic FLOPs of the backward are
    # the five products S, dP, dV, dQ, dK per kept (query, key) cube pair
    lse = torch.empty((w.B, w.heads, nt, 64), dtype=torch.float32, device=dev)
    out32 = torch.empty(q.shape, dtype=torch.float32, device=dev)
    g_out = torch.randn(q.shape, device=dev).mul_(0.5).to(torch.bfloat16)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    rows += [
        ("sparse_attn_fwd_train (training forward)", lambda: ops.vsa_sparse_attn_fwd_train(
            q, k, v, attn.block_idx, out, out32, lse, w.T, w.H, w.W, w.topk, attn.workspace, w.tile),
         "tensor", w.fine_flops()),
        ("sparse_attn_bwd (backward)", lambda: ops.vsa_sparse_attn_bwd(
            q, k, v, out32, g_out, attn.block_idx, lse, dq, dk, dv, w.T, w.H, w.W, w.topk,
            attn.workspace, w.tile),
         "tensor", 2.5 * w.fine_flops()),
        # linear branch backward: reads q, k, v, dout and writes dq, dk, dv
        # (the d x d states are a few MB); its products are ~10 d^2 FLOPs per
        # token, far below the tensor-core ridge, so HBM bounds it
        ("linear_branch_bwd (linear branch backward)", lambda: ops.vsa_linear_branch_bwd(
            q, k, v, g_out, attn.lin_S, attn.lin_z, dq, dk, dv, w.T, w.H, w.W, attn.workspace),
         "hbm", 7 * elem),
    ]
    # low-precision fine pass: E4M3 codes of q and k (one byte each) with
    # per-cube scales, then the fine kernel with Q K^T in E4M3; its FLOPs
    # are the same effective count, its fraction is of the bf16 peak (half
    # of the products run at the E4M3 rate, so a mixed ceiling is 4/3 of it)
    q8, k8 = (torch.empty(q.shape, dtype=torch.uint8, device=dev) for _ in range(2))
    sq, sk = (torch.empty((w.B, w.heads, nt), dtype=torch.float32, device=dev) for _ in range(2))
    rows += [
        ("quantize_qk_e4m3 (low-precision pre-pass)", lambda: ops.vsa_quantize_qk_e4m3(
            q, k, q8, k8, sq, sk, w.T, w.H, w.W, w.tile), "hbm", 3 * elem),
        ("sparse_attn_fwd_e4m3 (E4M3 Q K^T, bf16 P V)", lambda: ops.vsa_sparse_attn_fwd_e4m3(
            q8, k8, sq, sk, v, attn.block_idx, out, w.T, w.H, w.W, w.topk, attn.workspace, w.tile),
         "tensor", w.fine_flops()),
        ("sparse_linear_attn_fwd_e4m3 (SageSLA: E4M3 sparse + linear apply)",
         lambda: ops.vsa_sparse_linear_attn_fwd_e4m3(
             q8, k8, sq, sk, q, v, attn.block_idx, attn.lin_S, attn.lin_z, out, w.T, w.H, w.W, w.topk,
             attn.workspace, w.tile),
         "tensor", w.fine_flops()),
    ]
    for name, fn, bound, units in rows:
        ms = timed(fn)
        if bound == "hbm":
            achieved, peak, unit = units / (ms * 1e-3) / 1e9, peaks["hbm_gbs"], "GB/s"
        else:
            achieved, peak, unit = units / (ms * 1e-3) / 1e12, peaks["bf16_tflops"], "TFLOP/s"
        print(json.dumps({"kernel": name, "workload": w.name, "ms": round(ms, 4), "bound": bound,
                          "achieved": round(achieved, 2), "peak": peak, "unit": unit,
                          "frac": round(achieved / peak, 4), "peak_source": src,
                          "algorithmic": units}), flush=True)
    if attn.status() != 0:
        raise RuntimeError("device status not OK")


# -------------------------------------------------------------------- oracle

def oracle_sample(w, q, k, v, heads):
    """Select + fine (+ linear) of the oracle on the first `heads` heads (all
    query cubes of each); returns (seconds, fine FLOPs covered)."""
    from oracle import oracle as O
    qs, ks, vs = (x[:, :, :heads].contiguous() for x in (q, k, v))
    t0 = time.perf_counter()
    idx = O.select(qs, ks, w.B, heads, w.head_dim, w.T, w.H, w.W, w.topk, w.tile)
    out = O.fine(qs, ks, vs, idx, w.B, heads, w.head_dim, w.T, w.H, w.W, w.tile)
    if w.linear:
        S, z = O.linear_state(ks, vs, w.B, heads, w.head_dim, w.N)
        out = out + O.linear_apply(qs, S, z, w.B, heads, w.head_dim, w.N)
    dt = time.perf_counter() - t0
    return dt, w.fine_flops() * heads / w.heads


def cpu_baseline(w, q, k, v, heads):
    from oracle import oracle as O
    heads = min(heads, w.heads)
    dt, flops = oracle_sample(w, q, k, v, heads)
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": O.num_threads(),
            "kind": "oracle", "seconds": round(dt, 2),
            "sample": f"{heads} of {w.heads} heads, all {w.num_tiles} query cubes each: "
                      f"fp64 select + fine{' + linear' if w.linear else ''}"}


def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return                                   # rank 0 alone runs the CPU oracle
    from oracle import oracle as O
    w = WORKLOADS[args.workload]
    q, k, v = synth.make_workload_inputs(w)
    heads = min(args.cpu_heads, w.heads)
    for _ in range(args.warmup):
        oracle_sample(w, q, k, v, 1)
    times = []
    flops = 0.0
    for _ in range(args.steps):
        dt, flops = oracle_sample(w, q, k, v, heads)
        times.append(dt)
    sec = sum(times) / len(times)
    value = flops / sec / 1e12
    cb = {"value": round(value, 6), "unit": "TFLOP/s", "cores": O.num_threads(), "kind": "oracle",
          "sample": f"{heads} of {w.heads} heads per step, all {w.num_tiles} query cubes each: "
                    f"fp64 select + fine{' + linear' if w.linear else ''}"}
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(sec * 1e3, 2), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "heads": w.heads, "head_dim": w.head_dim,
                   "grid": [w.T, w.H, w.W], "topk": w.topk, "sample_heads": heads},
        "cpu_baseline": cb,
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-heads", type=int, default=4, help="heads in the oracle's timed sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernels", action="store_true",
                    help="print one roofline line per hot-path kernel instead of the step line")
    ap.add_argument("--sharded", action="store_true",
                    help="sequence-sharded inputs over the ranks, heads exchanged by all-to-all "
                         "(strong scaling); default: one independent workload per rank")
    ap.add_argument("--traffic", type=float, default=None,
                    help="DRAM bytes per fine launch from an ncu capture (reported as-is)")
    args = ap.parse_args()
    _, _, world = dist_env()
    if world != args.gpus:
        if args.gpus > 1 and world == 1:
            sys.exit("for --gpus > 1 launch with torch.distributed.run --nproc-per-node N")
    if args.impl == "reference":
        run_reference(args)
    elif args.kernels:
        if not torch.cuda.is_available():
            sys.exit("bench.py --kernels needs a CUDA device")
        run_kernels(args)
    else:
        if not torch.cuda.is_available():
            sys.exit("bench.py needs a CUDA device for --impl ours")
        if args.sharded:
            run_sharded(args)
        else:
            run_gpu(args)


if __name__ == "__main__":
    main()

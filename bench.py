"""Benchmark of the block-sparse / piecewise attention hot path on B200.

One step = one pass of the whole PISA path over one batch of the workload:
bsa_precompute -> bsa_route -> bsa_forward (the fixed-mask builder is built once per
model and is not part of a PISA step). Default workload: video PISA, batch 1, 40 heads,
L = 16384 (16 frames x 32 x 32), d = 128, block 128, density 12.5% (top-16 of 128).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--shard replicas|heads] [--no-e2e] [--no-cpu]

Prints ONE JSON line on rank 0. With torchrun (N > 1) every rank runs the same
workload on its own GPU (replicas, weak scaling; the path needs no data exchange), or
with --shard heads its own contiguous range of the workload's heads (strong scaling; the
optional all-gather of O is timed apart from the step). The time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from piecewise_attention_diffusion_b200 import synth  # noqa: E402

METRIC = "bsa_forward effective TFLOPS (executed FLOPs) over precompute+route+forward"
LAMBDA = 1.0


# ------------------------------------------------------------------ FLOP counting
def forward_flops(w, k_top: int, mode: str, row_lens=None) -> float:
    """Executed FLOPs of bsa_forward: per (batch, head, query block i)
    |S_i| * 4 B^2 d  (+ PISA: B * (4 d |U_i| + 2 d^2)); exps and softmax not counted.
    |S_i| = k_top for routed lists, the row length for a fixed mask (row_lens)."""
    M, B, d = w.n_blocks, w.block, w.head_dim
    lens = [k_top] * M if row_lens is None else list(row_lens)
    total = 0.0
    for n in lens:
        if mode == "pisa_block":  # every block is a tile (exact or linearised)
            total += M * 4.0 * B * B * d
            continue
        total += n * 4.0 * B * B * d
        if mode == "pisa":
            total += B * (4.0 * d * (M - n) + 2.0 * d * d)
    return w.batch * w.heads * total


GENERATOR_TEXT = {
    "iid": "N(0,1)",
    "block_centres": "K = per-block centre + 0.5 N(0,1), V = N(0,1)",
    "field2d_hot": "smooth 2-D field + 0.3 N(0,1), 4 hot blocks x3",
    "field3d": "smooth 3-D field + 0.3 N(0,1)",
}


def needs_precompute(w) -> bool:
    """The statistics feed the routing and PISA's Taylor tail; a fixed mask in the other
    modes needs neither."""
    return not w.mask or w.mode == "pisa"


def launches_per_step(w) -> int:
    """Kernels one step launches: precompute 3 (statistics, reduce, norm; skipped for a
    fixed keep-or-drop mask), route 2 (pooling, scoring; not for a fixed mask), forward:
    list validation, the PISA statistics' bf16 conversion, the forward kernel."""
    pre = 3 if needs_precompute(w) else 0
    route = 0 if w.mask else 2
    fwd = 3 if w.mode == "pisa" else 2
    return pre + route + fwd


def precompute_flops(w) -> float:
    """K_j^T V_j per block (2 B d^2), counted once."""
    return w.batch * w.heads * w.n_blocks * 2.0 * w.block * w.head_dim ** 2


def route_flops(w) -> float:
    """pooled-query x centroid scores (2 M^2 d per head)."""
    return w.batch * w.heads * 2.0 * w.n_blocks ** 2 * w.head_dim


def forward_bytes(w, mode: str) -> float:
    """Algorithmic HBM bytes of bsa_forward: Q, K, V read and O written once (bf16),
    plus the fp32 statistics for PISA."""
    BH, L, d, M = w.batch * w.heads, w.seq_len, w.head_dim, w.n_blocks
    b = 4.0 * BH * L * d * 2
    if mode == "pisa":
        b += BH * (2 * M * d + d * d) * 4
    return b


# ---------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples (every 50 ms, timestamped) of SM clock and throttle reasons;
    summary() keeps the samples that fall inside the timed region (widened by 0.25 s
    on both sides so that a short region still gets samples taken under load)."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def stop(self):
        if self.proc is not None:
            time.sleep(0.3)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self) -> dict:
        import datetime
        if self.proc is None or self.path is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for ln in f:
                p = [x.strip() for x in ln.split(",")]
                if len(p) < 10 or not p[2].replace(".", "").isdigit():
                    continue
                try:
                    ts = datetime.datetime.strptime(p[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                except ValueError:
                    continue
                rows.append([ts] + p[1:])
        os.unlink(self.path)
        inside = [r for r in rows if self.t0 - 0.25 <= r[0] <= self.t1 + 0.25]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None,
                    "reasons": [f"no samples in the timed region ({len(rows)} outside)"]}
        sm = [float(r[2]) for r in inside]
        mx = max(float(r[3]) for r in inside)
        reasons = sorted({self.REASONS[i] for r in inside for i in range(4)
                          if r[6 + i] == "Active"})
        pw = [float(r[4]) for r in inside if r[4].replace(".", "").isdigit()]
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(inside), "power_w_max": max(pw) if pw else None,
                "window_s": round(self.t1 - self.t0, 3)}


# ------------------------------------------------------------------ dist helpers
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest of every rank's x (the slowest rank's time), on every rank. The tensor
    lives where the process group's backend needs it (NCCL: this rank's GPU)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def replica_value(flops_per_rank: float, ms_slowest: float, world: int) -> float:
    """Whole-job TFLOP/s of `world` replicas that each ran `flops_per_rank` per step, timed
    by the slowest rank (weak scaling: every rank does the full workload)."""
    return world * flops_per_rank / (ms_slowest * 1e-3) / 1e12


def sum_over_ranks(x: float, world: int) -> float:
    """The sum of every rank's x, on every rank."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def job_value(flops_this_rank: float, ms_slowest: float, world: int, shard: str) -> float:
    """Whole-job TFLOP/s, timed by the slowest rank. Replicas: every rank ran the whole
    workload (weak scaling). Head shards: the ranks' FLOPs add up to the workload's (strong
    scaling)."""
    if shard == "heads":
        return sum_over_ranks(flops_this_rank, world) / (ms_slowest * 1e-3) / 1e12
    return replica_value(flops_this_rank, ms_slowest, world)


def shard_workload(w, world: int, rank: int):
    """This rank's part of `w` under head sharding: the workload restricted to the rank's
    contiguous range of flattened (batch * heads) indices (batch 1), and that range."""
    import dataclasses
    from piecewise_attention_diffusion_b200.shard import head_range
    BH = w.batch * w.heads
    if world > BH:
        raise SystemExit(f"--shard heads: {world} ranks for {BH} heads")
    h0, h1 = head_range(BH, world, rank)
    return dataclasses.replace(w, batch=1, heads=h1 - h0), (h0, h1)


def peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"bf16_tflops": d["bf16_tflops"], "hbm_gbs": d["hbm_gbs"], "source": "measured"}
    return {"bf16_tflops": 1590.0, "hbm_gbs": 6650.0, "source": "fallback"}


def load_traffic(w) -> float | None:
    """DRAM bytes per launch of the forward kernel from the committed ncu summary, only
    while the kernel source is the one that was captured and the head count matches
    (None otherwise: counters of another kernel do not describe this one)."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    src = os.path.join(ROOT, "piecewise_attention_diffusion_b200", "csrc", "forward_tc.cu")
    if not os.path.exists(p) or not os.path.exists(src):
        return None
    with open(p) as f:
        e = json.load(f).get(w.name)
    if e is None or e.get("scaled_to_heads") != w.heads:
        return None
    with open(src, "rb") as f:
        h = hashlib.sha256(f.read()).hexdigest()
    if not h.startswith(e.get("source_sha256_prefix", "?")):
        return None
    return e.get("bytes_per_launch")


# -------------------------------------------------------------- CPU oracle timing
def _steps_done(w) -> str:
    done = (["precomputed"] if (not w.mask or w.mode != "keep_or_drop") else []) \
        + ([] if w.mask else ["routed"]) + ["attended"]
    return ", ".join(done[:-1]) + (" and " if len(done) > 1 else "") + done[-1]



def oracle_sample(w, k_top, heads_sample: int, seed: int = 0) -> dict:
    """Time the fp64 oracle (as it stands) on `heads_sample` full heads and scale to
    the whole workload by the head count."""
    import oracle as orc
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = 1
    heads = list(range(heads_sample))
    q, k, v = synth.make_qkv(w, seed=seed, heads=heads)
    scale = 1 / math.sqrt(w.head_dim)
    fixed = orc.dense_to_csr(orc.mask_dense(**w.mask)) if w.mask else None
    kv = w.valid_tokens()
    t0 = time.perf_counter()
    for h in heads:
        qf, kf, vf = (x[h].to(torch.float64).numpy() for x in (q, k, v))
        if fixed is not None and w.mode == "keep_or_drop":
            orc.keep_or_drop_head(qf, kf, vf, fixed[0], fixed[1], w.block, scale, key_valid=kv)
            continue
        kbar, vsum, H, Hbar, Mn = orc.precompute_head(kf, vf, w.block, kv)
        if fixed is not None:
            rp, ci = fixed
        else:
            rp, ci, _ = orc.route_head(qf, kbar, Mn, w.block, k_top, LAMBDA, scale, kv)
        if w.mode == "pisa":
            orc.pisa_head(qf, kf, vf, rp, ci, w.block, scale, kbar, vsum, Hbar, key_valid=kv)
        elif w.mode == "pisa_block":
            orc.pisa_head(qf, kf, vf, rp, ci, w.block, scale, kbar, vsum, Hbar, Hblocks=H,
                          key_valid=kv)
        else:
            orc.keep_or_drop_head(qf, kf, vf, rp, ci, w.block, scale, key_valid=kv)
    dt = time.perf_counter() - t0
    BH = w.batch * w.heads
    return {"seconds_sample": dt, "seconds_full_est": dt * BH / len(heads), "cores": threads,
            "sample": f"{len(heads)} of {BH} heads, each fully {_steps_done(w)} (all "
                      f"{w.n_blocks} query blocks{', fixed mask' if w.mask else ''}); "
                      f"time scaled by heads"}


# --------------------------------------------------------------------- our arm
L2_BYTES = 126 * 2 ** 20
# the forward of these workloads is reported beside the headline: the long-sequence
# sweep's 4K, 16K and 32K points at 12.5% density in both modes, and the other configs
SWEEP_WORKLOADS = ("sweep_L4096_d125_pisa", "sweep_L4096_d125_keep_or_drop",
                   "sweep_L16384_d125_pisa", "sweep_L16384_d125_keep_or_drop",
                   "sweep_L32768_d125_pisa", "sweep_L32768_d125_keep_or_drop",
                   "tiny_pisa", "multimodal_dit", "image_pisa")


def input_bytes(w) -> int:
    """Bytes of Q, K and V (bf16) of a workload."""
    return 3 * w.batch * w.heads * w.seq_len * w.head_dim * 2


def needs_flush(w) -> bool:
    """Inputs that fit twice in L2 are timed with an L2 flush before every step."""
    return input_bytes(w) < 2 * L2_BYTES


def config_of(w, world: int, shard: str = "replicas") -> dict:
    """The workload as both arms name it (identical keys and values)."""
    k_top = 0 if w.mask else w.top_k()
    l2 = (f"inputs larger than L2 (Q+K+V = {input_bytes(w) / 1e6:.0f} MB)" if not needs_flush(w)
          else f"L2 flushed before every step (Q+K+V = {input_bytes(w) / 1e6:.0f} MB)")
    return {"workload": w.name, "batch": w.batch, "heads": w.heads, "seq_len": w.seq_len,
            "head_dim": w.head_dim, "block": w.block, "mode": w.mode, "density": w.density,
            "k_top": None if w.mask else k_top, "lambda": LAMBDA,
            "lists": "fixed multimodal mask (shared)" if w.mask else "bsa_route top-k",
            "real_tokens_per_block": w.valid_tokens() if w.key_valid else None,
            "parallelism": f"{shard} x{world}", "l2": l2}


class Path:
    """Device buffers and the launch sequence of one step of a workload:
    bsa_precompute -> bsa_route -> bsa_forward (the statistics and routing are skipped
    where the workload does not need them)."""

    def __init__(self, w, q, k, v, dev):
        from piecewise_attention_diffusion_b200 import bsattn as b
        self.b, self.w, self.dev = b, w, dev
        self.k_top = 0 if w.mask else w.top_k()  # a fixed mask has no top-k
        BH, M, L, d = w.batch * w.heads, w.n_blocks, w.seq_len, w.head_dim
        self.qd, self.kd, self.vd = q.to(dev), k.to(dev), v.to(dev)
        self.st = torch.zeros(1, dtype=torch.int32, device=dev)
        # real tokens per block (token padding), a constant of the workload like its mask
        self.kv = None if not w.key_valid else torch.tensor(w.valid_tokens(), dtype=torch.int32,
                                                            device=dev)
        f32 = dict(dtype=torch.float32, device=dev)
        self.stats = dict(kbar=torch.empty(BH, M, d, **f32), vsum=torch.empty(BH, M, d, **f32),
                          Hbar=torch.empty(BH, d, d, **f32), Mnorm=torch.empty(BH, M, **f32))
        if w.mask:
            # fixed multimodal pattern: one shared list for every head, built once
            self.rp, self.ci = b.build_mask(b.MaskDesc(**w.mask), device=dev, status=self.st)
            torch.cuda.synchronize()
            self.row_lens = np.diff(self.rp.cpu().numpy()).tolist()
            self.per_head = 0
        else:
            self.rp = torch.empty(BH * (M + 1), dtype=torch.int32, device=dev)
            self.ci = torch.empty(BH * M * self.k_top, dtype=torch.int32, device=dev)
            self.row_lens = None
            self.per_head = 1
        self.O = torch.empty_like(self.qd)
        self.ws_p = b.workspace(b.CALL_PRECOMPUTE, w.batch, w.heads, L, d, w.block, dev)
        self.ws_r = b.workspace(b.CALL_ROUTE, w.batch, w.heads, L, d, w.block, dev)
        self.ws_f = b.workspace(b.CALL_FORWARD, w.batch, w.heads, L, d, w.block, dev)
        self.mode = {"pisa": b.MODE_PISA, "pisa_block": b.MODE_PISA_BLOCK}.get(
            w.mode, b.MODE_KEEP_OR_DROP)
        self.stream = torch.cuda.current_stream(dev)

    def step(self, qx=None, kx=None, vx=None, ev=None, out=None):
        b, w, st, s = self.b, self.w, self.st, self.stats
        qx = self.qd if qx is None else qx
        kx = self.kd if kx is None else kx
        vx = self.vd if vx is None else vx
        if ev:
            ev[0].record(self.stream)
        if needs_precompute(w):
            b.bsa_precompute(kx, vx, w.block, s["kbar"], s["vsum"], s["Hbar"], s["Mnorm"], None,
                             self.ws_p, st, key_valid=self.kv)
        if ev:
            ev[1].record(self.stream)
        if not w.mask:
            b.bsa_route(qx, s["kbar"], s["Mnorm"], w.block, self.k_top, LAMBDA, 0.0, self.rp,
                        self.ci, None, self.ws_r, st, key_valid=self.kv)
        if ev:
            ev[2].record(self.stream)
        b.bsa_forward(qx, kx, vx, w.block, self.rp, self.ci, self.per_head, self.mode,
                      s["kbar"], s["vsum"], s["Hbar"], 0.0, self.O if out is None else out,
                      None, self.ws_f, st, key_valid=self.kv)
        if ev:
            ev[3].record(self.stream)

    def check_status(self):
        if self.st.item() != 0:
            raise RuntimeError(f"device status {self.b.status_string(self.st.item())}")

    def measure(self, steps: int, warmup: int, world: int = 1) -> dict:
        """Time `steps` steps after `warmup` untimed ones, CUDA events on the launching
        stream around every phase of every step, max over ranks. Workloads whose inputs
        fit in L2 get an L2 flush (a 256 MB write) before every step, outside the
        events; the step time is then the sum of the per-step event spans."""
        flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=self.dev) \
            if needs_flush(self.w) else None
        for _ in range(warmup):
            self.step()
        torch.cuda.synchronize()
        self.check_status()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
        t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        t0 = time.time()
        t_start.record(self.stream)
        for n in range(steps):
            if flush is not None:
                flush.zero_()
            self.step(ev=evs[n])
        t_end.record(self.stream)
        torch.cuda.synchronize()
        t1 = time.time()
        barrier(world)
        self.check_status()
        span = lambda a, z: sum(e[a].elapsed_time(e[z]) for e in evs) / steps
        ms_step = t_start.elapsed_time(t_end) / steps if flush is None else span(0, 3)
        F_fwd = forward_flops(self.w, self.k_top, self.w.mode, self.row_lens)
        F_step = F_fwd + (precompute_flops(self.w) if needs_precompute(self.w) else 0.0) \
            + (0.0 if self.w.mask else route_flops(self.w))
        return {"ms_step": max_over_ranks(ms_step, world),
                "fwd_ms": max_over_ranks(span(2, 3), world),
                "pre_ms": span(0, 1), "route_ms": span(1, 2), "F_fwd": F_fwd, "F_step": F_step,
                "t0": t0, "t1": t1, "flushed": flush is not None}


def run_sweep(args, world, rank, local) -> dict:
    """Forward (and step) numbers of the other workloads, measured in the same run: per
    workload its own inputs, 3 warm-up steps and `--sweep-steps` timed steps."""
    dev = torch.device("cuda", local)
    pk = peaks()
    out, cache = {}, {}
    for name in SWEEP_WORKLOADS:
        w = synth.workloads()[name]
        key = (w.seq_len, w.heads, w.batch, w.head_dim, w.block, w.generator, w.grid,
               w.key_valid)
        if key not in cache:
            cache.clear()
            cache[key] = synth.make_qkv(w, seed=args.seed + rank)
        path = Path(w, *cache[key], dev)
        m = path.measure(args.sweep_steps, 3, world)
        tf = m["F_fwd"] / (m["fwd_ms"] * 1e-3) / 1e12
        out[name] = {"seq_len": w.seq_len, "heads": w.heads, "mode": w.mode,
                     "density": w.density, "k_top": None if w.mask else path.k_top,
                     "forward_ms": round(m["fwd_ms"], 4), "forward_tflops": round(tf, 2),
                     "frac": round(tf / pk["bf16_tflops"], 4),
                     "precompute_ms": round(m["pre_ms"], 4), "route_ms": round(m["route_ms"], 4),
                     "step_ms": round(m["ms_step"], 4), "forward_gflop": round(m["F_fwd"] / 1e9, 3),
                     "l2": "flushed before every step" if m["flushed"] else "inputs larger than L2"}
        del path
    return {"steps": args.sweep_steps, "warmup": 3, "peak_tflops": pk["bf16_tflops"],
            "peak_source": f"{pk['source']} bf16_tflops (burst)", "points": out}


def run_ours(args, w, world, rank, local):
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w_full, shard = w, args.shard
    if shard == "heads":
        # this rank's heads of the one workload (the same bytes the whole run would hold)
        w, (h0, h1) = shard_workload(w_full, world, rank)
        q, k, v = (x.unsqueeze(0) for x in synth.make_qkv(w_full, seed=args.seed,
                                                          heads=range(h0, h1)))
    else:
        # replicas: every rank runs the whole workload on its own seed
        q, k, v = synth.make_qkv(w, seed=args.seed + rank)
    path = Path(w, q, k, v, dev)
    BH, L, d = w.batch * w.heads, w.seq_len, w.head_dim

    clk = ClockSampler(local).start()
    time.sleep(0.5)  # let nvidia-smi start sampling before the GPU work begins
    m = path.measure(args.steps, args.warmup, world)
    clk.t0, clk.t1 = m["t0"], m["t1"]
    ms_step, fwd_ms, F_fwd, F_step = m["ms_step"], m["fwd_ms"], m["F_fwd"], m["F_step"]
    value = job_value(F_step, ms_step, world, shard)
    pk = peaks()
    achieved = F_fwd / (fwd_ms * 1e-3) / 1e12

    # ---- end to end: host (pinned) inputs -> device -> path -> host output. Every step
    # copies its Q, K, V in and its O out; the steps are pipelined as a serving loop would
    # run them: two device buffer sets, the copies in on one stream and out on another,
    # so that step i's copies overlap step i-1's compute and each other (PCIe is full
    # duplex). Events order each buffer's reuse. The latency of one step run alone (its
    # copies and compute in sequence on one stream) is reported beside it.
    e2e = None
    if not args.no_e2e:
        stream = path.stream
        qd, kd, vd, O = path.qd, path.kd, path.vd, path.O
        qh, kh, vh = (x.pin_memory() for x in (q, k, v))
        Oh = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
        sets = [(qd, kd, vd, O),
                (torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd),
                 torch.empty_like(O))]
        # one input stream per tensor, so that the three copies can run on separate copy
        # engines at once
        s_ins = [torch.cuda.Stream(dev) for _ in range(3)]
        s_out = torch.cuda.Stream(dev)

        def e2e_steps(n, start_ev=None):
            ev = lambda: torch.cuda.Event()
            in_done = [[ev(), ev(), ev()], [ev(), ev(), ev()]]
            comp_done, out_done = [ev(), ev()], [ev(), ev()]
            if start_ev is not None:
                for s_in in s_ins:
                    s_in.wait_event(start_ev)
            for i in range(n):
                x = i % 2
                qx, kx, vx, ox = sets[x]
                for s_in, dst, src, done in zip(s_ins, (qx, kx, vx), (qh, kh, vh), in_done[x]):
                    with torch.cuda.stream(s_in):
                        if i >= 2:
                            s_in.wait_event(comp_done[x])  # step i-2 has read this set
                        dst.copy_(src, non_blocking=True)
                        done.record(s_in)
                for done in in_done[x]:
                    stream.wait_event(done)
                if i >= 2:
                    stream.wait_event(out_done[x])     # step i-2's output has been read
                path.step(qx, kx, vx, out=ox)
                comp_done[x].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(comp_done[x])
                    Oh.copy_(ox, non_blocking=True)
                    out_done[x].record(s_out)
            stream.wait_event(out_done[(n - 1) % 2])

        e2e_steps(2)
        torch.cuda.synchronize()
        e_s, e_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        e_s.record(stream)
        e2e_steps(args.steps, e_s)
        e_e.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        e2e_ms = max_over_ranks(e_s.elapsed_time(e_e) / args.steps, world)
        # one step at a time: copies in, the path, copy out, all on the launching stream
        n_serial = min(args.steps, 10)
        s_s, s_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        s_s.record(stream)
        for _ in range(n_serial):
            qd.copy_(qh, non_blocking=True)
            kd.copy_(kh, non_blocking=True)
            vd.copy_(vh, non_blocking=True)
            path.step()
            Oh.copy_(O, non_blocking=True)
        s_e.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        serial_ms = max_over_ranks(s_s.elapsed_time(s_e) / n_serial, world)
        e2e = {"value": round(job_value(F_step, e2e_ms, world, shard), 3), "unit": "TFLOP/s",
               "ms_per_step": round(e2e_ms, 4), "pipelined": True, "depth": 2,
               "serial_ms_per_step": round(serial_ms, 4),
               "serial_value": round(job_value(F_step, serial_ms, world, shard), 3),
               "h2d_bytes_per_step": int(3 * q.numel() * 2),
               "d2h_bytes_per_step": int(O.numel() * 2)}

    # head shards: the optional collective, an all-gather of O onto every rank, timed on
    # its own after the steps (the path itself exchanges nothing)
    o_gather = None
    if shard == "heads" and world > 1:
        from piecewise_attention_diffusion_b200.shard import gather_heads
        n_all = w_full.batch * w_full.heads
        full = gather_heads(path.O, n_all, world, rank)
        torch.cuda.synchronize()
        barrier(world)
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(path.stream)
        for _ in range(5):
            full = gather_heads(path.O, n_all, world, rank)
        g1.record(path.stream)
        torch.cuda.synchronize()
        o_gather = {"ms": round(max_over_ranks(g0.elapsed_time(g1) / 5, world), 4),
                    "bytes_per_rank": int(full.numel() * full.element_size()),
                    "in_step": False}

    clk.stop()
    clocks = clk.summary()
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "strong" if shard == "heads" else "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded: Q ~ N(0,1); K, V: " + GENERATOR_TEXT[w.generator] + ")",
        "config": config_of(w_full, world, shard),
        "forward_ms": round(fwd_ms, 4), "forward_tflops": round(achieved, 3),
        "precompute_ms": round(m["pre_ms"], 4), "route_ms": round(m["route_ms"], 4),
        "forward_gflop": round(F_fwd / 1e9, 3),
        "dense_equiv_tflops": round(4.0 * BH * L * L * d / (fwd_ms * 1e-3) / 1e12, 3),
        "roofline": {"kernel": "bsa_forward", "bound": "tensor", "achieved": round(achieved, 3),
                     "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(achieved / pk["bf16_tflops"], 4),
                     "peak_source": f"{pk['source']} bf16_tflops (burst)",
                     "traffic": load_traffic(w),
                     "algorithmic_bytes": forward_bytes(w, w.mode)},
        "clocks": clocks,
        "gpu_launches": launches_per_step(w) * args.steps,
    }
    if e2e:
        line["e2e"] = e2e
    if o_gather:
        line["o_gather"] = o_gather
    del path
    if not args.no_sweep:
        line["sweep"] = run_sweep(args, world, rank, local)
    if rank == 0 and world == 1 and not args.no_cpu:
        k_top = 0 if w.mask else w.top_k()
        cs = oracle_sample(w, k_top, args.cpu_heads, args.seed)
        line["cpu_baseline"] = {"value": round(F_step / cs["seconds_full_est"] / 1e12, 6),
                                "unit": "TFLOP/s", "cores": cs["cores"], "kind": "oracle",
                                "sample": cs["sample"],
                                "seconds_full_est": round(cs["seconds_full_est"], 2)}
    return line


# --------------------------------------------------------------- reference arm
def run_reference(args, w, world, rank):
    """The fp64 oracle, as it stands, on the host cores: each step a bounded sample."""
    k_top = 0 if w.mask else w.top_k()  # a fixed mask has no top-k
    row_lens = None
    if w.mask:
        import oracle as orc
        rp, _ = orc.dense_to_csr(orc.mask_dense(**w.mask))
        row_lens = np.diff(rp).tolist()
    F_step = forward_flops(w, k_top, w.mode, row_lens) \
        + (precompute_flops(w) if needs_precompute(w) else 0.0) \
        + (0.0 if w.mask else route_flops(w))
    for _ in range(args.warmup):
        oracle_sample(w, k_top, 1, args.seed)
    times, info = [], None
    for _ in range(args.steps):
        info = oracle_sample(w, k_top, args.ref_heads, args.seed)
        times.append(info["seconds_full_est"])
    sec = float(np.mean(times))
    value = F_step / sec / 1e12
    cpu = {"value": round(value, 6), "unit": "TFLOP/s", "cores": info["cores"], "kind": "oracle",
           "sample": info["sample"]}
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(sec * 1e3, 2), "higher_is_better": True,
            "scaling": "strong" if args.shard == "heads" else "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (same generator and seed)",
            "config": config_of(w, world, args.shard),
            "cpu_baseline": cpu,
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="video_pisa")
    ap.add_argument("--heads", type=int, default=0,
                    help="override the head count (smaller profiling captures)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads"],
                    help="N > 1: every rank runs the whole workload (replicas, weak scaling) "
                         "or its own range of the heads (strong scaling)")
    ap.add_argument("--cpu-heads", type=int, default=8)
    ap.add_argument("--ref-heads", type=int, default=2)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the per-workload forward numbers reported beside the headline")
    ap.add_argument("--sweep-steps", type=int, default=20)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = synth.workloads()[args.workload]
    if args.heads > 0:
        import dataclasses
        w = dataclasses.replace(w, heads=args.heads)

    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return
        print(json.dumps(run_reference(args, w, world, rank)), flush=True)
        return

    world, rank, local = dist_setup()
    try:
        line = run_ours(args, w, world, rank, local)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()

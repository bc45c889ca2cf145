"""Benchmark of the R-KV decode-time KV compression step on B200.

One step = one rkv_compress_step call over every layer, sequence and KV head
of the workload (plan kernel + fused per-unit kernel), on a cache that is due
for compression.  The default workload is the largest single-GPU one, the
ragged batch (64 sequences x 32 layers x 8 KV heads, budgets 512..2048 + 128,
lambda cycling 0 / 0.1 / 1 over the sequences).  The step compacts the cache
in place, so every warm-up and timed step starts from a pristine copy of the
inputs in HBM: its own replica when the replicas fit in memory, else one
working copy restored (outside the per-step events) before every step.  Every
replica is larger than the 126 MB L2, and a 256 MB buffer is written before
each timed region (and after each restore), so steps start from a cold L2.

Metric: cached tokens compressed per second (sum over compressed units of
their cached length N), and microseconds per step.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl rkv|reference]
                  [--workload NAME] [--redundancy mean|max]

Under torchrun (N > 1) every rank compresses its own batch (weak scaling,
no collective on the data path); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from rkv_synth import WORKLOADS, bf16_bits, make_inputs, pack_ragged  # noqa: E402

METRIC = "cached tokens compressed/sec (all layers×heads); µs per compress step"
UNIT = "tokens/s"
def profile_traffic_path(kernel, workload, variant=""):
    """The committed ncu traffic summary of `kernel` on `workload`; `variant` ("max")
    names a run whose kernel does different work (the step kernel reading r in MAX
    mode instead of computing the MEAN row sums)."""
    tag = f".{variant}" if variant else ""
    return os.path.join(ROOT, "profiles", f"{kernel}.{workload}{tag}.traffic.txt")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="rkv", choices=["rkv", "reference"])
    ap.add_argument("--workload", default="ragged_batch", choices=sorted(WORKLOADS))
    ap.add_argument("--redundancy", default="mean", choices=["mean", "max"])
    ap.add_argument("--e2e-steps", type=int, default=12)
    ap.add_argument("--layers", type=int, default=0,
                    help="run the workload with this many layers instead of its own (a smaller "
                         "case of the same shape, for profiler captures); 0 = the workload's")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the lambda sweep and the single-layer graph-replay figure")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cluster-size", type=int, default=0,
                    help="CTAs per unit: 0 = the library's choice, 1 = one CTA per unit, "
                         "2/4/8/16 = a cluster per unit")
    ap.add_argument("--mode", default="step", choices=["step", "shared", "paged"],
                    help="step: rkv_compress_step (the headline); shared: one kept set per "
                         "(layer, sequence) across the KV heads (rkv_score_shared, all-reduce "
                         "over ranks, rkv_select_compact_shared); paged: rkv_compress_step_paged")
    ap.add_argument("--page-rows", type=int, default=16)
    ap.add_argument("--layout", default="auto", choices=["auto", "uniform", "ragged"],
                    help="cache layout of the step: uniform [batch][Hkv][cap] caches "
                         "(rkv_compress_step) or per-sequence capacities in one pool per layer "
                         "(rkv_compress_step_ragged); auto = ragged when budgets differ")
    ap.add_argument("--loop", action="store_true",
                    help="run the whole decode loop of the workload (append + compress steps)")
    ap.add_argument("--generated", type=int, default=16384,
                    help="tokens generated per sequence in --loop mode")
    return ap.parse_args()


# ----------------------------------------------------------------------------- helpers
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def measured_bf16_tflops():
    """Dense bf16 tensor peak: the measured burst figure (kernels of a few hundred
    microseconds, timed inside short steps), else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured (burst)"
    return 1590.0, "fallback (burst)"


# The sources each timed kernel is compiled from (its file and the headers it includes).
KERNEL_SOURCES = {
    "rkv_unit_kernel": ("rkv_unit.cu", "rkv_block.cuh", "rkv_internal.h", "rkv_post.cuh",
                        "rkv_ptx.cuh"),
    "rkv_step_kernel": ("rkv_step.cu", "rkv_block.cuh", "rkv_internal.h", "rkv_post.cuh",
                        "rkv_ptx.cuh"),
    "rkv_gram_max_kernel": ("rkv_gram.cu", "rkv_block.cuh", "rkv_internal.h", "rkv_ptx.cuh"),
}


def kernel_source_digest(kernel):
    """sha256 (16 hex digits) of the kernel's own sources."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "decode_kv_cache_head_b200", "csrc")
    for name in sorted(KERNEL_SOURCES[kernel]):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel, workload, units_per_launch, variant=""):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    path = profile_traffic_path(kernel, workload, variant)
    if not os.path.exists(path):
        return None
    kv = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
    if kv.get("kernel_source_sha256_16") != kernel_source_digest(kernel):
        return None
    try:
        per_unit = float(kv["dram_bytes_per_unit"])
    except (KeyError, ValueError):
        return None
    return per_unit * units_per_launch


class ClockSampler:
    """nvidia-smi clocks and throttle reasons of this rank's GPU, sampled in the background."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.path = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            gid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            gid = str(device_index)
        self.gid = gid

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="rkv_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gid, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[0]), float(parts[1]), float(parts[2]),
                                 float(parts[3]), parts[4:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        busy = [r for r in rows if r[3] > 0] or rows
        names = ["active", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        reasons = sorted({names[i] for r in busy for i in range(1, 5)
                          if r[4][i].lower() in ("active", "1")})
        return {"sm_mhz": statistics.median(r[0] for r in busy),
                "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows),
                "samples": len(rows), "samples_busy": len([r for r in rows if r[3] > 0]),
                "reasons": reasons}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# ----------------------------------------------------------------------------- reference arm
ORACLE_SAMPLE_UNITS = 64        # units of layer 0 one oracle step computes (all threads)
ORACLE_SAMPLE_UNITS_1T = 8      # the same, single-threaded


def oracle_sample(w, red_mode, max_units):
    """Inputs for the oracle: up to max_units (sequence, KV head) units of layer 0 of
    the workload, taken at an even stride over the batch so that every budget of a
    ragged batch is represented."""
    x = make_inputs(w, layers=[0])
    G = w.n_q_heads // w.n_kv_heads
    qb, kb = bf16_bits(x["Q"]), bf16_bits(x["K"])
    allu = [(b, h) for b in range(w.batch) for h in range(w.n_kv_heads)]
    stride = max(1, -(-len(allu) // max_units))
    units = allu[::stride][:max_units]
    q = np.stack([qb[0, b, h * G:(h + 1) * G] for (b, h) in units])
    k = np.stack([kb[0, b, h] for (b, h) in units])
    N = np.array([int(x["cur_len"][b]) for (b, _) in units], dtype=np.int32)
    bud = np.array([w.budget_of(b) for (b, _) in units], dtype=np.int32)
    lam = np.array([lambda_of(w, b) for (b, _) in units], dtype=np.float64)
    return q, k, N, bud, lam


def time_oracle(w, red_mode, reps, threads, max_units):
    import oracle
    q, k, N, bud, lam = oracle_sample(w, red_mode, max_units)
    oracle.build()
    times = []
    for _ in range(reps):
        t0 = time.perf_counter()
        oracle.units(q, k, N, bud, lam, red_mode=red_mode, n_threads=threads)
        times.append(time.perf_counter() - t0)
    tokens = int(N.sum())
    return tokens, times, len(N)


def oracle_sample_text(w, units, tokens, threads):
    return (f"{units} (sequence, KV head) units of layer 0 of {w.name} at an even stride over "
            f"the batch, {tokens} cached tokens per run; C oracle, fp64, "
            + ("OpenMP over units" if threads > 1 else "one thread"))


def run_reference(args, w, red_mode):
    world, rank, _ = dist_setup(args)
    if rank != 0:
        return
    threads = os.cpu_count() or 1
    if args.warmup:
        time_oracle(w, red_mode, args.warmup, threads, ORACLE_SAMPLE_UNITS)
    tokens, times, units = time_oracle(w, red_mode, args.steps, threads, ORACLE_SAMPLE_UNITS)
    per = sum(times) / len(times)
    value = tokens / per
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, red_mode, args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": oracle_sample_text(w, units, tokens, threads) + " per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def lambda_of(w, b):
    """mix_lambda of sequence b: the ragged batch cycles 0 / 0.1 / 1 over its sequences
    (the two ablation extremes and the pages' value); other workloads use w.mix_lambda."""
    if w.name == "ragged_batch":
        return RAGGED_LAMBDAS[b % 3]
    return w.mix_lambda


RAGGED_LAMBDAS = (0.0, 0.1, 1.0)


def workload_config(w, red_mode, args):
    lam = (f"per sequence, cycling {list(RAGGED_LAMBDAS)}" if w.name == "ragged_batch"
           else w.mix_lambda)
    return {"workload": w.name, "n_layers": w.n_layers, "batch": w.batch,
            "n_kv_heads": w.n_kv_heads, "n_q_heads": w.n_q_heads, "head_dim": w.head_dim,
            "budget": list(w.budgets) if len(w.budgets) > 1 else w.budgets[0],
            "buffer": w.buffer, "window": w.window, "mix_lambda": lam,
            "redundancy": "max" if red_mode else "mean", "gqa_pool": "max",
            "cached_len": w.n_tokens()[0] if len(set(w.n_tokens())) == 1 else "ragged",
            "near_duplicate_frac": list(w.dup_frac) if len(w.dup_frac) > 1 else w.dup_frac[0],
            "l2": "pristine in-HBM caches every step (a fresh replica, or the working copy "
                  "restored outside the per-step events when replicas do not fit; K+V larger "
                  "than L2) and a 256 MB L2 flush before the timed region and after every restore",
            "layout": ("per-sequence capacities: one pool per layer, each sequence's block "
                       "budget + buffer rows per KV head (rkv_compress_step_ragged)"
                       if use_ragged_layout(args, w) else
                       "uniform [batch][Hkv][cap] caches (rkv_compress_step)"),
            "parallelism": f"dp{args.gpus} (independent sequences per rank)"}


def algorithmic_bytes(n_tok, budgets, n_layers, n_kv, G, window, moved):
    """HBM bytes the step must move, per the step's byte count: per unit the scoring
    reads K once (N rows of 256 B) and the G * w query rows, the select reads two
    fp32 scores per candidate and writes one int32 per kept row, and every kept row
    whose destination differs from its source is read and written once for each of
    K and V (4 x 256 B).  `moved` counts those rows exactly over the whole launch."""
    per_seq = [256 * (n + G * window) + 8 * (n - window) + 4 * bud
               for n, bud in zip(n_tok, budgets)]
    return n_layers * n_kv * sum(per_seq) + 1024 * moved


ALG_BYTES_DEFINITION = ("per unit 256*(N + G*w) (K read once, window queries) + 8*(N - w) + "
                        "4*budget (select) + 1024 per kept row that moves (K and V read and "
                        "written), moved rows counted exactly")


# ----------------------------------------------------------------------------- rkv arm
def graph_replay_single_layer(rkv, dev, stream, reps=50):
    """The single-layer step (8 units, N = 1152) as a captured CUDA graph of
    (reset cur_len, rkv_compress_step), replayed `reps` times with events around each
    replay; the same two calls issued eagerly for comparison.  Every replay compresses
    the cache again from N = 1152 rows, so each does the full step's work."""
    w1 = WORKLOADS["single_layer"]
    x = make_inputs(w1, device=str(dev))
    K, V, Q, cur0 = x["K"], x["V"], x["Q"], x["cur_len"].to(dev)
    cur = cur0.clone()
    L, B, H, cap, _ = K.shape
    cfg = rkv.make_config(w1.budget_of(0), w1.buffer, w1.window, 128, w1.n_kv_heads,
                          w1.n_q_heads, w1.mix_lambda)
    ws = torch.zeros(rkv.rkv_workspace_size(cfg, L, B, cap), dtype=torch.uint8, device=dev)

    def body(s):
        cur.copy_(cur0)
        rkv.rkv_compress_step(cfg, K, V, Q, cur, ws, stream=s)

    for _ in range(3):
        body(stream)
    torch.cuda.synchronize()
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(stream)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            body(side)
    stream.wait_stream(side)
    torch.cuda.synchronize()

    def timed(fn):
        out = []
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            out.append(a.elapsed_time(b) * 1e3)
        return statistics.median(out)

    g_us = timed(graph.replay)
    e_us = timed(lambda: body(stream))
    assert rkv.rkv_workspace_status(ws) == 0
    del graph
    return {"workload": "single_layer", "graph_replay_us_median": g_us,
            "eager_us_median": e_us, "replays": reps,
            "what": "CUDA graph of (cur_len reset, rkv_compress_step) on 1 layer x 8 KV heads, "
                    "N = 1152; events around each replay"}


def use_ragged_layout(args, w):
    if args.layout == "auto":
        return len(set(w.budget_of(b) for b in range(w.batch))) > 1
    return args.layout == "ragged"


def run_rkv(args, w, red_mode):
    world, rank, local = dist_setup(args)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=dev)
    from decode_kv_cache_head_b200 import build
    build.build()
    import decode_kv_cache_head_b200 as rkv
    from decode_kv_cache_head_b200 import dist as rdist

    seed = rdist.rank_seed(w.seed, rank)
    x = make_inputs(w, device=str(dev), seed=seed)
    L, B, H, cap, D = x["K"].shape
    Q, cur0 = x["Q"], x["cur_len"].to(dev)
    G = w.n_q_heads // w.n_kv_heads
    ragged = use_ragged_layout(args, w)
    caps = [w.budget_of(b) + w.buffer for b in range(B)]
    if ragged:
        # one pool per layer, every sequence's block exactly budget + buffer rows per head
        K0, V0 = pack_ragged(x["K"], caps), pack_ragged(x["V"], caps)
        rows, pool_rows = rkv.ragged_rows(caps, H)
        seq_row = torch.tensor(rows, dtype=torch.int64, device=dev)
        seq_cap = torch.tensor(caps, dtype=torch.int32, device=dev)
        cap = max(caps)
    else:
        K0, V0 = x["K"], x["V"]
    del x
    cfg = rkv.make_config(w.budget_of(0), w.buffer, w.window, 128, w.n_kv_heads, w.n_q_heads,
                          w.mix_lambda, redundancy_mode=red_mode)
    budgets = None
    if len(w.budgets) > 1:
        budgets = torch.tensor([w.budget_of(b) for b in range(B)], dtype=torch.int32, device=dev)
    lambdas = None
    if w.name == "ragged_batch":
        lambdas = torch.tensor([lambda_of(w, b) for b in range(B)], dtype=torch.float32,
                               device=dev)
    ws = torch.zeros(rkv.rkv_workspace_size(cfg, L, B, cap), dtype=torch.uint8, device=dev)
    shape = rkv.rkv_query_step_shape(cfg, L * B * H, cap)
    if args.cluster_size or ragged:
        cs = args.cluster_size or 1
        shape = (cs, cap if cs == 1 else shape[1], shape[2])
    kernel_name = "rkv_unit_kernel" if shape[0] == 1 else "rkv_step_kernel"
    stream = torch.cuda.current_stream()

    def call(cfg_, Kr, Vr, Qr, cr, lambdas_, events=None, kept=None, sim_events=None, strm=None):
        if ragged:
            rkv.rkv_compress_step_ragged(cfg_, Kr, Vr, Qr, cr, ws, seq_row, seq_cap, cap,
                                         budgets=budgets, lambdas=lambdas_, kept_out=kept,
                                         events=events, sim_events=sim_events,
                                         cluster_size=args.cluster_size, stream=strm or stream)
        else:
            rkv.rkv_compress_step(cfg_, Kr, Vr, Qr, cr, ws, budgets=budgets, lambdas=lambdas_,
                                  kept_out=kept, cluster_size=args.cluster_size,
                                  events=events, stream=strm or stream, sim_events=sim_events)

    def step(Kr, Vr, cr, events=None, kept=None, sim_events=None, cfg_=None, lambdas_=lambdas):
        call(cfg_ or cfg, Kr, Vr, Q, cr, lambdas_, events=events, kept=kept,
             sim_events=sim_events)

    # exact moved-row count (rows whose destination differs from their source)
    kept = torch.full((L, B, H, cap), -1, dtype=torch.int32, device=dev)
    Kt, Vt, ct = K0.clone(), V0.clone(), cur0.clone()
    step(Kt, Vt, ct, kept=kept)
    torch.cuda.synchronize()
    assert rkv.rkv_workspace_status(ws) == 0
    moved = 0
    for b in range(B):
        bud = w.budget_of(b)
        kb = kept[:, b, :, :bud]
        moved += int((kb != torch.arange(bud, device=dev, dtype=torch.int32)).sum().item())
    del Kt, Vt, ct, kept
    units = L * B * H
    n_tok = [w.budget_of(b) + w.buffer for b in range(B)]
    token_heads = int(L * H * sum(n_tok))
    alg_bytes = algorithmic_bytes(n_tok, [w.budget_of(b) for b in range(B)], L, H, G, w.window,
                                  moved)

    # replicas: one pristine copy per warm-up and timed step when they fit in memory
    # (restored between the two timed passes); otherwise one working copy restored
    # from the pristine one before every step, with the restore outside per-step events
    n_rep = args.warmup + args.steps
    rep_bytes = 2 * K0.numel() * K0.element_size()
    fits = n_rep * rep_bytes < 0.7 * torch.cuda.mem_get_info(dev)[0]
    reps = [(K0.clone(), V0.clone(), cur0.clone()) for _ in range(n_rep if fits else 1)]
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    # MAX redundancy: the similarity kernel is timed too (it is the longer kernel there)
    ev_sim = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)] if red_mode == 1 else None
    st = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    for a, b in ev + (ev_sim or []):   # materialise the events before handing them to the library
        a.record(stream); b.record(stream)

    def restore(r):
        r[0].copy_(K0); r[1].copy_(V0); r[2].copy_(cur0)
        flush.fill_(1.0)

    t_start, t_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed_pass(kernel_events, n_steps=None, **kw):
        """n_steps over pristine caches after an L2 flush; returns the elapsed ms.
        kernel_events: the library records ev[i] around the main kernel of step i."""
        n_steps = n_steps or args.steps
        flush.fill_(1.0)
        torch.cuda.synchronize()
        rdist.barrier(dev)
        torch.cuda.synchronize()
        t_start.record(stream)
        # an NVTX range around the timed steps (profilers can restrict a capture to it)
        torch.cuda.nvtx.range_push("timed_steps")
        for i in range(n_steps):
            if not fits:
                restore(reps[0])
                st[i][0].record(stream)
            step(*reps[args.warmup + i if fits else 0], events=ev[i] if kernel_events else None,
                 sim_events=ev_sim[i] if (kernel_events and ev_sim) else None, **kw)
            if not fits:
                st[i][1].record(stream)
        torch.cuda.nvtx.range_pop()
        t_stop.record(stream)
        torch.cuda.synchronize()
        rdist.barrier(dev)
        assert rkv.rkv_workspace_status(ws) == 0
        if fits:
            return t_start.elapsed_time(t_stop)
        return sum(a.elapsed_time(b) for a, b in st[:n_steps])

    def restore_all():
        if fits:
            for r in reps[args.warmup:]:
                restore(r)

    sampler = ClockSampler(local)
    sampler.start()
    for i in range(args.warmup):
        if not fits:
            restore(reps[0])
        step(*reps[i if fits else 0])
    # throughput: the steps back to back, nothing recorded between their kernels
    elapsed_ms = timed_pass(False)
    # the main kernel's duration: the same steps again on restored caches, with
    # events around the kernel (they cost the step a few microseconds)
    restore_all()
    timed_pass(True)
    clocks = sampler.stop()
    kern_ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps
    elapsed_ms, kern_ms = rdist.max_over_ranks([elapsed_ms, kern_ms], dev)
    ms_per_step = elapsed_ms / args.steps
    value = world * token_heads / (ms_per_step / 1e3)

    # the ragged batch is also timed with one scalar lambda per call: the two ablation
    # extremes and the pages' value
    lambda_sweep = None
    if w.name == "ragged_batch" and not args.no_extras:
        lambda_sweep = {}
        n_sw = min(args.steps, 10)
        for lam in RAGGED_LAMBDAS:
            c_l = rkv.make_config(w.budget_of(0), w.buffer, w.window, 128, w.n_kv_heads,
                                  w.n_q_heads, lam, redundancy_mode=red_mode)
            restore_all()
            ms = timed_pass(False, n_steps=n_sw, cfg_=c_l, lambdas_=None)
            lambda_sweep[str(lam)] = rdist.max_over_ranks([ms], dev)[0] / n_sw * 1e3
        lambda_sweep = {"us_per_step": lambda_sweep, "steps": n_sw}
    del reps

    graph1 = None
    if rank == 0 and world == 1 and not args.no_extras:
        graph1 = graph_replay_single_layer(rkv, dev, stream)

    # end to end through host buffers: every step copies its inputs host -> device, runs
    # the step and copies its result device -> host.  Consecutive steps overlap: two
    # device buffer sets, the copies in on one stream and out on another, so the H2D of
    # step i + 1 and the D2H of step i - 1 run while step i computes (the two copy
    # directions use the link at the same time).
    e2e = None
    # pinned inputs + pinned outputs, with headroom, for every rank on this host
    local_ranks = int(os.environ.get("LOCAL_WORLD_SIZE", "1"))
    host_need = 2.5 * rep_bytes * local_ranks
    try:
        import psutil
        host_free = psutil.virtual_memory().available
    except Exception:
        host_free = float("inf")
    # every rank takes the same branch (the timed e2e steps hold collectives)
    fits = rdist.max_over_ranks([0.0 if host_need <= host_free else 1.0], dev)[0] == 0.0
    if args.e2e_steps > 0 and not fits:
        e2e = {"skipped": f"host RAM: {host_need / 1e9:.1f} GB of pinned buffers needed on this "
                          f"host, {host_free / 1e9:.1f} GB available"}
    elif args.e2e_steps > 0:
        def pinned_copy(t):
            h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
            h.copy_(t)
            return h
        hK, hV, hQ, hc = pinned_copy(K0), pinned_copy(V0), pinned_copy(Q), pinned_copy(cur0)
        oK = torch.empty(K0.shape, dtype=K0.dtype, pin_memory=True)
        oV = torch.empty(V0.shape, dtype=V0.dtype, pin_memory=True)
        oc = torch.empty(cur0.shape, dtype=cur0.dtype, pin_memory=True)
        sets = [(torch.empty_like(K0), torch.empty_like(V0), torch.empty_like(Q),
                 torch.empty_like(cur0)) for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_step = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        used = [False, False]

        def e2e_step(i):
            k = i % 2
            dK, dV, dQ, dc = sets[k]
            with torch.cuda.stream(s_in):
                if used[k]:
                    s_in.wait_event(ev_out[k])      # this set's previous result is out
                dK.copy_(hK, non_blocking=True); dV.copy_(hV, non_blocking=True)
                dQ.copy_(hQ, non_blocking=True); dc.copy_(hc, non_blocking=True)
                ev_in[k].record(s_in)
            stream.wait_event(ev_in[k])
            call(cfg, dK, dV, dQ, dc, lambdas)
            ev_step[k].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_step[k])
                oK.copy_(dK, non_blocking=True); oV.copy_(dV, non_blocking=True)
                oc.copy_(dc, non_blocking=True)
                ev_out[k].record(s_out)
            used[k] = True

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        rdist.barrier(dev)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        s_in.wait_event(a)
        for i in range(args.e2e_steps):
            e2e_step(i)
        for k in range(2):
            stream.wait_event(ev_out[k])
        b.record(stream)
        torch.cuda.synchronize()
        assert rkv.rkv_workspace_status(ws) == 0
        e_ms = rdist.max_over_ranks([a.elapsed_time(b) / args.e2e_steps], dev)[0]
        h2d = sum(t.numel() * t.element_size() for t in (hK, hV, hQ, hc))
        d2h = sum(t.numel() * t.element_size() for t in (oK, oV, oc))
        e2e = {"value": world * token_heads / (e_ms / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms,
               "steps": args.e2e_steps,
               "overlap": "copies of consecutive steps overlap (two buffer sets, copy streams)"}
        del sets, hK, hV, oK, oV

    peak, peak_kind = measured_peaks()
    achieved = alg_bytes / (kern_ms / 1e3) / 1e9
    # a step launches the main kernel once per 32-layer chunk: the per-launch figures
    # are the step's totals over its launches (their ratio, `achieved`, is the same)
    n_chunks = (L + 31) // 32
    traffic = profiled_traffic(kernel_name, w.name, units, "max" if red_mode else "")
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak,
                "traffic": traffic / n_chunks if traffic is not None else None,
                "kernel": kernel_name, "launches_per_step": n_chunks,
                "kernel_us_per_launch": kern_ms * 1e3 / n_chunks,
                "algorithmic_bytes_per_launch": alg_bytes / n_chunks,
                "algorithmic_bytes_definition": ALG_BYTES_DEFINITION,
                "moved_rows": moved, "kept_rows": L * H * sum(w.budget_of(b) for b in range(B)),
                "peak_source": peak_kind,
                "kernel_source_sha256_16": kernel_source_digest(kernel_name),
                "cluster_size": shape[0], "rows_per_cta": shape[1], "smem_per_cta": shape[2]}
    roofline_unit = None
    if ev_sim:
        # MAX redundancy: the similarity kernel is the dominant one.  Algorithmic flops are
        # the symmetric Gram N (N - 1) D per unit.
        sim_ms = sum(a.elapsed_time(b) for a, b in ev_sim) / args.steps
        sim_ms = rdist.max_over_ranks([sim_ms], dev)[0]
        alg_flops = L * H * sum(n * (n - 1) * D for n in n_tok)
        exe_flops = L * H * sum(gram_executed_flops(n, w.window) for n in n_tok)
        tpeak, tkind = measured_bf16_tflops()
        t_ach = alg_flops / (sim_ms / 1e3) / 1e12
        roofline_unit = roofline
        n_sim = n_chunks * gram_launches_per_chunk()
        sim_traffic = profiled_traffic("rkv_gram_max_kernel", w.name, units)
        roofline = {"bound": "tensor", "achieved": t_ach, "peak": tpeak, "unit": "TFLOP/s",
                    "frac": t_ach / tpeak,
                    "traffic": sim_traffic / n_sim if sim_traffic is not None else None,
                    "kernel": "rkv_gram_max_kernel",
                    "kernel_source_sha256_16": kernel_source_digest("rkv_gram_max_kernel"),
                    "launches_per_step": n_sim, "kernel_us_per_launch": sim_ms * 1e3 / n_sim,
                    "algorithmic_flops_per_launch": alg_flops / n_sim,
                    "executed_flops_per_launch": exe_flops / n_sim,
                    "executed_tflops": exe_flops / (sim_ms / 1e3) / 1e12, "peak_source": tkind}

    cpu = cpu1 = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = os.cpu_count() or 1
        tokens, times, nu = time_oracle(w, red_mode, 3, threads, ORACLE_SAMPLE_UNITS)
        per = sorted(times)[1]
        cpu = {"value": tokens / per, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": oracle_sample_text(w, nu, tokens, threads) + ", median of 3 runs"}
        tokens, times, nu = time_oracle(w, red_mode, 1, 1, ORACLE_SAMPLE_UNITS_1T)
        cpu1 = {"value": tokens / times[0], "unit": UNIT, "cores": 1, "kind": "oracle",
                "sample": oracle_sample_text(w, nu, tokens, 1) + ", one run"}

    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return
    # per 32-layer chunk: the step kernel, plus the similarity kernel(s) in MAX mode
    n_main_launches = ((L + 31) // 32) * (1 + gram_launches_per_chunk() if red_mode else 1)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "us_per_step": ms_per_step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": workload_config(w, red_mode, args),
        "e2e": e2e, "gpu_launches": args.steps * (1 + n_main_launches),
        "roofline": roofline, "cpu_baseline": cpu, "cpu_baseline_single_thread": cpu1,
        "clocks": clocks,
        **({"roofline_unit_kernel": roofline_unit} if roofline_unit else {}),
        **({"lambda_sweep": lambda_sweep} if lambda_sweep else {}),
        **({"single_layer_graph": graph1} if graph1 else {}),
        "token_heads_per_step_per_gpu": token_heads,
    }
    print(json.dumps(line), flush=True)


def gram_launches_per_chunk():
    """Kernels the MAX-mode redundancy launches per 32-layer chunk (the similarity
    kernel computes the inverse norms itself)."""
    return 1


def gram_executed_flops(n, window):
    """Flops the similarity kernel executes for one unit of n cached rows: the tile
    pairs (I, J >= I) of 128 x 128 x 128 (the symmetric half, diagonal tiles whole)."""
    t = -(-n // 128)
    return t * (t + 1) // 2 * 2 * 128 ** 3


# ----------------------------------------------------------------------------- decode loop
def run_loop(args, w, red_mode):
    """Steady-state decode loop: fill the cache to budget + buffer, compress, then
    append `buffer` tokens and compress again until `--generated` tokens.  Only the
    compression steps are timed (CUDA events around each call); the same cycle is
    also replayed as a captured CUDA graph of (append + compress)."""
    from decode_kv_cache_head_b200 import build
    build.build()
    import decode_kv_cache_head_b200 as rkv
    from rkv_synth import DecodeTrace

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    L, B, H, D = w.n_layers, w.batch, w.n_kv_heads, w.head_dim
    bud, buf, cap = w.budget_of(0), w.buffer, w.cap
    cfg = rkv.make_config(bud, buf, w.window, D, H, w.n_q_heads, w.mix_lambda,
                          redundancy_mode=red_mode)
    K = torch.zeros((L, B, H, cap, D), dtype=torch.bfloat16, device=dev)
    V = torch.zeros_like(K)
    cur = torch.zeros(B, dtype=torch.int32, device=dev)
    ws = torch.zeros(rkv.rkv_workspace_size(cfg, L, B, cap), dtype=torch.uint8, device=dev)
    trace = DecodeTrace(w, device=str(dev))
    stream = torch.cuda.current_stream()
    evs = []

    def compress(Q):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        rkv.rkv_compress_step(cfg, K, V, Q, cur, ws, cluster_size=args.cluster_size, stream=stream)
        b.record(stream)
        evs.append((a, b))

    k_new, v_new = trace.chunk(cap, K, V, [0] * B)
    rkv.rkv_append_kv(cfg, K, V, k_new, v_new, cur, ws, stream=stream)
    del k_new, v_new
    compress(trace.queries())
    t = cap
    while t + buf <= args.generated:
        k_new, v_new = trace.chunk(buf, K, V, [bud] * B)
        rkv.rkv_append_kv(cfg, K, V, k_new, v_new, cur, ws, stream=stream)
        t += buf
        compress(trace.queries())
    torch.cuda.synchronize()
    assert rkv.rkv_workspace_status(ws) == 0
    assert cur.tolist() == [bud] * B
    step_ms = [a.elapsed_time(b) for a, b in evs]
    total_ms = sum(step_ms)

    # the same cycle as a CUDA graph (append + compress), replayed on fixed buffers
    kb = torch.empty((L, B, H, buf, D), dtype=torch.bfloat16, device=dev)
    vb = torch.empty_like(kb)
    Qb = torch.empty((L, B, w.n_q_heads, w.window, D), dtype=torch.bfloat16, device=dev)
    kb.copy_(k_new); vb.copy_(v_new); Qb.copy_(trace.queries())
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            rkv.rkv_append_kv(cfg, K, V, kb, vb, cur, ws, stream=side)
            rkv.rkv_compress_step(cfg, K, V, Qb, cur, ws, cluster_size=args.cluster_size,
                                  stream=side)
    stream.wait_stream(side)
    reps = 20
    g_ms = []
    for _ in range(reps):
        k_new, v_new = trace.chunk(buf, K, V, [bud] * B)
        kb.copy_(k_new); vb.copy_(v_new); Qb.copy_(trace.queries())
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        graph.replay()
        b.record(stream)
        torch.cuda.synchronize()
        g_ms.append(a.elapsed_time(b))
    assert rkv.rkv_workspace_status(ws) == 0
    del graph

    token_heads = L * B * H * cap
    full = L * B * H * args.generated * D * 2 * 2
    line = {
        "metric": METRIC, "value": len(step_ms) * token_heads / (total_ms / 1e3), "unit": UNIT,
        "n_gpus": 1, "steps": len(step_ms), "warmup": 0, "ms_per_step": total_ms / len(step_ms),
        "us_per_step": 1e3 * total_ms / len(step_ms), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_config(w, red_mode, args), mode="decode_loop",
                       layout="uniform [batch][Hkv][cap] caches",
                       generated_tokens=args.generated),
        "loop": {"compress_steps": len(step_ms), "total_compress_ms": total_ms,
                 "step_us_median": 1e3 * statistics.median(step_ms),
                 "graph_append_plus_compress_us_median": 1e3 * statistics.median(g_ms),
                 "full_cache_bytes": full,
                 "capacity_cache_bytes": L * B * H * cap * D * 2 * 2,
                 "compacted_cache_bytes": L * B * H * bud * D * 2 * 2,
                 "capacity_fraction": cap / args.generated,
                 "compacted_fraction": bud / args.generated},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- other modes
def run_mode(args, w, red_mode):
    """The shared-selection or paged-cache variant of the step on the same workload:
    device-timed with CUDA events over the whole call sequence, a fresh replica per step."""
    world, rank, local = dist_setup(args)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=dev)
    from decode_kv_cache_head_b200 import build
    build.build()
    import decode_kv_cache_head_b200 as rkv
    from decode_kv_cache_head_b200 import dist as rdist

    tp = args.mode == "shared" and world > 1
    # shared selection across ranks is tensor parallelism: every rank holds the same
    # sequences and its own share of the KV heads; the other modes shard sequences
    x = make_inputs(w, device=str(dev), seed=w.seed if tp else rdist.rank_seed(w.seed, rank))
    K0, V0, Q, cur0 = x["K"], x["V"], x["Q"], x["cur_len"].to(dev)
    G = w.n_q_heads // w.n_kv_heads
    if tp:
        h0, h1 = rdist.head_range(w.n_kv_heads, world, rank)
        K0, V0 = K0[:, :, h0:h1].contiguous(), V0[:, :, h0:h1].contiguous()
        Q = Q[:, :, h0 * G:h1 * G].contiguous()
    L, B, H, cap, D = K0.shape
    cfg = rkv.make_config(w.budget_of(0), w.buffer, w.window, 128, H, H * G,
                          w.mix_lambda, redundancy_mode=red_mode)
    budgets = None
    if len(w.budgets) > 1:
        budgets = torch.tensor([w.budget_of(b) for b in range(B)], dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()
    n_rep = args.warmup + args.steps
    extra = {}
    if args.mode == "shared":
        ws = torch.zeros(rkv.rkv_workspace_size_shared(cfg, L, B, cap), dtype=torch.uint8,
                         device=dev)
        z = torch.empty((L, B, cap), dtype=torch.float32, device=dev)
        reps = [(K0.clone(), V0.clone(), cur0.clone()) for _ in range(n_rep)]

        def call(r):
            rdist.compress_step_shared(rkv, cfg, r[0], r[1], Q, r[2], z, ws, budgets=budgets,
                                       stream=stream)
        extra["all_reduce_bytes_per_step"] = z.numel() * 4 if world > 1 else 0
    else:
        P = args.page_rows
        assert cap % P == 0, "cache length must be a multiple of the page size"
        mb = cap // P
        pages = B * mb
        perm = torch.randperm(pages, generator=torch.Generator().manual_seed(7)).to(torch.int32)
        bt = perm.view(B, mb).to(dev)
        pk = torch.empty((L, pages, H, P, D), dtype=torch.bfloat16, device=dev)
        pv = torch.empty_like(pk)
        idx = bt.view(-1).long()
        pk[:, idx] = K0.view(L, B, H, mb, P, D).permute(0, 1, 3, 2, 4, 5).reshape(L, pages, H, P, D)
        pv[:, idx] = V0.view(L, B, H, mb, P, D).permute(0, 1, 3, 2, 4, 5).reshape(L, pages, H, P, D)
        ws = torch.zeros(rkv.rkv_workspace_size(cfg, L, B, cap), dtype=torch.uint8, device=dev)
        freed = torch.empty((B, mb), dtype=torch.int32, device=dev)
        n_freed = torch.empty((B,), dtype=torch.int32, device=dev)
        reps = [(pk.clone(), pv.clone(), cur0.clone()) for _ in range(n_rep)]
        del pk, pv

        def call(r):
            rkv.rkv_compress_step_paged(cfg, r[0], r[1], Q, r[2], ws, bt, P, freed, n_freed,
                                        budgets=budgets, stream=stream)
        extra["page_rows"] = P
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    sampler = ClockSampler(local)
    sampler.start()
    for i in range(args.warmup):
        call(reps[i])
    flush.fill_(1.0)
    torch.cuda.synchronize()
    rdist.barrier(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    torch.cuda.nvtx.range_push("timed_steps")
    for i in range(args.steps):
        call(reps[args.warmup + i])
    torch.cuda.nvtx.range_pop()
    b.record(stream)
    torch.cuda.synchronize()
    rdist.barrier(dev)
    clocks = sampler.stop()
    assert rkv.rkv_workspace_status(ws) == 0
    ms = rdist.max_over_ranks([a.elapsed_time(b) / args.steps], dev)[0]
    token_heads = w.token_heads() * (1 if tp else world)   # whole job
    if rank == 0:
        line = {
            "metric": METRIC, "value": token_heads / (ms / 1e3), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "us_per_step": ms * 1e3, "higher_is_better": True,
            "scaling": "strong" if tp else "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(workload_config(w, red_mode, args), mode=args.mode, **extra,
                           layout=("paged pools" if args.mode == "paged"
                                   else "uniform [batch][Hkv][cap] caches"),
                           **({"parallelism": f"tp{world} (KV heads split over ranks)"}
                              if tp else {})),
            # shared: plan, scoring kernels, head sum, plan, select+compact per 32-layer chunk;
            # paged: plan, freed pages, step kernel per chunk (+ the similarity kernel in MAX)
            "gpu_launches": args.steps * (
                3 + ((L + 31) // 32) * (2 + (1 if red_mode else 0)) if args.mode == "shared"
                else 2 + ((L + 31) // 32) * (2 if red_mode else 1)),
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    args = parse_args()
    w = WORKLOADS[args.workload]
    if args.layers:
        w = dataclasses.replace(w, n_layers=args.layers)
    red_mode = 1 if args.redundancy == "max" else 0
    if args.impl == "reference":
        run_reference(args, w, red_mode)
    elif args.loop:
        run_loop(args, w, red_mode)
    elif args.mode != "step":
        run_mode(args, w, red_mode)
    else:
        run_rkv(args, w, red_mode)


if __name__ == "__main__":
    main()

"""Benchmark of the SAGA + Atop-N decode attention step on B200.

One step = one decode token through the workload's attention stack: for every
layer, either a plain Atop-N step (saga_decode_step) or, when t mod R == 0, a
refresh (saga_refresh_threshold with V and out, which also runs that step).
The default workload is the Llama-3.2-1B-shaped 16-layer stack at batch 8 and
128K context (h_q=32, h_k=2, h_v=8, d=64, bf16 caches, N=2048, R=32).

Prints one JSON line (rank 0):
  value      the R-cycle average of the whole job in steps/s:
             R / (t_refresh + (R - 1) t_plain), t_plain and t_refresh the
             medians over at least ten replays of CUDA graphs of consecutive
             plain and consecutive refresh steps (CUDA events on the launching
             stream, max over ranks), inputs resident in HBM; both parts are
             in step_times. timed_steps: exactly --steps steps of the real
             schedule (refresh at t mod R == 0, t from 0) in one graph.
  e2e        the same metric with each step's queries copied in from pinned
             host memory and its outputs read back;
  roofline   the plain-step call (the dominant one): algorithmic bytes per
             call / its median duration, against the measured HBM copy peak;
  dense_gqa  the library's dense GQA stack at the same shape, same metric;
  saga_full  full attention over the same SAGA-headed caches (the ablation arm
             between dense GQA and SAGA + Atop-N);
  cpu_baseline  the float64 oracle on the host cores, on a bounded sample;
  workloads  the same figures for the other workloads (the Qwen2.5-1.5B- and
             Llama-3.2-1B-shaped single layers, the ragged refresh-every-step
             batch at each N, the tiny fp32 case), unless --primary-only.

With --impl reference the oracle alone is timed (the reference arm).
--gpus N starts N ranks (torch.distributed.run) unless already launched by
it; every rank runs its own batch of the same workload (weak scaling), with
no collective on the data path.
"""
import argparse
import hashlib
import json
import math
import os
import re
import socket
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

DEFAULT_WORKLOAD = "llama1b_stack16_b8_128k"
EXTRA_WORKLOADS = ("qwen1p5b_128k", "llama1b_32k", "ragged_refresh_b16", "tiny_f32")
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
MIN_REPLAYS = 10
METRIC = "SAGA+Atop-N decode-attn steps/s at 128K ctx; HBM GB/s vs peak"
PAGES_CONTEXT = ("the SAGA paper reports an end-to-end decode speedup above 2x over "
                 "full-attention GQA at 128K context on Llama 3.2-1B and Qwen2.5-1.5B "
                 "(model level, hardware not tied to the figure); its key-head merge "
                 "alone gives up to 1.47x at batch 16 and 128K")


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--primary-only", action="store_true",
                    help="measure the --workload alone, without the other workloads")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=None,
                    help="override the stack depth (same per-layer launch, smaller footprint)")
    ap.add_argument("--merge", default=None,
                    help="time the closed-form GQA-to-SAGA key merge on this calibration "
                         "workload instead (synth.merge_workload.MERGE_WORKLOADS)")
    return ap.parse_args(argv)


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def spawn_ranks(args, argv):
    """--gpus N > 1 outside torch.distributed.run: start N ranks through it
    (one process per GPU, rendezvous on 127.0.0.1) and return their exit
    status; None when this process is a rank already or N == 1."""
    if args.gpus <= 1 or "WORLD_SIZE" in os.environ:
        return None
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={args.gpus}", "--master-addr=127.0.0.1",
           f"--master-port={free_port()}", os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def dist_init(backend=None):
    """One process per GPU: NCCL over the node's GPUs (gloo for CPU-only
    checks). Returns (world, rank, local_rank)."""
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if backend is None:
        backend = "nccl" if torch.cuda.is_available() else "gloo"
    if world > 1 and not dist.is_initialized():
        import datetime
        kw = {"device_id": torch.device("cuda", local)} if backend == "nccl" else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    if backend == "nccl":
        torch.cuda.set_device(local)
    return world, rank, local


def _reduce(x, world, op):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=op)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    import torch.distributed as dist
    return _reduce(x, world, dist.ReduceOp.MAX if world > 1 else None)


def sum_over_ranks(x, world):
    import torch.distributed as dist
    return _reduce(x, world, dist.ReduceOp.SUM if world > 1 else None)


def finish_dist(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def rank_workload(w, rank):
    """Each rank decodes its own batch of the same workload (weak scaling):
    rank 0 keeps the canonical seed, rank r > 0 draws independent inputs."""
    return w if rank == 0 else w.with_(seed=w.seed + 7919 * rank)


def aggregate_value(steps, max_ms, world):
    """Whole-job steps/s: every rank ran `steps` steps of its own batch; the
    job takes as long as the slowest rank."""
    return world * steps / (max_ms / 1e3)


def r_cycle(t_plain_ms, t_refresh_ms, R):
    """Steps/s of one rank averaged over a refresh cycle of R steps: one
    refresh step and R - 1 plain steps."""
    return R / ((t_refresh_ms + (R - 1) * t_plain_ms) / 1e3)


def step_schedule(n, R):
    """Refresh flags of steps 0 .. n-1 (t mod R == 0)."""
    return [t % R == 0 for t in range(n)]


# ---------------------------------------------------------------------------
# measurement helpers
# ---------------------------------------------------------------------------
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        # raw samples; the JSON line carries their summary
        self.path = os.environ.get("SAGA_CLOCK_LOG") or os.path.join(
            tempfile.gettempdir(), f"saga_clocks_gpu{index}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(smax)),
                "samples": len(sm), "reasons": sorted(reasons)}


def source_hash(paths):
    """Hash of the kernel sources with comments and blank lines removed, so a
    change of wording alone does not void counters taken on the same code."""
    h = hashlib.sha256()
    for p in paths:
        text = open(p, encoding="utf-8").read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        lines = [ln.rstrip() for ln in text.splitlines() if ln.strip()]
        h.update("\n".join(lines).encode())
    return h.hexdigest()[:16]


def step_kernel_sources():
    """The sources the decode step's kernels and plan are built from."""
    here = os.path.join(ROOT, "sparse_decode_attention_step_b200", "csrc")
    return [os.path.join(here, f) for f in ("common.cuh", "sm100.cuh", "kernels.h",
                                            "saga_api.cu", "saga_tc.cu", "gather.cu", "combine.cu")]


def ncu_traffic(kernel_sources):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("source_hash") != source_hash(kernel_sources):
        return None
    return d.get("dram_bytes_per_call")


# ---------------------------------------------------------------------------
# the oracle on the host cores (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------
class OracleSample:
    """One (sequence, key-head group) of one layer, the bounded sample the
    oracle is timed on; scaled by the number of such groups per step."""

    def __init__(self, w, steps=2):
        self.w = w
        L = int(synth.seq_lens(w)[0])
        G = w.h_q // w.h_k
        hv_g = w.h_v // w.h_k
        self.L, self.G = L, G
        self.groups_per_step = w.layers * w.B * w.h_k
        K = synth.widen(synth.cache_rows(w, 0, "K", 0, 0, 0, L))
        V = np.stack([synth.widen(synth.cache_rows(w, 0, "V", 0, v, 0, L)) for v in range(hv_g)])
        self.K = K[None, None]             # [1][1][L][d]
        self.V = V[None]                   # [1][hv_g][L][d]
        self.l = np.array([L])
        self.qs = synth.widen(synth.queries(w, 0, max(2, steps), B=1, h_q=G))   # [steps][1][G][d]
        self.tau = None

    def step(self, t, refresh):
        import oracle
        q = self.qs[t % len(self.qs)]
        if refresh or self.tau is None:
            self.tau = oracle.refresh(q, self.K, self.l, self.w.N)
        oracle.decode_step(q, self.K, self.V, self.l, self.tau)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def time_oracle(w, n_plain=2, n_refresh=1):
    """Seconds per full step (every layer, sequence and key-head group), from
    timing the sample's plain and refresh steps, averaged over a refresh cycle."""
    s = OracleSample(w)
    s.step(0, True)                                   # warm
    t0 = time.perf_counter()
    for i in range(n_refresh):
        s.step(i, True)
    t_ref = (time.perf_counter() - t0) / n_refresh
    t0 = time.perf_counter()
    for i in range(n_plain):
        s.step(i + 1, False)
    t_plain = (time.perf_counter() - t0) / n_plain
    per_group = (t_ref + (w.R - 1) * t_plain) / w.R
    return per_group * s.groups_per_step, t_plain, t_ref, s


def cpu_baseline_entry(w):
    step_s, t_plain, t_ref, s = time_oracle(w)
    return {"value": 1.0 / step_s, "unit": "steps/s", "cores": os.cpu_count(),
            "blas_threads": blas_threads(), "kind": "oracle",
            "sample": (f"layer 0, sequence 0, key head 0 ({s.G} query heads, l_kv={s.L}): "
                       f"1 refresh + 2 plain steps timed, R-cycle average, scaled by "
                       f"{s.groups_per_step} groups per step"),
            "sample_plain_s": t_plain, "sample_refresh_s": t_ref}


def workload_config(w, world, replicas=1):
    return {"workload": w.name, "batch_per_gpu": w.B, "global_batch": w.B * world,
            "layers": w.layers, "h_q": w.h_q, "h_k": w.h_k, "h_v": w.h_v, "d": w.d,
            "l_kv": w.l_kv if w.l_kv_range is None else list(w.l_kv_range), "N": w.N,
            "R": w.R, "dense_gqa_h_kv": w.dense_hkv,
            "parallelism": f"weak: {world} independent batch replica(s)",
            "l2": ("inputs larger than L2" if replicas == 1 else
                   f"{replicas} bit-identical cache replicas rotated"),
            "timed_region": ("CUDA graphs of consecutive steps of one kind (R-cycle value); "
                             "the --steps schedule in one graph (timed_steps)")}


def reference_arm(args, w):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return                     # rank 0 alone times the oracle; no process group
    s = OracleSample(w, steps=args.warmup + args.steps)
    for t in range(args.warmup):
        s.step(t, t % w.R == 0)
    t0 = time.perf_counter()
    for t in range(args.steps):
        s.step(args.warmup + t, t % w.R == 0)
    sample_s = time.perf_counter() - t0
    step_s = sample_s / args.steps * s.groups_per_step
    v = 1.0 / step_s
    sample = (f"layer 0, sequence 0, key head 0 ({s.G} query heads, l_kv={s.L}) of each "
              f"step, scaled by {s.groups_per_step} groups per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "steps/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, world, replicas_for(w)),
        "cpu_baseline": {"value": v, "unit": "steps/s", "cores": os.cpu_count(),
                         "blas_threads": blas_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": v, "unit": "steps/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def stack_cap(w):
    """Cache capacity: the longest sequence rounded up to 128 positions."""
    return int(math.ceil(int(synth.seq_lens(w).max()) / 128) * 128)


def replicas_for(w, dense=False):
    """Single-layer workloads rotate bit-identical cache replicas so the
    working set stays well above L2."""
    if w.layers > 1:
        return 1
    h = w.dense_hkv if dense else w.h_k
    hv = w.dense_hkv if dense else w.h_v
    layer_bytes = w.B * (h + hv) * stack_cap(w) * w.d * w.elem_bytes
    return max(1, math.ceil(4 * L2_BYTES / layer_bytes))


class Stack:
    """Device state of one attention stack: per-layer caches, thresholds,
    outputs, the static query buffer and the workspace."""

    def __init__(self, w, saga, dense=False):
        import torch
        from synth import device as sdev
        self.w, self.dense = w, dense
        h_k = w.dense_hkv if dense else w.h_k
        h_v = w.dense_hkv if dense else w.h_v
        kk, vk = ("KD", "VD") if dense else ("K", "V")
        self.lens = synth.seq_lens(w)
        cap = stack_cap(w)
        self.cap = cap
        self.shape = saga.shape(w.B, w.h_q, h_k, h_v, w.d, w.dtype, cap, cap)
        self.replicas = replicas_for(w, dense)
        self.nl = w.layers
        dt = torch.float32 if w.dtype == synth.F32 else torch.int16
        self.K, self.V = [], []
        for r in range(self.replicas):
            for l in range(self.nl):
                if r == 0:
                    K = torch.empty(w.B, h_k, cap, w.d, dtype=dt, device="cuda")
                    V = torch.empty(w.B, h_v, cap, w.d, dtype=dt, device="cuda")
                    sdev.fill(K, w, l, kk)
                    sdev.fill(V, w, l, vk)
                else:
                    K = self.K[l].clone()
                    V = self.V[l].clone()
                self.K.append(K)
                self.V.append(V)
        self.l = torch.from_numpy(self.lens).cuda()
        self.tau = torch.zeros(self.nl, w.B, w.h_q, dtype=torch.float32, device="cuda")
        self.out = torch.zeros(self.nl, w.B, w.h_q, w.d, dtype=torch.float32, device="cuda")
        self.q = torch.zeros(self.nl, w.B, w.h_q, w.d, dtype=dt, device="cuda")
        self.ws = saga.Workspace(self.shape, w.N)
        self.saga = saga

    def layer_call(self, t, l, refresh, sel_mask=None, N=None):
        r = t % self.replicas
        K, V = self.K[r * self.nl + l], self.V[r * self.nl + l]
        s = self.saga
        if self.dense:
            s.gqa_dense_decode(self.shape, self.q[l], K, V, self.l, self.out[l], self.ws)
        elif refresh:
            s.refresh_threshold(self.shape, self.q[l], K, self.l, self.w.N if N is None else N,
                                self.tau[l], self.ws, V=V, out=self.out[l], sel_mask=sel_mask)
        else:
            s.decode_step(self.shape, self.q[l], K, V, self.l, self.tau[l], self.out[l], self.ws,
                          sel_mask=sel_mask)

    def step(self, t, refresh, N=None):
        for l in range(self.nl):
            self.layer_call(t, l, refresh, N=N)

    def full_step(self, t):
        """Full attention over the same (SAGA-headed) caches, every layer."""
        r = t % self.replicas
        for l in range(self.nl):
            self.saga.dense_decode(self.shape, self.q[l], self.K[r * self.nl + l],
                                   self.V[r * self.nl + l], self.l, self.out[l], self.ws)

    def free(self):
        import torch
        self.K, self.V = [], []
        torch.cuda.empty_cache()


def kernels_per_call(dense, refresh):
    if dense:
        return 2                  # dense split + combine
    return 4 if refresh else 2    # (dump, radix,) step + combine


def graph_of(fn):
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def replay_ms(g, n, stream):
    """Device time of each of n back-to-back replays of graph g (CUDA events
    on the launching stream; the host is kept ahead of the GPU)."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n)]
    torch.cuda.synchronize()
    torch.cuda._sleep(int(2e7))
    for a, b in evs:
        a.record(stream)
        g.replay()
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def call_ms(fn, n, stream):
    """Device time of each of n direct calls of fn (host kept ahead)."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n)]
    torch.cuda.synchronize()
    torch.cuda._sleep(int(2e8))
    for i, (a, b) in enumerate(evs):
        a.record(stream)
        fn(i)
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def measure_saga(w, args, saga, world, rank, N=None, st=None, with_dense=True, with_cpu=True):
    """All figures of one workload (and one N): the R-cycle value and its
    parts, the --steps schedule, e2e, roofline, dense GQA, SAGA full
    attention and the CPU baseline. Returns (dict, stack)."""
    import torch
    N = w.N if N is None else N
    R, nl = w.R, w.layers
    own = st is None
    if own:
        st = Stack(w, saga)
    esz = w.elem_bytes
    reps = 4 if nl > 1 else 32                     # steps per graph replay
    W, K = max(3, args.warmup), args.steps
    n_q = W + K + 2 * reps
    qh = np.stack([synth.queries(w, l, n_q) for l in range(nl)], axis=1)
    if w.dtype != synth.F32:
        qh = qh.view(np.int16)
    Q = torch.from_numpy(qh).cuda()                # [step][layer][B][h_q][d]
    Qpin = torch.from_numpy(qh).pin_memory()
    stream = torch.cuda.current_stream()
    sched = step_schedule(K, R)

    def run_steps(idx0, n, kind):
        # n steps with queries idx0.., refresh by `kind` (a list of flags or a bool)
        for i in range(n):
            st.q.copy_(Q[idx0 + i], non_blocking=True)
            st.step(idx0 + i, kind[i] if isinstance(kind, list) else kind, N=N)

    # warm-up: every kernel loaded and tau set before any capture
    run_steps(0, W, step_schedule(W, R))
    torch.cuda.synchronize()
    g_timed = graph_of(lambda: run_steps(W, K, sched))
    g_plain = graph_of(lambda: run_steps(W + K, reps, False))
    g_ref = graph_of(lambda: run_steps(W + K + reps, reps, True))
    torch.cuda.synchronize()
    barrier(world)

    # ---- the --steps schedule, then the R-cycle parts ---------------------
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda._sleep(int(2e7))
    ev0.record(stream)
    g_timed.replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    timed_ms = max_over_ranks(ev0.elapsed_time(ev1), world)
    n_plain = max(MIN_REPLAYS, 64 // reps)
    plain = replay_ms(g_plain, n_plain, stream) if R > 1 else []
    refr = replay_ms(g_ref, max(MIN_REPLAYS, 16 // reps), stream)
    t_plain = max_over_ranks(float(np.median(plain)) / reps, world) if plain else None
    t_ref = max_over_ranks(float(np.median(refr)) / reps, world)
    per_rank = r_cycle(t_plain, t_ref, R) if R > 1 else 1e3 / t_ref
    value = world * per_rank
    n_refresh = sum(sched)
    launches = nl * (n_refresh * kernels_per_call(False, True)
                     + (K - n_refresh) * kernels_per_call(False, False))
    del g_timed, g_plain, g_ref

    # ---- roofline of the dominant call: the plain step (the refresh at R = 1)
    dom_refresh = R == 1
    n_calls = 24

    def one_call(i):
        st.q.copy_(Q[W + K + i % (2 * reps)])
        st.layer_call(i, i % nl, dom_refresh, N=N)
    ms = call_ms(one_call, n_calls, stream)
    call = float(np.median(ms))
    B, h_q, h_k, h_v, d = w.B, w.h_q, w.h_k, w.h_v, w.d
    lens = st.lens.astype(np.int64)
    k_bytes = float(np.sum(h_k * lens * d * esz))
    qo_bytes = B * h_q * d * (esz + 4) + B * h_q * 4
    mask = torch.zeros(B, h_q, st.cap, dtype=torch.uint8, device="cuda")
    v_bytes, v_nodedup = [], []
    for i in range(4):
        st.q.copy_(Q[W + K + i])
        mask.zero_()
        st.layer_call(i, i % nl, dom_refresh, sel_mask=mask, N=N)
        m = mask.view(B, h_v, h_q // h_v, st.cap)
        v_bytes.append(int(m.amax(dim=2).sum().item()) * d * esz)
        v_nodedup.append(int(mask.sum().item()) * d * esz)
    torch.cuda.synchronize()
    del mask
    alg = k_bytes + float(np.mean(v_bytes)) + qo_bytes
    peak, peak_kind = measured_peaks()
    achieved = alg / (call / 1e3) / 1e9
    roof = {"bound": "hbm",
            "kernel": ("saga_refresh_threshold (score pass, select, stored-score step, combine)"
                       if dom_refresh else "saga_decode_step (step kernel + combine)"),
            "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
            "peak_source": peak_kind,
            "traffic": None if dom_refresh else ncu_traffic(step_kernel_sources()),
            "alg_bytes_per_call": alg, "call_ms": call, "calls_timed": n_calls,
            "v_bytes_per_call_distinct": float(np.mean(v_bytes)),
            "v_bytes_per_call_nodedup": float(np.mean(v_nodedup)),
            "frac_of_8000_nominal": achieved / 8000.0}

    # ---- e2e: each step's queries in from pinned host memory, outputs back
    out_pin = torch.empty(st.out.shape, dtype=torch.float32).pin_memory()
    l_pin = torch.from_numpy(st.lens).pin_memory()
    g1 = {}
    for r in range(st.replicas):
        for kind in ((True, False) if R > 1 else (True,)):
            g1[(kind, r)] = graph_of(lambda r=r, kind=kind: st.step(r, kind, N=N))
    torch.cuda.synchronize()
    barrier(world)
    e2e = {True: [], False: []}
    n_e2e = MIN_REPLAYS + 2
    for kind in g1and_kinds(R):
        for i in range(n_e2e):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            st.q.copy_(Qpin[W + K + i % (2 * reps)], non_blocking=True)
            st.l.copy_(l_pin, non_blocking=True)
            g1[(kind, i % st.replicas)].replay()
            out_pin.copy_(st.out, non_blocking=True)
            b.record(stream)
            stream.synchronize()
            e2e[kind].append(a.elapsed_time(b))
    e2e_p = max_over_ranks(float(np.median(e2e[False])), world) if R > 1 else None
    e2e_f = max_over_ranks(float(np.median(e2e[True])), world)
    e2e_value = world * (r_cycle(e2e_p, e2e_f, R) if R > 1 else 1e3 / e2e_f)
    h2d = Q[0].numel() * Q.element_size() + l_pin.numel() * 4
    d2h = st.out.numel() * 4
    del g1

    res = {
        "value": value, "unit": "steps/s", "ms_per_step": 1e3 / value * world,
        "tokens_per_s": value * B,
        "step_times": {"plain_ms": t_plain, "refresh_ms": t_ref, "refresh_every": R,
                       "steps_per_replay": reps, "replays": [len(plain), len(refr)],
                       "statistic": "median per step, max over ranks"},
        "timed_steps": {"steps": K, "refresh_steps": n_refresh, "ms": timed_ms,
                        "steps_per_s": aggregate_value(K, timed_ms, world)},
        "gpu_launches": launches * world,
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": "steps/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "plain_ms": e2e_p, "refresh_ms": e2e_f},
        "N": N,
    }

    # ---- dense GQA stack at the same shape, and SAGA full attention --------
    if with_dense and not args.no_dense and w.dense_hkv is not None:
        dst = Stack(w, saga, dense=True)
        dst.q.copy_(Q[0])
        dst.step(0, False)
        torch.cuda.synchronize()
        dreps = 2 if nl > 1 else 16

        def dense_steps():
            for i in range(dreps):
                dst.q.copy_(Q[i], non_blocking=True)
                dst.step(i, False)
        gd = graph_of(dense_steps)
        dms = max_over_ranks(float(np.median(replay_ms(gd, MIN_REPLAYS, stream))) / dreps, world)
        del gd
        dbytes = nl * (2 * w.dense_hkv * float(np.sum(lens)) * d * esz + qo_bytes)
        dgbs = dbytes / (dms / 1e3) / 1e9
        dvalue = world * 1e3 / dms
        res["dense_gqa"] = {"value": dvalue, "unit": "steps/s", "ms_per_step": dms,
                            "tokens_per_s": dvalue * B, "achieved_gbs": dgbs,
                            "frac_of_peak": dgbs / peak, "h_kv": w.dense_hkv,
                            "speedup_saga_over_dense": value / dvalue}
        dst.free()
        del dst
    if with_dense and not args.no_dense and w.h_k != w.h_v:
        freps = 2 if nl > 1 else 16

        def full_steps():
            for i in range(freps):
                st.q.copy_(Q[i], non_blocking=True)
                st.full_step(i)
        full_steps()
        torch.cuda.synchronize()
        gf = graph_of(full_steps)
        fms = max_over_ranks(float(np.median(replay_ms(gf, MIN_REPLAYS, stream))) / freps, world)
        del gf
        fbytes = nl * ((w.h_k + w.h_v) * float(np.sum(lens)) * d * esz + qo_bytes)
        fgbs = fbytes / (fms / 1e3) / 1e9
        fvalue = world * 1e3 / fms
        res["saga_full"] = {"value": fvalue, "unit": "steps/s", "ms_per_step": fms,
                            "tokens_per_s": fvalue * B, "achieved_gbs": fgbs,
                            "frac_of_peak": fgbs / peak, "h_k": w.h_k, "h_v": w.h_v,
                            "speedup_saga_atopn_over_full": value / fvalue}
        if "dense_gqa" in res:
            res["saga_full"]["speedup_full_over_dense_gqa"] = fvalue / res["dense_gqa"]["value"]
    if with_cpu and rank == 0 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline_entry(w.with_(N=N))
    res["config"] = workload_config(w, world, st.replicas)
    res["config"]["N"] = N
    del Q, Qpin
    if own:
        st.free()
    return res, (None if own else st)


def g1and_kinds(R):
    return (True, False) if R > 1 else (True,)


def run_ours(args, w):
    import torch
    import sparse_decode_attention_step_b200 as saga
    saga.load()
    world, rank, local = dist_init()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but {world} ranks were started")
    torch.manual_seed(0)
    names = [w.name] + ([] if args.primary_only else [n for n in EXTRA_WORKLOADS if n != w.name])
    results = {}
    with ClockSampler(local) as clk:
        for name in names:
            ww = w if name == w.name else synth.WORKLOADS[name]
            ww = rank_workload(ww, rank)
            if ww.N_sweep:
                st = Stack(ww, saga)
                for N in ww.N_sweep:
                    results[f"{name}_N{N}"], st = measure_saga(ww, args, saga, world, rank, N=N, st=st,
                                                               with_dense=False)
                st.free()
                del st
            else:
                results[name], _ = measure_saga(ww, args, saga, world, rank)
            torch.cuda.empty_cache()
    clocks = clk.summary()
    if rank == 0:
        primary_key = w.name if w.name in results else f"{w.name}_N{w.N}"
        p = results.pop(primary_key)
        line = {
            "metric": METRIC, "value": p["value"], "unit": "steps/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": 1e3 / p["value"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype != synth.F32 else "f32", "accumulate": "f32",
            "data": "synthetic (seeded Philox N(0,1) K/V, 1% planted keys, AR(1) queries)",
            "config": p.pop("config"),
            "tokens_per_s": p.pop("tokens_per_s"), "refresh_every": w.R,
        }
        p.pop("value"), p.pop("unit"), p.pop("ms_per_step")
        line.update(p)
        line["clocks"] = clocks
        line["pages_context"] = PAGES_CONTEXT
        line["workloads"] = results
        print(json.dumps(line), flush=True)
    finish_dist(world)


# ---------------------------------------------------------------------------
# the closed-form key merge (one layer's conversion)
# ---------------------------------------------------------------------------
MERGE_METRIC = "GQA-to-SAGA closed-form key merges/s (one layer)"


def merge_oracle_seconds(w, X, W, Q):
    """The float64 oracle on the host cores: one pair's Eq. (13) weight at its
    Eq. (15) optimum, timed, scaled by the number of pairs (the matching and
    the merged projection are negligible beside it)."""
    from oracle import key_merge as km
    n_pairs = w.h_k * (w.h_k - 1) // 2
    t0 = time.perf_counter()
    km.pair_weights(X, W, Q, w.h_q, w.h_k, w.d, 1e-6, pairs=[(0, 1)])
    one = time.perf_counter() - t0
    return one * n_pairs, one, n_pairs


def bench_merge(args):
    import torch
    import sparse_decode_attention_step_b200 as saga
    from synth import merge_workload as mw
    saga.load()
    w = mw.MERGE_WORKLOADS[args.merge]
    Xb, Wb, Qb = mw.merge_inputs(w)
    host = [torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).pin_memory()
            for a in (Xb, Wb, Qb)]
    X, W, Q = (h.cuda() for h in host)
    ms = saga.merge_shape(w.T, w.d_model, w.h_q, w.h_k, w.d)
    ws = saga.MergeWorkspace(ms)
    n2 = w.h_k // 2
    wout = torch.empty((w.h_k, w.h_k), dtype=torch.float64, device="cuda")
    pairs = torch.empty((n2, 2), dtype=torch.int32, device="cuda")
    total = torch.empty(1, dtype=torch.float64, device="cuda")
    W_S = torch.empty((n2 * w.d, w.d_model), dtype=torch.float32, device="cuda")
    outs_h = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (wout, pairs, W_S)]
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def call(x, wk, q):
        saga.merge_keys(ms, x, wk, q, 1e-6, wout, pairs, W_S, ws, total=total)

    for _ in range(max(3, args.warmup)):
        call(X, W, Q)
    torch.cuda.synchronize()
    assert saga.read_device_error(ws) == 0
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    ee = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    with ClockSampler(torch.cuda.current_device()) as clk:
        for i in range(args.steps):
            flush.zero_()                       # every call starts with a cold L2
            ev[i][0].record(stream)
            call(X, W, Q)
            ev[i][1].record(stream)
        # end to end: inputs in from pinned host memory, results back
        for i in range(args.steps):
            flush.zero_()
            ee[i][0].record(stream)
            X.copy_(host[0], non_blocking=True)
            W.copy_(host[1], non_blocking=True)
            Q.copy_(host[2], non_blocking=True)
            call(X, W, Q)
            for h, t in zip(outs_h, (wout, pairs, W_S)):
                h.copy_(t, non_blocking=True)
            ee[i][1].record(stream)
        torch.cuda.synchronize()
    call_ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    e2e_ms = float(np.mean([a.elapsed_time(b) for a, b in ee]))
    assert saga.read_device_error(ws) == 0
    HD = w.h_k * w.d
    flops = (2.0 * w.T * w.d_model * HD          # K = X W^T
             + 3 * 2.0 * w.T * HD * HD            # C = K^T K as three bf16 products
             + 2.0 * w.T * w.d * w.d * w.h_q)     # the S_r
    h2d = sum(h.numel() * h.element_size() for h in host)
    d2h = sum(h.numel() * h.element_size() for h in outs_h)
    cpu = None
    if not args.no_cpu_baseline:
        Xw, Ww, Qw = (synth.widen(a) for a in (Xb, Wb, Qb))
        secs, one, n_pairs = merge_oracle_seconds(w, Xw, Ww, Qw)
        cpu = {"value": 1.0 / secs, "unit": "merges/s", "cores": blas_threads(),
               "kind": "oracle",
               "sample": f"the weight of pair (0, 1) (Eq. 13 from explicit logits at the "
                         f"Eq. 15 optimum) timed once, {one:.2f} s, scaled by {n_pairs} pairs"}
    line = {
        "metric": MERGE_METRIC, "value": 1e3 / call_ms, "unit": "merges/s", "n_gpus": 1,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": call_ms,
        "higher_is_better": True, "scaling": "none", "vs_baseline": None,
        "dtype": "bf16 GEMMs (f32 accumulate), f64 pair algebra", "data": "synthetic",
        "config": {"workload": w.name, "T": w.T, "d_model": w.d_model, "h_q": w.h_q,
                   "h_k": w.h_k, "d": w.d, "l2": "flushed before every call"},
        "gpu_launches": 8 * args.steps,
        "gemm_tflops_algorithmic": flops / (call_ms / 1e3) / 1e12,
        "e2e": {"value": 1e3 / e2e_ms, "unit": "merges/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "pairs": [tuple(p) for p in pairs.cpu().tolist()],
        "clocks": clk.summary(),
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def main():
    argv = sys.argv[1:]
    args = parse(argv)
    rc = spawn_ranks(args, argv)
    if rc is not None:
        sys.exit(rc)
    if args.merge is not None:
        bench_merge(args)
        return
    w = synth.WORKLOADS[args.workload]
    if args.layers is not None:
        w = w.with_(layers=args.layers)
    if args.steps < 1 or args.warmup < 0:
        raise SystemExit("--steps must be >= 1")
    if args.impl == "reference":
        reference_arm(args, w)
        return
    run_ours(args, w)


if __name__ == "__main__":
    main()

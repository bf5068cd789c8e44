#!/usr/bin/env python
"""Throughput of the log-linear attention forward (Mamba-2 form) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--path auto|simt|tcgen05]

One step is one forward over one batch of the workload (all of: decay scan,
chunk states, Fenwick block merge, intra-chunk part, lam-weighted readout), with
inputs resident in HBM.  Default workload: B=4, H=32, T=8192, d_k=d_v=64, bf16
q/k/v, fp32 log_a/lam (L=14), fp32 out; synthetic seeded inputs.  The metric is
tokens/s (tokens = sum of sequence lengths; heads are inside a token).  Under
torchrun each rank runs its own batch (weak scaling, no collective on the data
path); the time is the max over ranks.

Prints ONE JSON line (rank 0) with the throughput, the dominant kernel's
roofline fraction against the measured HBM bandwidth, the CPU oracle baseline,
the end-to-end figure through the host-buffer C entry point, launch count and
SM clocks sampled during the timed region.

--pass bwd times the backward pass over the same workload: dq, dk, dv, dlog_a and dlam from
q, k, v, log_a, lam and the output gradient (tokens/s of gradient computation).

--workload decode_b64_h32_d64_bf16 times the decoding step instead: one new token for each of
64 sequences whose positions are spread over [0, 8192), H=32, d=64, reading the level states
the positions occupy and writing the carried one (tokens/s = sequences x steps / time).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "log-linear attn fwd tokens/s at T=8K,H=32,d=64; % of roofline (1×B200)"
DEFAULT_WORKLOAD = "t8k_d64_bf16"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--path", default="auto", choices=["auto", "simt", "tcgen05"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--graph", default="auto", choices=["auto", "on", "off"],
                    help="replay the forward step as a CUDA graph (auto and on: yes; off: every "
                         "step issued from Python through the binding)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--segment-chunks", type=int, default=0,
                    help="force the tensor-core path's segment length in chunks (0: automatic)")
    ap.add_argument("--pass", dest="which", choices=["fwd", "bwd"], default="fwd",
                    help="bwd times the backward pass (gradients of all inputs) instead")
    return ap.parse_args()


# ---------------------------------------------------------------------------------------------
# accounting
# ---------------------------------------------------------------------------------------------
def algorithmic_bytes(w, total_tokens):
    """Bytes the method must move: read q, k, v, log_a, lam; write out (fp32)."""
    esz = 2 if w.dtype == "bf16" else 4
    per = (2 * w.dk + w.dv) * esz + 4 * w.dv + 4 + 4 * w.L
    return per * total_tokens * w.H, per


def algorithmic_flops(w, lengths, chunk):
    """Dense-tile FLOPs of the chunkwise form: intra 2C^2(dk+dv), chunk state 2C dk dv,
    readout 2C dk dv per set bit of the chunk index."""
    tot = 0
    for n in lengths:
        nch = (n + chunk - 1) // chunk
        pc = sum(bin(c).count("1") for c in range(nch))
        tot += nch * (2 * chunk * chunk * (w.dk + w.dv) + 2 * chunk * w.dk * w.dv) \
            + pc * 2 * chunk * w.dk * w.dv
    return tot * w.H


def decode_algorithmic_bytes(d):
    """Bytes one decoding step must move, summed over (sequence, head): the occupied level
    states read (popcount(n) of them), the carried state written (unless n is the last position
    the slots hold), each slot's pending-gate scalar read and the new ones written, the token's
    q, k, v, log_a and lam, and the fp32 output."""
    esz = 2 if d.dtype == "bf16" else 4
    nslot = d.L - 1
    state = 4 * d.dk * d.dv
    tot = 0
    for n in (int(x) for x in d.pos):
        occ = bin(n).count("1")
        m = 0
        while (n >> m) & 1:
            m += 1
        carry = 1 if m < nslot else 0
        new_gates = bin((n + 1) & ((1 << nslot) - 1)).count("1")
        per = (occ + carry) * state + 4 * (occ + new_gates) \
            + (2 * d.dk + d.dv) * esz + 4 + 4 * d.L + 4 * d.dv
        tot += per * d.H + 4   # + the position
    return tot


def bwd_algorithmic(w, lengths):
    """Bytes and FLOPs of one backward step.  Bytes: read q, k, v, dout (input type), log_a, lam;
    write dq, dk, dv, dlog_a, dlam (fp32).  FLOPs of the level-by-level form: every causal pair
    inside an aligned 32-token tile costs two dot products and three product terms (10 d); at
    each level l >= 6, every token of a block with both halves present adds its outer product
    to a d x d state (2 d^2) and applies the other half's state (2 d^2 on the right half,
    4 d^2 on the left)."""
    esz = 2 if w.dtype == "bf16" else 4
    d = w.dk
    per = (2 * w.dk + 2 * w.dv) * esz + 4 + 4 * w.L + (2 * w.dk + w.dv) * 4 + 4 + 4 * w.L
    flops = 0
    for n in lengths:
        for t0 in range(0, n, 32):
            m = min(32, n - t0)
            flops += m * (m + 1) // 2 * 10 * d
        for lvl in range(6, w.L):
            half = 1 << (lvl - 1)
            for lo in range(0, n, 2 * half):
                nl = min(half, n - lo)
                nr = max(0, min(2 * half, n - lo) - half)
                if nr:
                    flops += (nl + nr) * 2 * d * d + nr * 2 * d * d + nl * 4 * d * d
    return per * sum(lengths) * w.H, flops * w.H, per


def alu_peak_tflops():
    """fp32 FMA peak of a B200: 148 SMs x 128 fp32 lanes x 2 FLOPs x 1965 MHz (max SM clock)."""
    return 148 * 128 * 2 * 1.965e9 / 1e12


def bwd_on_tensor_cores(inp):
    """Whether llattn_bwd runs this problem's pair interactions on the tensor cores (bf16
    inputs at d = 64), as the library dispatches it."""
    return inp.dtype == "bf16" and inp.dk == 64 and inp.dv == 64


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


# The CUDA sources each measured kernel is built from.  A stored ncu capture stays valid while
# these files' code is unchanged; code elsewhere in the library (other kernels, the host API)
# does not move that kernel's DRAM traffic.
KERNEL_SOURCES = {
    "tcgen05": ["llattn_tc.cu", "llattn_tc_ptx.cuh", "llattn_common.cuh", "llattn_internal.h"],
    "simt": ["llattn_simt.cu", "llattn_common.cuh", "llattn_internal.h"],
    "decode": ["llattn_decode.cu", "llattn_decode.h", "llattn_common.cuh", "llattn_internal.h"],
    "bwd": ["llattn_bwd.cu", "llattn_bwd.h", "llattn_bwd_tc.cu", "llattn_tc_ptx.cuh",
            "llattn_common.cuh", "llattn_internal.h"],
}


def source_hash(kernel_key):
    """Hash of the code of the sources a kernel is built from (``kernel_key`` is
    "<kernel>:<workload>"): comments and whitespace are left out, so that only a change of the
    code itself makes a stored ncu capture stale."""
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "hierarchical_fenwick_state_b200", "csrc")
    for name in sorted(KERNEL_SOURCES[kernel_key.split(":")[0]]):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(name.encode() + " ".join(text.split()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key):
    """DRAM bytes per launch from the committed ncu summary, if it matches these sources."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    ent = d.get(kernel_key)
    if not ent or ent.get("source_hash") != source_hash(kernel_key):
        return None
    return ent.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, device_index):
        self.dev = device_index
        self.samples = []
        self.reasons = 0
        self.err = None
        self._stop = threading.Event()
        self._t = None
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001
            self.err = f"nvml unavailable: {e}"
            self.nv = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception as e:  # noqa: BLE001
                self.err = str(e)
                return
            time.sleep(0.005)

    def start(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        self._stop.set()
        if self._t is not None:
            self._t.join()
        names = [n for n, bit in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples),
                **({"error": self.err} if self.err else {})}


# ---------------------------------------------------------------------------------------------
# CPU oracle timing (the baseline and the reference arm)
# ---------------------------------------------------------------------------------------------
def oracle_sample_rate(inp, heads, seconds_hint=None):
    """Time the recurrent fp64 oracle on one sequence x `heads` heads; return (tok/s, desc, s)."""
    import numpy as np
    import oracle as O
    try:
        from threadpoolctl import threadpool_limits
    except Exception:  # noqa: BLE001
        threadpool_limits = None
    start, n = inp.seq_slices()[0]
    qf = inp.q.reshape(-1, inp.H, inp.dk)[start:start + n, :heads].transpose(1, 0, 2)
    kf = inp.k.reshape(-1, inp.H, inp.dk)[start:start + n, :heads].transpose(1, 0, 2)
    vf = inp.v.reshape(-1, inp.H, inp.dv)[start:start + n, :heads].transpose(1, 0, 2)
    la = inp.log_a.reshape(-1, inp.H)[start:start + n, :heads].T
    lm = inp.lam.reshape(-1, inp.H, inp.L)[start:start + n, :heads].transpose(1, 0, 2)
    ctx = threadpool_limits(limits=1) if threadpool_limits else None
    if ctx:
        ctx.__enter__()
    t0 = time.perf_counter()
    O.llattn_recurrent_seq(np.ascontiguousarray(qf), np.ascontiguousarray(kf),
                           np.ascontiguousarray(vf), np.ascontiguousarray(la),
                           np.ascontiguousarray(lm))
    dt = time.perf_counter() - t0
    if ctx:
        ctx.__exit__(None, None, None)
    # tokens/s of the whole workload = (tokens of the sample * heads/H) / time
    rate = n * (heads / inp.H) / dt
    desc = (f"recurrent fp64 oracle form, 1 sequence x {heads} of {inp.H} heads x {n} tokens, "
            f"{dt:.2f} s, numpy single thread")
    return rate, desc, dt


def _oracle_head_worker(arrs):
    """One head of the recurrent fp64 oracle in a worker process (single-threaded BLAS)."""
    import oracle as O
    t0 = time.perf_counter()
    O.llattn_recurrent_seq(*arrs)
    return time.perf_counter() - t0


def _host_info():
    info = {"cpu_count": os.cpu_count()}
    try:
        from threadpoolctl import threadpool_info
        blas = [d for d in threadpool_info() if d.get("user_api") == "blas"]
        info["blas_threads"] = int(sum(d.get("num_threads", 0) for d in blas)) if blas else None
    except Exception:  # noqa: BLE001
        info["blas_threads"] = None
    return info


class OraclePool:
    """Worker processes for the recurrent fp64 oracle, one head per task, each with a
    single-threaded BLAS (spawn context: safe after CUDA has been initialised)."""

    def __init__(self, cores=None):
        import multiprocessing as mp
        self.cores = max(1, cores or os.cpu_count() or 1)
        keep = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS",
                                                "MKL_NUM_THREADS")}
        for k in keep:
            os.environ[k] = "1"          # inherited by the spawned workers
        try:
            self.pool = mp.get_context("spawn").Pool(self.cores)
        finally:
            for k, v in keep.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v

    def close(self):
        self.pool.close()
        self.pool.join()

    def rate(self, inp, heads=None, tokens=None):
        """`heads` heads (default: all) of the first sequence, its first `tokens` tokens
        (default: all), spread over the cores, one head per task; returns (tok/s of the whole
        workload, cores used, description, wall seconds)."""
        import numpy as np
        start, n = inp.seq_slices()[0]
        sl = slice(start, start + n)

        def head(h, m=None):
            e = sl if m is None else slice(start, start + m)
            return (np.ascontiguousarray(inp.q.reshape(-1, inp.H, inp.dk)[e, h][None]),
                    np.ascontiguousarray(inp.k.reshape(-1, inp.H, inp.dk)[e, h][None]),
                    np.ascontiguousarray(inp.v.reshape(-1, inp.H, inp.dv)[e, h][None]),
                    np.ascontiguousarray(inp.log_a.reshape(-1, inp.H)[e, h][None]),
                    np.ascontiguousarray(inp.lam.reshape(-1, inp.H, inp.L)[e, h][None]))

        # every worker started (imports done) before the clock: a tiny task each
        self.pool.map(_oracle_head_worker, [head(0, min(n, 8))] * self.cores)
        nh = inp.H if heads is None else max(1, min(heads, inp.H))
        m = n if tokens is None else max(1, min(tokens, n))
        work = [head(h, m) for h in range(nh)]
        used = min(self.cores, nh)
        t0 = time.perf_counter()
        self.pool.map(_oracle_head_worker, work, chunksize=1)
        wall = time.perf_counter() - t0
        which = f"all {inp.H}" if nh == inp.H else f"{nh} of {inp.H}"
        desc = (f"recurrent fp64 oracle form, 1 sequence x {which} heads x {m} tokens, one "
                f"head per task on {used} host cores (spawned pool, single-threaded BLAS each), "
                f"{wall:.2f} s wall")
        # tokens/s of the whole workload: the sample is m tokens x nh / H of the heads
        return m * nh / inp.H / wall, used, desc, wall


def oracle_allcores_rate(inp):
    pool = OraclePool()
    try:
        return pool.rate(inp)
    finally:
        pool.close()


def oracle_quadratic_rate(inp, max_tokens=4096):
    """The quadratic (masked) fp64 oracle form on one head of the first sequence's first
    `max_tokens` tokens, with the process's BLAS threads; tok/s of the workload at that
    prefix length (the form's cost grows with T^2, so the full length is slower still)."""
    import numpy as np
    import oracle as O
    start, n = inp.seq_slices()[0]
    m = min(n, max_tokens)
    sl = slice(start, start + m)
    t0 = time.perf_counter()
    O.llattn_quadratic_seq(inp.q.reshape(-1, inp.H, inp.dk)[sl, 0],
                           inp.k.reshape(-1, inp.H, inp.dk)[sl, 0],
                           inp.v.reshape(-1, inp.H, inp.dv)[sl, 0],
                           inp.log_a.reshape(-1, inp.H)[sl, 0],
                           inp.lam.reshape(-1, inp.H, inp.L)[sl, 0])
    dt = time.perf_counter() - t0
    return {"value": m / inp.H / dt, "unit": "tokens/s", "kind": "oracle (quadratic form)",
            "sample": f"1 head x first {m} tokens of one sequence, {dt:.2f} s, BLAS threads of "
                      f"the process; cost grows as T^2"}


def run_reference(args, w, rank, world):
    """The oracle as it stands, timed on the host cores (rank 0 only)."""
    from hierarchical_fenwick_state_b200 import inputs as I
    if rank != 0:
        return None
    inp = I.make_inputs(w, seed=args.seed)
    pool = OraclePool()
    # one round of the pool per step: as many heads of the first sequence as there are cores,
    # so the default run (100 steps) stays within a few minutes; warm-up steps on a short sample
    heads = min(inp.H, pool.cores)
    try:
        for _ in range(args.warmup):
            pool.rate(inp, heads=heads, tokens=256)
        times, rates = [], []
        for _ in range(args.steps):
            r, cores, desc, dt = pool.rate(inp, heads=heads)
            times.append(dt)
            rates.append(r)
    finally:
        pool.close()
    value = float(statistics.mean(rates))
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * statistics.mean(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": workload_config(w, None, None),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": desc + " per step", "host": _host_info()},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    return line


def max_over_ranks(x: float, dist, device) -> float:
    """The largest per-rank value over all ranks (the slowest rank sets the step time);
    `dist` is torch.distributed or None for a single process."""
    if dist is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(seed: int, rank: int) -> int:
    """Each rank draws its own batch (weak scaling: per-GPU work fixed as N grows)."""
    return seed + rank


def workload_config(w, chunk, path):
    cfg = {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "dk": w.dk, "dv": w.dv, "L": w.L,
           "inputs": f"{w.dtype} q/k/v, f32 log_a/lam, f32 out",
           "log_a": f"-exp(N({w.log_a_mu},0.5))", "lam": "softplus(N(0,1))",
           "l2": "inputs larger than L2 (no flush between steps)"}
    if w.varlen:
        cfg["varlen"] = f"{w.B} sequences, lengths U[{w.len_lo},{w.len_hi}]"
    if chunk:
        cfg["chunk"] = chunk
    if path:
        cfg["path"] = path
    return cfg


# ---------------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------------
def run_ours(args, w, rank, world, local_rank):
    import numpy as np
    import torch

    from hierarchical_fenwick_state_b200 import binding
    from hierarchical_fenwick_state_b200 import inputs as I

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    binding.lib()
    inp = I.make_inputs(w, seed=rank_seed(args.seed, rank))
    dt = torch.bfloat16 if inp.dtype == "bf16" else torch.float32
    q = torch.from_numpy(inp.q).to(dev).to(dt)
    k = torch.from_numpy(inp.k).to(dev).to(dt)
    v = torch.from_numpy(inp.v).to(dev).to(dt)
    la = torch.from_numpy(inp.log_a).to(dev)
    lm = torch.from_numpy(inp.lam).to(dev)
    cu = torch.from_numpy(inp.cu_seqlens).to(dev) if inp.cu_seqlens is not None else None
    out = torch.empty(inp.v.shape, dtype=torch.float32, device=dev)
    lengths = [n for _, n in inp.seq_slices()]
    total_tokens = int(sum(lengths))
    path = args.path
    # resolve the path and chunk the call will use
    if path == "auto":
        try:
            binding.workspace_bytes(1 if dt == torch.bfloat16 else 0, "tcgen05", 0, inp.B, inp.H,
                                    inp.T, inp.dk, inp.dv, cu is not None)
            path = "tcgen05" if dt == torch.bfloat16 else "simt"
        except binding.LLAttnError:
            path = "simt"
    chunk = 128 if path == "tcgen05" else (16 if inp.T <= 256 else 64)
    nws = binding.workspace_bytes(1 if dt == torch.bfloat16 else 0, path, chunk, inp.B, inp.H,
                                  inp.T, inp.dk, inp.dv, cu is not None)
    ws = torch.empty(max(nws, 256), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    # the automatic choice is called as a user calls it (path and chunk left to the library);
    # on CUDA cores it runs short sequences (T <= 512) as the one-launch masked form
    automatic = args.path == "auto"
    short_form = automatic and path == "simt" and inp.T <= 512

    def step():
        if automatic:
            binding.forward(q, k, v, la, lm, cu_seqlens=cu, T=inp.T, out=out, workspace=ws)
        else:
            binding.forward(q, k, v, la, lm, cu_seqlens=cu, T=inp.T, out=out, path=path,
                            chunk=chunk, workspace=ws)

    seg_chunks = 0
    if path == "tcgen05":
        seg_chunks = binding.segment_plan(inp.B, inp.H, inp.T, inp.dk, inp.dv, cu is not None)

    dist = None
    if world > 1:
        import torch.distributed as dist
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    # The step is captured once as a CUDA graph after the warm-up calls and replayed: the same
    # kernels on the same resident inputs, without the per-call host cost (argument checks and
    # marshalling in Python, the driver's launches), which bounds short steps.  The capture
    # checks only this thread's calls: under torchrun the process group's own threads may query
    # events meanwhile.
    use_graph = args.graph != "off"
    graph = None
    if use_graph:
        binding.profile_read(reset=True)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, capture_error_mode="thread_local"):
            step()
        torch.cuda.synchronize()
        launches_per_step = binding.profile_read(reset=True)[2]
        for _ in range(max(args.warmup, 3)):
            graph.replay()
        torch.cuda.synchronize()
    binding.profile_read(reset=True)
    clocks = ClockSampler(local_rank)
    clocks.start()
    binding.profile(True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        if graph is not None:
            graph.replay()
        else:
            step()
    e1.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    binding.profile(False)
    clk = clocks.stop()
    ms_total = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    main_ms, main_n, launches = binding.profile_read(reset=True)
    if graph is not None:
        # replays do not pass through the library: its launches are those captured, per step;
        # the step's device time stands for the dominant kernel's
        launches, main_n = launches_per_step * args.steps, 0
        del graph
    status = binding.device_status(clear=True)
    if status:
        raise RuntimeError(f"device status flags {status:#x} after the timed region")

    ms_step = ms_total / args.steps
    value = total_tokens * world / (ms_step / 1000.0)

    # roofline of the dominant kernel
    hbm_gbs, tflops, peak_kind = measured_peaks()
    abytes, per_tok = algorithmic_bytes(w, total_tokens)
    aflops = algorithmic_flops(w, lengths, chunk)
    main_avg_s = (main_ms / main_n) / 1000.0 if main_n else ms_step / 1000.0
    t_mem = abytes / (hbm_gbs * 1e9)
    t_cmp = aflops / (tflops * 1e12)
    kernel_key = f"{path}:{w.name}"
    if t_mem >= t_cmp:
        roof = {"bound": "hbm", "achieved": abytes / main_avg_s / 1e9, "peak": hbm_gbs,
                "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": aflops / main_avg_s / 1e12, "peak": tflops,
                "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = ncu_traffic(kernel_key)
    roof["peak_source"] = f"{peak_kind} (MEASURED_PEAKS.json)" if peak_kind == "measured" \
        else "profiling-recipe fallback"
    roof["kernel"] = kernel_key
    roof["algorithmic_bytes_per_launch"] = abytes
    roof["bytes_per_token_head"] = per_tok
    roof["main_kernel_ms"] = main_avg_s * 1000.0
    if use_graph:
        # replays bypass the library's event pair around its dominant kernel: the time is the
        # whole step's (every kernel of it), which bounds the kernel's own from above
        roof["timed"] = "whole step (CUDA graph replay)"

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if inp.dtype == "bf16" else "f32", "data": "synthetic",
        "config": {**workload_config(w, None if short_form else chunk,
                                     "simt, one launch (masked form, T <= 512)" if short_form
                                     else path),
                   **({"segment_chunks": seg_chunks} if path == "tcgen05" else {}),
                   **({"launch": "CUDA graph of one step, replayed"} if use_graph else {})},
        "roofline": roof, "gpu_launches": launches, "clocks": clk,
    }

    # end to end through the host-buffer entry point (pinned host memory)
    if not args.no_e2e:
        in_dtype = 1 if inp.dtype == "bf16" else 0
        if inp.dtype == "bf16":
            hq = torch.from_numpy(I.bf16_bits(inp.q).view(np.int16)).pin_memory()
            hk = torch.from_numpy(I.bf16_bits(inp.k).view(np.int16)).pin_memory()
            hv = torch.from_numpy(I.bf16_bits(inp.v).view(np.int16)).pin_memory()
        else:
            hq = torch.from_numpy(inp.q).pin_memory()
            hk = torch.from_numpy(inp.k).pin_memory()
            hv = torch.from_numpy(inp.v).pin_memory()
        hla = torch.from_numpy(inp.log_a).pin_memory()
        hlm = torch.from_numpy(inp.lam).pin_memory()
        hout = torch.empty(inp.v.shape, dtype=torch.float32).pin_memory()
        hcu = torch.from_numpy(inp.cu_seqlens) if inp.cu_seqlens is not None else None
        h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hla, hlm))
        h2d += hcu.numel() * 4 if hcu is not None else 0
        d2h = hout.numel() * 4

        def e2e_step():
            binding.fwd_host(in_dtype, hq, hk, hv, hla, hlm, hout, inp.B, inp.H, inp.T, inp.dk,
                             inp.dv, cu_seqlens=hcu, stream=stream)

        for _ in range(2):
            e2e_step()
        n_e2e = max(3, min(args.steps, 20))
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        # device-timed on the stream the host entry point copies and computes on; each call
        # synchronises that stream, so host-side gaps between calls are inside the bracket too
        e0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_s = max_over_ranks(e0.elapsed_time(e1) / 1000.0 / n_e2e, dist, dev)
        ref_host = hout.numpy()
        if not np.isfinite(ref_host).all():
            raise RuntimeError("non-finite output through the host entry point")
        line["e2e"] = {"value": total_tokens * world / e2e_s, "unit": "tokens/s",
                       "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                       "steps": n_e2e, "entry": "llattn_fwd_host (pinned host buffers)"}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, cores, desc, _ = oracle_allcores_rate(inp)
        line["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": cores,
                                "kind": "oracle", "sample": desc, "host": _host_info(),
                                "quadratic_form": oracle_quadratic_rate(inp)}
    return line


# ---------------------------------------------------------------------------------------------
# decoding step
# ---------------------------------------------------------------------------------------------
DECODE_METRIC = "log-linear attn decode tokens/s, 64 sequences at positions < 8192, H=32, d=64 (1×B200)"


def decode_config(w, d):
    return {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "dk": w.dk, "dv": w.dv,
            "positions": f"U[0, {1 << (w.L - 1)}) per sequence, seeded",
            "inputs": f"{w.dtype} q/k/v, f32 log_a/lam, f32 out, f32 level states",
            "state_bytes": int(d.B * d.H * (d.L - 1) * (d.dk * d.dv + 2) * 4),
            "l2": "inputs larger than L2: each step reads "
                  f"{decode_algorithmic_bytes(d) / 1e6:.0f} MB of level states (no flush)"}


def oracle_decode_rate(d, pairs):
    """Time the fp64 oracle's decoding step on `pairs` (sequence, head) pairs; tokens/s."""
    import oracle as O
    try:
        from threadpoolctl import threadpool_limits
        ctx = threadpool_limits(limits=1)
    except Exception:  # noqa: BLE001
        ctx = None
    if ctx:
        ctx.__enter__()
    t0 = time.perf_counter()
    for b, h in pairs:
        O.llattn_decode_step(d.states[b, h], int(d.pos[b]), d.q[b, h], d.k[b, h], d.v[b, h],
                             d.log_a[b, h], d.lam[b, h])
    dt = time.perf_counter() - t0
    if ctx:
        ctx.__exit__(None, None, None)
    rate = (len(pairs) / d.H) / dt
    whole = "the whole step" if len(pairs) == d.B * d.H else f"a sample of {d.B * d.H}"
    desc = (f"fp64 oracle decoding step on {len(pairs)} (sequence, head) pairs ({whole}), "
            f"{dt:.2f} s, numpy single thread; tokens/s = pairs / H / time")
    return rate, desc, dt


def _decode_pairs(d, n):
    import numpy as np
    rng = np.random.default_rng(1)
    return list(zip(rng.integers(0, d.B, n).tolist(), rng.integers(0, d.H, n).tolist()))


def run_decode_reference(args, w, rank, world):
    from hierarchical_fenwick_state_b200 import inputs as I
    if rank != 0:
        return None
    d = I.make_decode_inputs(w, seed=args.seed)
    pairs = _decode_pairs(d, 512)
    for _ in range(args.warmup):
        oracle_decode_rate(d, pairs[:64])
    times, rates = [], []
    for _ in range(args.steps):
        r, desc, dt = oracle_decode_rate(d, pairs)
        times.append(dt)
        rates.append(r)
    value = float(statistics.mean(rates))
    return {
        "metric": DECODE_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * statistics.mean(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference", "config": decode_config(w, d),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": desc + " per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def run_decode(args, w, rank, world, local_rank):
    import numpy as np
    import torch

    from hierarchical_fenwick_state_b200 import binding
    from hierarchical_fenwick_state_b200 import inputs as I

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    binding.lib()
    d = I.make_decode_inputs(w, seed=rank_seed(args.seed, rank))
    B, H, L, dk, dv = d.B, d.H, d.L, d.dk, d.dv
    dt = torch.bfloat16 if d.dtype == "bf16" else torch.float32
    q = torch.from_numpy(d.q).to(dev).to(dt)
    k = torch.from_numpy(d.k).to(dev).to(dt)
    v = torch.from_numpy(d.v).to(dev).to(dt)
    la = torch.from_numpy(d.log_a).to(dev)
    lm = torch.from_numpy(d.lam).to(dev)
    pos = torch.from_numpy(d.pos).to(dev)
    nst = binding.decode_state_bytes(B, H, L, dk, dv) // 4
    state = torch.empty(nst, dtype=torch.float32, device=dev)
    nlev = B * H * (L - 1) * dk * dv
    # each level stored without its pending gate, the gate row of the position's parity set
    state[:nlev].view(B, H, L - 1, dk, dv).copy_(
        torch.from_numpy(d.states * np.exp(-d.pending)[..., None, None]).to(dev))
    gate = np.zeros((B, H, 2, L - 1), np.float32)
    gate[np.arange(B), :, d.pos & 1] = d.pending
    state[nlev:].copy_(torch.from_numpy(gate.reshape(-1)).to(dev))
    out = torch.empty((B, H, dv), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    # Re-running a step from the same positions reads the same slots and rewrites the same
    # carried slot and gate row with the same values, so every timed step does the full work.
    def step():
        binding.decode_step(q, k, v, la, lm, pos, state, out, B, H, L, dk, dv)

    dist = None
    if world > 1:
        import torch.distributed as dist
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    binding.profile_read(reset=True)
    clocks = ClockSampler(local_rank)
    clocks.start()
    binding.profile(True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    binding.profile(False)
    clk = clocks.stop()
    ms_total = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    main_ms, main_n, launches = binding.profile_read(reset=True)
    status = binding.device_status(clear=True)
    if status:
        raise RuntimeError(f"device status flags {status:#x} after the timed region")
    ms_step = ms_total / args.steps
    value = B * world / (ms_step / 1000.0)

    hbm_gbs, _, peak_kind = measured_peaks()
    abytes = decode_algorithmic_bytes(d)
    main_avg_s = (main_ms / main_n) / 1000.0 if main_n else ms_step / 1000.0
    kernel_key = f"decode:{w.name}"
    roof = {"bound": "hbm", "achieved": abytes / main_avg_s / 1e9, "peak": hbm_gbs,
            "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = ncu_traffic(kernel_key)
    roof["peak_source"] = f"{peak_kind} (MEASURED_PEAKS.json)" if peak_kind == "measured" \
        else "profiling-recipe fallback"
    roof["kernel"] = kernel_key
    roof["algorithmic_bytes_per_launch"] = abytes
    roof["main_kernel_ms"] = main_avg_s * 1000.0
    line = {
        "metric": DECODE_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if d.dtype == "bf16" else "f32", "data": "synthetic",
        "config": decode_config(w, d), "roofline": roof, "gpu_launches": launches,
        "clocks": clk,
    }

    if not args.no_e2e:
        # per step: this step's token inputs and positions up from pinned host memory, the step,
        # the outputs back; the level states stay on the device between steps
        if d.dtype == "bf16":
            hq = torch.from_numpy(I.bf16_bits(d.q).view(np.int16)).pin_memory()
            hk = torch.from_numpy(I.bf16_bits(d.k).view(np.int16)).pin_memory()
            hv = torch.from_numpy(I.bf16_bits(d.v).view(np.int16)).pin_memory()
        else:
            hq, hk, hv = (torch.from_numpy(x).pin_memory() for x in (d.q, d.k, d.v))
        hla = torch.from_numpy(d.log_a).pin_memory()
        hlm = torch.from_numpy(d.lam).pin_memory()
        hpos = torch.from_numpy(d.pos).pin_memory()
        hout = torch.empty((B, H, dv), dtype=torch.float32).pin_memory()
        dq, dk_, dv_ = (torch.empty(x.shape, dtype=x.dtype, device=dev) for x in (hq, hk, hv))
        dla, dlm, dpos = (torch.empty_like(x, device=dev) for x in (hla, hlm, hpos))
        h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hla, hlm, hpos))
        d2h = hout.numel() * 4

        def e2e_step():
            for dst, src in ((dq, hq), (dk_, hk), (dv_, hv), (dla, hla), (dlm, hlm), (dpos, hpos)):
                dst.copy_(src, non_blocking=True)
            binding.decode_step(dq, dk_, dv_, dla, dlm, dpos, state, out, B, H, L, dk, dv)
            hout.copy_(out, non_blocking=True)
            stream.synchronize()

        for _ in range(3):
            e2e_step()
        n_e2e = max(10, min(args.steps, 100))
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_s = max_over_ranks(e0.elapsed_time(e1) / 1000.0 / n_e2e, dist, dev)
        if not np.isfinite(hout.numpy()).all():
            raise RuntimeError("non-finite decoding output")
        line["e2e"] = {"value": B * world / e2e_s, "unit": "tokens/s",
                       "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                       "steps": n_e2e,
                       "entry": "llattn_decode_step, token inputs from pinned host memory"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, desc, _ = oracle_decode_rate(d, [(b, h) for b in range(B) for h in range(H)])
        line["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                "sample": desc}
    return line


# ---------------------------------------------------------------------------------------------
# backward pass
# ---------------------------------------------------------------------------------------------
BWD_METRIC = "log-linear attn bwd tokens/s at T=8K,H=32,d=64 (1×B200)"


def oracle_bwd_rate(inp, do, n_pairs):
    """Time the oracle's direct-sum gradients (dq, dk, dv, dlam rows and columns) on n_pairs
    (token, head) pairs; tokens/s of gradient rows = pairs / H / time."""
    import numpy as np
    import oracle as O
    try:
        from threadpoolctl import threadpool_limits
        ctx = threadpool_limits(limits=1)
    except Exception:  # noqa: BLE001
        ctx = None
    rng = np.random.default_rng(1)
    total = inp.total_tokens
    samples = list(zip(rng.integers(0, total, n_pairs).tolist(),
                       rng.integers(0, inp.H, n_pairs).tolist()))
    if ctx:
        ctx.__enter__()
    t0 = time.perf_counter()
    O.llattn_backward_sampled(inp, do, samples)
    dt = time.perf_counter() - t0
    if ctx:
        ctx.__exit__(None, None, None)
    desc = (f"fp64 oracle, direct sums of the dq, dk, dv and dlam rows of {n_pairs} sampled "
            f"(token, head) pairs (dlog_a not included), {dt:.2f} s, numpy single thread; "
            f"tokens/s = pairs / H / time")
    return (n_pairs / inp.H) / dt, desc, dt


def bwd_config(w, path):
    cfg = workload_config(w, None, path)
    cfg["pass"] = "bwd"
    cfg["inputs"] = f"{w.dtype} q/k/v/dout (dout ~ N(0,1)), f32 log_a/lam, f32 gradients"
    return cfg


def _bwd_do(inp, seed):
    import numpy as np
    from hierarchical_fenwick_state_b200 import inputs as I
    do = np.random.default_rng(seed + 1000).standard_normal(inp.v.shape).astype(np.float32)
    return I.round_to_bf16(do) if inp.dtype == "bf16" else do


def run_bwd_reference(args, w, rank, world):
    from hierarchical_fenwick_state_b200 import inputs as I
    if rank != 0:
        return None
    inp = I.make_inputs(w, seed=args.seed)
    do = _bwd_do(inp, args.seed)
    for _ in range(args.warmup):
        oracle_bwd_rate(inp, do, 32)
    times, rates = [], []
    for _ in range(args.steps):
        r, desc, dt = oracle_bwd_rate(inp, do, 256)
        times.append(dt)
        rates.append(r)
    value = float(statistics.mean(rates))
    return {
        "metric": BWD_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * statistics.mean(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference", "config": bwd_config(w, None),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": desc + " per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def run_bwd(args, w, rank, world, local_rank):
    import numpy as np
    import torch

    from hierarchical_fenwick_state_b200 import binding
    from hierarchical_fenwick_state_b200 import inputs as I

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    binding.lib()
    inp = I.make_inputs(w, seed=rank_seed(args.seed, rank))
    do = _bwd_do(inp, rank_seed(args.seed, rank))
    dt = torch.bfloat16 if inp.dtype == "bf16" else torch.float32
    names = ("q", "k", "v", "log_a", "lam")
    x = {n: torch.from_numpy(getattr(inp, n)).to(dev) for n in names}
    for n in ("q", "k", "v"):
        x[n] = x[n].to(dt)
    tdo = torch.from_numpy(do).to(dev).to(dt)
    cu = torch.from_numpy(inp.cu_seqlens).to(dev) if inp.cu_seqlens is not None else None
    grads = {n: torch.empty(getattr(inp, n).shape, dtype=torch.float32, device=dev) for n in names}
    nws = binding.bwd_workspace_bytes(inp.B, inp.H, inp.T, inp.dk, inp.dv)
    ws = torch.empty(max(nws, 256), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    lengths = [n for _, n in inp.seq_slices()]
    total_tokens = int(sum(lengths))

    def step():
        binding.backward(x["q"], x["k"], x["v"], x["log_a"], x["lam"], tdo, cu_seqlens=cu,
                         T=inp.T, grads=grads, workspace=ws)

    dist = None
    if world > 1:
        import torch.distributed as dist
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    # as for the forward: the call captured once as a CUDA graph and replayed (--graph off:
    # every call issued from Python)
    use_graph = args.graph != "off"
    graph = None
    if use_graph:
        binding.profile_read(reset=True)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, capture_error_mode="thread_local"):
            step()
        torch.cuda.synchronize()
        launches_per_step = binding.profile_read(reset=True)[2]
        for _ in range(max(args.warmup, 3)):
            graph.replay()
        torch.cuda.synchronize()
    binding.profile_read(reset=True)
    clocks = ClockSampler(local_rank)
    clocks.start()
    binding.profile(True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        if graph is not None:
            graph.replay()
        else:
            step()
    e1.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    binding.profile(False)
    clk = clocks.stop()
    ms_total = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    main_ms, main_n, launches = binding.profile_read(reset=True)
    if graph is not None:
        launches, main_n = launches_per_step * args.steps, 0   # the step's time is the call's
        del graph
    status = binding.device_status(clear=True)
    if status:
        raise RuntimeError(f"device status flags {status:#x} after the timed region")
    ms_step = ms_total / args.steps
    value = total_tokens * world / (ms_step / 1000.0)

    hbm_gbs, bf16_tflops, peak_kind = measured_peaks()
    abytes, aflops, per_tok = bwd_algorithmic(w, lengths)
    main_avg_s = (main_ms / main_n) / 1000.0 if main_n else ms_step / 1000.0
    kernel_key = f"bwd:{w.name}"
    peak_src = f"{peak_kind} (MEASURED_PEAKS.json)" if peak_kind == "measured" \
        else "profiling-recipe fallback"
    # bf16 at d = 64 runs every pair interaction on the tensor cores: its FLOPs count against
    # the bf16 tensor peak; the other shapes compute in fp32 on CUDA cores
    tensor = bwd_on_tensor_cores(inp)
    if tensor:
        cpeak, cunit, csrc = bf16_tflops, "TFLOP/s", peak_src + ", dense bf16 tensor"
    else:
        cpeak, cunit = alu_peak_tflops(), "TFLOP/s"
        csrc = "derived: 148 SMs x 128 fp32 lanes x 2 x 1965 MHz (fp32 FMA)"
    if aflops / (cpeak * 1e12) >= abytes / (hbm_gbs * 1e9):
        roof = {"bound": "tensor" if tensor else "alu", "achieved": aflops / main_avg_s / 1e12,
                "peak": cpeak, "unit": cunit, "peak_source": csrc}
    else:
        roof = {"bound": "hbm", "achieved": abytes / main_avg_s / 1e9, "peak": hbm_gbs,
                "unit": "GB/s", "peak_source": peak_src}
        roof["compute_frac"] = aflops / main_avg_s / 1e12 / cpeak
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = ncu_traffic(kernel_key)
    roof["kernel"] = kernel_key + " (all backward kernels of one call, one event pair)"
    roof["algorithmic_bytes_per_launch"] = abytes
    roof["algorithmic_flops_per_launch"] = aflops
    roof["hbm_frac"] = abytes / main_avg_s / 1e9 / hbm_gbs
    roof["bytes_per_token_head"] = per_tok
    roof["main_kernel_ms"] = main_avg_s * 1000.0
    line = {
        "metric": BWD_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if inp.dtype == "bf16" else "f32", "data": "synthetic",
        "config": {**bwd_config(w, "tensor cores: chunk pairs, then level by level" if tensor
                                else "simt level-by-level"),
                   **({"launch": "CUDA graph of one step, replayed"} if use_graph else {})},
        "roofline": roof, "gpu_launches": launches, "clocks": clk,
    }

    if not args.no_e2e:
        # inputs and the output gradient up from pinned host memory, the backward, all five
        # gradients back, every step
        hx = {}
        for n in names:
            a = getattr(inp, n)
            if n in ("q", "k", "v") and inp.dtype == "bf16":
                hx[n] = torch.from_numpy(I.bf16_bits(a).view(np.int16)).pin_memory()
            else:
                hx[n] = torch.from_numpy(a).pin_memory()
        hdo = (torch.from_numpy(I.bf16_bits(do).view(np.int16)) if inp.dtype == "bf16"
               else torch.from_numpy(do)).pin_memory()
        hg = {n: torch.empty(getattr(inp, n).shape, dtype=torch.float32).pin_memory()
              for n in names}
        dx = {n: torch.empty(hx[n].shape, dtype=hx[n].dtype, device=dev) for n in names}
        ddo = torch.empty(hdo.shape, dtype=hdo.dtype, device=dev)
        h2d = sum(t.numel() * t.element_size() for t in list(hx.values()) + [hdo])
        d2h = sum(t.numel() * 4 for t in hg.values())

        def e2e_step():
            for n in names:
                dx[n].copy_(hx[n], non_blocking=True)
            ddo.copy_(hdo, non_blocking=True)
            qv = {n: (dx[n].view(torch.bfloat16) if n in ("q", "k", "v") and inp.dtype == "bf16"
                      else dx[n]) for n in names}
            binding.backward(qv["q"], qv["k"], qv["v"], qv["log_a"], qv["lam"],
                             ddo.view(torch.bfloat16) if inp.dtype == "bf16" else ddo,
                             cu_seqlens=cu, T=inp.T, grads=grads, workspace=ws)
            for n in names:
                hg[n].copy_(grads[n], non_blocking=True)
            stream.synchronize()

        for _ in range(2):
            e2e_step()
        n_e2e = max(3, min(args.steps, 10))
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_s = max_over_ranks(e0.elapsed_time(e1) / 1000.0 / n_e2e, dist, dev)
        if not all(np.isfinite(hg[n].numpy()).all() for n in names):
            raise RuntimeError("non-finite gradients through the host copies")
        line["e2e"] = {"value": total_tokens * world / e2e_s, "unit": "tokens/s",
                       "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                       "steps": n_e2e, "entry": "llattn_bwd, inputs and gradients through pinned "
                                                "host memory"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, desc, _ = oracle_bwd_rate(inp, do, 1024)
        line["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                "sample": desc}
    return line


# ---------------------------------------------------------------------------------------------
# Log-Linear Gated DeltaNet forward
# ---------------------------------------------------------------------------------------------
GDN_METRIC = "log-linear gated deltanet fwd tokens/s (1×B200)"


def gdn_algorithmic(w, lengths):
    """Bytes: read q, k, v (input type), log_alpha, beta, lam (fp32); write out (fp32).  FLOPs of
    the recurrent form: at token t every occupied level l >= 1 (popcount(t) of them) takes the
    transition (k . s and the rank-1 update: 4 d_k d_v), the write is 2 d_k d_v, and each of the
    popcount(t) + 1 levels read out costs 2 d_k d_v."""
    esz = 2 if w.dtype == "bf16" else 4
    per = (2 * w.dk + w.dv) * esz + 4 + 4 + 4 * w.L + 4 * w.dv
    flops = 0
    for n in lengths:
        pc = sum(bin(t).count("1") for t in range(n))
        flops += (4 * pc + 2 * n + 2 * (pc + n)) * w.dk * w.dv
    return per * sum(lengths) * w.H, flops * w.H, per


def run_gdn(args, w, rank, world, local_rank):
    import numpy as np
    import torch

    from hierarchical_fenwick_state_b200 import binding
    from hierarchical_fenwick_state_b200 import inputs as I

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    binding.lib()
    inp = I.make_gdn_inputs(w, seed=rank_seed(args.seed, rank))
    dt = torch.bfloat16 if inp.dtype == "bf16" else torch.float32
    t = {n: torch.from_numpy(getattr(inp, n)).to(dev) for n in ("q", "k", "v", "log_a", "beta", "lam")}
    for n in ("q", "k", "v"):
        t[n] = t[n].to(dt)
    out = torch.empty(inp.v.shape, dtype=torch.float32, device=dev)
    lengths = [n for _, n in inp.seq_slices()]
    total_tokens = int(sum(lengths))
    stream = torch.cuda.current_stream()

    def step():
        binding.gdn_forward(t["q"], t["k"], t["v"], t["log_a"], t["beta"], t["lam"], out=out)

    dist = None
    if world > 1:
        import torch.distributed as dist
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    binding.profile_read(reset=True)
    clocks = ClockSampler(local_rank)
    clocks.start()
    binding.profile(True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    binding.profile(False)
    clk = clocks.stop()
    ms_total = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    main_ms, main_n, launches = binding.profile_read(reset=True)
    if binding.device_status(clear=True):
        raise RuntimeError("device status flags set after the timed region")
    ms_step = ms_total / args.steps
    value = total_tokens * world / (ms_step / 1000.0)
    hbm_gbs, _, peak_kind = measured_peaks()
    abytes, aflops, per_tok = gdn_algorithmic(w, lengths)
    main_avg_s = (main_ms / main_n) / 1000.0 if main_n else ms_step / 1000.0
    alu = alu_peak_tflops()
    if abytes / (hbm_gbs * 1e9) >= aflops / (alu * 1e12):
        roof = {"bound": "hbm", "achieved": abytes / main_avg_s / 1e9, "peak": hbm_gbs,
                "unit": "GB/s"}
    else:
        roof = {"bound": "alu", "achieved": aflops / main_avg_s / 1e12, "peak": alu,
                "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = None
    roof["peak_source"] = ("derived fp32 FMA peak: 148 SMs x 128 lanes x 2 x 1965 MHz"
                           if roof["bound"] == "alu" else
                           (f"{peak_kind} (MEASURED_PEAKS.json)" if peak_kind == "measured"
                            else "profiling-recipe fallback"))
    roof["kernel"] = f"gdn:{w.name}"
    roof["algorithmic_bytes_per_launch"] = abytes
    roof["algorithmic_flops_per_launch"] = aflops
    roof["main_kernel_ms"] = main_avg_s * 1000.0
    cfg = workload_config(w, None, "cuda cores (recurrent form)")
    cfg["beta"] = "sigmoid(N(0,1))"
    cfg["log_a"] = f"log alpha = -exp(N({w.log_a_mu},0.5))"
    line = {
        "metric": GDN_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if inp.dtype == "bf16" else "f32", "data": "synthetic", "config": cfg,
        "roofline": roof, "gpu_launches": launches, "clocks": clk,
    }
    if not args.no_e2e:
        # per step: inputs up from pinned host memory, the forward, out back
        if inp.dtype == "bf16":
            hs = {n: torch.from_numpy(I.bf16_bits(getattr(inp, n)).view(np.int16)).pin_memory()
                  for n in ("q", "k", "v")}
        else:
            hs = {n: torch.from_numpy(getattr(inp, n)).pin_memory() for n in ("q", "k", "v")}
        for n in ("log_a", "beta", "lam"):
            hs[n] = torch.from_numpy(getattr(inp, n)).pin_memory()
        hout = torch.empty(inp.v.shape, dtype=torch.float32).pin_memory()
        ds = {n: torch.empty(x.shape, dtype=x.dtype, device=dev) for n, x in hs.items()}
        h2d = sum(x.numel() * x.element_size() for x in hs.values())

        def e2e_step():
            for n in hs:
                ds[n].copy_(hs[n], non_blocking=True)
            qd, kd, vd = ((ds[n].view(torch.bfloat16) if inp.dtype == "bf16" else ds[n])
                          for n in ("q", "k", "v"))
            binding.gdn_forward(qd, kd, vd, ds["log_a"], ds["beta"], ds["lam"], out=out)
            hout.copy_(out, non_blocking=True)
            stream.synchronize()

        e2e_step()
        n_e2e = max(3, min(args.steps, 10))
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_s = max_over_ranks(e0.elapsed_time(e1) / 1000.0 / n_e2e, dist, dev)
        line["e2e"] = {"value": total_tokens * world / e2e_s, "unit": "tokens/s",
                       "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(hout.numel() * 4),
                       "steps": n_e2e, "entry": "llattn_gdn_fwd, inputs from pinned host memory"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle as O
        start, n = inp.seq_slices()[0]
        heads = min(inp.H, 4)
        sl = slice(start, start + n)
        q_ = inp.q.reshape(-1, inp.H, inp.dk)[sl, :heads].transpose(1, 0, 2)
        k_ = inp.k.reshape(-1, inp.H, inp.dk)[sl, :heads].transpose(1, 0, 2)
        v_ = inp.v.reshape(-1, inp.H, inp.dv)[sl, :heads].transpose(1, 0, 2)
        la_ = inp.log_a.reshape(-1, inp.H)[sl, :heads].T
        b_ = inp.beta.reshape(-1, inp.H)[sl, :heads].T
        lm_ = inp.lam.reshape(-1, inp.H, inp.L)[sl, :heads].transpose(1, 0, 2)
        t0 = time.perf_counter()
        O.gdn_recurrent_seq(q_, k_, v_, la_, b_, lm_)
        dts = time.perf_counter() - t0
        line["cpu_baseline"] = {
            "value": n * (heads / inp.H) / dts, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"recurrent fp64 Gated DeltaNet oracle, 1 sequence x {heads} of {inp.H} "
                      f"heads x {n} tokens batched, {dts:.2f} s, numpy", "host": _host_info()}
    return line


def run_gdn_reference(args, w, rank, world):
    """The Gated DeltaNet oracle (recurrent form) on the host: one sequence x 4 heads per step."""
    import numpy as np
    import oracle as O
    from hierarchical_fenwick_state_b200 import inputs as I
    if rank != 0:
        return None
    inp = I.make_gdn_inputs(w, seed=args.seed)
    start, n = inp.seq_slices()[0]
    heads = min(inp.H, 4)
    sl = slice(start, start + n)
    arrs = (inp.q.reshape(-1, inp.H, inp.dk)[sl, :heads].transpose(1, 0, 2),
            inp.k.reshape(-1, inp.H, inp.dk)[sl, :heads].transpose(1, 0, 2),
            inp.v.reshape(-1, inp.H, inp.dv)[sl, :heads].transpose(1, 0, 2),
            inp.log_a.reshape(-1, inp.H)[sl, :heads].T, inp.beta.reshape(-1, inp.H)[sl, :heads].T,
            inp.lam.reshape(-1, inp.H, inp.L)[sl, :heads].transpose(1, 0, 2))
    arrs = tuple(np.ascontiguousarray(a) for a in arrs)
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        O.gdn_recurrent_seq(*arrs)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    dt = statistics.mean(times)
    value = n * (heads / inp.H) / dt
    desc = (f"recurrent fp64 Gated DeltaNet oracle, 1 sequence x {heads} of {inp.H} heads x {n} "
            f"tokens batched, {dt:.2f} s per step, numpy")
    return {
        "metric": GDN_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * dt,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference", "config": workload_config(w, None, None),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": desc, "host": _host_info()},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    from hierarchical_fenwick_state_b200 import inputs as I
    decoding = args.workload in I.DECODE_WORKLOADS
    gdn = args.workload in I.GDN_WORKLOADS
    w = (I.DECODE_WORKLOADS if decoding else I.GDN_WORKLOADS if gdn else
         I.PROFILE_WORKLOADS if args.workload in I.PROFILE_WORKLOADS else I.WORKLOADS)[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if gdn:
            line = run_gdn_reference(args, w, rank, world)
        elif args.which == "bwd" and not decoding:
            line = run_bwd_reference(args, w, rank, world)
        else:
            line = (run_decode_reference if decoding else run_reference)(args, w, rank, world)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    if args.segment_chunks:
        from hierarchical_fenwick_state_b200 import binding
        binding.set_segment_chunks(args.segment_chunks)
    try:
        if gdn:
            line = run_gdn(args, w, rank, world, local_rank)
        elif args.which == "bwd" and not decoding:
            line = run_bwd(args, w, rank, world, local_rank)
        else:
            line = (run_decode if decoding else run_ours)(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""HeadQ decode benchmark on B200: cached tokens/s, HBM GB/s and roofline fraction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl headq|reference]
                    [--workload NAME]

One *step* is one serving decode step of one layer over a synthetic batch:
``headq_decode_append`` writes the step's new token of every (sequence, KV
head) into position T-1 (base code + side code, bit-exact with the cache
write) and attends over the T cached tokens (query projection, streaming the
packed cache, logits with the side-code correction, online softmax, value
readout and the split merge) -- one kernel on the tensor-core path.  The default workload is the long-context GQA layer (batch 1,
32 query heads over 8 KV heads, d=128, T=131072, r=16, 2-bit keys + 4-bit side
code + bf16 values), the bandwidth-bound case.  Calibration (one-off, offline)
and the KL diagnostic (needs the full-precision cache) are timed beside the
step and reported under "rows".

Timing: W untimed warm-up steps, then exactly K steps replayed from a CUDA
graph, bracketed by a barrier and a device synchronise, measured with CUDA
events on the launching stream; the maximum over ranks is reported.  Two
copies of the cache (2 x 348 MB > the 126 MB L2) alternate between steps, so
every step reads its cache from HBM.  ``e2e`` is the same step through the
public Python API with the step's inputs (query, new key/value) copied from
pinned host memory and the output read back to the host every step, the host
waiting for each step; the step (copies, decode, copy back) is captured once in
a CUDA graph per cache copy and replayed, as a serving loop runs it.

With --gpus N under torchrun every rank runs its own independent layer (weak
scaling, no collective on the data path).  ``--impl reference`` times the CPU
oracle on the host cores instead (rank 0 only).
"""

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from bit_decode_attention_sm_b200 import configs, synth  # noqa: E402

DEFAULT_WORKLOAD = configs.WORKLOADS[3].name
METRIC = "HeadQ decode-attn cached tokens/s and HBM GB/s (% of B200 peak), 1 GPU"
UNIT = "cached tokens/s"
FALLBACK_HBM_GBS = 6650.0


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["headq", "reference"], default="headq")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-rows", action="store_true", help="skip calibrate/write/kl rows")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the rows of the other workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args(argv)


# ---------------------------------------------------------------------------
# distributed plumbing (one process per GPU, NCCL; gloo in CPU tests)
# ---------------------------------------------------------------------------

def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def rank_seed(base_seed, rank):
    """Each rank decodes its own independent layer (weak scaling)."""
    return base_seed + 1000 * rank


def max_over_ranks(x, device=None):
    """Maximum of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------------------
# measurement helpers
# ---------------------------------------------------------------------------

def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def recorded_traffic(kernel_files, summary_file):
    """DRAM bytes per launch from a committed ncu summary, if the kernel source
    (the given files, concatenated) is still the one that was profiled (else None)."""
    try:
        if isinstance(kernel_files, str):
            kernel_files = [kernel_files]
        src = b"".join(open(os.path.join(ROOT, "bit_decode_attention_sm_b200", "csrc", f),
                            "rb").read() for f in kernel_files)
        sha = hashlib.sha256(src).hexdigest()
        fields = {}
        for line in open(os.path.join(ROOT, "profiles", summary_file)):
            if ":" in line and line.strip().startswith("- "):
                k, v = line.strip()[2:].split(":", 1)
                v = v.strip()
                if v.startswith("`"):
                    v = v[1:].split("`", 1)[0]
                else:
                    v = v.split()[0] if v else v
                fields[k.strip()] = v
        if fields.get("kernel_source_sha256") != sha:
            return None
        return float(fields["dram_bytes_per_launch"])
    except Exception:
        return None


def gpu_smi_id(ordinal):
    """nvidia-smi identifier (UUID) of CUDA device `ordinal` in this process."""
    import torch
    try:
        u = str(torch.cuda.get_device_properties(ordinal).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        return ids[ordinal] if ordinal < len(ids) else str(ordinal)


class ClockSampler:
    """nvidia-smi clock and throttle-reason samples while the GPU is busy."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]),
                                 power=float(parts[3]) if parts[3] not in ("", "[N/A]") else 0.0,
                                 hw=parts[5], hwt=parts[6], swt=parts[7], swp=parts[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        busy = [r for r in rows if r["power"] >= 0.5 * max(x["power"] for x in rows)] or rows
        reasons = set()
        for r in busy:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("swp", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in busy),
                "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(busy)}


# ---------------------------------------------------------------------------
# the CPU oracle, timed on the host cores (cpu_baseline / --impl reference)
# ---------------------------------------------------------------------------

def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def oracle_decode_rate(w, L, U, budget_s=12.0, max_T=None):
    """Cached tokens/s of the oracle's cache read on a bounded sample of the layer:
    the first T_s tokens of every (sequence, KV head), all query heads."""
    import oracle
    cores = oracle.set_threads(host_cores())
    T_full = L.keys.shape[2]
    max_T = T_full if max_T is None else min(max_T, T_full)
    T_s = min(256, max_T)

    def sample(Ts):
        k = L.keys[:, :, :Ts]
        v = L.values[:, :, :Ts]
        planes = oracle.cache_write(k, U, v=v, vmode=w.vmode)
        return planes, v

    planes, v = sample(T_s)
    t0 = time.perf_counter()
    oracle.decode(L.queries, planes, U, v=v, vmode=w.vmode)
    dt = time.perf_counter() - t0
    # grow the sample until one call takes about a third of the budget
    while T_s < max_T and dt < budget_s / 3:
        T_s = min(max_T, int(T_s * max(2.0, (budget_s / 3) / max(dt, 1e-3))))
        planes, v = sample(T_s)
        t0 = time.perf_counter()
        oracle.decode(L.queries, planes, U, v=v, vmode=w.vmode)
        dt = time.perf_counter() - t0
    reps, total = 1, dt
    while total < budget_s * 0.66:
        t0 = time.perf_counter()
        oracle.decode(L.queries, planes, U, v=v, vmode=w.vmode)
        total += time.perf_counter() - t0
        reps += 1
    B = L.keys.shape[0]
    return {"value": B * T_s * reps / total, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": "oracle cache read (fp64 attention from the exact fp32 codec) of the "
                      "first %d of %d tokens of every sequence and KV head, all %d query "
                      "heads, %d call(s), %.1f s" % (T_s, T_full, L.queries.shape[1], reps,
                                                      total)}


def _oracle_sample_timed(prepare, run, T_full, budget_s, T0=256):
    """Grow a token-prefix sample T_s until one run() takes about a third of
    budget_s, then repeat it until about two thirds of the budget is spent;
    prepare(T_s) sets up a sample size outside the timing.  Returns (T_s,
    calls, seconds)."""

    def once():
        t0 = time.perf_counter()
        run()
        return time.perf_counter() - t0

    T_s = min(T0, T_full)
    prepare(T_s)
    dt = once()
    while T_s < T_full and dt < budget_s / 3:
        T_s = min(T_full, int(T_s * max(2.0, (budget_s / 3) / max(dt, 1e-3))))
        prepare(T_s)
        dt = once()
    reps, total = 1, dt
    while total < budget_s * 0.66:
        total += once()
        reps += 1
    return T_s, reps, total


def oracle_op_rates(w, L, U, budget_s=4.0):
    """The oracle's cache write and KL diagnostic on the host cores, each on a
    bounded token-prefix sample of every (sequence, KV head): cached tokens/s
    (B * T_s per call, the decode metric's unit)."""
    import oracle
    cores = oracle.set_threads(host_cores())
    T_full = L.keys.shape[2]
    B = L.keys.shape[0]
    st = {}

    def prep_write(Ts):
        st["k"] = np.ascontiguousarray(L.keys[:, :, :Ts])
        st["v"] = np.ascontiguousarray(L.values[:, :, :Ts])

    def write():
        oracle.cache_write(st["k"], U, v=st["v"], vmode=w.vmode)

    T_s, reps, total = _oracle_sample_timed(prep_write, write, T_full, budget_s)
    out = {"cache_write": {
        "value": B * T_s * reps / total, "unit": UNIT, "cores": cores, "kind": "oracle",
        "sample": "oracle cache write (exact fp32 codec: base code, residual, projection, "
                  "side code%s) of the first %d of %d tokens of every sequence and KV head, "
                  "%d call(s), %.1f s" % (", 2-bit values" if w.vmode == "2bit" else "",
                                          T_s, T_full, reps, total)}}

    def prep_kl(Ts):
        prep_write(Ts)
        st["planes"] = oracle.cache_write(st["k"], U, v=st["v"], vmode=w.vmode)

    def kl():
        oracle.attn_kl(L.queries, st["planes"], U, st["k"], st["v"], v=st["v"], vmode=w.vmode)

    T_s, reps, total = _oracle_sample_timed(prep_kl, kl, T_full, budget_s)
    out["attn_kl"] = {
        "value": B * T_s * reps / total, "unit": UNIT, "cores": cores, "kind": "oracle",
        "sample": "oracle KL / Fisher / A^2 diagnostic (fp64) of the first %d of %d tokens of "
                  "every sequence and KV head, all %d query heads, %d call(s), %.1f s"
                  % (T_s, T_full, L.queries.shape[1], reps, total)}
    return out


def run_reference(args):
    """--impl reference: the oracle on the host cores, same metric and config."""
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    import oracle
    w = configs.workload(args.workload)
    L = synth.make_layer(w)
    U, _ = oracle.calibrate(L.q_cal, w.Hkv, w.r)
    cores = oracle.set_threads(host_cores())
    budget = max(1.0, 150.0 / max(1, args.steps + args.warmup))
    T_s = 256
    planes, v = None, None
    while True:
        planes = oracle.cache_write(L.keys[:, :, :T_s], U, v=L.values[:, :, :T_s],
                                    vmode=w.vmode)
        v = L.values[:, :, :T_s]
        t0 = time.perf_counter()
        oracle.decode(L.queries, planes, U, v=v, vmode=w.vmode)
        dt = time.perf_counter() - t0
        if dt >= budget / 2 or T_s >= w.T:
            break
        T_s = min(w.T, T_s * 2)
    for _ in range(args.warmup):
        oracle.decode(L.queries, planes, U, v=v, vmode=w.vmode)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.decode(L.queries, planes, U, v=v, vmode=w.vmode)
        times.append(time.perf_counter() - t0)
    ms = 1e3 * sum(times) / len(times)
    value = w.B * T_s / (ms / 1e3)
    sample = ("oracle cache read of the first %d of %d tokens of every sequence and KV head "
              "per step" % (T_s, w.T))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, note="CPU oracle; L2 not applicable"),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, note):
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "T": w.T,
            "r": w.r, "keys": "2-bit group-32 base code + %d x 4-bit side code" % w.r,
            "values": "bf16 dense" if w.vmode == "dense" else "2-bit group-32",
            "l2": note}


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------

def _events(torch):
    return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)


def run_headq(args):
    import torch
    import torch.distributed as dist
    from bit_decode_attention_sm_b200 import headq as hq

    rank, local_rank, world = dist_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    w = configs.workload(args.workload)
    L = synth.make_layer(w, seed=rank_seed(w.seed, rank))
    dt = torch.bfloat16 if w.kv_dtype == "bf16" else torch.float32
    B, Hq, Hkv, d, T = w.B, w.Hq, w.Hkv, w.d, w.T
    stream = torch.cuda.current_stream()

    # calibration on the GPU (row C1), then the full prefill write of both copies
    q_cal = torch.from_numpy(L.q_cal).to(dev).to(dt)
    U, _ = hq.headq_calibrate(q_cal, Hkv, w.r)
    k_all = torch.from_numpy(L.keys).to(dev).to(dt)
    v_all = torch.from_numpy(L.values).to(dev).to(dt)
    caches = []
    for _ in range(2):
        c = hq.HeadQCache(B, Hkv, T, d, w.r, vmode=w.vmode, v_dtype=dt, device=dev)
        hq.headq_cache_write(c, k_all, v_all, U)
        caches.append(c)
    q = torch.from_numpy(L.queries).to(dev).to(dt)
    k_new = k_all[:, :, T - 1].contiguous()   # [B, Hkv, d]: the step's new token
    v_new = v_all[:, :, T - 1].contiguous()
    out = torch.empty((B, Hq, d), dtype=torch.float32, device=dev)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    ws = hq.decode_workspace(caches[0], Hq, T)
    splits, chunk, n_dec, n_step = hq.decode_plan(caches[0], Hq, T)
    torch.cuda.synchronize()

    def step(c):
        # append the new token at position T-1 and attend over the T cached tokens
        hq.headq_decode_append(c, k_new, v_new, q, U, T=T, out=out, lse=lse, ws=ws)

    for i in range(max(args.warmup, 3)):
        step(caches[i % 2])
    torch.cuda.synchronize()
    hq.headq_workspace_status(ws)

    # capture one step per cache copy
    graphs = []
    use_graph = True
    try:
        for c in caches:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step(c)
            graphs.append(g)
        for g in graphs:
            g.replay()
        torch.cuda.synchronize()
    except Exception:
        use_graph = False
        graphs = []

    def run_step(i):
        if use_graph:
            graphs[i % 2].replay()
        else:
            step(caches[i % 2])

    sampler = ClockSampler(gpu_smi_id(local_rank))
    sampler.start()
    K = args.steps
    barrier(dev)
    torch.cuda.synchronize()
    e0, e1 = _events(torch)
    e0.record(stream)
    for i in range(K):
        run_step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(dev)
    ms_local = e0.elapsed_time(e1) / K
    # keep the same step running for a short soak so the clock record has samples
    t_end = time.time() + 1.5
    i = 0
    while time.time() < t_end:
        run_step(i)
        i += 1
        if i % 200 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = max_over_ranks(ms_local, dev)
    hq.headq_workspace_status(ws)

    # decode call alone, back to back from a graph, for the roofline
    dec_ms = None
    try:
        M = 20
        gd = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gd):
            for j in range(M):
                hq.headq_decode_attn(caches[j % 2], q, U, T=T, out=out, lse=lse, ws=ws)
        gd.replay()
        torch.cuda.synchronize()
        a, b_ = _events(torch)
        R = max(5, min(100, 2000 // M))
        a.record(stream)
        for _ in range(R):
            gd.replay()
        b_.record(stream)
        torch.cuda.synchronize()
        dec_ms = a.elapsed_time(b_) / (R * M)
        del gd
    except Exception:
        a, b_ = _events(torch)
        a.record(stream)
        for j in range(50):
            hq.headq_decode_attn(caches[j % 2], q, U, T=T, out=out, lse=lse, ws=ws)
        b_.record(stream)
        torch.cuda.synchronize()
        dec_ms = a.elapsed_time(b_) / 50
    dec_ms = max_over_ranks(dec_ms, dev)

    # end to end through the public API: pinned host inputs in, output out, every
    # step.  The step's inputs (query, new key, new value) sit in one pinned host
    # buffer and move in one copy, as a serving loop batches them; the device
    # tensors are views of one buffer (each 16-byte aligned).
    n_q, n_kv = q.numel(), k_new.numel()
    in_h = torch.empty(n_q + 2 * n_kv, dtype=dt).pin_memory()
    in_h[:n_q].copy_(torch.from_numpy(L.queries).to(dt).reshape(-1))
    in_h[n_q:n_q + n_kv].copy_(k_new.reshape(-1).cpu())
    in_h[n_q + n_kv:].copy_(v_new.reshape(-1).cpu())
    in_d = torch.empty_like(in_h, device=q.device)
    q_d = in_d[:n_q].view(q.shape)
    kn_d = in_d[n_q:n_q + n_kv].view(k_new.shape)
    vn_d = in_d[n_q + n_kv:].view(v_new.shape)
    out_h = torch.empty((B, Hq, d), dtype=torch.float32).pin_memory()

    def e2e_eager(c):
        in_d.copy_(in_h, non_blocking=True)
        hq.headq_decode_append(c, kn_d, vn_d, q_d, U, T=T, out=out, lse=lse, ws=ws)
        out_h.copy_(out, non_blocking=True)

    # a serving loop captures the step once (copies in, decode with append, copy
    # out) and replays it: every replay still moves the step's inputs from pinned
    # host memory and its output back, and the host waits for each step
    e2e_graphs = []
    if use_graph:
        try:
            for j in range(2):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    e2e_eager(caches[j])
                e2e_graphs.append(g)
            for g in e2e_graphs:
                g.replay()
            torch.cuda.synchronize()
        except Exception:
            e2e_graphs = []
    Ke = max(10, min(K, 200))
    barrier(dev)
    torch.cuda.synchronize()
    a, b_ = _events(torch)
    a.record(stream)
    for i in range(Ke):
        if e2e_graphs:
            e2e_graphs[i % 2].replay()
        else:
            e2e_eager(caches[i % 2])
        stream.synchronize()
    b_.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a.elapsed_time(b_) / Ke, dev)
    e2e_graph = bool(e2e_graphs)
    e2e_graphs.clear()
    h2d = in_h.numel() * in_h.element_size()
    d2h = out_h.numel() * out_h.element_size()

    # rows beside the step: calibration, the full prefill write, the KL diagnostic
    rows = None
    if not args.no_rows and rank == 0:
        with_cpu = world == 1 and not args.no_cpu_baseline
        rows = measure_rows(torch, hq, w, q_cal, k_all, v_all, q, U, caches[0], dt, stream, L,
                            with_cpu=with_cpu)
        if not args.no_workloads:
            rows["workloads"] = measure_workloads(torch, hq, stream, w.name, with_cpu)

    if world > 1:
        barrier(dev)
    bytes_tok = caches[0].nbytes_per_token()
    alg_bytes = B * Hkv * T * bytes_tok
    peak, peak_kind = measured_hbm_peak()
    achieved = alg_bytes / (dec_ms * 1e-3) / 1e9
    traffic = (recorded_traffic(["decode_mma.cu", "decode_pipe.cuh", "decode_common.cuh", "codec.cuh"],
                                "decode_mma_longctx.md")
               if w.name == DEFAULT_WORKLOAD else None)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        U_np = U.cpu().numpy()
        cpu = oracle_decode_rate(w, L, U_np)
    value = world * B * T / (ms * 1e-3)
    line = {
        "impl": "headq", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(w, note="inputs larger than L2: two 348 MB cache copies "
                                          "alternate between steps" if w.T == 131072 else
                                          "two cache copies alternate between steps"),
        "parallelism": "independent layer per rank" if world > 1 else "1 GPU",
        "hbm_gbs_per_step": world * alg_bytes / (ms * 1e-3) / 1e9,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": "headq_decode_attn, %d kernel(s), %d splits of %d tokens"
                               % (n_dec, splits, chunk),
                     "algorithmic_bytes_per_launch": alg_bytes,
                     "launch_ms": dec_ms, "peak_kind": peak_kind + " copy bandwidth"},
        "cpu_baseline": cpu,
        "e2e": {"value": world * B * T / (e2e_ms * 1e-3), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "cuda_graph": e2e_graph},
        "gpu_launches": K * n_step,
        "cuda_graph": use_graph,
        "clocks": clocks,
        "rows": rows,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    for c in caches:
        del c
    graphs.clear()
    if world > 1:
        dist.destroy_process_group()
    return 0


# fp64 FMA lanes per SM per clock on B200 (148 SMs, 1965 MHz max clock):
# 148 x 64 x 2 x 1.965e9 = 37.2 TFLOP/s, the published fp64 figure
FP64_FMA_PER_SM_CLK = 64


def fp64_peak_tflops(sm_count=148, mhz=1965.0):
    return sm_count * FP64_FMA_PER_SM_CLK * 2 * mhz * 1e6 / 1e12


PAGE_SIZE = 256
PLANE_ATTRS = ("k_codes", "k_scale", "k_min", "z_codes", "z_scale", "v", "v_codes", "v_scale",
               "v_min")


def paged_decode_row(torch, hq, w, q, U, cache, timed, hbm_row):
    """Decode over the same cache held as PAGE_SIZE-token pages of a pool in a
    shuffled order (block table a random permutation), timed like the
    contiguous layout beside it."""
    B, Hkv, T = w.B, w.Hkv, w.T
    if cache.T_cap % PAGE_SIZE:
        return None
    P = cache.T_cap // PAGE_SIZE
    gen = torch.Generator().manual_seed(0)
    table = torch.randperm(B * P, generator=gen).to(torch.int32).view(B, P)
    pc = hq.PagedHeadQCache(B, Hkv, w.d, w.r, PAGE_SIZE, B * P, P, vmode=cache.vmode,
                            v_dtype=cache.v_dtype, block_table=table)
    dst_idx = pc.block_table.reshape(-1).long()
    for name in PLANE_ATTRS:
        src = getattr(cache, name)
        if src is None:
            continue
        tail = tuple(src.shape[3:])
        pages = src.reshape((B, Hkv, P, PAGE_SIZE) + tail).transpose(1, 2)
        getattr(pc, name)[dst_idx] = pages.reshape((B * P, Hkv, PAGE_SIZE) + tail)
    ws_c = hq.decode_workspace(cache, w.Hq, T)
    ws_p = hq.decode_workspace(pc, w.Hq, T)
    out = torch.empty((B, w.Hq, w.d), dtype=torch.float32, device=q.device)
    lse = torch.empty((B, w.Hq), dtype=torch.float32, device=q.device)
    ms_c = timed(lambda: hq.headq_decode_attn(cache, q, U, T=T, out=out, lse=lse, ws=ws_c), 20)
    ms_p = timed(lambda: hq.headq_decode_attn(pc, q, U, T=T, out=out, lse=lse, ws=ws_p), 20)
    hq.headq_workspace_status(ws_p)
    splits, chunk, _, _ = hq.decode_plan(pc, w.Hq, T)
    row = hbm_row(ms_p, B * Hkv * T * cache.nbytes_per_token(), page_size=PAGE_SIZE,
                  contiguous_ms=ms_c, plan="%d splits of %d tokens" % (splits, chunk),
                  note="headq_decode_attn over a shuffled page pool; contiguous_ms is the "
                       "same call on the contiguous planes, timed the same way (CUDA graph "
                       "of 20 back-to-back calls)")
    del pc
    return row


CP_WORLD = 8


def cp_rank_row(torch, hq, w, q, U, cache, timed, hbm_row):
    """One rank of a CP_WORLD-way split-T decode of this workload: the local
    decode over its token range (the first range, as a cache holding T/CP_WORLD
    tokens) and the merge of CP_WORLD exchanged partials.  The all-gather
    between them crosses NVLink and is not part of this one-GPU measurement."""
    from bit_decode_attention_sm_b200 import context_parallel as cp
    B, Hq, d, T = w.B, w.Hq, w.d, w.T
    t_lo, n = cp.shard_range(T, 0, CP_WORLD)
    BH = B * Hq
    stride = cp.part_stride(BH, d)
    buf = torch.zeros(CP_WORLD * stride, dtype=torch.float32, device=q.device)
    o = buf[:BH * d].view(B, Hq, d)
    lse = buf[BH * d:BH * d + BH].view(B, Hq)
    ws = hq.decode_workspace(cache, Hq, n)
    hq.headq_decode_attn(cache, q, U, T=n, out=o, lse=lse, ws=ws)
    for r in range(1, CP_WORLD):  # stand-in partials for the other ranks
        buf[r * stride:(r + 1) * stride].copy_(buf[:stride])
    out = torch.empty((BH, d), dtype=torch.float32, device=q.device)
    lse_m = torch.empty(BH, dtype=torch.float32, device=q.device)
    ms_dec = timed(lambda: hq.headq_decode_attn(cache, q, U, T=n, out=o, lse=lse, ws=ws), 20)
    ms_merge = timed(lambda: hq.headq_merge_partials(buf, CP_WORLD, BH, d, stride, out=out,
                                                     lse=lse_m), 20)
    splits, chunk, _, _ = hq.decode_plan(cache, Hq, n)
    return hbm_row(ms_dec + ms_merge, B * w.Hkv * n * cache.nbytes_per_token(), world=CP_WORLD,
                   local_tokens=n, decode_ms=ms_dec, merge_ms=ms_merge,
                   exchange_bytes_per_rank=4 * stride,
                   plan="%d splits of %d tokens" % (splits, chunk),
                   note="rank-local work of a split-T step: decode over T/world tokens, "
                        "then headq_merge_partials, each from a CUDA graph of 20 calls; the "
                        "all-gather is not measured on one GPU")


A2_OBS = 16        # observation queries per sequence
A2_KEEP = 0.05     # fraction of each sequence's tokens whose values stay exact
def a2_policy_row(torch, hq, w, q, U, cache, k_all, v_all, dt, L, timed, gtimed, hbm_row):
    """The A^2 value policy on this workload: scores from A2_OBS observation
    queries per sequence (two logit passes, on tensor cores for bf16, plus the
    per-token value error; CUDA graph of 5 calls, against HBM), the top-K
    selection with the copy of the kept values, and the decode followed by the
    value fixup (against HBM, the cache plus the kept values)."""
    B, Hq, Hkv, d, T = w.B, w.Hq, w.Hkv, w.d, w.T
    qo = torch.from_numpy(synth.make_observation_queries(w, L, A2_OBS)).to(q.device).to(dt)
    K = max(1, int(A2_KEEP * T))
    ws = hq.a2_workspace(cache, A2_OBS, Hq, T)
    scores = torch.empty((B, Hkv, T), dtype=torch.float32, device=q.device)
    keep_idx = torch.empty((B, Hkv, K), dtype=torch.int32, device=q.device)
    keep_v = torch.empty((B, Hkv, K, d), dtype=dt, device=q.device)
    ms_sc = gtimed(lambda: hq.headq_a2_scores(cache, qo, k_all, v_all, ws=ws, out=scores),
                   reps=5, replays=3)
    ms_sel = timed(lambda: hq.headq_a2_select(scores, K, v_all, keep_idx=keep_idx, keep_v=keep_v), 5)
    hq.headq_workspace_status(ws)
    out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    dws = hq.decode_workspace(cache, Hq, T)

    def dec_fix():
        hq.headq_decode_attn(cache, q, U, T=T, out=out, lse=lse, ws=dws)
        hq.headq_a2_value_fixup(cache, q, U, keep_idx, keep_v, out, lse, T=T)

    ms_dec = gtimed(lambda: hq.headq_decode_attn(cache, q, U, T=T, out=out, lse=lse, ws=dws))
    ms_df = gtimed(dec_fix)
    # the scores must read the exact keys and values, the cached 2-bit value
    # planes, and write one score per token (the second pass's re-read of the
    # keys is not algorithmic)
    esz = k_all.element_size()
    sc_bytes = B * Hkv * T * (2 * d * esz + (d // 4 + 8 * (d // min(32, d))) + 4)
    sc_gbs = sc_bytes / (ms_sc * 1e-3) / 1e9
    keep_bytes = B * Hkv * K * (4 + d * keep_v.element_size())
    row = hbm_row(ms_df, B * Hkv * T * cache.nbytes_per_token() + keep_bytes, kept_per_seq=K,
                  observation_queries=A2_OBS, decode_ms=ms_dec, fixup_ms=ms_df - ms_dec,
                  select_ms=ms_sel, note="ms = decode + value fixup (CUDA graph of 20); "
                  "scores_roofline: the observation-logit passes (tensor cores for bf16)")
    row["scores_ms"] = ms_sc
    row["scores_roofline"] = dict(row["roofline"], achieved=sc_gbs,
                                  frac=sc_gbs / row["roofline"]["peak"], traffic=None,
                                  work="exact K and V, cached 2-bit value planes, scores")
    row["scores_algorithmic_bytes"] = sc_bytes
    return row


def channel_keys_row(torch, hq, w, q, U, k_all, v_all, dt, timed, gtimed, hbm_row):
    """The alternative base code (per-channel keys over 64-token blocks) on this
    workload: the prefill write and the tensor-core decode, each against HBM."""
    B, Hkv, T, d = w.B, w.Hkv, w.T, w.d
    if T % 64:
        return None
    c = hq.HeadQCache(B, Hkv, T, d, w.r, vmode=w.vmode, v_dtype=dt, device=q.device,
                      kmode="channel")
    ms_w = timed(lambda: hq.headq_cache_write(c, k_all, v_all, U), 3)
    ws = hq.decode_workspace(c, w.Hq, T)
    out = torch.empty((B, w.Hq, d), dtype=torch.float32, device=q.device)
    lse = torch.empty((B, w.Hq), dtype=torch.float32, device=q.device)
    ms_d = gtimed(lambda: hq.headq_decode_attn(c, q, U, T=T, out=out, lse=lse, ws=ws), reps=5,
                  replays=3)
    tok = B * Hkv * T
    planes = tok * c.nbytes_per_token()
    row = hbm_row(ms_d, planes, write_ms=ms_w, bytes_per_token=c.nbytes_per_token(),
                  note="ms: headq_decode_attn (tensor-core kernel) on the per-channel code; "
                       "write_roofline: the prefill write")
    gbs = (tok * d * 2 * k_all.element_size() + planes) / (ms_w * 1e-3) / 1e9
    row["write_roofline"] = dict(row["roofline"], achieved=gbs, frac=gbs / row["roofline"]["peak"])
    del c
    return row


class Timing:
    """CUDA-event timing on one stream, and rows against the HBM roofline."""

    def __init__(self, torch, stream):
        self.torch, self.stream = torch, stream
        self.peak, self.peak_kind = measured_hbm_peak()
        self.l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
        self._flush = None

    def timed(self, fn, reps):
        """Mean time of reps back-to-back calls (after one untimed call)."""
        torch = self.torch
        fn()
        torch.cuda.synchronize()
        a, b = _events(torch)
        a.record(self.stream)
        for _ in range(reps):
            fn()
        b.record(self.stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    def gtimed(self, fn, reps=20, replays=10):
        """Per-call time of fn from a CUDA graph of `reps` back-to-back calls
        (no host launch cost between them); plain calls if capture fails."""
        torch = self.torch
        try:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for _ in range(reps):
                    fn()
            g.replay()
            torch.cuda.synchronize()
            a, b = _events(torch)
            a.record(self.stream)
            for _ in range(replays):
                g.replay()
            b.record(self.stream)
            torch.cuda.synchronize()
            del g
            return a.elapsed_time(b) / (replays * reps)
        except Exception:
            return self.timed(fn, reps)

    def flushed(self, fn, reps=20):
        """Mean time of single calls, each after the L2 is flushed (a buffer of
        twice the L2 size written between the calls, outside the timing)."""
        torch = self.torch
        if self._flush is None:
            self._flush = torch.empty(2 * self.l2, dtype=torch.uint8, device="cuda")
        fn()
        total = 0.0
        for _ in range(reps):
            self._flush.zero_()
            a, b = _events(torch)
            a.record(self.stream)
            fn()
            b.record(self.stream)
            torch.cuda.synchronize()
            total += a.elapsed_time(b)
        return total / reps

    def hbm_row(self, ms, nbytes, **extra):
        gbs = nbytes / (ms * 1e-3) / 1e9
        return dict(ms=ms, algorithmic_bytes=nbytes,
                    roofline={"bound": "hbm", "achieved": gbs, "peak": self.peak,
                              "unit": "GB/s", "frac": gbs / self.peak,
                              "peak_kind": self.peak_kind + " copy bandwidth"},
                    **extra)


def measure_rows(torch, hq, w, q_cal, k_all, v_all, q, U, cache, dt, stream, L,
                 with_cpu=False):
    """The other rows of the path, timed with CUDA events, each against its roofline:
    the prefill cache write and the KL diagnostic against HBM bandwidth (bytes they
    must move), calibration against the fp64 ALU peak (its Gram matrix FLOPs); with
    with_cpu, the oracle's cache write and diagnostic on the host cores beside them."""
    rows = {}
    tm = Timing(torch, stream)
    timed, gtimed, hbm_row = tm.timed, tm.gtimed, tm.hbm_row
    B, Hkv, T, d = w.B, w.Hkv, w.T, w.d
    tok = B * Hkv * T
    kv_in = tok * d * 2 * k_all.element_size()          # the bf16 K and V read
    planes = tok * cache.nbytes_per_token()              # the packed cache
    # inputs larger than L2; CUDA graphs of back-to-back calls, as for the decode
    ms = gtimed(lambda: hq.headq_cache_write(cache, k_all, v_all, U), reps=5, replays=3)
    rows["cache_write_prefill"] = hbm_row(ms, kv_in + planes, tokens=B * T,
                                          note="reads K,V and writes every plane (CUDA graph "
                                               "of 5 calls)")
    ws = hq.attn_kl_workspace(cache, w.Hq, T)
    ms = gtimed(lambda: hq.headq_attn_kl(cache, q, U, k_all, v_all, ws=ws), reps=5, replays=3)
    rows["attn_kl"] = hbm_row(ms, kv_in + planes, note="reads the packed cache and full K,V "
                                                       "(CUDA graph of 5 calls)")
    if with_cpu:
        cpu = oracle_op_rates(w, L, U.cpu().numpy())
        rows["cache_write_prefill"]["cpu_baseline"] = cpu["cache_write"]
        rows["attn_kl"]["cpu_baseline"] = cpu["attn_kl"]
    rows["decode_paged"] = paged_decode_row(torch, hq, w, q, U, cache, gtimed, hbm_row)
    rows["context_parallel_rank"] = cp_rank_row(torch, hq, w, q, U, cache, gtimed, hbm_row)
    rows["channel_keys"] = channel_keys_row(torch, hq, w, q, U, k_all, v_all, dt, timed, gtimed,
                                            hbm_row)
    if w.vmode == "2bit":  # the policy chooses which 2-bit values to keep exact
        rows["a2_policy"] = a2_policy_row(torch, hq, w, q, U, cache, k_all, v_all, dt, L, timed,
                                          gtimed, hbm_row)
    ms = timed(lambda: hq.headq_calibrate(q_cal, Hkv, w.r), 3)
    M = q_cal.shape[0] * w.G
    flops = 2.0 * Hkv * M * d * d
    pk = fp64_peak_tflops(torch.cuda.get_device_properties(0).multi_processor_count)
    tf = flops / (ms * 1e-3) / 1e12
    rows["calibrate"] = dict(ms=ms, queries=int(q_cal.shape[0]),
                             roofline={"bound": "alu", "achieved": tf, "peak": pk,
                                       "unit": "TFLOP/s", "frac": tf / pk,
                                       "peak_kind": "fp64 from unit counts and max clock",
                                       "work": "Gram matrix, 2*Hkv*N*G*d^2 flops"})
    return rows


COPIES_MAX = 16  # cache copies rotated to keep a small cache's reads out of L2


def workload_rows(torch, hq, w, stream, with_cpu):
    """Every row of the path on one more workload: the serving step and the
    decode call (HBM roofline: the packed cache), the prefill cache write and
    the KL diagnostic (HBM roofline: K and V read, every plane written or read),
    the A^2 value policy on 2-bit-value workloads, and with with_cpu the
    oracle's decode, cache write and diagnostic on the host cores.  The decode
    rotates cache copies whose total exceeds twice the L2 (at least two, at
    most COPIES_MAX) in a CUDA graph; a cache too small for that is timed call
    by call with the L2 flushed before each call."""
    tm = Timing(torch, stream)
    L = synth.make_layer(w)
    dt = torch.bfloat16 if w.kv_dtype == "bf16" else torch.float32
    B, Hq, Hkv, d, T = w.B, w.Hq, w.Hkv, w.d, w.T
    q_cal = torch.from_numpy(L.q_cal).cuda().to(dt)
    U, _ = hq.headq_calibrate(q_cal, Hkv, w.r)
    k_all = torch.from_numpy(L.keys).cuda().to(dt)
    v_all = torch.from_numpy(L.values).cuda().to(dt)
    q = torch.from_numpy(L.queries).cuda().to(dt)
    k_new = k_all[:, :, T - 1].contiguous()
    v_new = v_all[:, :, T - 1].contiguous()
    c0 = hq.HeadQCache(B, Hkv, T, d, w.r, vmode=w.vmode, v_dtype=dt)
    hq.headq_cache_write(c0, k_all, v_all, U)
    tok = B * Hkv * T
    planes = tok * c0.nbytes_per_token()
    kv_in = tok * d * 2 * k_all.element_size()
    ncopies = max(2, -(-2 * tm.l2 // planes))
    big = ncopies <= COPIES_MAX
    caches = [c0]
    for _ in range(ncopies - 1 if big else 0):
        c1 = hq.HeadQCache(B, Hkv, T, d, w.r, vmode=w.vmode, v_dtype=dt)
        hq.headq_cache_write(c1, k_all, v_all, U)
        caches.append(c1)
    out = torch.empty((B, Hq, d), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    ws = hq.decode_workspace(c0, Hq, T)
    splits, chunk, n_dec, n_step = hq.decode_plan(c0, Hq, T)
    ctr = [0]

    def alternating(call):
        def fn():
            call(caches[ctr[0] % len(caches)])
            ctr[0] += 1
        return fn

    dec = alternating(lambda c: hq.headq_decode_attn(c, q, U, T=T, out=out, lse=lse, ws=ws))
    stp = alternating(lambda c: hq.headq_decode_append(c, k_new, v_new, q, U, T=T, out=out,
                                                        lse=lse, ws=ws))
    if big:
        dec_ms, step_ms = tm.gtimed(dec, reps=max(20, 2 * ncopies)), tm.gtimed(stp, reps=max(20, 2 * ncopies))
        l2 = ("%d cache copies (%.0f MB in all, more than twice the L2) rotate, CUDA graph of "
              "%d calls" % (ncopies, ncopies * planes / 1e6, max(20, 2 * ncopies)))
    else:
        dec_ms, step_ms = tm.flushed(dec), tm.flushed(stp)
        l2 = "cache smaller than L2: L2 flushed before each timed call"
    hq.headq_workspace_status(ws)
    row = tm.hbm_row(dec_ms, planes, value=B * T / (step_ms * 1e-3), unit=UNIT,
                     step_ms=step_ms, bytes_per_token_kv_head=c0.nbytes_per_token(),
                     plan="%d splits of %d tokens, %d kernel(s) per decode call"
                          % (splits, chunk, n_dec), l2=l2,
                     note="ms / roofline: headq_decode_attn; value: cached tokens/s of the "
                          "serving step (headq_decode_append)")
    ops = {}
    wr = lambda: hq.headq_cache_write(c0, k_all, v_all, U)
    ms_w = tm.gtimed(wr, reps=5, replays=3) if kv_in + planes > 2 * tm.l2 else tm.flushed(wr)
    ops["cache_write_prefill"] = tm.hbm_row(ms_w, kv_in + planes, tokens_per_sequence=T,
                                            note="prefill of every sequence: reads K,V and "
                                                 "writes every plane")
    kws = hq.attn_kl_workspace(c0, Hq, T)
    kl = lambda: hq.headq_attn_kl(c0, q, U, k_all, v_all, ws=kws)
    ms_k = tm.gtimed(kl, reps=5, replays=3) if kv_in + planes > 2 * tm.l2 else tm.flushed(kl, 5)
    ops["attn_kl"] = tm.hbm_row(ms_k, kv_in + planes,
                                note="reads the packed cache and full K,V")
    if w.vmode == "2bit":
        ops["a2_policy"] = a2_policy_row(torch, hq, w, q, U, c0, k_all, v_all, dt, L, tm.timed,
                                         tm.gtimed, tm.hbm_row)
    if with_cpu:
        U_np = U.cpu().numpy()
        row["cpu_baseline"] = oracle_decode_rate(w, L, U_np, budget_s=4.0)
        cpu = oracle_op_rates(w, L, U_np)
        ops["cache_write_prefill"]["cpu_baseline"] = cpu["cache_write"]
        ops["attn_kl"]["cpu_baseline"] = cpu["attn_kl"]
    row.update(ops)
    del caches, c0
    return row


def measure_workloads(torch, hq, stream, skip, with_cpu):
    """workload_rows for every workload but `skip` (the headline's own)."""
    res = {}
    for w in configs.WORKLOADS:
        if w.name == skip:
            continue
        try:
            res[w.name] = workload_rows(torch, hq, w, stream, with_cpu)
        except Exception as e:  # reported in the line, never silently dropped
            res[w.name] = {"error": "%s: %s" % (type(e).__name__, e)}
        torch.cuda.empty_cache()
    return res


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_headq(args)


if __name__ == "__main__":
    sys.exit(main())

"""Benchmark: BasisKV routed decode attention over a compressed paged KV cache.

One step = one ``basiskv_decode_attn`` call (routing scores + top-k, exact QK
on the selected pages, softmax, latent sum, combine and B_v) for every
(sequence, KV head) of the workload, inputs resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--keys int8]
    python bench.py --impl reference ...     # the float64 CPU oracle arm

``--keys int8`` stores the original keys as int8 codes with a per-token scale
(quantised on the device before timing) instead of bf16.

Prints one JSON line (rank 0).  Multi-GPU: one process per GPU under
torchrun; every rank runs its own replica of the workload (no collective on
the data path: the units are independent), weak scaling.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "compressed-KV decode attn context-tokens/s; HBM GB/s vs ~8 TB/s peak (1 B200)"
UNIT = "context-tokens/s"
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama3_8b_decode")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (smaller profiling cases)")
    ap.add_argument("--keys", choices=["native", "int8"], default="native",
                    help="int8: keys as int8 codes with a per-token scale")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="skip the long-context, high-concurrency and dense-limit lines")
    ap.add_argument("--per-workload-steps", type=int, default=300)
    ap.add_argument("--cpu-budget-s", type=float, default=15.0)
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(world, backend):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Largest value of x over all ranks (the slowest rank sets the time)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def replica_spec(spec, rank: int):
    """Rank r of a multi-GPU run processes its own replica of the workload
    (weak scaling): same shapes, its own seed."""
    return spec.with_(seed=spec.seed + 1000 * rank) if rank else spec


def aggregate(tokens_per_rank: int, ms_per_step: float, world: int, device=None):
    """Whole-job throughput: every rank's tokens over the slowest rank's step
    time.  Returns (value, max ms per step)."""
    ms_max = max_over_ranks(ms_per_step, world, device)
    return tokens_per_rank * world / (ms_max * 1e-3), ms_max


def workload_config(args, w, world):
    """The workload part of the JSON line's config, the same for both arms."""
    s = w.spec
    int8 = getattr(args, "keys", "native") == "int8"
    name = args.workload if not args.batch else f"{args.workload}[batch={s.batch}]"
    return {"workload": name + ("+int8_keys" if int8 else ""),
            "keys": "int8 codes + fp32 scale per token" if int8 else s.dtype,
            "batch": s.batch, "kv_heads": s.num_kv_heads, "q_heads": s.num_q_heads, "head_dim": s.head_dim,
            "page": s.page_size, "rank_r": s.rank_r, "rank_s": s.rank_s, "topk": s.topk,
            "context_tokens": w.context_tokens, "algorithmic_bytes": w.algorithmic_bytes(int8)["total"],
            "parallelism": f"replicas x{world}, no data-path collective"}


def peaks():
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed loop runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                self.out = ""

    def summary(self):
        rows = []
        for line in (self.out or "").strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, fl in rows for i, v in enumerate(fl) if v == "Active"})
        return {"sm_mhz": float(np.median([r[0] for r in rows])), "sm_max_mhz": rows[0][1],
                "reasons": reasons, "samples": len(rows)}


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch recorded by an ncu capture of this kernel, if the
    capture matches the current kernel source (profiles/traffic.json)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        e = rec.get(f"{kernel}:{workload}")
        if not e:
            return None
        import hashlib
        h = hashlib.sha256()
        for fn in sorted(e["sources"]):
            with open(os.path.join(ROOT, fn), "rb") as f:
                h.update(f.read())
        return float(e["dram_bytes_per_launch"]) if h.hexdigest() == e["sources_sha256"] else None
    except Exception:
        return None


def oracle_problem(w, int8_keys=False):
    """Host copies of a workload's stored tensors for the oracle; with
    int8_keys, the keys quantised by the oracle's own quantiser."""
    import torch
    from oracle import oracle
    s = w.spec
    bf16 = s.dtype == "bf16"

    def host(t):
        t = t.detach().cpu().contiguous()
        return t.view(torch.int16).numpy() if bf16 else t.numpy()

    k = host(w.k_pool)
    k_scale = None
    if int8_keys:
        codes = np.empty(k.shape, np.int8)
        k_scale = np.empty(k.shape[:3], np.float32)
        for i in range(0, k.shape[0], 256):  # slot chunks bound the float temporaries
            kf = (k[i:i + 256].view(np.uint16).astype(np.uint32) << 16).view(np.float32) if bf16 \
                else k[i:i + 256]
            codes[i:i + 256], k_scale[i:i + 256] = oracle.quantize_keys(kf)
        k = codes
    return oracle.Problem(
        q=host(w.q), z_pool=host(w.z_pool), r_pool=host(w.r_pool), k_pool=k,
        w_zk=w.w_zk.cpu().numpy(), b_r=w.b_r.cpu().numpy(), b_v=w.b_v.cpu().numpy(),
        page_table=np.where(w.page_table >= 0, w.page_table, 0).astype(np.int32),
        seq_lens=w.seq_lens, gqa_group=s.gqa_group, topk=s.topk, softmax_scale=s.softmax_scale,
        dtype=oracle.BF16 if bf16 else oracle.F32, k_scale=k_scale)


def cpu_oracle_timing(prob, w, budget_s: float):
    """Time the oracle on a bounded sample of units: grow the sample until it
    costs about budget_s of wall time.  Returns (tokens/s, cores, sample text)."""
    from oracle import oracle
    s = w.spec
    U = s.batch * s.num_kv_heads
    cores = oracle.max_threads()
    order = np.random.default_rng(0).permutation(U)
    done, spent, tokens = 0, 0.0, 0.0
    n = max(1, min(U, cores))
    while done < U and spent < budget_s:
        units = order[done:done + n].tolist()
        t0 = time.perf_counter()
        oracle.decode(prob, units=units)
        spent += time.perf_counter() - t0
        tokens += sum(float(w.seq_lens[u // s.num_kv_heads]) / s.num_kv_heads for u in units)
        done += len(units)
        n = min(U - done, n * 2)
    sample = (f"{done} of {U} (sequence, KV head) units of {s.name}, {cores} OpenMP threads, "
              f"{spent:.1f} s; tokens counted as L_b/Hkv per unit")
    return tokens / spent, cores, sample


def run_reference(args, rank, world):
    """The oracle arm: the float64 CPU oracle on this workload, each step a
    bounded sample (one unit, its sequence cut to fit the time budget)."""
    if rank != 0:
        return 0
    import torch
    from compressed_kv_cache_routing_b200 import workloads as W
    from oracle import oracle
    spec = W.SPECS[args.workload]
    if args.batch:
        spec = spec.with_(batch=args.batch)
    w = W.generate(spec, device="cuda" if torch.cuda.is_available() else "cpu")
    prob = oracle_problem(w, args.keys == "int8")
    cores = oracle.max_threads()
    # per-step sample: unit 0 on every thread, sequence cut so the whole run
    # stays near two minutes
    total_steps = args.steps + args.warmup
    L0 = int(w.seq_lens[0])
    per_step_budget = 120.0 / max(1, total_steps)
    units = list(range(min(cores, spec.num_kv_heads)))
    probe = oracle.Problem(**{**prob.__dict__, "seq_lens": np.array([min(L0, spec.page_size * 8)] +
                                                                   [0] * (spec.batch - 1), np.int32)})
    t0 = time.perf_counter()
    oracle.decode(probe, units=units)
    t_probe = max(time.perf_counter() - t0, 1e-4)
    L = int(min(L0, max(spec.page_size, spec.page_size * 8 * per_step_budget / t_probe)))
    lens = np.zeros(spec.batch, np.int32)
    lens[0] = L
    step_prob = oracle.Problem(**{**prob.__dict__, "seq_lens": lens})
    for _ in range(args.warmup):
        oracle.decode(step_prob, units=units)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.decode(step_prob, units=units)
        times.append(time.perf_counter() - t0)
    ms = 1e3 * float(np.mean(times))
    tokens = L * len(units) / spec.num_kv_heads
    value = tokens / (ms * 1e-3)
    sample = (f"sequence 0 cut to {L} tokens, KV heads {units}, {cores} OpenMP threads per step "
              f"(tokens counted as L/Hkv per (sequence, KV head))")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {**workload_config(args, w, world),
                       "l2": "host run; the oracle reads host memory",
                       "timing": "host wall clock around each step, mean of K steps"},
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def aux_measurements(kv, w, stream, dev, int8_codes=None):
    """Device time of the write-side entry points, after the timed region:
    basiskv_encode_rows for one page of P tokens of every KV head (a prefill
    chunk) and for one token, into the last pool slot; basiskv_encode_tokens
    for one token of every sequence (the decode-time append) into the last
    slots;
    with int8 keys, basiskv_quantize_keys over the whole key pool.  CUDA
    events around 20 calls each, after one untimed call (the first encode
    call computes the bases' pseudo-inverses on the host)."""
    import torch
    from compressed_kv_cache_routing_b200 import basiskv as bk
    s = w.spec
    g = torch.Generator(device=dev).manual_seed(99)
    dt = w.k_pool.dtype
    slot = int(w.k_pool.shape[0]) - 1

    def timed(fn, n=20):
        fn()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / n * 1e3  # us per call

    out = {}
    for name, rows in (("encode_rows_page", s.page_size), ("encode_rows_token", 1)):
        k = torch.randn((s.num_kv_heads, rows, s.head_dim), generator=g, device=dev).to(dt)
        v = torch.randn((s.num_kv_heads, rows, s.head_dim), generator=g, device=dev).to(dt)
        us = timed(lambda: bk.basiskv_encode_rows(kv.handle, slot, 0, k, v, stream=stream))
        out[name] = {"us_per_call": us, "rows_per_call": rows * s.num_kv_heads,
                     "rows_per_s": rows * s.num_kv_heads / (us * 1e-6)}
    # the decode-time append: one new token per sequence, one launch
    nb = s.batch
    slots = torch.arange(slot, slot - nb, -1, device=dev, dtype=torch.int32).clamp_(min=0)
    rows = torch.zeros(nb, device=dev, dtype=torch.int32)
    k = torch.randn((nb, s.num_kv_heads, s.head_dim), generator=g, device=dev).to(dt)
    v = torch.randn((nb, s.num_kv_heads, s.head_dim), generator=g, device=dev).to(dt)
    us = timed(lambda: bk.basiskv_encode_tokens(kv.handle, slots, rows, k, v, stream=stream))
    out["encode_tokens_batch"] = {"us_per_call": us, "rows_per_call": nb * s.num_kv_heads,
                                  "rows_per_s": nb * s.num_kv_heads / (us * 1e-6)}
    if int8_codes is not None:
        nbytes = w.k_pool.numel() * w.k_pool.element_size() + int8_codes.numel() + 4 * int8_codes.numel() // s.head_dim
        us = timed(lambda: bk.basiskv_quantize_keys(kv.handle, w.k_pool, stream=stream), n=5)
        out["quantize_keys_pool"] = {"us_per_call": us, "rows": int8_codes.numel() // s.head_dim,
                                     "gb_per_s": nbytes / (us * 1e-6) / 1e9,
                                     "bytes": int(nbytes)}
    if bk.basiskv_get_status(kv.handle, clear=True):
        raise SystemExit("device status error in the write-side measurements")
    return out


def make_handle(w, int8, dev):
    """A library handle over w's pools; with int8, the keys quantised on the
    device into int8 codes and per-token scales first.  Returns (handle
    object, codes or None)."""
    import torch
    from compressed_kv_cache_routing_b200 import basiskv as bk
    if not int8:
        return bk.BasisKV.for_workload(w), None
    codes = torch.empty(tuple(w.k_pool.shape), dtype=torch.int8, device=dev)
    k_scale = torch.empty(tuple(w.k_pool.shape[:3]), dtype=torch.float32, device=dev)
    kv = bk.BasisKV(z_pool=w.z_pool, r_pool=w.r_pool, k_pool=codes, w_zk=w.w_zk, b_r=w.b_r, b_v=w.b_v,
                    gqa_group=w.spec.gqa_group, max_batch=w.spec.batch,
                    max_pages_per_seq=max(1, w.page_table.shape[1]), max_topk=w.spec.topk, k_scale=k_scale)
    bk.basiskv_quantize_keys(kv.handle, w.k_pool)
    bk.basiskv_load_page_table(kv.handle, np.where(w.page_table >= 0, w.page_table, 0), w.seq_lens)
    torch.cuda.synchronize(dev)
    return kv, codes


class L2Flush:
    """Between steps: write a buffer of twice the L2 size, then read another
    one of the same size.  The write evicts the workload's lines; the read
    evicts the written (dirty) lines, so their write-back to HBM happens here,
    outside the timed region, and the next step starts with an L2 holding only
    clean lines of neither."""

    def __init__(self, dev):
        import torch
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        self.wbuf = torch.empty(2 * l2 // 4 + 1, device=dev, dtype=torch.float32)
        self.rbuf = torch.zeros(2 * l2 // 4 + 1, device=dev, dtype=torch.float32)
        self.sink = torch.empty((), device=dev, dtype=torch.float32)

    def __call__(self):
        import torch
        self.wbuf.zero_()
        torch.sum(self.rbuf, dim=0, out=self.sink)


def measure_workload(name, int8, dev, local, steps, warmup):
    """Another workload in the same process and with the same protocol as the
    main line (L2 flushed between steps, a CUDA event pair around each call,
    clock samples during the timed loop, per-grid events in a second loop)."""
    import torch
    from compressed_kv_cache_routing_b200 import basiskv as bk
    from compressed_kv_cache_routing_b200 import workloads as W
    w = W.generate(name, device=dev)
    kv, codes = make_handle(w, int8, dev)
    s = w.spec
    out = torch.empty((s.batch, s.num_q_heads, s.head_dim), device=dev, dtype=torch.float32)
    sel = torch.empty((s.batch, s.num_kv_heads, s.topk), device=dev, dtype=torch.int32)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        bk.basiskv_decode_attn(kv.handle, w.q, s.topk, s.softmax_scale, out, sel, stream=stream)

    for _ in range(max(3, warmup)):
        flush()
        step()
    torch.cuda.synchronize(dev)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    with ClockSampler(local) as clk:
        time.sleep(0.3)
        torch.cuda.synchronize(dev)
        for k in range(steps):
            flush()
            starts[k].record(stream)
            step()
            ends[k].record(stream)
        torch.cuda.synchronize(dev)
    step_ms = np.array([a.elapsed_time(b) for a, b in zip(starts, ends)])
    bk.basiskv_profile_begin(kv.handle, steps)
    for _ in range(steps):
        flush()
        step()
    torch.cuda.synchronize(dev)
    prof = bk.basiskv_profile_end(kv.handle, steps)
    status = bk.basiskv_get_status(kv.handle, clear=True)
    launch = bk.basiskv_last_launch(kv.handle)
    kv.close()
    ms = float(np.mean(step_ms))
    nbytes = w.algorithmic_bytes(int8)["total"]
    hbm_peak, peak_kind = peaks()
    gbs = nbytes / (ms * 1e-3) / 1e9
    res = {"ms_per_step": ms, "step_ms_p10_p50_p90": [float(np.percentile(step_ms, q)) for q in (10, 50, 90)],
           "value": w.context_tokens / (ms * 1e-3), "unit": UNIT, "context_tokens": w.context_tokens,
           "algorithmic_bytes": nbytes, "achieved_gbs": gbs, "frac_of_measured": gbs / hbm_peak,
           "frac_of_8tbs": gbs / 8000.0, "peak_kind": peak_kind, "steps": steps,
           "kernels_ms": {k: float(np.mean(v)) for k, v in prof.items()},
           "launch": launch, "clocks": clk.summary(), "device_status": status,
           "config": {"batch": s.batch, "page": s.page_size, "rank_r": s.rank_r, "rank_s": s.rank_s,
                      "topk": s.topk, "keys": "int8" if int8 else s.dtype}}
    del w, codes, out, sel, flush
    torch.cuda.empty_cache()
    return res


def run_ours(args, rank, world, local):
    import torch
    from compressed_kv_cache_routing_b200 import basiskv as bk
    from compressed_kv_cache_routing_b200 import build
    from compressed_kv_cache_routing_b200 import workloads as W

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    build.build()
    spec = W.SPECS[args.workload]
    if args.batch:
        spec = spec.with_(batch=args.batch)
    spec = replica_spec(spec, rank)
    w = W.generate(spec, device=dev)
    int8 = args.keys == "int8"
    kv, codes = make_handle(w, int8, dev)
    s = w.spec
    out = torch.empty((s.batch, s.num_q_heads, s.head_dim), device=dev, dtype=torch.float32)
    sel = torch.empty((s.batch, s.num_kv_heads, s.topk), device=dev, dtype=torch.int32)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        bk.basiskv_decode_attn(kv.handle, w.q, s.topk, s.softmax_scale, out, sel, stream=stream)

    for _ in range(max(3, args.warmup)):
        flush()
        step()
    torch.cuda.synchronize(dev)
    if bk.basiskv_get_status(kv.handle, clear=True):
        raise SystemExit("device status error during warm-up")

    K = args.steps
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    with ClockSampler(local) as clk:
        time.sleep(0.3)  # let the sampler start before the timed loop
        # timed region: K steps, a CUDA event pair around each whole call on
        # the launching stream (the L2 flush between steps stays outside)
        barrier(world, dev)
        torch.cuda.synchronize(dev)
        wall0 = time.perf_counter()
        for k in range(K):
            flush()
            starts[k].record(stream)
            step()
            ends[k].record(stream)
        torch.cuda.synchronize(dev)
        wall = time.perf_counter() - wall0
        barrier(world, dev)
        step_ms = np.array([a.elapsed_time(b) for a, b in zip(starts, ends)])
        # per-grid times: a second K-step loop with the library's events
        # between its grids (those events keep the grids from overlapping)
        bk.basiskv_profile_begin(kv.handle, K)
        for _ in range(K):
            flush()
            step()
        torch.cuda.synchronize(dev)
        prof = bk.basiskv_profile_end(kv.handle, K)
    clocks = clk.summary()
    status = bk.basiskv_get_status(kv.handle, clear=True)
    launch = bk.basiskv_last_launch(kv.handle)

    ms_step = float(np.mean(step_ms))
    tokens = w.context_tokens
    value, ms_step_max = aggregate(tokens, ms_step, world, dev)
    nbytes = w.algorithmic_bytes(int8)
    hbm_peak, peak_kind = peaks()
    route_mean = float(np.mean(prof["route"])) if launch["route_ctas"] else 0.0
    attn_mean = float(np.mean(prof["attn"]))
    if route_mean > 0 and nbytes["route"] >= nbytes["attn"]:
        dom_bytes, dom_ms = nbytes["route"], route_mean
        kname = "route_mma_kernel" if launch["route_tensor_core"] else "route_generic_kernel"
    else:
        dom_bytes, dom_ms = nbytes["attn"], attn_mean
        kname = ("attn_coop_kernel" if launch["attn_shared_ring"] else "attn_mma_kernel") \
            if launch["attn_tensor_core"] else "attn_generic_kernel"
    # routing (+ its selection grid on the tensor-core path), attention, prep past 512 sequences
    launches_per_step = (1 + launch["route_tensor_core"] if launch["route_ctas"] else 0) + 1 + \
        (1 if s.batch > 512 else 0)
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
    traffic = ncu_traffic(kname, args.workload + ("+int8_keys" if int8 and kname.startswith("attn") else ""))

    # end to end through the host-buffer entry point: q in, out (+ selection) back
    q_host = w.q.cpu().pin_memory()
    out_host = torch.empty(out.shape, dtype=torch.float32).pin_memory()
    sel_host = torch.empty(sel.shape, dtype=torch.int32).pin_memory()
    for _ in range(3):
        bk.basiskv_decode_attn_host(kv.handle, q_host, s.topk, s.softmax_scale, out_host, sel_host,
                                    stream=stream)
    e2e_steps = max(5, min(K, 50))
    e2e_times = []
    for _ in range(e2e_steps):
        flush()
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        bk.basiskv_decode_attn_host(kv.handle, q_host, s.topk, s.softmax_scale, out_host, sel_host,
                                    stream=stream)
        e2e_times.append(time.perf_counter() - t0)
    e2e_s = max_over_ranks(float(np.mean(e2e_times)), world, dev)
    h2d = q_host.numel() * q_host.element_size()
    d2h = out_host.numel() * 4 + sel_host.numel() * 4
    aux = aux_measurements(kv, w, stream, dev, codes if int8 else None)

    # the other workloads of the same family, same protocol (one GPU only)
    per_workload = None
    if world == 1 and not args.batch and not args.no_per_workload and args.workload == "llama3_8b_decode":
        per_workload = {name: measure_workload(name, int8, dev, local, min(K, args.per_workload_steps), args.warmup)
                        for name in ("long_context", "high_concurrency", "dense_limit")}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        prob = oracle_problem(w, int8)
        v, cores, sample = cpu_oracle_timing(prob, w, args.cpu_budget_s)
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_step_max, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": s.dtype, "data": "synthetic",
            "config": {**workload_config(args, w, world),
                       "l2": "flushed between steps, outside the per-step events: a 2x L2 buffer written, then another read (its dirty lines written back before the step)",
                       "timing": "CUDA event pair around each call on the launching stream, mean of K steps"},
            "hbm": {"achieved_gbs": nbytes["total"] / (ms_step_max * 1e-3) / 1e9, "peak_gbs": hbm_peak,
                    "frac": nbytes["total"] / (ms_step_max * 1e-3) / 1e9 / hbm_peak,
                    "frac_of_8tbs": nbytes["total"] / (ms_step_max * 1e-3) / 8e12, "peak_kind": peak_kind},
            "roofline": {"bound": "hbm", "kernel": kname, "achieved": achieved, "peak": hbm_peak,
                         "unit": "GB/s", "frac": achieved / hbm_peak, "traffic": traffic,
                         "algorithmic_bytes_per_launch": dom_bytes, "launch_ms": dom_ms,
                         "launch_ms_from": "per-grid CUDA events (second K-step loop)",
                         "peak_kind": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"},
            "kernels_ms": {k: float(np.mean(v)) for k, v in prof.items()},
            "kernels_ms_note": "second K-step loop, events between grids (no PDL overlap there)",
            "step_ms_p10_p50_p90": [float(np.percentile(step_ms, q)) for q in (10, 50, 90)],
            "launch": launch,
            "gpu_launches": K * launches_per_step,
            "e2e": {"value": tokens * world / e2e_s, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_s * 1e3,
                    "how": "basiskv_decode_attn_host: pinned q H2D, decode writing out+sel into pinned host memory, stream sync; host wall clock"},
            "wall_ms_per_step_incl_flush": wall * 1e3 / K,
            "clocks": clocks,
            "device_status": status,
            "cpu_baseline": cpu,
            "aux": aux,
            "per_workload": per_workload,
        }
        print(json.dumps(line), flush=True)
    kv.close()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    rank, world, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, rank, world)
    return run_ours(args, rank, world, local)


if __name__ == "__main__":
    sys.exit(main())

#!/usr/bin/env python
"""AB-Attention hot-path benchmark on B200.

One step = one pass of the whole path over one synthetic layer:
abattn_plan (mean keys -> k-means -> scores -> water-fill + Poisson
sampling + compaction) followed by the gathered sparse forward (the plan is
used by `forwards_per_plan` forwards: 1 for the 14B-like layer, 4 for the
HunyuanVideo-like one).  The metric is the executed tensor-core TFLOP/s of
the sparse forward over the step time; the forward alone, every kernel's
time, the in-house dense kernel and the CPU oracle are reported beside it.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
        [--workload wan14b-720p|wan1.3b-480p|hunyuan-720p|sweep-75k|tiny]
For N > 1 launch under torchrun: every rank runs its own full layer (weak
scaling, no data-path collective; each (b, h, q-block) row is independent).
"""
from __future__ import annotations

import argparse
import concurrent.futures
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from block_sparse_attention_12_b200 import inputs, multigpu  # noqa: E402

METRIC = "AB-Attn fwd ms & executed TFLOPS (% bf16 TC peak), 75.6K tok × 40 heads"
UNIT = "TFLOP/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="wan14b-720p", choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--heads", type=int, default=0,
                    help="run only this many heads of the layer (small cases for ncu captures)")
    ap.add_argument("--e2e-steps", type=int, default=16)
    ap.add_argument("--dense-iters", type=int, default=3)
    ap.add_argument("--cpu-rows", type=int, default=64)
    ap.add_argument("--cpu-rows-one-core", type=int, default=12)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--denoise", action="store_true",
                    help="synthetic denoising loop: dense warm-up steps and first block, a plan every 4 steps")
    ap.add_argument("--denoise-steps", type=int, default=50)
    ap.add_argument("--denoise-layers", type=int, default=2)
    ap.add_argument("--model-layers", type=int, default=40)
    ap.add_argument("--strong", action="store_true",
                    help="one layer's heads sharded over the ranks (head_offset plans, all-gather of O)")
    ap.add_argument("--gather-bench", action="store_true",
                    help="microbenchmark of the sparse forward's gather: cp.async, 4-row TMA boxes, TMA gather4")
    ap.add_argument("--e4m3", action="store_true",
                    help="the E4M3 forward beside the bf16 forward on the same plan (ms, TFLOP/s, error)")
    ap.add_argument("--mma-bench", action="store_true",
                    help="tensor-core rate microbenchmark (cycles per MMA by operand source and N)")
    ap.add_argument("--sweep", action="store_true",
                    help="budget x kv_block x (SIP, top-k) sweep on the sweep-75k layer, one JSON line per point")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=p["hbm_gbs"], bf16=p["bf16_tflops"], bf16_sus=p["bf16_tflops_sustained"],
                    sm_mhz=p.get("sm_max_mhz", 1965.0), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, sm_mhz=1965.0, src="fallback")


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        sel = []
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            pass
        try:
            self.p = subprocess.Popen(["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "50"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        try:
            self.p.wait(5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.count(",") >= 7]
        os.unlink(self.f.name)
        sm, mx, pw, reasons = [], None, [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[0]))
                mx = float(r[1])
                pw.append(float(r[2]))
            except ValueError:
                continue
            for n, v in zip(names, r[4:8]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        loaded = [s for s, p in zip(sm, pw) if p > 0.3 * max(pw)] if pw else sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- oracle leg
def oracle_sample(w, n_rows: int, seed_offset: int = 0, n_heads: int = 4):
    """A bounded seeded sample of rows of the workload: n_rows q-blocks spread
    over n_heads heads, plus those heads' Q, K, V as float64 (drawn and
    converted outside any timed region)."""
    import oracle
    g = np.random.default_rng(4321 + seed_offset)
    nqb = math.ceil(w.N / 128)
    flat_heads = g.choice(w.B * w.H, size=min(n_heads, w.B * w.H), replace=False)
    heads = [divmod(int(x), w.H) for x in flat_heads]
    rows = []
    for i in range(n_rows):
        b, h = heads[i % len(heads)]
        rows.append((b, h, int(g.integers(nqb))))
    data = {bh: tuple(oracle.f64(t) for t in inputs.make_head(w, bh[0], bh[1])) for bh in heads}
    return rows, data


def executed_flops_row(n_sel: int, kb: int, d: int) -> float:
    return 4.0 * 128 * 128 * d * math.ceil(n_sel * kb / 128)


def run_oracle_rows(w, rows, data, threads: int):
    """Plan + forward of the listed rows with the CPU oracle; returns
    (seconds, executed-equivalent FLOPs)."""
    import oracle
    oracle.set_num_threads(1)
    t0 = time.perf_counter()
    kbars = {}

    def kbar(bh):
        if bh not in kbars:
            kbars[bh] = oracle.meanpool(data[bh][1], w.kv_block)
        return kbars[bh]

    for bh in {(b, h) for b, h, _ in rows}:
        kbar(bh)
    f64 = data

    def one(r):
        b, h, qb = r
        q, k, v = f64[(b, h)]
        out = oracle.plan_forward_row(q, k, v, kbars[(b, h)], b, h, qb, w.kv_block, w.budget, w.seed,
                                      w.n_clusters, w.kmeans_iters)
        flops = executed_flops_row(out["idx"].size, w.kv_block, w.d) * w.forwards_per_plan
        if w.forwards_per_plan > 1:  # the extra forwards reuse the plan
            for _ in range(w.forwards_per_plan - 1):
                oracle.sparse_block(q[qb * 128:qb * 128 + 128], k, v, w.kv_block, out["idx"], out["pi_sel"],
                                    1 / math.sqrt(w.d))
        return flops

    with concurrent.futures.ThreadPoolExecutor(threads) as ex:
        flops = sum(ex.map(one, rows))
    return time.perf_counter() - t0, flops


def cpu_baseline(w, n_rows: int, n_rows_one: int):
    """The oracle on a bounded seeded sample of the workload's rows, on all
    host cores and on one core.  Rows are independent and their work is
    proportional to their selected blocks, so the whole layer's time is
    extrapolated linearly from each sample (reported as such)."""
    threads = os.cpu_count() or 1
    total_rows = w.B * w.H * math.ceil(w.N / 128)
    rows, data = oracle_sample(w, n_rows)
    secs, flops = run_oracle_rows(w, rows, data, threads)
    rows1, data1 = oracle_sample(w, n_rows_one, seed_offset=1)
    secs1, flops1 = run_oracle_rows(w, rows1, data1, 1)
    return {"value": flops / secs / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{len(rows)} (head, q-block) rows of {w.name} (of {total_rows}), "
                      f"k-means + scores + water-fill + sampling + gathered forward in fp64, "
                      f"{secs:.2f} s wall on {threads} threads",
            "one_core": {"value": flops1 / secs1 / 1e12, "unit": UNIT, "cores": 1,
                         "sample": f"{len(rows1)} rows, {secs1:.2f} s on 1 thread"},
            "extrapolated_layer_ms": {"all_cores": 1e3 * secs * total_rows / len(rows),
                                      "one_core": 1e3 * secs1 * total_rows / len(rows1),
                                      "how": "extrapolated: sample time x (layer rows / sampled rows)"}}


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    threads = os.cpu_count() or 1
    rows_per_step = max(threads, 16)
    samples = [oracle_sample(w, rows_per_step, seed_offset=s) for s in range(args.warmup + args.steps)]
    for s in range(args.warmup):
        run_oracle_rows(w, *samples[s], threads)
    tot_s, tot_f = 0.0, 0.0
    for s in range(args.warmup, args.warmup + args.steps):
        sec, fl = run_oracle_rows(w, *samples[s], threads)
        tot_s += sec
        tot_f += fl
    value = tot_f / tot_s / 1e12
    line = {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_s / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": w.name, "tokens": w.N, "heads": w.H, "d": w.d,
                                           "kv_block": w.kv_block, "budget": w.budget},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": f"each step: {rows_per_step} seeded (head, q-block) rows of {w.name}, "
                                       f"plan + gathered forward in fp64"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU leg
def source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_sparse_attention_12_b200", "csrc")
    for n in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, units: float):
    """DRAM bytes per launch from the committed ncu summary, scaled to this
    launch's units, if it was captured from the current sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    e = t.get(kernel)
    if not e or e.get("source_hash") != source_hash():
        return None
    return e["bytes_per_unit"] * units


def timed(fn, iters, stream):
    # two untimed calls first: the caching allocator then holds every buffer
    # the call allocates, so no cudaMalloc lands inside the timed loop
    fn()
    fn()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(iters):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / iters


def run_strong(args):
    """Strong scaling of one layer: rank r holds heads head_shard(H, r, N),
    plans them with head_offset = the slice's first head (so the plan equals
    those rows of the one-GPU plan) and runs the forward; a step ends with the
    all-gather of O over NCCL.  Timing as in the default mode (barrier and
    synchronize around K steps, max over ranks); value = the layer's executed
    TFLOP per step over that time."""
    from block_sparse_attention_12_b200 import abi, build
    build.build()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    w = inputs.WORKLOADS[args.workload]
    hs = multigpu.head_shard(w.H, rank, world)
    Q, K, V = inputs.make_qkv_heads(w, hs, device=f"cuda:{local}")
    shape = tuple(Q.shape)
    cfg = abi.Config(kv_block=w.kv_block, budget=w.budget, n_clusters=w.n_clusters,
                     kmeans_iters=w.kmeans_iters, seed=w.seed, head_offset=hs.start)
    planner = abi.Planner(shape, cfg)
    O = torch.empty_like(Q)
    stream = torch.cuda.current_stream()

    def step():
        plan = planner(Q, K)
        abi.forward(Q, K, V, plan, cfg, O=O, want_lse=False)
        return multigpu.gather_heads(O, w.H, world)

    for _ in range(max(args.warmup, 3)):
        step()
    abi.check()
    fl = torch.tensor([abi.executed_flops(planner.plan, shape)], dtype=torch.float64, device=Q.device)
    if dist:
        dist.all_reduce(fl)  # the layer's executed FLOP: the ranks' shards summed
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    ms = multigpu.max_over_ranks(e0.elapsed_time(e1) / args.steps, Q.device)
    abi.check()
    if rank == 0:
        print(json.dumps({
            "metric": METRIC, "value": float(fl.item()) / (ms / 1e3) / 1e12, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "tokens": w.N, "heads": w.H, "heads_per_rank": len(hs),
                       "kv_block": w.kv_block, "budget": w.budget,
                       "step": "abattn_plan + abattn_forward on the rank's heads + all-gather of O",
                       "parallelism": f"heads sharded over {world} GPUs"},
        }), flush=True)
    if dist:
        dist.destroy_process_group()


def run_denoise(args):
    """One JSON line: the denoising-loop policy (first 10 of 50 steps and the
    first block dense, a plan every 4 steps) over `--denoise-layers` synthetic
    layers of the workload whose activations drift between steps; attention
    time per step measured with CUDA events, per-call times solved from it,
    and the same policy extrapolated to `--model-layers` blocks."""
    from block_sparse_attention_12_b200 import build, denoise
    build.build()
    w = inputs.WORKLOADS[args.workload]
    if args.heads:
        import dataclasses
        w = dataclasses.replace(w, H=args.heads, name=f"{w.name}-{args.heads}heads")
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    pol = denoise.Policy(steps=args.denoise_steps)
    res = denoise.run(w, pol, layers=args.denoise_layers)
    dense_ms, sparse_ms, plan_ms = denoise.per_call_ms(pol, res, args.denoise_layers)
    out = denoise.summary(w, pol, res, args.denoise_layers, dense_ms, sparse_ms, plan_ms, args.model_layers)
    out["data"] = "synthetic (seeded base + seeded drift per step)"
    print(json.dumps(out))


def run_sweep(args):
    """Budget 5/8/11/25/50/100% x kv_block 4/128 x (SIP, top-k) on the
    75,600-token x 10-head layer: plan and forward time, executed TFLOP/s,
    relative-L2 error of O against the in-house dense kernel, and the ratio
    of the sparse to the dense softmax normaliser (top-k: the retained
    attention mass; SIP: about 1, the Horvitz-Thompson normaliser being
    unbiased)."""
    from block_sparse_attention_12_b200 import abi, build
    build.build()
    torch.cuda.set_device(0)
    w = inputs.SWEEP
    Q, K, V = inputs.make_qkv(w, device="cuda")
    shape = tuple(Q.shape)
    stream = torch.cuda.current_stream()
    Od = torch.empty_like(Q)
    _, lse_d = abi.dense_forward(Q, K, V, O=Od)
    dense_ms = timed(lambda: abi.dense_forward(Q, K, V, O=Od, want_lse=False), 3, stream)
    dfl = 4.0 * w.B * w.H * w.N * w.N * w.d
    print(json.dumps({"sweep": "dense", "workload": w.name, "ms": dense_ms, "tflops": dfl / dense_ms / 1e9}), flush=True)
    O = torch.empty_like(Q)
    lse = torch.empty(shape[:3], dtype=torch.float32, device="cuda")
    odn = Od.float().norm()
    for kb in (4, 128):
        for budget in (0.05, 0.08, 0.11, 0.25, 0.5, 1.0):
            for mode in (abi.MODE_SIP, abi.MODE_TOPK):
                cfg = abi.Config(kv_block=kb, budget=budget, mode=mode, seed=w.seed)
                planner = abi.Planner(shape, cfg)
                plan = planner(Q, K)
                abi.forward(Q, K, V, plan, cfg, O=O, lse=lse)
                abi.check()
                plan_ms = timed(lambda: planner(Q, K), 3, stream)
                fwd_ms = timed(lambda: abi.forward(Q, K, V, plan, cfg, O=O, lse=lse), 5, stream)
                abi.check()
                efl = abi.executed_flops(plan, shape)
                err = float((O.float() - Od.float()).norm() / odn)
                ratio = torch.exp(lse.double() - lse_d.double())
                nkvb = -(-w.N // kb)
                print(json.dumps({
                    "sweep": "point", "workload": w.name, "kv_block": kb, "budget": budget,
                    "mode": "SIP" if mode == abi.MODE_SIP else "TOPK",
                    "selected_blocks_mean": float(plan.counts.float().mean()), "nkvb": nkvb,
                    "plan_ms": plan_ms, "fwd_ms": fwd_ms, "executed_tflops": efl / fwd_ms / 1e9,
                    "fwd_vs_dense_speedup": dense_ms / fwd_ms, "rel_l2_vs_dense": err,
                    "normaliser_ratio_mean": float(ratio.mean()), "normaliser_ratio_p05": float(ratio.quantile(0.05)) if ratio.numel() < 2**24 else None,
                }), flush=True)
                del planner, plan
                torch.cuda.empty_cache()


def run_e4m3(args):
    """The E4M3 forward (QK^T in 8-bit floats, per-block scales) beside the
    bf16 forward on the same plan of the benchmark's layer: forward ms and
    executed TFLOP/s of both (CUDA events, inputs larger than L2), the
    quantisation of Q and K, and the E4M3 output's rel-L2 against the bf16
    forward's.  One JSON line."""
    import dataclasses
    from block_sparse_attention_12_b200 import abi, build
    build.build()
    torch.cuda.set_device(0)
    w = inputs.WORKLOADS[args.workload]
    if args.heads:
        w = dataclasses.replace(w, H=args.heads)
    Q, K, V = inputs.make_qkv(w, device="cuda:0")
    cfg = abi.Config(kv_block=w.kv_block, budget=w.budget, n_clusters=w.n_clusters,
                     kmeans_iters=w.kmeans_iters, seed=w.seed)
    stream = torch.cuda.current_stream()
    plan = abi.plan(Q, K, cfg)
    O, lse = abi.forward(Q, K, V, plan, cfg)
    Q8, qs = abi.quantize_e4m3(Q, 128)
    K8, ks = abi.quantize_e4m3(K, w.kv_block)
    O8, lse8 = abi.forward_e4m3(Q8, qs, K8, ks, V, plan, cfg)
    abi.check()
    n_it = max(3, args.steps)
    t_bf = timed(lambda: abi.forward(Q, K, V, plan, cfg, O=O, lse=lse), n_it, stream)
    t_q = timed(lambda: (abi.quantize_e4m3(Q, 128, codes=Q8, scales=qs),
                         abi.quantize_e4m3(K, w.kv_block, codes=K8, scales=ks)), n_it, stream)
    t_8 = timed(lambda: abi.forward_e4m3(Q8, qs, K8, ks, V, plan, cfg, O=O8, lse=lse8), n_it, stream)
    abi.check()
    fl = abi.executed_flops(plan, tuple(Q.shape))
    d = O8.float() - O.float()
    print(json.dumps({
        "e4m3_forward": w.name, "heads": w.H, "tokens": w.N,
        "bf16_forward_ms": t_bf, "bf16_forward_tflops": fl / (t_bf / 1e3) / 1e12,
        "e4m3_forward_ms": t_8, "e4m3_forward_tflops": fl / (t_8 / 1e3) / 1e12,
        "quantize_q_and_k_ms": t_q,
        "e4m3_vs_bf16_output_rel_l2": float(d.norm() / O.float().norm()),
        "note": "QK^T in E4M3 (Q scaled per 128-query block, K per KV block); P and V bf16",
    }), flush=True)


def run_gather_bench(args):
    """Cycles per 128-key tile to gather the 32 selected 4-row blocks of K and
    V (64 KB) into a 3-stage shared-memory ring, for each copy method and
    number of issuing warps; one CTA per SM, blocks spread over two heads of
    75,600 tokens (K and V L2-resident, as in the forward's head-major order).
    One JSON line per configuration; the microbenchmark also checks the last
    tile's bytes against global memory."""
    import ctypes
    from block_sparse_attention_12_b200 import build
    lib = ctypes.CDLL(build.build_gatherbench())
    f = lib.abattn_gather_bench
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p] + [ctypes.c_int] * 5 + [
        ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_longlong)]
    torch.cuda.set_device(0)
    BH, N = 2, 75600
    g = torch.Generator(device="cuda").manual_seed(11)
    K = torch.randn(BH, N, 128, device="cuda", generator=g).to(torch.bfloat16)
    V = torch.randn(BH, N, 128, device="cuda", generator=g).to(torch.bfloat16)
    names = {1: "cp.async 16B/lane", 0: "TMA tiled box 4x64", 2: "TMA tile::gather4"}
    for mode in (1, 0, 2):
        for warps in (1, 2, 4, 7, 8, 16):
            cyc, bad = ctypes.c_double(), ctypes.c_longlong()
            rc = f(K.data_ptr(), V.data_ptr(), BH, N, mode, warps, 200, ctypes.byref(cyc), ctypes.byref(bad))
            print(json.dumps({"gather_bench": names[mode], "issuing_warps": warps, "rc": rc,
                              "cycles_per_tile": cyc.value if rc == 0 else None,
                              "bytes_per_cycle": 65536 / cyc.value if rc == 0 and cyc.value > 0 else None,
                              "last_tile_mismatched_chunks": bad.value}), flush=True)


def run_mma_bench(args):
    """Clock cycles per bf16 tcgen05.mma (M = 128, K = 16) issued back to back
    by one thread per SM, one CTA per SM: operands in shared memory at N = 64,
    128 and 256, A in TMEM at N = 128, the score and forward kernels' own
    issue patterns, and N = 128 beside four warps loading or storing shared
    memory (with the bytes per cycle those warps get).  Full rate is
    2*128*N*16 / 8192 cycles per MMA (64 at N = 128).  One JSON line per
    mode."""
    import ctypes
    from block_sparse_attention_12_b200 import build
    lib = ctypes.CDLL(build.build_mmabench())
    f = lib.abattn_mma_bench
    f.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_double),
                  ctypes.POINTER(ctypes.c_double)]
    torch.cuda.set_device(0)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    modes = [(0, "smem A and B, N=128", 128), (1, "smem A and B, N=256", 256), (2, "A in TMEM, N=128", 128),
             (3, "smem A and B, N=64", 64), (4, "score kernel issue pattern (N=128)", 128),
             (5, "forward kernel issue pattern (N=128)", 128),
             (6, "smem A and B, N=128, 4 warps loading shared memory", 128),
             (7, "A in TMEM, N=128, 4 warps loading shared memory", 128),
             (8, "smem A and B, N=128, 4 warps storing shared memory", 128)]
    for mode, name, n in modes:
        cyc, tr = ctypes.c_double(), ctypes.c_double()
        rc = f(mode, 1024, sms, ctypes.byref(cyc), ctypes.byref(tr))
        line = {"mma_bench": name, "rc": rc, "cycles_per_mma": cyc.value if rc == 0 else None,
                "flop_per_cycle_per_sm": 2 * 128 * n * 16 / cyc.value if rc == 0 and cyc.value > 0 else None,
                "full_rate_cycles": 2 * 128 * n * 16 / 8192}
        if mode >= 6:
            line["other_warps_smem_bytes_per_cycle"] = tr.value if rc == 0 else None
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.gather_bench:
        run_gather_bench(args)
        return
    if args.mma_bench:
        run_mma_bench(args)
        return
    if args.e4m3:
        run_e4m3(args)
        return
    if args.sweep:
        run_sweep(args)
        return
    if args.denoise:
        run_denoise(args)
        return
    if args.strong:
        run_strong(args)
        return
    w = inputs.WORKLOADS[args.workload]
    if args.heads:
        import dataclasses
        w = dataclasses.replace(w, H=args.heads, name=f"{w.name}-{args.heads}heads")
    if args.impl == "reference":
        run_reference(args, w)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    from block_sparse_attention_12_b200 import abi, build
    build.build()
    P = peaks()
    shape = (w.B, w.H, w.N, w.d)
    Q, K, V = inputs.make_qkv(w, device=f"cuda:{local}", seed=w.seed + 1000 * rank)
    cfg = abi.Config(kv_block=w.kv_block, budget=w.budget, n_clusters=w.n_clusters,
                     kmeans_iters=w.kmeans_iters, seed=w.seed)
    planner = abi.Planner(shape, cfg)
    O = torch.empty_like(Q)
    lse = torch.empty(shape[:3], dtype=torch.float32, device=Q.device)
    stream = torch.cuda.current_stream()

    def step():
        plan = planner(Q, K)
        for _ in range(w.forwards_per_plan):
            abi.forward(Q, K, V, plan, cfg, O=O, lse=lse)

    for _ in range(max(args.warmup, 3)):
        step()
    abi.check()
    plan = planner.plan
    exec_fl = abi.executed_flops(plan, shape) * w.forwards_per_plan
    useful_fl = abi.useful_flops(plan, shape) * w.forwards_per_plan

    # ---- the timed region: K whole steps, barrier + sync on both sides
    clocks = ClockSampler(local)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clk = clocks.stop()
    ms = multigpu.max_over_ranks(e0.elapsed_time(e1) / args.steps, Q.device)
    abi.check()
    value = multigpu.job_throughput(exec_fl, ms, world) / 1e12

    # ---- per-kernel breakdown (separate loops, same stream, after the timed region)
    kb_ms = {}
    n_it = max(3, min(args.steps, 10))
    Kbar = abi.meanpool(K, w.kv_block)
    kb_ms["meanpool"] = timed(lambda: abi.meanpool(K, w.kv_block, out=Kbar), n_it, stream)
    C, wt, _ = abi.kmeans(Q, cfg)
    kb_ms["kmeans"] = timed(lambda: abi.kmeans(Q, cfg), n_it, stream)
    S = abi.score(C, wt, Kbar, shape, cfg)
    kb_ms["score"] = timed(lambda: abi.score(C, wt, Kbar, shape, cfg), n_it, stream)
    p2 = abi.plan_from_scores(S, shape, cfg)
    kb_ms["planner"] = timed(lambda: abi.plan_from_scores(S, shape, cfg, plan=p2), n_it, stream)
    kb_ms["plan_total"] = timed(lambda: planner(Q, K), n_it, stream)
    kb_ms["forward"] = timed(lambda: abi.forward(Q, K, V, plan, cfg, O=O, lse=lse), n_it, stream)
    abi.check()
    del S, p2
    fwd_fl = abi.executed_flops(plan, shape)
    fwd_tf = fwd_fl / (kb_ms["forward"] / 1e3) / 1e12

    dense = None
    if not args.no_dense and rank == 0:
        Od = torch.empty_like(Q)
        abi.dense_forward(Q, K, V, O=Od, want_lse=False)
        dms = timed(lambda: abi.dense_forward(Q, K, V, O=Od, want_lse=False), args.dense_iters, stream)
        abi.check()
        dfl = 4.0 * w.B * w.H * w.N * w.N * w.d
        dense = {"ms": dms, "tflops": dfl / (dms / 1e3) / 1e12, "frac_of_bf16_peak": dfl / (dms / 1e3) / 1e12 / P["bf16"]}
        del Od

    # ---- rooflines (algorithmic work per launch / measured launch time)
    BH = w.B * w.H
    nqb, nkvb = math.ceil(w.N / 128), math.ceil(w.N / w.kv_block)
    rows = BH * nqb
    sel_cnt = float(plan.counts.sum().item())
    roofs = {
        # against the burst peak; the forward is timed right after the step loop, under the
        # power cap, so its fraction of the sustained (seconds-long) peak is given beside it
        "forward": {"bound": "tensor", "achieved": fwd_tf, "peak": P["bf16"], "unit": "TFLOP/s",
                    "work": fwd_fl, "traffic": traffic_for("forward", rows),
                    "frac_of_sustained_peak": fwd_tf / P["bf16_sus"]},
        "meanpool": {"bound": "hbm", "unit": "GB/s", "peak": P["hbm"],
                     "work": BH * w.N * w.d * 2 + BH * nkvb * w.d * 4,
                     "traffic": traffic_for("meanpool", BH * nkvb)},
        # k-means (both Lloyd steps on tcgen05) is bound by the latency of its
        # dependent iterations; its roofline is its one read of the queries (and
        # the centroid, weight and label writes)
        "kmeans": {"bound": "hbm", "unit": "GB/s", "peak": P["hbm"],
                   "work": rows * (128 * w.d * 2 + w.n_clusters * w.d * 4 + w.n_clusters * 4 + 128 * 4),
                   "traffic": traffic_for("kmeans", rows)},
        # tensor cores, bf16 hi/lo split: 3 MMAs per product, 2 passes over 8 cluster slots
        "score": {"bound": "tensor", "unit": "TFLOP/s", "peak": P["bf16"],
                  "work": 3 * 2 * (2.0 * rows * 8 * nkvb * w.d), "traffic": traffic_for("score", rows),
                  # its HBM side: the mean keys once per head, the centroids, the scores written
                  "hbm_bytes": BH * nkvb * w.d * 4 + rows * 8 * w.d * 4 + rows * nkvb * 4},
        "planner": {"bound": "hbm", "unit": "GB/s", "peak": P["hbm"],
                    "work": rows * nkvb * 4 + rows * 4 + sel_cnt * 8, "traffic": traffic_for("planner", rows)},
    }
    for k, r in roofs.items():
        t = kb_ms[k] / 1e3
        if k != "forward":
            r["achieved"] = r["work"] / t / (1e9 if r["unit"] == "GB/s" else 1e12)
        r["frac"] = r["achieved"] / r["peak"]
        r["ms"] = kb_ms[k]
        if "hbm_bytes" in r:
            r["hbm_gbs"] = r["hbm_bytes"] / t / 1e9
            r["hbm_frac"] = r["hbm_gbs"] / P["hbm"]
    step_share = {k: kb_ms[k] * (w.forwards_per_plan if k == "forward" else 1) for k in roofs}
    dom = max(step_share, key=step_share.get)
    rd = roofs[dom]
    roofline = {"kernel": dom, "bound": rd["bound"], "achieved": rd["achieved"], "peak": rd["peak"],
                "unit": rd["unit"], "frac": rd["frac"], "traffic": rd["traffic"],
                "peak_source": P["src"] + (" bf16 burst" if rd["bound"] == "tensor" else " hbm copy")}

    # ---- end to end through the public API with host buffers: every step
    # copies its Q, K, V from pinned host memory and its O back; steps are
    # pipelined on three streams (the upload of step k+1 and the download of
    # step k-1 run while step k computes), with two device buffer sets
    e2e = None
    if not args.no_e2e:
        Qh, Kh, Vh = (t.cpu().pin_memory() for t in (Q, K, V))
        Oh = [torch.empty(O.shape, dtype=O.dtype, pin_memory=True) for _ in range(2)]
        dev = [tuple(torch.empty_like(t) for t in (Q, K, V, O)) for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        s_cmp = stream

        def e2e_run(n_steps):
            ev_in = [torch.cuda.Event() for _ in range(n_steps)]
            ev_cmp = [torch.cuda.Event() for _ in range(n_steps)]
            ev_out = [torch.cuda.Event() for _ in range(n_steps)]
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record(s_in)
            for k in range(n_steps):
                Qd, Kd, Vd, Od = dev[k % 2]
                with torch.cuda.stream(s_in):
                    if k >= 2:
                        s_in.wait_event(ev_cmp[k - 2])  # step k-2 is done with this buffer set
                    Qd.copy_(Qh, non_blocking=True)
                    Kd.copy_(Kh, non_blocking=True)
                    Vd.copy_(Vh, non_blocking=True)
                    ev_in[k].record(s_in)
                s_cmp.wait_event(ev_in[k])
                if k >= 2:
                    s_cmp.wait_event(ev_out[k - 2])  # O of step k-2 has been read back
                pl = planner(Qd, Kd, stream=s_cmp)
                for _ in range(w.forwards_per_plan):
                    abi.forward(Qd, Kd, Vd, pl, cfg, O=Od, lse=lse, stream=s_cmp)
                ev_cmp[k].record(s_cmp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_cmp[k])
                    Oh[k % 2].copy_(Od, non_blocking=True)
                    ev_out[k].record(s_out)
            e1.record(s_out)
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) / n_steps

        e2e_run(2)
        if dist:
            dist.barrier()
        e2e_ms = multigpu.max_over_ranks(e2e_run(args.e2e_steps), Q.device)
        abi.check()
        h2d = 3 * Q.numel() * Q.element_size()

        # the host link alone: one step's uploads with nothing else running
        # (best of three), the bound that the pipelined steps approach
        def upload_ms():
            ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            ea.record(s_in)
            with torch.cuda.stream(s_in):
                for t_d, t_h in zip(dev[0][:3], (Qh, Kh, Vh)):
                    t_d.copy_(t_h, non_blocking=True)
            eb.record(s_in)
            torch.cuda.synchronize()
            return ea.elapsed_time(eb)

        up_ms = min(upload_ms() for _ in range(3))
        e2e = {"value": multigpu.job_throughput(exec_fl, e2e_ms, world) / 1e12, "unit": UNIT, "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": O.numel() * O.element_size(),
               "steps": args.e2e_steps,
               "pipelining": "upload of step k+1 and download of step k-1 overlap step k (3 streams); "
                             "the time includes the pipeline's fill and drain",
               "h2d_gbs_alone": h2d / (up_ms * 1e6),
               "link_bound_ms": up_ms,
               "link_frac": up_ms / e2e_ms}
        del Qh, Kh, Vh, Oh, dev

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, args.cpu_rows, args.cpu_rows_one_core)

    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "tokens": w.N, "heads": w.H, "d": w.d, "grid": list(w.grid),
                   "kv_block": w.kv_block, "budget": w.budget, "q_block": 128, "clusters": w.n_clusters,
                   "kmeans_iters": w.kmeans_iters, "forwards_per_plan": w.forwards_per_plan,
                   "step": "abattn_plan + forwards_per_plan x abattn_forward",
                   "l2": "inputs larger than L2 (Q, K, V %.2f GB per GPU)" % (3 * Q.numel() * 2 / 1e9),
                   "parallelism": f"weak x{world}: one full layer per GPU"},
        "fwd_ms": kb_ms["forward"], "fwd_tflops": fwd_tf, "fwd_frac_of_bf16_peak": fwd_tf / P["bf16"],
        "plan_ms": kb_ms["plan_total"], "kernel_ms": kb_ms,
        "executed_tflop_per_step": exec_fl / 1e12, "useful_tflop_per_step": useful_fl / 1e12,
        "selected_blocks_mean": sel_cnt / rows, "sparsity": 1.0 - sel_cnt / rows / nkvb,
        "dense": dense, "roofline": roofline,
        "rooflines": {k: {kk: vv for kk, vv in r.items() if kk != "work"} for k, r in roofs.items()},
        "cpu_baseline": cpu, "e2e": e2e, "clocks": clk,
        # per step: abattn_plan launches mean keys, k-means, scores and the planner;
        # then one forward per plan use
        "gpu_launches": (4 + w.forwards_per_plan) * args.steps,
        "peaks": P,
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()

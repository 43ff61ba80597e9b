#!/usr/bin/env python3
"""Benchmark of the DDTree verification round on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one full verification round (top-k -> tree build -> tree attention
-> tree walk) over one batch of the "b64" workload: batch 1, L=16 draft
positions, V=151936, top-k 8, budget B=64, context 4096, GQA 32/8, d=128,
bf16 draft logits and KV, f32 target logits.  Inputs are synthetic and
resident in HBM when the timed region starts; R input sets (each a different
sequence) rotate so that the bytes a step touches are not left in the 126 MB
L2 by the previous step.  Each set's round is one CUDA graph; the last step
of every set in the timed region replays a copy of that graph with event
nodes between the kernels, which gives the per-kernel durations.

Multi-GPU (torchrun): every rank runs its own sequences (the round shards by
sequence, nothing is exchanged); the time is the max over ranks and the value
counts the rounds of all ranks.

``--impl reference`` times the CPU oracle (fp64, single thread) on the same
workload instead, as the reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "verify rounds/sec and tree-attn HBM GB/s (% of B200 peak) at B=64–512"
WORKLOAD = "b64"
PER_WORKLOAD_MAX_STEPS = 2000  # graph replays per workload of `per_workload` (long512: ~5 s)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--sets", type=int, default=5, help="rotating input sets")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extensions", action="store_true",
                    help="skip the measurements beyond the round (e.g. for a launch list)")
    ap.add_argument("--profile", action="store_true",
                    help="no timing: four rounds of one input set with an L2 flush before each, "
                         "for an ncu capture filtered by kernel name (-k)")
    ap.add_argument("--workload", default=None, help="workload for --profile (default: the bench's)")
    ap.add_argument("--sweep", action="store_true",
                    help="budget sweep: round time and acceptance for each B in --budgets")
    ap.add_argument("--budgets", default="16,32,64,128,256,512")
    ap.add_argument("--sweep-batch", type=int, default=8)
    ap.add_argument("--sweep-draws", type=int, default=40)
    ap.add_argument("--sweep-invt", type=float, default=3.0,
                    help="inverse temperature of the drafter's marginals in the sweep (the b64 "
                         "logits at 1.0 give the top token < 0.2%%; 3.0 gives ~0.8)")
    ap.add_argument("--stage-sweep", action="store_true",
                    help="each stage kernel timed alone on every workload, with its roofline")
    ap.add_argument("--stage-workloads", default="b64,b256,paged128,long512")
    ap.add_argument("--extensions", action="store_true",
                    help="with --profile: also run the sampled walk and the KV commit after "
                         "each round")
    ap.add_argument("--no-budget-sweep", action="store_true",
                    help="skip the budget sweep and the adaptive round in the bench line")
    ap.add_argument("--line-budgets", default="16,32,64,128,256")
    ap.add_argument("--line-sweep-draws", type=int, default=16)
    ap.add_argument("--no-per-workload", action="store_true",
                    help="skip the rounds of the other workloads (b256, paged128, long512)")
    ap.add_argument("--per-workload", default="b256,paged128,long512")
    ap.add_argument("--clock-window-s", type=float, default=0.5,
                    help="untimed replays before and after the timed region, so that the clock "
                         "sampler sees the GPU under load around it")
    ap.add_argument("--cpu-threads", type=int, default=0,
                    help="threads of the threaded oracle baseline (0: every core of the host)")
    ap.add_argument("--selftest-ranks", action="store_true",
                    help="no GPU: each rank only exercises the multi-rank host logic on gloo")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


def input_set_bytes(w):
    """Bytes of one input set of a round: draft logits, root tokens and
    context lengths, queries, the context K/V, the tree K/V, target logits."""
    es_draft = 4 if w.draft_dtype == "f32" else 2
    return (w.batch * w.L * w.V * es_draft + 8 * w.batch + w.batch * w.n_max * w.hq * w.d * 2 +
            2 * w.batch * w.ctx * w.hkv * w.d * 2 + 2 * w.batch * w.n_max * w.hkv * w.d * 2 +
            w.batch * w.n_max * w.V * 4)


def workload_config(w, sets, set_bytes):
    return {"workload": "%s: batch %d, L=%d, V=%d, top-k %d, B=%d, ctx %d, GQA %d/%d, d=%d, "
                        "bf16 draft/KV, f32 target logits" % (w.name, w.batch, w.L, w.V, w.k, w.B,
                                                              w.ctx, w.hq, w.hkv, w.d),
            "batch": w.batch, "L": w.L, "V": w.V, "k": w.k, "B": w.B, "ctx": w.ctx,
            "hq": w.hq, "hkv": w.hkv, "d": w.d,
            "l2": "inputs larger than L2: %d rotating input sets, %.0f MB in total (L2 126 MB)"
                  % (sets, sets * set_bytes / 1e6)}


# ----------------------------------------------------------------------------
# clocks during the timed region
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, dev_index):
        self.proc = None
        self.lines = []
        import torch
        try:
            uuid = str(torch.cuda.get_device_properties(dev_index).uuid)
            self.sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.sel = str(dev_index)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.sel, "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------
def max_over_ranks(value, world, device):
    """The largest of every rank's value (a job's time is its slowest rank's)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def host_cores():
    """Cores this process may run on, and the host's core count."""
    try:
        usable = len(os.sched_getaffinity(0))
    except Exception:
        usable = os.cpu_count() or 1
    return usable, os.cpu_count() or usable


def relaunch_command(argv, n, port):
    """The torchrun command that runs this script as n ranks on this node."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            "--nproc-per-node", str(n), "--master-addr", "127.0.0.1",
            "--master-port", str(port), os.path.abspath(__file__)] + list(argv)


def relaunch_as_ranks(n):
    """`bench.py --gpus N` started without a launcher: run it again under
    torchrun as N ranks (one per GPU) and return their exit status."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    return subprocess.call(relaunch_command(sys.argv[1:], n, port))


def run_selftest_ranks(args):
    """Each rank: a gloo process group, the max-over-ranks time and the job
    throughput of the real path, on the CPU; rank 0 prints one JSON line."""
    import datetime
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world > 1:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    local_ms = 2.0 + rank
    ms = max_over_ranks(local_ms, world, "cpu")
    line = {"selftest": True, "n_gpus": world, "rank_ms": local_ms, "job_ms": ms,
            "value": job_throughput(world, 1, args.steps, ms)}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def job_throughput(world, batch, steps, elapsed_ms):
    """Rounds of all ranks per second: every rank runs `steps` rounds of its own
    `batch` sequences (weak scaling), all within the slowest rank's time."""
    return world * batch * steps / (elapsed_ms * 1e-3)


def make_inputs(w, rank, s):
    """Host-side (numpy) inputs of one set: a different sequence per (rank, set)."""
    from block_draft_tree_b200 import synth
    seed = w.seed + 1000 * rank + 17 * s + 1
    x = {"draft": synth.draft_logits(w, seed), "root": synth.root_tokens(w, seed)}
    x.update(synth.attention_inputs(w, seed))
    return x, seed


def to_device(x, w, torch):
    bf = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).cuda()
    d = {"draft": bf(x["draft"]) if x["draft"].dtype == np.uint16 else torch.from_numpy(x["draft"]).cuda(),
         "root": torch.from_numpy(x["root"]).cuda(), "ctx_len": torch.from_numpy(x["ctx_len"]).cuda(),
         "q": bf(x["q"]), "k_cache": bf(x["k_cache"]), "v_cache": bf(x["v_cache"]),
         "k_tree": bf(x["k_tree"]), "v_tree": bf(x["v_tree"])}
    if "page_table" in x:
        d["page_table"] = torch.from_numpy(x["page_table"]).cuda()
    return d


def stage_bytes(w, n_nodes_total):
    """Algorithmic HBM bytes of each stage for one round of the workload."""
    rows = w.batch * w.L
    topk = rows * w.V * 2 + rows * w.k * 12 + rows * 4
    kv = w.batch * w.ctx * w.hkv * w.d * 2 * 2
    q_o = 2 * w.batch * w.n_max * w.hq * w.d * 2
    tree_kv = 2 * w.batch * w.n_max * w.hkv * w.d * 2
    attn = kv + q_o + tree_kv
    walk = n_nodes_total * w.V * 4
    flops = 4.0 * sum([w.ctx] * w.batch) * w.n_max * w.hq * w.d  # context part dominates
    return {"topk": topk, "tree": 0, "attn": attn, "walk": walk, "attn_flops": flops}


def kernel_nodes(rnd, torch, cudart):
    """Kernels one round launches: captured once more into a kept graph whose
    kernel nodes are counted."""
    try:
        g = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(g):
            rnd.launch()
        err, nodes, n = cudart.cudaGraphGetNodes(g.raw_cuda_graph(), 0)
        err, nodes, n = cudart.cudaGraphGetNodes(g.raw_cuda_graph(), n)
        kinds = [cudart.cudaGraphNodeGetType(nd)[1] for nd in nodes]
        return sum(1 for t in kinds if t == cudart.cudaGraphNodeType.cudaGraphNodeTypeKernel)
    except Exception:
        return 4


def traffic_for(kernel_tag):
    """DRAM bytes per launch of a kernel from the committed ncu summary, if the
    kernel's source is unchanged since the counters were taken."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
        e = t[kernel_tag]
        src = os.path.join(ROOT, e["source"])
        sha = hashlib.sha1(open(src, "rb").read()).hexdigest()
        return e["dram_bytes_per_launch"] if sha == e["source_sha1"] else None
    except Exception:
        return None


def _chunks(n, parts):
    step = max(1, -(-n // max(1, parts)))
    return [(i, min(n, i + step)) for i in range(0, n, step)]


def cpu_baseline(w, x_host, attn_fraction=1.0, threads=1):
    """Time the CPU oracle on one round of the workload (attention on a
    bounded sample of its (sequence, row, head) items, scaled to the round).
    With threads > 1 the oracle's calls run on that many host threads over
    independent pieces (rows of the top-k, sequences of the tree and the
    walk, items of the attention); the oracle's arithmetic is unchanged and
    its C calls release the interpreter lock."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle
    from block_draft_tree_b200 import synth
    ex = ThreadPoolExecutor(max_workers=threads) if threads > 1 else None

    def pmap(fn, pieces):
        return list(ex.map(fn, pieces)) if ex else [fn(p) for p in pieces]

    z = x_host["draft"]
    t0 = time.perf_counter()
    rows = z.reshape(-1, z.shape[-1])
    parts = pmap(lambda r: oracle.topk(rows[r[0]:r[1]], w.k, w.inv_temperature),
                 _chunks(rows.shape[0], threads))
    ids = np.concatenate([p[0] for p in parts]).reshape(w.batch, w.L, w.k)
    zk = np.concatenate([p[1] for p in parts]).reshape(w.batch, w.L, w.k)
    lse = np.concatenate([p[3] for p in parts]).reshape(w.batch, w.L)
    t1 = time.perf_counter()
    bud, kps = w.budget_per_seq(), w.k_per_seq()
    seq_parts = _chunks(w.batch, threads)
    trees = pmap(lambda r: oracle.build_tree(ids[r[0]:r[1]], zk[r[0]:r[1]], lse[r[0]:r[1]],
                                             bud[r[0]:r[1]], w.inv_temperature,
                                             root_token=x_host["root"][r[0]:r[1]],
                                             ctx_len=x_host["ctx_len"][r[0]:r[1]],
                                             k_per_seq=kps[r[0]:r[1]], n_max=w.n_max), seq_parts)
    tree = {k: np.concatenate([t[k] for t in trees]) for k in trees[0]}
    t2 = time.perf_counter()
    items = [(b, j, h) for b in range(w.batch) for j in range(int(tree["n_nodes"][b]))
             for h in range(w.hq)]
    n_all = len(items)
    n_s = max(1, int(round(n_all * attn_fraction)))
    items = np.array(items[:n_s], np.int32)
    pmap(lambda r: oracle.tree_attn(items[r[0]:r[1]], x_host["q"], x_host["k_cache"],
                                    x_host["v_cache"], x_host["ctx_len"], x_host["k_tree"],
                                    x_host["v_tree"], tree["mask"], tree["n_nodes"],
                                    1.0 / np.sqrt(w.d), page_table=x_host.get("page_table"),
                                    page_size=x_host.get("page_size", 64)),
         _chunks(n_s, 4 * threads))
    t3 = time.perf_counter()
    tgt = synth.target_logits(w, tree["tok"], tree["parent"], tree["depth"], tree["n_nodes"])
    t4 = time.perf_counter()
    pmap(lambda r: oracle.tree_walk(tgt[r[0]:r[1]], tree["tok"][r[0]:r[1]],
                                    tree["parent"][r[0]:r[1]], tree["depth"][r[0]:r[1]],
                                    tree["n_nodes"][r[0]:r[1]], w.L), seq_parts)
    t5 = time.perf_counter()
    if ex:
        ex.shutdown()
    round_s = (t1 - t0) + (t2 - t1) + (t3 - t2) * n_all / n_s + (t5 - t4)
    return round_s, {"topk_s": t1 - t0, "tree_s": t2 - t1, "attn_s": (t3 - t2) * n_all / n_s,
                     "walk_s": t5 - t4, "attn_rows_timed": n_s, "attn_rows": n_all}


# ----------------------------------------------------------------------------
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from block_draft_tree_b200 import synth
    w = synth.WORKLOADS[WORKLOAD]
    x, _ = make_inputs(w, 0, 0)
    usable, total = host_cores()
    threads = args.cpu_threads or usable
    # size the attention sample so that the whole run stays within a few minutes
    probe_s, parts = cpu_baseline(w, x, attn_fraction=0.02, threads=threads)
    per_step_budget = 150.0 / max(1, args.steps + args.warmup)
    fixed = parts["topk_s"] + parts["tree_s"] + parts["walk_s"]
    per_row = parts["attn_s"] / parts["attn_rows"]
    frac = min(1.0, max(1.0 / parts["attn_rows"], (per_step_budget - fixed) / max(per_row * parts["attn_rows"], 1e-9)))
    for _ in range(args.warmup):
        cpu_baseline(w, x, attn_fraction=frac, threads=threads)
    times = []
    for _ in range(args.steps):
        s_, parts = cpu_baseline(w, x, attn_fraction=frac, threads=threads)
        times.append(s_)
    round_s = statistics.mean(times)
    value = w.batch / round_s
    sample = ("full top-k, tree and walk; attention on %d of %d (row, head) items per step, "
              "scaled to the full round; %d threads on a host of %d cores"
              % (parts["attn_rows_timed"], parts["attn_rows"], threads, total))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "rounds/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round_s * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, args.sets, input_set_bytes(w)),
            "cpu_baseline": {"value": value, "unit": "rounds/s", "cores": threads,
                             "host_cores": total, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "rounds/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


LM_HIDDEN = 4096  # synthetic target hidden size for the LM-head call


def measure_extensions(w, sets, graphs, hbm_peak, reps=30):
    """Per-launch device time of the library's calls beyond the round proper
    (the sampled walk), each launch after an L2 flush, on the round's own
    target logits and trees.  Not part of the timed region."""
    import torch

    from block_draft_tree_b200 import api

    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    inv_t = 1.0
    times = []
    n_rows = []
    for rep in range(reps + 3):
        j = rep % len(sets)
        o = graphs[j][1].out
        tgt = sets[j]["target"]
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        api.tree_walk_sample(tgt, o["tok"], o["parent"], o["depth"], o["n_nodes"], w.L, inv_t,
                             seed=12345, step=rep)
        b.record()
        torch.cuda.synchronize()
        if rep >= 3:
            times.append(a.elapsed_time(b) * 1e3)
            n_rows.append(int(o["n_nodes"].sum().item()))
    us = statistics.median(times)
    alg = statistics.mean(n_rows) * w.V * 4  # every tree row's fp32 target logits, read once
    gbs = alg / (us * 1e-6) / 1e9
    ext = {"walk_sample": {"us": round(us, 3), "alg_bytes": int(alg), "gbs": round(gbs, 1),
                           "frac_hbm": round(gbs / hbm_peak, 4), "inv_temperature": inv_t,
                           "launches": len(times), "l2": "flushed before each launch"}}

    # KV commit of each round's accepted path, into copies of the cache (the
    # timed rounds' own buffers stay as they were)
    kc = sets[0]["k_cache"].clone()
    vc = sets[0]["v_cache"].clone()
    pt = sets[0].get("page_table")
    cl = torch.empty_like(sets[0]["ctx_len"])
    times, rows = [], []
    for rep in range(reps + 3):
        j = rep % len(sets)
        o = graphs[j][1].out
        cl.copy_(sets[j]["ctx_len"])
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        api.kv_commit(sets[j]["k_tree"], sets[j]["v_tree"], o["acc_len"], o["acc_nodes"], cl,
                      kc, vc, page_table=pt, page_size=w.page_size or 64)
        b.record()
        torch.cuda.synchronize()
        if rep >= 3:
            times.append(a.elapsed_time(b) * 1e3)
            rows.append(int(o["acc_len"].sum().item()) + w.batch)
    us = statistics.median(times)
    alg = statistics.mean(rows) * w.hkv * w.d * 2 * 2 * 2  # K and V rows, read and written
    ext["kv_commit"] = {"us": round(us, 3), "alg_bytes": int(alg),
                        "gbs": round(alg / (us * 1e-6) / 1e9, 2), "launches": len(times),
                        "bound": "launch latency (a few KB per sequence)"}

    # the greedy walk straight from the target's hidden states: LM head on the
    # tensor cores + argmax + walk (synthetic hidden size 4096, random head)
    K = LM_HIDDEN
    g = torch.Generator(device="cuda")
    g.manual_seed(77)
    hid = (torch.randn(w.batch, w.n_max, K, device="cuda", generator=g) * 0.5).bfloat16()
    head = (torch.randn(w.V, K, device="cuda", generator=g) / K ** 0.5).bfloat16()
    o = graphs[0][1].out
    times = []
    for rep in range(reps + 3):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        api.lm_head_walk(hid, head, o["tok"], o["parent"], o["depth"], o["n_nodes"], w.L)
        b.record()
        torch.cuda.synchronize()
        if rep >= 3:
            times.append(a.elapsed_time(b) * 1e3)
    us = statistics.median(times)
    alg = w.V * K * 2 + w.batch * w.n_max * K * 2  # the head and the hidden rows, read once
    flops = 2.0 * w.batch * w.n_max * w.V * K
    gbs = alg / (us * 1e-6) / 1e9
    ext["lm_head_walk"] = {"us": round(us, 3), "alg_bytes": int(alg), "gbs": round(gbs, 1),
                           "frac_hbm": round(gbs / hbm_peak, 4),
                           "tflops": round(flops / (us * 1e-6) / 1e12, 1), "hidden": K,
                           "launches": len(times),
                           "l2": "the %.2f GB head exceeds L2" % (w.V * K * 2 / 1e9)}
    del hid, head
    return ext


def device_inputs(w, seed):
    """One input set of a workload generated on the GPU (seeded torch
    generator): the same distributions as the seeded host generator
    (block_draft_tree_b200.synth) -- N(0,1) drafts with +6/+4/+3 spikes at
    distinct tokens, or Zipf(1.1) drafts over a fresh permutation per row;
    N(0,1) bf16 queries and K/V; ragged contexts and a random page placement
    for the paged workload -- drawn where the large workloads live, so that
    building them takes milliseconds.  Target logits are N(0,1) here and
    planted from the GPU's own tree (plant_greedy) once the tree exists."""
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    dev = "cuda"
    rows = w.batch * w.L
    if w.draft == "spikes":
        z = torch.randn(rows, w.V, device=dev, generator=g)
        t0 = torch.randint(0, w.V, (rows,), device=dev, generator=g)
        r = torch.arange(rows, device=dev)
        for i, sp in enumerate(w.spikes):  # distinct tokens: fixed offsets from a random start
            z[r, (t0 + 7919 * i) % w.V] += sp
    else:
        ranks = torch.arange(1, w.V + 1, device=dev, dtype=torch.float64)
        zipf = (-1.1 * torch.log(ranks)).float()
        perm = torch.argsort(torch.rand(rows, w.V, device=dev, generator=g), dim=1)
        z = torch.empty(rows, w.V, device=dev)
        z.scatter_(1, perm, zipf.expand(rows, w.V).contiguous())
    x = {"draft": z.reshape(w.batch, w.L, w.V).to(torch.bfloat16)}
    del z
    x["root"] = torch.randint(0, w.V, (w.batch,), device=dev, generator=g, dtype=torch.int32)
    if w.ctx_min is None:
        ctx = torch.full((w.batch,), w.ctx, device=dev, dtype=torch.int32)
    else:
        ctx = torch.randint(w.ctx_min, w.ctx + 1, (w.batch,), device=dev, generator=g,
                            dtype=torch.int32)
    x["ctx_len"] = ctx
    bf = lambda *shape: torch.randn(*shape, device=dev, generator=g).to(torch.bfloat16)
    x["q"] = bf(w.batch, w.n_max, w.hq, w.d)
    x["k_tree"] = bf(w.batch, w.n_max, w.hkv, w.d)
    x["v_tree"] = bf(w.batch, w.n_max, w.hkv, w.d)
    if w.page_size:
        ps = w.page_size
        npg = (ctx.long() + ps - 1) // ps
        total = int(npg.sum().item())
        max_pages = int(npg.max().item())
        perm = torch.randperm(total, device=dev, generator=g).to(torch.int32)
        pt = torch.full((w.batch, max_pages), -1, device=dev, dtype=torch.int32)
        off = 0
        for b, n in enumerate(npg.tolist()):
            pt[b, :n] = perm[off:off + n]
            off += n
        x["page_table"] = pt
        shape = (total, ps, w.hkv, w.d)
    else:
        shape = (w.batch, w.ctx, w.hkv, w.d)
    x["k_cache"] = bf(*shape)
    x["v_cache"] = bf(*shape)
    x["target"] = torch.randn(w.batch, w.n_max, w.V, device=dev, generator=g)
    return x, g


def plant_greedy(w, target, tok, parent, depth, n_nodes, g):
    """Planted agreement on the GPU, as synth.target_logits plants it on the
    host: every tree row with children, with probability max(0, p0 - decay *
    depth), gets logit (row max + 2) at the token of one of its children
    picked uniformly."""
    import torch
    b, n_max, V = target.shape
    rows = torch.arange(n_max, device=target.device)
    live = (rows[None, :] < n_nodes[:, None]) & (rows[None, :] > 0)
    par = parent.long().clamp(min=0)
    key = torch.rand(b, n_max, device=target.device, generator=g)
    key = torch.where(live, key, torch.full_like(key, -1.0))
    best = torch.full((b, n_max), -1.0, device=target.device)
    best.scatter_reduce_(1, par, key, reduce="amax")  # per parent: the largest child key
    chosen = live & (key == best.gather(1, par))
    p = (w.plant_p0 - w.plant_decay * depth.float()).clamp(min=0.0)
    u = torch.rand(b, n_max, device=target.device, generator=g)
    plant_row = (u < p) & (rows[None, :] < n_nodes[:, None])  # per parent row
    bi, ci = torch.nonzero(chosen, as_tuple=True)
    xi = par[bi, ci]
    keep = plant_row[bi, xi]
    bi, ci, xi = bi[keep], ci[keep], xi[keep]
    rowmax = target.amax(dim=2)
    target[bi, xi, tok[bi, ci].long()] = rowmax[bi, xi] + 2.0


def measure_per_workload(names, hbm_peak, tf_peak, steps, seed=5):
    """One full round of each named workload (one CUDA graph per workload,
    its inputs far larger than L2), timed like the headline: `steps` graph
    replays between CUDA events; then the same round with event nodes
    between the kernels, replayed a few times, for each stage's time and its
    fraction of the binding roofline."""
    import torch
    from cuda.bindings import runtime as cudart

    from block_draft_tree_b200 import api, synth
    from block_draft_tree_b200.round import VerifyRound

    out = {}
    for name in names:
        w = synth.WORKLOADS[name]
        x, g = device_inputs(w, seed + w.index)
        max_ctx = int(x["ctx_len"].max().item())
        ps = w.page_size or 64
        rnd = VerifyRound(batch=w.batch, L=w.L, V=w.V, k=w.k, B_max=w.B, hq=w.hq, hkv=w.hkv,
                          d=w.d, max_ctx=max_ctx, draft_dtype=torch.bfloat16,
                          target_dtype=torch.float32, inv_temperature=w.inv_temperature,
                          paged=w.page_size > 0, page_size=ps,
                          max_pages=(max_ctx + ps - 1) // ps)
        if w.chain_seq0:
            x["k_per_seq"] = torch.from_numpy(w.k_per_seq()).cuda()
            x["budget"] = torch.from_numpy(w.budget_per_seq()).cuda()
        rnd.bind(x)
        rnd.launch()
        torch.cuda.synchronize()
        o = rnd.out
        plant_greedy(w, x["target"], o["tok"], o["parent"], o["depth"], o["n_nodes"], g)
        graph = rnd.capture()
        evs = [cudart.cudaEventCreate()[1] for _ in range(5)]

        def marks(i, evs=evs):
            st = torch.cuda.current_stream().cuda_stream
            cudart.cudaEventRecordWithFlags(evs[i], st, cudart.cudaEventRecordExternal)

        timed = rnd.capture(marks)
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        assert int(o["status"].item()) == 0, "device status raised (%s)" % name
        a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            graph.replay()
        e.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(e) / steps
        per = {n: [] for n in ("topk", "tree", "attn", "walk")}
        for _ in range(5):
            timed.replay()
            torch.cuda.synchronize()
            for i, n in enumerate(per):
                per[n].append(cudart.cudaEventElapsedTime(evs[i], evs[i + 1])[1] * 1e3)
        us = {n: statistics.median(v) for n, v in per.items()}
        n_nodes = o["n_nodes"].long().cpu().numpy()
        ctx = x["ctx_len"].long().cpu().numpy()
        rows = w.batch * w.L
        topk_b = rows * w.V * 2 + rows * w.k * 12 + rows * 4
        attn_b = (int(ctx.sum()) * w.hkv * w.d * 2 * 2 + 2 * int(n_nodes.sum()) * w.hq * w.d * 2 +
                  2 * int(n_nodes.sum()) * w.hkv * w.d * 2)
        attn_f = 4.0 * w.d * w.hq * float((n_nodes * (ctx + n_nodes)).sum())
        acc = o["acc_len"].long().cpu().numpy()
        walk_mode = api.tree_walk_resolve_mode(rnd.walk_mode, torch.float32, w.batch, w.n_max,
                                               w.V, w.L)
        walk_rows = int(n_nodes.sum()) if walk_mode == api.WALK_ALL_ROWS else int((acc + 1).sum())
        walk_b = walk_rows * w.V * 4
        t_hbm, t_tc = attn_b / (hbm_peak * 1e9), attn_f / (tf_peak * 1e12)
        st = {"topk": {"us": round(us["topk"], 2), "alg_bytes": topk_b,
                       "gbs": round(topk_b / us["topk"] / 1e3, 1),
                       "frac_hbm": round(topk_b / us["topk"] / 1e3 / hbm_peak, 4)},
              "tree": {"us": round(us["tree"], 2), "bound": "latency"},
              "attn": {"us": round(us["attn"], 2), "alg_bytes": attn_b, "alg_flops": attn_f,
                       "gbs": round(attn_b / us["attn"] / 1e3, 1),
                       "tflops": round(attn_f / us["attn"] / 1e6, 1),
                       "bound": "tensor" if t_tc > t_hbm else "hbm",
                       "frac_binding": round(max(t_hbm, t_tc) / (us["attn"] * 1e-6), 4)},
              "walk": {"us": round(us["walk"], 2), "mode": "all rows" if walk_mode == 0 else
                       "path only", "alg_bytes": walk_b,
                       "gbs": round(walk_b / us["walk"] / 1e3, 1),
                       "rows_read": walk_rows}}
        out[name] = {"rounds_per_s": round(w.batch / (ms * 1e-3), 1), "ms_per_round": round(ms, 4),
                     "steps": steps, "batch": w.batch, "mean_accepted": round(float(acc.mean()), 3),
                     "stages": st,
                     "inputs": "generated on the GPU; %.2f GB per set, above L2"
                               % (sum(t.numel() * t.element_size() for t in x.values()) / 1e9)}
        for ev in evs:
            cudart.cudaEventDestroy(ev)
        del graph, timed, rnd, x
        torch.cuda.empty_cache()
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist
    from cuda.bindings import runtime as cudart

    from block_draft_tree_b200 import synth
    from block_draft_tree_b200.round import VerifyRound

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    w = synth.WORKLOADS[WORKLOAD]
    hbm_peak, tf_peak, peak_kind = peaks()

    rnd = VerifyRound(batch=w.batch, L=w.L, V=w.V, k=w.k, B_max=w.B, hq=w.hq, hkv=w.hkv, d=w.d,
                      max_ctx=w.ctx, draft_dtype=torch.bfloat16, target_dtype=torch.float32,
                      inv_temperature=w.inv_temperature)
    sets, hosts = [], []
    for s in range(args.sets):
        xh, seed = make_inputs(w, rank, s)
        xd = to_device(xh, w, torch)
        xd["target"] = torch.empty((w.batch, w.n_max, w.V), dtype=torch.float32, device="cuda")
        xd["target"].normal_()
        rnd.bind(xd)
        rnd.launch()
        torch.cuda.synchronize()
        o = rnd.out
        tgt = synth.target_logits(w, o["tok"].cpu().numpy(), o["parent"].cpu().numpy(),
                                  o["depth"].cpu().numpy(), o["n_nodes"].cpu().numpy(), seed=seed)
        xd["target"].copy_(torch.from_numpy(tgt))
        sets.append(xd)
        hosts.append((xh, tgt))
    set_bytes = input_set_bytes(w)

    # one graph per input set, with event nodes around the stages
    def make_events(n):
        evs = []
        for _ in range(n):
            err, e = cudart.cudaEventCreate()
            evs.append(e)
        return evs

    # per input set: a plain graph of the round, and the same round with
    # event-record nodes between the kernels (replayed once per set at the
    # end of the timed region, for the per-kernel durations)
    graphs, timed_graphs, stage_events = [], [], []
    for xd in sets:
        rnd_s = VerifyRound(batch=w.batch, L=w.L, V=w.V, k=w.k, B_max=w.B, hq=w.hq, hkv=w.hkv,
                            d=w.d, max_ctx=w.ctx, inv_temperature=w.inv_temperature)
        rnd_s.bind(xd)
        rnd_s.launch()  # allocate-free warm call outside capture
        torch.cuda.synchronize()
        evs = make_events(5)

        def marks(i, evs=evs):
            st = torch.cuda.current_stream().cuda_stream
            cudart.cudaEventRecordWithFlags(evs[i], st, cudart.cudaEventRecordExternal)

        graphs.append((rnd_s.capture(), rnd_s))
        timed_graphs.append(rnd_s.capture(marks))
        stage_events.append(evs)
    launches_per_step = kernel_nodes(graphs[0][1], torch, cudart)
    torch.cuda.synchronize()

    # correctness guard: every set's graph reproduces its eager round
    for (g, r), xd in zip(graphs, sets):
        g.replay()
    torch.cuda.synchronize()
    for g, r in graphs:
        assert int(r.out["status"].item()) == 0, "device status raised"

    n_sets = len(graphs)

    def load_for(seconds):
        """Untimed replays for `seconds`, so that the clock sampler sees the
        GPU under the same load just before and just after the timed region."""
        t_end = time.perf_counter() + seconds
        i = 0
        while time.perf_counter() < t_end:
            graphs[i % n_sets][0].replay()
            i += 1
            if i % 64 == 0:
                torch.cuda.synchronize()
        torch.cuda.synchronize()

    clocks = ClockSampler(local) if rank == 0 else None
    if clocks:
        clocks.start()
    for i in range(args.warmup):
        graphs[i % n_sets][0].replay()
    load_for(args.clock_window_s)
    if world > 1:
        dist.barrier()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    n_plain = max(0, args.steps - n_sets)
    start.record()
    for i in range(n_plain):
        graphs[i % n_sets][0].replay()
    for i in range(n_plain, args.steps):  # the last step of every set: instrumented
        timed_graphs[i % n_sets].replay()
    end.record()
    torch.cuda.synchronize()
    load_for(args.clock_window_s)
    clk = clocks.stop() if clocks else None
    if clk is not None:
        clk["window"] = ("nvidia-smi every 100 ms from %.1f s of untimed replays before the timed "
                         "region to %.1f s after it" % (args.clock_window_s, args.clock_window_s))
    elapsed_ms = max_over_ranks(start.elapsed_time(end), world, "cuda")
    if world > 1:
        dist.barrier()

    # per-stage durations: the instrumented replays that end the timed region
    names = ["topk", "tree", "attn", "walk"]
    per_stage = {n: [] for n in names}
    for evs in stage_events:
        for i, n in enumerate(names):
            err, ms = cudart.cudaEventElapsedTime(evs[i], evs[i + 1])
            per_stage[n].append(ms)
    stage_us = {n: 1e3 * statistics.mean(v) for n, v in per_stage.items()}
    n_nodes_total = statistics.mean(int(r.out["n_nodes"].sum().item()) for _, r in graphs)
    sb = stage_bytes(w, n_nodes_total)
    stages = {}
    for n in names:
        t_s = stage_us[n] * 1e-6
        gbs = sb[n] / t_s / 1e9 if sb[n] else None
        stages[n] = {"us": round(stage_us[n], 3), "alg_bytes": sb[n],
                     "gbs": round(gbs, 1) if gbs else None,
                     "frac_hbm": round(gbs / hbm_peak, 4) if gbs else None}
    stages["attn"]["tflops"] = round(sb["attn_flops"] / (stage_us["attn"] * 1e-6) / 1e12, 2)
    dom = max(["topk", "attn", "walk"], key=lambda n: stage_us[n])
    tags = {"topk": "topk", "attn": "attn", "walk": "walk"}  # keys of profiles/traffic.json
    roof = {"kernel": dom, "bound": "hbm", "achieved": stages[dom]["gbs"], "peak": hbm_peak,
            "unit": "GB/s", "frac": stages[dom]["frac_hbm"],
            "traffic": traffic_for(tags[dom]),
            "peak_kind": "%s (MEASURED_PEAKS.json hbm_gbs)" % peak_kind if peak_kind == "measured"
            else "fallback"}
    acc = [r.out["acc_len"].float().mean().item() for _, r in graphs]

    # end to end: pinned host inputs -> H2D -> round -> D2H of the result, every step
    e2e = None
    if rank == 0 or world > 1:
        pins = []
        for (xh, tgt), xd in zip(hosts, sets):
            ph = {k: torch.empty_like(v, device="cpu").pin_memory() for k, v in xd.items()
                  if k in ("draft", "q", "k_tree", "v_tree", "target", "root")}
            for k in ph:
                ph[k].copy_(xd[k].cpu())
            pins.append(ph)
        res_host = [torch.empty(w.batch * (2 + w.L), dtype=torch.int32).pin_memory() for _ in sets]
        h2d = sum(v.numel() * v.element_size() for v in pins[0].values())
        d2h = res_host[0].numel() * 4

        def e2e_step(i):
            j = i % len(graphs)
            xd, (g, r) = sets[j], graphs[j]
            for k, v in pins[j].items():
                xd[k].copy_(v, non_blocking=True)
            g.replay()
            o = r.out
            res = torch.cat([o["acc_len"], o["bonus"], o["acc_tok"].reshape(-1)])
            res_host[j].copy_(res, non_blocking=True)

        for i in range(max(3, args.warmup // 10)):
            e2e_step(i)
        torch.cuda.synchronize()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record()
        for i in range(args.e2e_steps):
            e2e_step(i)
        e2.record()
        torch.cuda.synchronize()
        ms = max_over_ranks(s2.elapsed_time(e2), world, "cuda")
        e2e = {"value": job_throughput(world, w.batch, args.e2e_steps, ms), "unit": "rounds/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps}
        # the graphs overwrote the target buffers with the same data: nothing to restore

    if world > 1:
        dist.barrier()
    if rank != 0:
        if world > 1:
            for g, _ in graphs:
                del g
            dist.destroy_process_group()
        return 0

    # Rank 0 alone, after the last collective: the other ranks never wait on
    # these in a collective, whatever the process group's timeout.
    ext = measure_extensions(w, sets, graphs, hbm_peak) if not args.no_extensions else None
    per_wl = (measure_per_workload(args.per_workload.split(","), hbm_peak, tf_peak,
                                   max(10, min(args.steps, PER_WORKLOAD_MAX_STEPS)))
              if not args.no_per_workload else None)
    sweep = (budget_sweep(w, [int(b) for b in args.line_budgets.split(",")], args.sweep_batch,
                          args.line_sweep_draws, args.sweep_invt)
             if not args.no_budget_sweep else None)

    cpu = None
    if not args.no_cpu_baseline and world == 1:
        xh, _ = hosts[0]
        usable, total = host_cores()
        threads = args.cpu_threads or usable
        t0 = time.perf_counter()
        round_mt, parts_mt = cpu_baseline(w, xh, attn_fraction=1.0, threads=threads)
        t1 = time.perf_counter()
        round_st, parts_st = cpu_baseline(w, xh, attn_fraction=1.0, threads=1)
        t2 = time.perf_counter()
        cpu = {"value": w.batch / round_mt, "unit": "rounds/s", "cores": threads,
               "host_cores": total, "kind": "oracle",
               "sample": "one full b64 round (all %d attention items) of input set 0, fp64 C "
                         "oracle on %d threads (%.1f s), and again on one thread (%.1f s)"
                         % (parts_mt["attn_rows"], threads, t1 - t0, t2 - t1),
               "stage_s": {k: round(v, 4) for k, v in parts_mt.items() if k.endswith("_s")},
               "single_thread": {"value": w.batch / round_st, "unit": "rounds/s", "cores": 1,
                                 "stage_s": {k: round(v, 4) for k, v in parts_st.items()
                                             if k.endswith("_s")}}}

    value = job_throughput(world, w.batch, args.steps, elapsed_ms)
    line = {"metric": METRIC, "value": value, "unit": "rounds/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": workload_config(w, args.sets, set_bytes),
            "roofline": roof, "stages": stages, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps, "clocks": clk,
            "mean_accepted": round(statistics.mean(acc), 3), "extensions": ext,
            "per_workload": per_wl, "budget_sweep": sweep,
            "parallelism": "dp%d (independent sequences per GPU)" % world}
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_profile(args):
    """Four rounds of one input set, each after an L2 flush (a target for ncu)."""
    import torch
    from block_draft_tree_b200 import synth
    from block_draft_tree_b200.round import VerifyRound

    w = synth.WORKLOADS[args.workload or WORKLOAD]
    xh, seed = make_inputs(w, 0, 0)
    ps = w.page_size or 64
    max_ctx = int(xh["ctx_len"].max())  # the page table covers the longest context drawn
    rnd = VerifyRound(batch=w.batch, L=w.L, V=w.V, k=w.k, B_max=w.B, hq=w.hq, hkv=w.hkv, d=w.d,
                      max_ctx=max_ctx, draft_dtype=torch.bfloat16, target_dtype=torch.float32,
                      inv_temperature=w.inv_temperature, paged=w.page_size > 0, page_size=ps,
                      max_pages=(max_ctx + ps - 1) // ps)
    xd = to_device(xh, w, torch)
    xd["target"] = torch.randn((w.batch, w.n_max, w.V), dtype=torch.float32, device="cuda")
    rnd.bind(xd)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    from block_draft_tree_b200 import api
    o = rnd.out
    if args.extensions:
        g = torch.Generator(device="cuda")
        g.manual_seed(77)
        hid = (torch.randn(w.batch, w.n_max, LM_HIDDEN, device="cuda", generator=g) * 0.5).bfloat16()
        head = (torch.randn(w.V, LM_HIDDEN, device="cuda", generator=g) / LM_HIDDEN ** 0.5).bfloat16()
    for i in range(4):
        flush.fill_(i)
        rnd.launch()
        if args.extensions:  # the calls beyond the round, on the round's own outputs
            api.tree_walk_sample(xd["target"], o["tok"], o["parent"], o["depth"], o["n_nodes"],
                                 w.L, 1.0, seed=12345, step=i)
            cl = xd["ctx_len"].clone()
            api.kv_commit(xd["k_tree"], xd["v_tree"], o["acc_len"], o["acc_nodes"], cl,
                          xd["k_cache"].clone(), xd["v_cache"].clone(),
                          page_table=xd.get("page_table"), page_size=w.page_size or 64)
            api.lm_head_walk(hid, head, o["tok"], o["parent"], o["depth"], o["n_nodes"], w.L)
    torch.cuda.synchronize()
    print(json.dumps({"profile": w.name, "rounds": 4, "status": int(rnd.out["status"].item()),
                      "extensions": bool(args.extensions)}))
    return 0


def plant_targets(target, probs, depth, n_nodes, L, gen):
    """Synthetic target logits for the budget sweep: every tree row of depth
    d < L gets, on top of ``target``'s N(0,1) noise, a logit of 100 at a token
    drawn from the drafter's marginal q_{d+1} (``probs`` [batch, L, V]), one
    independent draw per row; so a greedy walk accepts a path with exactly the
    probability the factorised draft gives it, and the expected accepted
    length is the tree's surrogate (DDTree page, 理論基礎, Proposition 1).
    Returns the planted tokens [batch, n_max] (-1 where nothing is planted)."""
    import torch
    b, n_max, _ = target.shape
    draws = torch.multinomial(probs.reshape(b * L, -1), n_max, replacement=True,
                              generator=gen).reshape(b, L, n_max)
    rows = torch.arange(n_max, device=target.device)
    live = (rows[None, :] < n_nodes[:, None]) & (depth < L)
    pos = depth.clamp(0, L - 1).long()
    tok = torch.gather(draws, 1, pos[:, None, :]).squeeze(1)
    tok = torch.where(live, tok, torch.full_like(tok, -1))
    bi, xi = torch.nonzero(live, as_tuple=True)
    target[bi, xi, tok[bi, xi]] = 100.0
    return tok


def budget_sweep(w0, budgets, batch, draws, invt, spread=(0.5, 1.5), seed=2024, adaptive=True):
    """Budget sweep (DDTree page, 實驗結果與權衡: acceptance grows with the node
    budget B while the verifier's cost grows too) on a batch whose sequences
    draft with different confidence (sequence b's draft logits scaled by a
    factor from ``spread``).  For each B: device time of one round (CUDA
    graph, median of launches after an L2 flush) and the mean accepted
    length over target resamplings planted from the drafter's own marginals
    (so that its expectation is the tree's surrogate, Proposition 1).  A
    linear fit of round time against the batch's draft nodes gives a cost
    model, and the adaptive round (ddt_plan_budget between two builds, the
    largest B as every sequence's cap) is measured the same way."""
    import torch
    from block_draft_tree_b200.round import VerifyRound

    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    Bmax = max(budgets)
    wmax = w0.scaled(batch=batch, B=Bmax, inv_temperature=invt)
    x, _ = device_inputs(wmax, seed)
    scale = torch.linspace(spread[0], spread[1], batch, device="cuda")
    x["draft"] = (x["draft"].float() * scale[:, None, None]).to(torch.bfloat16)
    probs = torch.softmax(x["draft"].float() * invt, dim=-1)

    def inputs_for(n_max):
        xd = dict(x)
        for key in ("q", "k_tree", "v_tree", "target"):
            xd[key] = x[key][:, :n_max].contiguous()
        return xd

    def measure(rnd, xd, n_max):
        rnd.bind(xd)
        rnd.launch()
        torch.cuda.synchronize()
        o = rnd.out
        acc, surr, nodes = [], [], []
        for _ in range(draws):
            xd["target"].normal_(generator=gen)
            plant_targets(xd["target"], probs, o["depth"], o["n_nodes"], w0.L, gen)
            rnd.launch()
            acc.append(o["acc_len"].double().mean().item())
            surr.append(o["surrogate"].mean().item())
            nodes.append(int(o["n_nodes"].sum().item()) - batch)
        g = rnd.capture()
        times = []
        for rep in range(23):
            flush.zero_()
            a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            g.replay()
            e.record()
            torch.cuda.synchronize()
            if rep >= 3:
                times.append(a.elapsed_time(e) * 1e3)
        assert int(o["status"].item()) == 0, "device status raised"
        us = statistics.median(times)
        mean_acc = statistics.mean(acc)
        row = {"round_us": round(us, 2), "draft_nodes": round(statistics.mean(nodes), 1),
               "mean_accepted": round(mean_acc, 3), "surrogate": round(statistics.mean(surr), 3),
               "accepted_se": round(statistics.pstdev(acc) / max(1, len(acc)) ** 0.5, 3),
               "tokens_per_s": round(batch * (mean_acc + 1) / (us * 1e-6), 1)}
        del g
        return row

    rows = []
    for B in budgets:
        w = w0.scaled(batch=batch, B=B, inv_temperature=invt)
        rnd = VerifyRound(batch=batch, L=w.L, V=w.V, k=w.k, B_max=B, hq=w.hq, hkv=w.hkv, d=w.d,
                          max_ctx=w.ctx, inv_temperature=invt)
        row = dict(B=B, **measure(rnd, inputs_for(B + 1), B + 1))
        rows.append(row)
        print("# sweep row", json.dumps(row), file=sys.stderr, flush=True)
        del rnd
    # round time against draft nodes: least squares c0 + c1 * nodes
    xs = np.array([r["draft_nodes"] for r in rows])
    ys = np.array([r["round_us"] for r in rows])
    c1, c0 = np.polyfit(xs, ys, 1)
    out = {"workload": "%s shapes at batch %d" % (w0.name, batch), "draws": draws,
           "draft_inv_temperature": invt,
           "confidence_spread": "draft logits of sequence b scaled by %.2f .. %.2f" % spread,
           "target": "argmax planted from the drafter's marginals per row", "rows": rows,
           "cost_model": {"c0_us": round(float(c0), 2), "c1_us_per_node": round(float(c1), 4)}}
    if adaptive and c1 > 0 and c0 > 0:
        rnd = VerifyRound(batch=batch, L=w0.L, V=w0.V, k=w0.k, B_max=Bmax, hq=w0.hq, hkv=w0.hkv,
                          d=w0.d, max_ctx=w0.ctx, inv_temperature=invt,
                          adaptive_budget={"total": -1, "cost_fixed": float(c0),
                                           "cost_per_node": float(c1)})
        row = measure(rnd, inputs_for(Bmax + 1), Bmax + 1)
        row["budgets"] = rnd.out["budget"].cpu().tolist()
        out["adaptive"] = dict(cap=Bmax, **row)
        best = max(rows, key=lambda r: r["tokens_per_s"])
        out["best_fixed"] = {"B": best["B"], "tokens_per_s": best["tokens_per_s"]}
        print("# adaptive", json.dumps(out["adaptive"]), file=sys.stderr, flush=True)
        del rnd
    del x, probs
    torch.cuda.empty_cache()
    return out


def run_sweep(args):
    """The budget sweep alone (see budget_sweep), one JSON line."""
    from block_draft_tree_b200 import synth
    w0 = synth.WORKLOADS[args.workload or WORKLOAD]
    budgets = [int(x) for x in args.budgets.split(",")]
    res = budget_sweep(w0, budgets, args.sweep_batch, args.sweep_draws, args.sweep_invt)
    print(json.dumps({"sweep": res}), flush=True)
    return 0


def run_stage_sweep(args):
    """Each stage kernel timed alone on every workload (CUDA events, an L2
    flush before each launch, median of 15), with its algorithmic bytes and
    flops and the fraction of its binding roofline (measured peaks)."""
    import torch
    from block_draft_tree_b200 import synth
    from block_draft_tree_b200.round import VerifyRound

    hbm_peak, tf_peak, peak_kind = peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    out = []
    for name in args.stage_workloads.split(","):
        w = synth.WORKLOADS[name]
        ps = w.page_size or 64
        xh, _ = make_inputs(w, 0, 0)
        max_ctx = int(xh["ctx_len"].max())  # the page table covers the longest context drawn
        rnd = VerifyRound(batch=w.batch, L=w.L, V=w.V, k=w.k, B_max=w.B, hq=w.hq, hkv=w.hkv,
                          d=w.d, max_ctx=max_ctx, draft_dtype=torch.bfloat16,
                          target_dtype=torch.float32, inv_temperature=w.inv_temperature,
                          paged=w.page_size > 0, page_size=ps, max_pages=(max_ctx + ps - 1) // ps)
        xd = to_device(xh, w, torch)
        xd["target"] = torch.randn((w.batch, w.n_max, w.V), dtype=torch.float32, device="cuda")
        rnd.bind(xd)
        rnd.launch()
        torch.cuda.synchronize()
        times = {}
        for i, stage in enumerate(("topk", "tree", "attn", "walk")):
            ts = []
            for rep in range(18):
                flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                rnd.launch_stage(i)
                b.record()
                torch.cuda.synchronize()
                if rep >= 3:
                    ts.append(a.elapsed_time(b) * 1e3)
            times[stage] = statistics.median(ts)
        assert int(rnd.out["status"].item()) == 0, "device status raised"
        n_nodes = rnd.out["n_nodes"].cpu().numpy().astype(np.int64)
        ctx = xh["ctx_len"].astype(np.int64)
        rows = w.batch * w.L
        topk_b = rows * w.V * 2 + rows * w.k * 12 + rows * 4
        kv_b = int(ctx.sum()) * w.hkv * w.d * 2 * 2
        attn_b = kv_b + 2 * int(n_nodes.sum()) * w.hq * w.d * 2 + 2 * int(n_nodes.sum()) * w.hkv * w.d * 2
        attn_f = 4.0 * w.d * w.hq * float((n_nodes * ctx).sum())
        walk_b = int(n_nodes.sum()) * w.V * 4
        row = {"workload": name}
        for stage, byts in (("topk", topk_b), ("walk", walk_b)):
            us = times[stage]
            gbs = byts / (us * 1e-6) / 1e9
            row[stage] = {"us": round(us, 2), "alg_bytes": byts, "gbs": round(gbs, 1),
                          "frac_hbm": round(gbs / hbm_peak, 3)}
        us = times["attn"]
        gbs = attn_b / (us * 1e-6) / 1e9
        tfl = attn_f / (us * 1e-6) / 1e12
        t_hbm, t_tc = attn_b / (hbm_peak * 1e9), attn_f / (tf_peak * 1e12)
        row["attn"] = {"us": round(us, 2), "alg_bytes": attn_b, "alg_flops": attn_f,
                       "gbs": round(gbs, 1), "tflops": round(tfl, 1),
                       "bound": "tensor" if t_tc > t_hbm else "hbm",
                       "frac_binding": round(max(t_hbm, t_tc) / (us * 1e-6), 3)}
        row["tree"] = {"us": round(times["tree"], 2), "bound": "latency (one CTA per sequence)"}
        out.append(row)
        print("# " + json.dumps(row), file=sys.stderr, flush=True)
        del rnd, xd
        torch.cuda.empty_cache()
    print(json.dumps({"stage_sweep": out, "peaks": {"hbm_gbs": hbm_peak, "bf16_tflops": tf_peak,
                                                    "kind": peak_kind},
                      "timing": "each kernel alone, L2 flushed before each launch, median of 15"}),
          flush=True)
    return 0


def main():
    args = parse()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return relaunch_as_ranks(args.gpus)
    if args.selftest_ranks:
        return run_selftest_ranks(args)
    if args.impl == "reference":
        return run_reference(args)
    if args.profile:
        return run_profile(args)
    if args.sweep:
        return run_sweep(args)
    if args.stage_sweep:
        return run_stage_sweep(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())

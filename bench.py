#!/usr/bin/env python3
"""Benchmark of the routed sparse-attention decode step (MSA) on B200.

Workload: batched decode on a shared 4.19M-token memory bank -- batch 8, 32
query heads / 8 KV heads, head_dim 128, 1024 documents x 4096 tokens, 4096-token
local context, 1 query token, top_k = 16 documents per (sequence, KV head),
bf16 storage, fp32 accumulation, seeded synthetic N(0,1) inputs.

One step = msa_route + msa_attend through the C ABI (identical to msa_forward):
q_r, cosine router over every chunk of K_r, top-k, split-KV attention, merge.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Multi-GPU: each rank runs an independent replica (the step does not shard);
value = all ranks' queries / max-over-ranks device time.
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

WORKLOAD = "decode_4m"
METRIC = "decode queries/s on 4M-tok bank; router+attn HBM GB/s as % of B200 peak"
L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="time only --workload (the default run also times prefill and the two host-tier banks)")
    ap.add_argument("--cpu-steps", type=int, default=3,
                    help="whole oracle steps timed for the cpu_baseline (after one untimed step)")
    ap.add_argument("--workload", default=WORKLOAD, choices=[WORKLOAD, "decode_512k", "prefill", "prefill_64docs", "prefill_short_docs", "ragged_planted", "bank_100m"],
                    help="decode_512k: the same step on a 128-document bank (profiling captures); "
                         "prefill: 4096 query tokens in 64-token routing blocks (tensor-bound)")
    ap.add_argument("--kv-cache-gb", type=float, default=0.0,
                    help="host-tier workloads: device-resident slab cache of this many GB (msa_set_kv_cache); "
                         "each step then takes one of --query-pool query batches at random")
    ap.add_argument("--query-pool", type=int, default=4)
    ap.add_argument("--host-fetch", default="gather", choices=["gather", "copy"],
                    help="host-tier workloads: move the selected slabs with the SM gather kernel through the "
                         "mapped pinned K/V (default) or with cudaMemcpyAsync copies (msa_set_host_fetch)")
    ap.add_argument("--backward", action="store_true",
                    help="time msa_attend_backward on --workload's selection (gradients of the queries, "
                         "local K/V and bank K/V)")
    ap.add_argument("--build-only", action="store_true",
                    help="time msa_build_bank (chunk-mean pooling of the routing keys + Parallel RoPE of the "
                         "bank keys, in place) over the whole bank of --workload")
    ap.add_argument("--kr-bf16", action="store_true",
                    help="the reduced-precision router: read only the bf16 high part of the normalised K_r "
                         "(msa_set_router_precision(MSA_KR_BF16)), half the router's bytes")
    ap.add_argument("--memory-parallel", type=int, default=0, metavar="S",
                    help="Memory Parallel: the bank split into document shards. With one process, S shard banks "
                         "on one GPU (stacks in place of the all-gathers); under torchrun, one shard per rank and "
                         "NCCL all-gathers (S is then the world size)")
    ap.add_argument("--route-only", action="store_true",
                    help="time msa_route alone on the full bank's K_r with a stand-in 1-document K/V "
                         "(routing keys streamed in slices; a few GB on the device, for profiling captures)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            m = json.load(f)
        return float(m["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def tensor_peak(sustained: bool = False):
    """Dense bf16 TFLOP/s: the burst figure (a kernel timed alone), or the sustained one
    (cuBLAS back to back under the power cap), for a kernel timed inside a long run."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            peaks_ = json.load(f)
        if sustained and "bf16_tflops_sustained" in peaks_:
            return float(peaks_["bf16_tflops_sustained"]), "measured, sustained (timed after >= 1 s of the same load)"
        return float(peaks_["bf16_tflops"]), "measured"
    return (1400.0, "fallback, sustained") if sustained else (1590.0, "fallback")


SETTLE_S = 1.0   # tensor-bound steps run this long before timing: the clocks under the power cap settle


def settle(fn, min_steps: int, min_s: float = SETTLE_S):
    """Runs fn at least min_steps times and for at least min_s seconds of GPU work."""
    import torch
    t0 = time.perf_counter()
    n = 0
    while n < min_steps or time.perf_counter() - t0 < min_s:
        fn()
        n += 1
        if n % 4 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()


def launches_per_step(w, batch=None, gather=False) -> int:
    """Kernels libmsa launches for one route + attend step of workload w (over `batch`
    sequences; msa_forward on a pinned-host bank runs micro-batches of up to 2 parts,
    each with one slab-gather launch when the SM gather moves the slabs)."""
    if batch is None and w.host_tier:
        parts = min(w.batch, 2)
        nb = -(-w.batch // parts)
        sizes = [min(nb, w.batch - b0) for b0 in range(0, w.batch, nb)]
        return sum(launches_per_step(w, b) + (1 if gather else 0) for b in sizes)
    batch = w.batch if batch is None else batch
    rows_route = batch * (w.q_tokens // w.route_block)
    n = (0 if w.route_block <= 4 else 1) + (rows_route + 15) // 16 + 1     # qr_prep, router passes, top-k
    rows = (w.n_q_heads // w.n_kv_heads) * w.route_block
    tc = w.head_dim == 128 and w.route_block in (64, 128) and rows % 128 == 0
    # decode kernel | rope_local (+ rope of the queries for the tcgen05 kernel) + prefill kernel
    n += 1 if rows <= 16 else (3 if tc else 2)
    return n


# ----------------------------------------------------------------- CPU oracle
# The oracle as it stands, run on whole decode steps of the bench workload. One
# step = every sequence of the batch: for each (sequence, KV head) the oracle's
# router over every chunk of K_r, its top-k, and its attention for the G query
# heads of that KV head. The (sequence, KV head) items are spread over worker
# processes (spawned; each single-threaded: BLAS threads pinned to 1), so the
# thread count is the worker count. K_r is pooled by the oracle from the
# workload's routing keys, and the selected documents' keys carry the oracle's
# Parallel RoPE: both are offline bank state, built before the first step.

_ONE_THREAD = {v: "1" for v in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS",
                                "NUMEXPR_NUM_THREADS", "VECLIB_MAXIMUM_THREADS")}
# the workers allocate and free many multi-MB numpy temporaries: keep glibc from
# returning each one to the kernel (mmap / munmap page-fault churn)
_ONE_THREAD.update({"MALLOC_MMAP_THRESHOLD_": "33554432", "MALLOC_TRIM_THRESHOLD_": "2147483647"})


def _oracle_worker(conn, wname, items):
    """Serves oracle steps for a fixed list of (sequence, KV head) items."""
    import synth
    from oracle import msa_oracle as O

    f64 = lambda bits: synth.bf16_bits_to_f32(bits).astype(np.float64)
    w = synth.WORKLOADS[wname]
    n, d, Hkv, Hq = w.n_docs, w.head_dim, w.n_kv_heads, w.n_q_heads
    G, lens = Hq // Hkv, w.doc_lens()
    off = np.concatenate([[0], np.cumsum(lens)])
    t_setup = time.perf_counter()
    kr, chunk_doc = {}, None
    for h in sorted({h for _, h in items}):   # offline bank build: pooling of the routing keys
        rows, owner = [], []
        for j in range(n):
            rows.append(O.chunk_mean_pool(f64(synth.bank_rows_bits(w, synth.T_R, h, int(off[j]), int(lens[j])))))
            owner.extend([j] * rows[-1].shape[0])
        kr[h], chunk_doc = np.concatenate(rows), np.asarray(owner, dtype=np.int64)
    Qr = f64(synth.query_bits(w, synth.T_QR, (w.batch, Hkv, w.q_tokens, d)))
    Q = f64(synth.query_bits(w, synth.T_Q, (w.batch, Hq, w.q_tokens, d)))
    k_off = O.k_offset(w.top_k, lens)
    conn.send(("ready", time.perf_counter() - t_setup))
    cache = {}
    while True:
        cmd = conn.recv()
        if cmd is None:
            break
        misses, excluded = 0, 0.0
        t0 = time.perf_counter()
        for b, h in items:
            for blk in range(w.q_tokens // w.route_block):
                qb = O.block_mean_query(Qr[b, h], w.route_block)[blk]
                sel = O.select_top_k(O.route_doc_scores(qb, kr[h], chunk_doc, n), w.top_k)
                key = (b, h, tuple(int(j) for j in sel))
                if key not in cache:
                    # bank keys with Parallel RoPE and the values of the selected documents
                    # (offline bank state), the local K/V: inputs, outside the step's time
                    t_in = time.perf_counter()
                    mk = np.concatenate([O.parallel_rope_bank(f64(synth.bank_rows_bits(w, synth.T_K, h, int(off[j]),
                                                                                        int(lens[j]))),
                                                              [int(lens[j])], w.rope_base) for j in sel])
                    mv = np.concatenate([f64(synth.bank_rows_bits(w, synth.T_V, h, int(off[j]), int(lens[j])))
                                         for j in sel])
                    base = (b * Hkv + h) * w.local_len * d
                    lk = f64(synth.normal_bf16_bits(w.seed, synth.T_LK, base, w.local_len * d)).reshape(-1, d)
                    lv = f64(synth.normal_bf16_bits(w.seed, synth.T_LV, base, w.local_len * d)).reshape(-1, d)
                    cache[key] = (mk, mv, lk, lv)
                    misses += 1
                    excluded += time.perf_counter() - t_in
                mk, mv, lk, lv = cache[key]
                for g in range(G):
                    for t in range(blk * w.route_block, (blk + 1) * w.route_block):
                        O.routed_attention_row(Q[b, h * G + g, t], w.local_len - w.q_tokens + t, k_off,
                                               w.rope_base, mk, mv, lk, lv)
        conn.send((time.perf_counter() - t0 - excluded, misses))


class OracleSteps:
    """Worker processes that run whole oracle steps of a workload on the host cores."""

    def __init__(self, wname: str):
        import multiprocessing as mp
        import synth
        w = synth.WORKLOADS[wname]
        self.units = w.batch * w.q_tokens          # queries (decode) per step
        items = [(b, h) for h in range(w.n_kv_heads) for b in range(w.batch)]
        try:
            avail = len(os.sched_getaffinity(0))
        except AttributeError:
            avail = os.cpu_count() or 1
        self.workers = max(1, min(avail, len(items)))
        ctx = mp.get_context("spawn")   # the parent may hold a CUDA context: never fork it
        saved = {k: os.environ.get(k) for k in _ONE_THREAD}
        os.environ.update(_ONE_THREAD)
        self.procs, self.conns = [], []
        try:
            for i in range(self.workers):
                a, b = ctx.Pipe()
                # contiguous blocks of the head-major item list: a worker pools as few heads as possible
                mine = items[i * len(items) // self.workers:(i + 1) * len(items) // self.workers]
                p = ctx.Process(target=_oracle_worker, args=(b, wname, mine), daemon=True)
                p.start()
                self.procs.append(p)
                self.conns.append(a)
        finally:
            for k, v in saved.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v
        self.setup_s = max(c.recv()[1] for c in self.conns)

    def step(self):
        """One whole step; returns (wall seconds, cache misses)."""
        t0 = time.perf_counter()
        for c in self.conns:
            c.send(1)
        replies = [c.recv() for c in self.conns]
        return time.perf_counter() - t0, sum(m for _, m in replies)

    def close(self):
        for c in self.conns:
            c.send(None)
        for p in self.procs:
            p.join(timeout=30)


def oracle_timed(wname: str, steps: int, warmup: int):
    """Runs `warmup` untimed and `steps` timed whole oracle steps; returns a dict."""
    runner = OracleSteps(wname)
    try:
        for _ in range(warmup):
            runner.step()
        walls, misses = [], 0
        for _ in range(steps):
            wall, m = runner.step()
            walls.append(wall)
            misses += m
    finally:
        runner.close()
    mean = sum(walls) / len(walls)
    return {"value": runner.units / mean, "ms_per_step": 1000.0 * mean, "steps": steps, "warmup": warmup,
            "cores": runner.workers, "setup_s": runner.setup_s, "timed_misses": misses,
            "total_s": sum(walls)}


def oracle_sample_text(r: dict, w) -> str:
    nch = int(sum(-(-int(L) // 256) for L in w.doc_lens()))
    return (f"{r['steps']} whole decode steps of {w.batch} queries after {r['warmup']} untimed "
            f"({r['total_s']:.1f} s timed): per (sequence, KV head) the oracle's router over all {nch} "
            f"chunks of K_r (pooled by the oracle from the routing keys), its top-{w.top_k}, and its "
            f"attention for the {w.n_q_heads // w.n_kv_heads} query heads; {r['cores']} single-threaded "
            f"worker processes; bank build (pooling, Parallel RoPE) not timed")


def step_bytes_estimate(w) -> float:
    """HBM bytes a step reads at most (no shared documents): K_r once, the selected
    documents' K/V per (sequence, routing block, KV head), the local K/V."""
    nblk = w.q_tokens // w.route_block
    nch = int(sum(-(-int(L) // 256) for L in w.doc_lens()))
    return (w.n_kv_heads * nch * w.route_dim * 4 + w.batch * nblk * w.n_kv_heads * w.top_k * w.max_len * w.head_dim * 4
            + w.batch * w.n_kv_heads * w.local_len * w.head_dim * 4)


def base_config(w, world: int = 1) -> dict:
    """The workload description both arms print (identical for the same workload and N)."""
    return {"workload": w.name, "batch": w.batch, "q_heads": w.n_q_heads, "kv_heads": w.n_kv_heads,
            "head_dim": w.head_dim, "bank_docs": w.n_docs, "doc_len": w.doc_len, "local_len": w.local_len,
            "q_tokens": w.q_tokens, "route_block": w.route_block, "top_k": w.top_k,
            "parallelism": f"replicas x{world}",
            "l2": f"inputs larger than L2: up to {step_bytes_estimate(w) / 1e9:.2f} GB read per step vs 126 MB L2"}


def run_reference(args):
    import synth
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = synth.WORKLOADS[WORKLOAD]
    r = oracle_timed(WORKLOAD, max(1, args.steps), max(0, args.warmup))
    line = {
        "impl": "reference", "metric": METRIC, "value": r["value"], "unit": "queries/s", "n_gpus": args.gpus,
        "steps": r["steps"], "warmup": r["warmup"], "ms_per_step": r["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": base_config(w, args.gpus),
        "cpu_baseline": {"value": r["value"], "unit": "queries/s", "cores": r["cores"], "kind": "oracle",
                         "sample": oracle_sample_text(r, w)},
        "e2e": {"value": r["value"], "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "reference_note": "the pages ship no code: the reference arm is the fp64 CPU oracle, timed as it stands",
        "setup_s": r["setup_s"],
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(gpu_index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        self.t_start = self.t_end = None

    def mark(self, start: bool):
        if start:
            self.t_start = time.time()
        else:
            self.t_end = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sms, maxes, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sms.append(float(parts[1]))
                maxes.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        load = [s for s in sms if s > 0.5 * (max(sms) if sms else 1)]
        return {"sm_mhz": statistics.median(load) if load else None,
                "sm_max_mhz": max(maxes) if maxes else None, "reasons": sorted(reasons), "samples": len(sms)}


# ----------------------------------------------------------------- ours
KERNEL_SOURCES = {
    "attend_decode": ["attend_decode.cu", "common.cuh", "pdl.cuh"],
    "attend_prefill_tc": ["attend_prefill_tc.cu", "common.cuh"],
}


def source_sha(kernel: str) -> str:
    """sha256 over the source files a kernel is compiled from (its .cu and the shared header)."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(ROOT, "sparse_attention_routed_b200", "csrc", f), "rb").read())
    return h.hexdigest()


def profile_traffic(profile: str, kernel: str):
    """DRAM bytes per launch from a committed ncu summary under profiles/, or None
    when the kernel's sources changed since the counters were taken."""
    prof = os.path.join(ROOT, "profiles", profile)
    if not os.path.exists(prof):
        return None
    vals = {}
    for line in open(prof):
        if ":" in line:
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    if vals.get("source_sha256") != source_sha(kernel):
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def max_over_ranks(values, device="cpu"):
    """Each timing's maximum over all ranks (the slowest replica sets the job's
    time); the values unchanged on a single process."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(world: int, units_per_step: float, steps: int, total_ms: float) -> float:
    """Whole-job throughput of `world` replicas that each processed `units_per_step`
    units in each of `steps` steps, over the max-over-ranks time `total_ms`."""
    return world * units_per_step * steps / (total_ms / 1000.0)


def measure_device(args, wname: str, n: int, warmup: int, world: int, rank: int, local: int,
                   with_e2e: bool = True):
    """Times n steps (msa_forward: route + attend through the C ABI) of a device-resident
    workload after `warmup` untimed ones, then n more as msa_route + msa_attend with an
    event between them for the two phases' times; returns the JSON line on rank 0
    (None elsewhere)."""
    import torch
    import torch.distributed as dist

    import synth
    from sparse_attention_routed_b200 import MSA_KR_BF16, msa_attend, msa_forward, msa_route, ptr
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors, query_tensors

    w = synth.WORKLOADS[wname]
    prefill = wname.startswith("prefill")
    K, V, R = bank_tensors(w)
    bank = Bank(K, V, w.doc_lens(), w.rope_base)
    bank.build(R)
    if args.kr_bf16:
        bank.set_router_precision(MSA_KR_BF16)
    torch.cuda.synchronize()
    del R
    torch.cuda.empty_cache()
    # the step's inputs and outputs live in a few contiguous device buffers (queries and
    # routing queries together, local K and V together, output and selection together),
    # so that the end-to-end run moves each group with one copy
    Q0, Qr0, LK0, LV0 = query_tensors(w)
    qin = torch.cat([Q0.reshape(-1), Qr0.reshape(-1)])
    Q, Qr = qin[:Q0.numel()].view(Q0.shape), qin[Q0.numel():].view(Qr0.shape)
    kvloc = torch.stack([LK0, LV0])
    LK, LV = kvloc[0], kvloc[1]
    del Q0, Qr0, LK0, LV0
    qry = bank.query(Q, Qr, LK, LV, w.route_block)
    bank.reserve(qry, w.top_k)
    B, k, Hkv, d = w.batch, w.top_k, w.n_kv_heads, w.head_dim
    nblk = w.q_tokens // w.route_block
    n_out, n_idx = B * w.n_q_heads * w.q_tokens * d, B * nblk * Hkv * k
    outbuf = torch.empty(4 * (n_out + n_idx), dtype=torch.uint8, device="cuda")
    out = outbuf[:4 * n_out].view(torch.float32).view(B, w.n_q_heads, w.q_tokens, d)
    idx = outbuf[4 * n_out:].view(torch.int32).view(B, nblk, Hkv, k)
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream

    def step():
        msa_forward(bank.handle, qry, k, idx.data_ptr(), out.data_ptr(), sh)

    for _ in range(max(3, warmup)):
        step()
        msa_route(bank.handle, qry, k, 0, idx.data_ptr(), 0, sh)
        msa_attend(bank.handle, qry, k, idx.data_ptr(), out.data_ptr(), sh)
    torch.cuda.synchronize()
    assert bank.device_error() == 0

    # algorithmic bytes and FLOPs of one step (the selection is fixed by the fixed inputs)
    sel = idx.cpu().numpy()
    lens = w.doc_lens()
    uniq = {(int(j), h) for b in range(B) for blk in range(nblk) for h in range(Hkv) for j in sel[b, blk, h]}
    kv_sel = sum(int(lens[j]) for j, _ in uniq) * d * 2 * 2
    kv_local = B * Hkv * w.local_len * d * 2 * 2
    q_out = B * w.n_q_heads * w.q_tokens * d * (2 + 4)
    nch = bank.info["n_chunks"]
    router = Hkv * nch * (d * (2 if args.kr_bf16 else 4)) + B * nblk * Hkv * w.n_docs * 4 * 2 + B * Hkv * w.q_tokens * d * 2
    attn_bytes = kv_sel + kv_local + q_out
    step_bytes = attn_bytes + router
    G = w.n_q_heads // w.n_kv_heads
    mem_keys = sum(int(lens[j]) for b in range(B) for blk in range(nblk) for h in range(Hkv)
                   for j in sel[b, blk, h]) * G * w.route_block
    first = w.local_len - w.q_tokens
    loc_keys = B * w.n_q_heads * sum(first + t + 1 for t in range(w.q_tokens))
    attn_flops = 4 * d * (mem_keys + loc_keys)

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    time.sleep(0.4)
    if prefill:
        # tensor-bound: the clocks under the 1 kW cap settle before anything is timed
        settle(step, 3)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(2 * n)]
    t_begin, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def phases(e):
        # the two phases on their own (not the headline): the router + top-k, then the attention
        for i in range(n):
            e[i][0].record(stream)
            msa_route(bank.handle, qry, k, 0, idx.data_ptr(), 0, sh)
            e[i][1].record(stream)
            msa_attend(bank.handle, qry, k, idx.data_ptr(), out.data_ptr(), sh)
            e[i][2].record(stream)

    clocks.mark(True)
    # n phase steps before and n after the timed steps, so that a clock that drifts under
    # the power cap weighs on the phase times as on the timed steps
    phases(ev[:n])
    t_begin.record(stream)
    for i in range(n):
        step()
    t_end.record(stream)
    phases(ev[n:])
    torch.cuda.synchronize()
    clocks.mark(False)
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    total_ms = t_begin.elapsed_time(t_end)
    route_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / len(ev)
    attend_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / len(ev)
    assert bank.device_error() == 0

    e2e_ms, n_e2e, h2d, d2h = None, 0, 0, 0
    if with_e2e:
        # e2e: pinned host inputs of each step copied in -- decode: queries, routing
        # queries and the newest local token's K/V; prefill: queries, routing queries
        # and the whole local K/V (the prompt) -- the step run, output + selection copied out.
        # Two buffer sets and two copy streams, as a server runs it: step i computes
        # while step i+1's inputs come in and step i-1's result goes out; every step
        # still moves its own bytes inside the timed region.
        qin_h = qin.cpu().pin_memory()
        kv_h = (kvloc if prefill else kvloc[:, :, :, -1]).cpu().pin_memory()  # decode: the newest token's K, V
        sets = [(qin, kvloc, outbuf, qry, out, idx)]
        qin1, kvloc1, outbuf1 = qin.clone(), kvloc.clone(), torch.empty_like(outbuf)
        Q1, Qr1 = qin1[:Q.numel()].view(Q.shape), qin1[Q.numel():].view(Qr.shape)
        qry1 = bank.query(Q1, Qr1, kvloc1[0], kvloc1[1], w.route_block)
        sets.append((qin1, kvloc1, outbuf1, qry1, outbuf1[:4 * n_out].view(torch.float32).view(out.shape),
                     outbuf1[4 * n_out:].view(torch.int32).view(idx.shape)))
        out_h = [torch.empty(outbuf.shape, dtype=outbuf.dtype, pin_memory=True) for _ in range(2)]
        h2d = qin_h.numel() * 2 + kv_h.numel() * 2
        d2h = out_h[0].numel()
        n_e2e = max(10, n)   # as many steps as the headline, so the pipeline's fill and drain weigh alike
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        def e2e_run(steps, timed):
            if timed:
                e0.record(stream)
            s_in.wait_stream(stream)
            s_out.wait_stream(stream)
            for i in range(steps):
                si = i % 2
                q_d, kv_d, ob_d, qy, o_d, ix_d = sets[si]
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(ev_comp[si])            # step i-2 has read this set's inputs
                    q_d.copy_(qin_h, non_blocking=True)
                    (kv_d if prefill else kv_d[:, :, :, -1]).copy_(kv_h, non_blocking=True)
                    ev_in[si].record(s_in)
                stream.wait_event(ev_in[si])
                if i >= 2:
                    stream.wait_event(ev_out[si])               # step i-2's result has left this set
                msa_forward(bank.handle, qy, k, ix_d.data_ptr(), o_d.data_ptr(), sh)
                ev_comp[si].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_comp[si])
                    out_h[si].copy_(ob_d, non_blocking=True)
                    ev_out[si].record(s_out)
            stream.wait_stream(s_out)
            if timed:
                e1.record(stream)

        e2e_run(4, False)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e2e_run(n_e2e, True)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1)
        assert bank.device_error() == 0

    total_ms, e2e_ms, route_ms, attend_ms = max_over_ranks([total_ms, e2e_ms or 0.0, route_ms, attend_ms], "cuda")
    if world > 1:
        dist.barrier()
    ms_step = total_ms / n
    units = B * (w.q_tokens if prefill else 1)   # queries (decode) or query tokens (prefill) per step
    value = job_throughput(world, units, n, total_ms)
    e2e_value = job_throughput(world, units, n_e2e, e2e_ms) if with_e2e else None

    if rank == 0:
        peak, peak_kind = peaks()
        if prefill:
            tpeak, tkind = tensor_peak(sustained=True)
            achieved = attn_flops / (attend_ms / 1000.0) / 1e12
            roofline = {"kernel": "sparse_attend (rope_local + attend_prefill launches)", "bound": "tensor",
                        "achieved": achieved, "peak": tpeak, "peak_kind": tkind, "unit": "TFLOP/s",
                        "frac": achieved / tpeak,
                        "traffic": profile_traffic("attend_prefill_tc.prefill.txt", "attend_prefill_tc"),
                        "algorithmic_flops_per_launch": attn_flops,
                        "hbm_bytes_algorithmic": attn_bytes}
            metric, unit = "prefill query tokens/s (4096-token prompt, 64-token routing blocks)", "tokens/s"
        else:
            achieved = attn_bytes / (attend_ms / 1000.0) / 1e9
            roofline = {"kernel": "sparse_attend (attend_decode launch)", "bound": "hbm",
                        "achieved": achieved, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                        "frac": achieved / peak, "traffic": profile_traffic("attend_decode.decode_4m.txt", "attend_decode"),
                        "algorithmic_bytes_per_launch": attn_bytes}
            metric, unit = METRIC, "queries/s"
        line = {
            "metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": n,
            "warmup": warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": base_config(w, world),
            "router_keys": "bf16" if args.kr_bf16 else "f32",
            "router_attn_hbm": {"bytes_per_step": step_bytes, "GBps": step_bytes / (ms_step / 1000.0) / 1e9,
                                "frac_of_peak": step_bytes / (ms_step / 1000.0) / 1e9 / peak,
                                "route_ms": route_ms, "attend_ms": attend_ms},
            "roofline": roofline,
            "clocks": clk,
            "gpu_launches": launches_per_step(w) * n,
        }
        if with_e2e:
            line["e2e"] = {"value": e2e_value, "unit": unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    bank.close()
    return line if rank == 0 else None


# The other workloads the default run also times once (after the headline), so that
# every configuration's figures come from the same run: (name, steps, warmup).
EXTRA_WORKLOADS = (("prefill", 20, 3), ("ragged_planted", 5, 2), ("bank_100m", 5, 2))


def extra_summary(line: dict) -> dict:
    keep = ("metric", "value", "unit", "steps", "warmup", "ms_per_step", "config", "roofline", "router",
            "router_attn_hbm", "planted_recall", "unpipelined_ms_per_step", "gpu_launches", "clocks", "setup_s")
    return {k: line[k] for k in keep if k in line}


def run_ours(args):
    import torch
    import torch.distributed as dist

    import synth
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    line = measure_device(args, args.workload, args.steps, args.warmup, world, rank, local)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    torch.cuda.empty_cache()
    if world == 1 and args.workload == WORKLOAD and not args.no_extras:
        extras = {}
        for name, steps, warm in EXTRA_WORKLOADS:
            try:
                if synth.WORKLOADS[name].host_tier:
                    r = measure_host(args, name, steps, warm)
                else:
                    r = measure_device(args, name, steps, warm, 1, 0, local, with_e2e=False)
                extras[name] = extra_summary(r)
            except Exception as e:  # reported in the line, never hidden
                extras[name] = {"error": f"{type(e).__name__}: {e}"}
            torch.cuda.synchronize()
            torch.cuda.empty_cache()
        line["workloads"] = extras
    if world == 1 and not args.no_cpu_baseline and args.workload == WORKLOAD:
        w = synth.WORKLOADS[WORKLOAD]
        r = oracle_timed(WORKLOAD, args.cpu_steps, 1)
        line["cpu_baseline"] = {"value": r["value"], "unit": "queries/s", "cores": r["cores"], "kind": "oracle",
                                "sample": oracle_sample_text(r, w)}
    print(json.dumps(line), flush=True)


def shard_tensors(w, lo: int, hi: int, device="cuda"):
    """K, V, R of documents [lo, hi) of a device workload, generated directly (each
    head's rows are one slice of the whole tensor's stream)."""
    import torch

    import synth
    from synth.device import fill_normal
    off = np.concatenate([[0], np.cumsum(w.doc_lens())])
    a, b = int(off[lo]), int(off[hi])
    out = []
    for tid, rows, dim in ((synth.T_K, w.kv_rows, w.head_dim), (synth.T_V, w.kv_rows, w.head_dim),
                           (synth.T_R, w.n_tokens, w.route_dim)):
        t = torch.empty((w.n_kv_heads, b - a, dim), dtype=torch.bfloat16, device=device)
        for h in range(w.n_kv_heads):
            fill_normal(t[h], w.seed, tid, (h * rows + a) * dim)
        out.append(t)
    return out


def run_memory_parallel(args):
    """The decode step with the bank split into document shards (Memory Parallel):
    every shard routes its own documents, the candidates are merged into the global
    top-k, every shard attends over the selected documents it holds (shard 0 also
    over the local context) and the partials are merged. One process: S shards on
    one GPU, timed against the single bank on the same GPU. Under torchrun: one
    shard per rank, NCCL all-gathers, max-over-ranks time (the bank is fixed and
    split: strong scaling)."""
    import torch
    import torch.distributed as dist

    import synth
    from sparse_attention_routed_b200.parallel import MemoryParallelStep, ShardedStep, shard_ranges
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import query_tensors

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    w = synth.WORKLOADS[args.workload]
    assert not w.host_tier and w.q_tokens == w.route_block, "Memory Parallel bench: device-tier decode workloads"
    S = world if world > 1 else max(1, args.memory_parallel)
    ranges = shard_ranges(w.n_docs, S)
    lens, max_len = w.doc_lens(), int(w.doc_lens().max())
    mine = [rank] if world > 1 else list(range(S))
    banks, keep = [], []
    for s in mine:
        lo, hi = ranges[s]
        K, V, R = shard_tensors(w, lo, hi)
        bank = Bank(K, V, lens[lo:hi], w.rope_base)
        bank.set_shard(lo, w.n_docs, max_len)
        bank.build(R)
        torch.cuda.synchronize()
        del R
        banks.append(bank)
        keep += [K, V]
    Q, Qr, LK, LV = query_tensors(w)
    queries = [b.query(Q, Qr, LK, LV, w.route_block) for b in banks]
    step = (MemoryParallelStep(banks[0], owner=0) if world > 1 else ShardedStep(banks, owner=0))
    run = (lambda: step(queries[0], w.top_k)) if world > 1 else (lambda: step(queries, w.top_k))
    stream = torch.cuda.current_stream()
    for _ in range(max(3, args.warmup)):
        run()
    torch.cuda.synchronize()
    for b in banks:
        assert b.device_error() == 0
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    time.sleep(0.4)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        run()
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    (total_ms,) = max_over_ranks([e0.elapsed_time(e1)], "cuda")
    line = None
    if rank == 0:
        ms = total_ms / args.steps
        line = {"metric": f"decode queries/s, Memory Parallel over {S} document shards",
                "value": w.batch / (ms / 1e3), "unit": "queries/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                "scaling": "strong" if world > 1 else "n/a (shards share one GPU)", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic",
                "config": dict(base_config(w, world), parallelism=f"memory parallel, {S} shards"),
                "clocks": clk}
    if world > 1:
        dist.destroy_process_group()
    else:
        # the same step on one bank holding every document, same GPU, same inputs
        for b in banks:
            b.close()
        banks.clear()
        keep.clear()
        torch.cuda.empty_cache()
        K, V, R = shard_tensors(w, 0, w.n_docs)
        whole = Bank(K, V, lens, w.rope_base)
        whole.build(R)
        del R
        qry = whole.query(Q, Qr, LK, LV, w.route_block)
        for _ in range(max(3, args.warmup)):
            whole.forward(qry, w.top_k)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            whole.forward(qry, w.top_k)
        e1.record(stream)
        torch.cuda.synchronize()
        line["single_bank_ms_per_step"] = e0.elapsed_time(e1) / args.steps
        whole.close()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_route_only(args):
    """msa_route alone over the full K_r of the workload (profiling aid, not the headline)."""
    import torch

    import synth
    from sparse_attention_routed_b200 import msa_route
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import fill_normal, query_tensors

    w = synth.WORKLOADS[args.workload]
    Hkv, d, L = w.n_kv_heads, w.head_dim, int(w.doc_lens().max())
    K = torch.zeros((Hkv, L, d), dtype=torch.bfloat16, device="cuda")   # every document aliases these rows
    V = torch.zeros_like(K)
    bank = Bank(K, V, w.doc_lens(), w.rope_base, doc_rows=np.zeros(w.n_docs, dtype=np.int64))
    off = np.concatenate([[0], np.cumsum(w.doc_lens())])
    step = 64
    for j0 in range(0, w.n_docs, step):
        j1 = min(w.n_docs, j0 + step)
        T = int(off[j1] - off[j0])
        R = torch.empty((Hkv, T, d), dtype=torch.bfloat16, device="cuda")
        for h in range(Hkv):
            fill_normal(R[h], w.seed, synth.T_R, (h * w.n_tokens + int(off[j0])) * d)
        bank.build(R, j0, j1, rope=False)
        torch.cuda.synchronize()
        del R
    Q, Qr, LK, LV = query_tensors(w)
    qry = bank.query(Q, Qr, LK, LV, w.route_block)
    idx = torch.empty((w.batch, 1, Hkv, w.top_k), dtype=torch.int32, device="cuda")
    sh = torch.cuda.current_stream().cuda_stream
    for _ in range(max(3, args.warmup)):
        msa_route(bank.handle, qry, w.top_k, 0, idx.data_ptr(), 0, sh)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        msa_route(bank.handle, qry, w.top_k, 0, idx.data_ptr(), 0, sh)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    kr_bytes = Hkv * bank.info["n_chunks"] * (d * 4 + 4)
    peak, kind = peaks()
    print(json.dumps({"mode": "route-only", "workload": args.workload, "route_ms": ms,
                      "k_r_bytes": kr_bytes, "GBps": kr_bytes / (ms / 1e3) / 1e9,
                      "frac_of_peak": kr_bytes / (ms / 1e3) / 1e9 / peak, "peak_kind": kind,
                      "device_error": bank.device_error()}), flush=True)
    bank.close()


def run_host_tier(args):
    if args.kv_cache_gb > 0:
        return measure_host(args, args.workload, args.steps, args.warmup, cache=True)
    print(json.dumps(measure_host(args, args.workload, args.steps, args.warmup)), flush=True)


def measure_host(args, wname: str, n: int, warmup: int, cache: bool = False):
    """Decode steps on a bank whose K/V live in pinned host memory (69M / 100M tokens):
    msa_forward routes on the device, copies the selected documents' K/V slabs over
    PCIe and attends, pipelined over micro-batches of sequences. Also timed: the
    routing alone, and routing then attention without the pipeline. Returns the line."""
    import torch

    import synth
    from sparse_attention_routed_b200 import (MSA_FETCH_COPY_ENGINE, MSA_FETCH_SM_GATHER, MSA_KV_PINNED_HOST,
                                              msa_attend, msa_forward, msa_route)
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import fill_normal, host_kv_pool, query_tensors

    w = synth.WORKLOADS[wname]
    Hkv, d, B, k = w.n_kv_heads, w.head_dim, w.batch, w.top_k
    t0 = time.time()
    Kh, Vh = host_kv_pool(w)
    bank = Bank(Kh, Vh, w.doc_lens(), w.rope_base, kv_location=MSA_KV_PINNED_HOST, doc_rows=w.doc_kv_rows())
    lens = w.doc_lens()
    off = np.concatenate([[0], np.cumsum(lens)])
    for j0 in range(0, w.n_docs, 64):          # routing keys streamed through the build
        j1 = min(w.n_docs, j0 + 64)
        T = int(off[j1] - off[j0])
        R = torch.empty((Hkv, T, d), dtype=torch.bfloat16, device="cuda")
        for h in range(Hkv):
            fill_normal(R[h], w.seed, synth.T_R, (h * w.n_tokens + int(off[j0])) * d)
        bank.build(R, j0, j1, rope=False)
        del R
    torch.cuda.synchronize()
    setup_s = time.time() - t0
    bank.set_host_fetch(MSA_FETCH_SM_GATHER if args.host_fetch == "gather" else MSA_FETCH_COPY_ENGINE)
    if cache:
        return run_host_cache(args, w, bank, setup_s, Kh)
    Q, Qr, LK, LV = query_tensors(w)
    qry = bank.query(Q, Qr, LK, LV, w.route_block)
    idx = torch.empty((B, 1, Hkv, k), dtype=torch.int32, device="cuda")
    out = torch.empty((B, w.n_q_heads, 1, d), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream
    for _ in range(max(2, warmup)):
        msa_forward(bank.handle, qry, k, idx.data_ptr(), out.data_ptr(), sh)
    msa_route(bank.handle, qry, k, 0, idx.data_ptr(), 0, sh)
    msa_attend(bank.handle, qry, k, idx.data_ptr(), out.data_ptr(), sh)
    torch.cuda.synchronize()
    assert bank.device_error() == 0
    sel = idx.cpu().numpy()
    uniq = {(int(j), h) for b in range(B) for h in range(Hkv) for j in sel[b, 0, h]}
    pcie_bytes = sum(int(lens[j]) for j, _ in uniq) * d * 2 * 2
    recall = None
    if w.planted:
        tg = synth.planted_targets(w.seed, B, w.n_docs, w.planted)
        recall = float(np.mean([tg[b, h % w.planted] in sel[b, 0, h] for b in range(B) for h in range(Hkv)]))
    # pinned H2D reference bandwidth (1 GiB, best of 3)
    hbuf = torch.empty(1 << 30, dtype=torch.uint8, pin_memory=True)
    dbuf = torch.empty(1 << 30, dtype=torch.uint8, device="cuda")
    best = 1e9
    for _ in range(3):
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        dbuf.copy_(hbuf, non_blocking=True)
        a1.record(stream)
        a1.synchronize()
        best = min(best, a0.elapsed_time(a1))
    h2d_peak = (1 << 30) / (best / 1e3) / 1e9
    del hbuf, dbuf
    clocks = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    time.sleep(0.4)
    torch.cuda.synchronize()
    t_begin, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_begin.record(stream)
    for i in range(n):
        msa_forward(bank.handle, qry, k, idx.data_ptr(), out.data_ptr(), sh)
    t_end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    step_ms = t_begin.elapsed_time(t_end) / n
    assert bank.device_error() == 0
    # the routing alone, and routing then attention without the pipeline (a few steps each)
    n2 = max(3, n // 3)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n2)]
    for i in range(n2):
        ev[i][0].record(stream)
        msa_route(bank.handle, qry, k, 0, idx.data_ptr(), 0, sh)
        ev[i][1].record(stream)
        msa_attend(bank.handle, qry, k, idx.data_ptr(), out.data_ptr(), sh)
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    route_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / n2
    unpipelined_ms = sum(e[0].elapsed_time(e[2]) for e in ev) / n2
    router_bytes = Hkv * bank.info["n_chunks"] * d * 4
    peak, kind = peaks()
    line = {
        "metric": f"decode queries/s, pinned-host K/V tier ({w.n_tokens / 1e6:.1f}M-token bank)",
        "value": B / (step_ms / 1e3), "unit": "queries/s", "n_gpus": 1, "steps": n, "warmup": warmup,
        "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wname, "batch": B, "q_heads": w.n_q_heads, "kv_heads": Hkv,
                   "head_dim": d, "bank_docs": w.n_docs, "bank_tokens": w.n_tokens, "local_len": w.local_len,
                   "top_k": k, "kv_slabs_pinned": w.kv_slabs, "pinned_kv_bytes": 2 * Kh.numel() * 2,
                   "host_fetch": args.host_fetch},
        "roofline": {"kernel": "selected K/V slabs over PCIe (" + FETCH_DESC[args.host_fetch] + "), "
                               "whole pipelined step", "bound": "pcie",
                     "achieved": pcie_bytes / (step_ms / 1e3) / 1e9, "peak": h2d_peak,
                     "peak_kind": "measured pinned H2D copy, 1 GiB", "unit": "GB/s",
                     "frac": pcie_bytes / (step_ms / 1e3) / 1e9 / h2d_peak, "bytes_per_step": pcie_bytes},
        "router": {"ms": route_ms, "bytes": router_bytes, "GBps": router_bytes / (route_ms / 1e3) / 1e9,
                   "frac_of_hbm_peak": router_bytes / (route_ms / 1e3) / 1e9 / peak},
        "unpipelined_ms_per_step": unpipelined_ms,
        "planted_recall": recall, "setup_s": setup_s, "clocks": clk,
        "gpu_launches": launches_per_step(w, gather=args.host_fetch == "gather") * n,
    }
    bank.close()
    del Kh, Vh
    if hasattr(torch._C, "_host_emptyCache"):
        torch._C._host_emptyCache()   # hand the pinned pool back before the next workload pins its own
    return line


FETCH_DESC = {"gather": "host_gather_kernel: the SMs read the mapped pinned K/V, one launch per micro-batch",
              "copy": "cudaMemcpyAsync per host-contiguous run of slabs"}


def run_host_cache(args, w, bank, setup_s, Kh):
    """Host-tier decode with a device-resident slab cache: each step takes one of
    --query-pool seeded query batches uniformly at random, so the cache sees the
    locality of a pool of recurring queries; hit rate and PCIe bytes per step are
    reported with the throughput."""
    import torch

    import synth
    from sparse_attention_routed_b200 import msa_forward
    from synth.device import fill_normal, query_tensors

    B, Hkv, d, k = w.batch, w.n_kv_heads, w.head_dim, w.top_k
    bank.set_kv_cache(int(args.kv_cache_gb * 1e9))
    pool = []
    for i in range(args.query_pool):
        Q, Qr, LK, LV = query_tensors(w)
        if i:
            for t, tid in ((Q, synth.T_Q), (Qr, synth.T_QR), (LK, synth.T_LK), (LV, synth.T_LV)):
                fill_normal(t, w.seed + 7919 * i, tid)
        pool.append((bank.query(Q, Qr, LK, LV, w.route_block), (Q, Qr, LK, LV)))
    idx = torch.empty((B, 1, Hkv, k), dtype=torch.int32, device="cuda")
    out = torch.empty((B, w.n_q_heads, 1, d), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream
    rng = np.random.RandomState(w.seed)
    for _ in range(max(3, args.warmup)):
        msa_forward(bank.handle, pool[rng.randint(len(pool))][0], k, idx.data_ptr(), out.data_ptr(), sh)
    torch.cuda.synchronize()
    assert bank.device_error() == 0
    n = args.steps
    picks = rng.randint(len(pool), size=n)
    slabs = hits = copied = 0
    clocks = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    time.sleep(0.4)
    torch.cuda.synchronize()
    t_begin, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_begin.record(stream)
    for i in range(n):
        msa_forward(bank.handle, pool[picks[i]][0], k, idx.data_ptr(), out.data_ptr(), sh)
        st = bank.cache_stats()  # host-side figures of the step just planned
        slabs += st["slabs"]
        hits += st["hits"]
        copied += st["bytes_copied"]
    t_end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    assert bank.device_error() == 0
    step_ms = t_begin.elapsed_time(t_end) / n
    slab_bytes = 2 * w.max_len * d * 2
    line = {
        "metric": f"decode queries/s, pinned-host K/V tier with a device slab cache ({w.n_tokens / 1e6:.1f}M-token bank)",
        "value": B / (step_ms / 1e3), "unit": "queries/s", "n_gpus": 1, "steps": n, "warmup": args.warmup,
        "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": f"synthetic; each step one of {len(pool)} seeded query batches, uniform at random",
        "config": dict(base_config(w), bank_tokens=w.n_tokens, kv_slabs_pinned=w.kv_slabs,
                       kv_cache_bytes=int(args.kv_cache_gb * 1e9),
                       kv_cache_slots=int(args.kv_cache_gb * 1e9) // slab_bytes, query_pool=len(pool),
                       host_fetch=args.host_fetch),
        "cache": {"hit_rate": hits / max(1, slabs), "slabs_per_step": slabs / n,
                  "pcie_bytes_per_step": copied / n, "pcie_GBps": copied / n / (step_ms / 1e3) / 1e9},
        "setup_s": setup_s, "clocks": clk,
        "gpu_launches": launches_per_step(w, gather=args.host_fetch == "gather") * n,
    }
    print(json.dumps(line), flush=True)
    bank.close()


def run_backward(args):
    """The backward of the routed attention on the workload's own selection, timed
    with CUDA events. Algorithmic FLOPs: 2.5 x the forward's (the five matmuls
    S, dP, dV, dK, dQ of 2 d FLOP per (query row, visible key)), no credit for
    recomputation."""
    import torch

    import synth
    from sparse_attention_routed_b200 import msa_attend_backward, msa_attend_backward_saved, msa_attend_lse
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors, normal, query_tensors

    w = synth.WORKLOADS[args.workload]
    K, V, R = bank_tensors(w)
    bank = Bank(K, V, w.doc_lens(), w.rope_base)
    bank.build(R)
    del R
    Q, Qr, LK, LV = query_tensors(w)
    qry = bank.query(Q, Qr, LK, LV, w.route_block)
    idx, out = bank.forward(qry, w.top_k)
    d_out = normal(tuple(out.shape), w.seed, 77).float()
    dq = torch.empty_like(out)
    dlk = torch.empty(LK.shape, dtype=torch.float32, device="cuda")
    dlv = torch.empty(LV.shape, dtype=torch.float32, device="cuda")
    dbk = torch.zeros(K.shape, dtype=torch.float32, device="cuda")
    dbv = torch.zeros(V.shape, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream
    # the forward's state a training step keeps: the output and each row's log-sum-exp
    lse = torch.empty(out.shape[:-1], dtype=torch.float32, device="cuda")
    msa_attend_lse(bank.handle, qry, w.top_k, idx.data_ptr(), out.data_ptr(), lse.data_ptr(), sh)

    def step():
        msa_attend_backward_saved(bank.handle, qry, w.top_k, idx.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                  d_out.data_ptr(), dq.data_ptr(), dlk.data_ptr(), dlv.data_ptr(), dbk.data_ptr(),
                                  dbv.data_ptr(), sh)

    def step_recompute():
        msa_attend_backward(bank.handle, qry, w.top_k, idx.data_ptr(), d_out.data_ptr(), dq.data_ptr(),
                            dlk.data_ptr(), dlv.data_ptr(), dbk.data_ptr(), dbv.data_ptr(), sh)

    for _ in range(max(3, args.warmup)):
        step()
        step_recompute()
    torch.cuda.synchronize()
    assert bank.device_error() == 0
    sel = idx.cpu().numpy()
    lens = w.doc_lens()
    nblk = w.q_tokens // w.route_block
    G = w.n_q_heads // w.n_kv_heads
    mem_keys = sum(int(lens[j]) for b in range(w.batch) for blk in range(nblk) for h in range(w.n_kv_heads)
                   for j in sel[b, blk, h]) * G * w.route_block
    first = w.local_len - w.q_tokens
    loc_keys = w.batch * w.n_q_heads * sum(first + t + 1 for t in range(w.q_tokens))
    flops = 10 * w.head_dim * (mem_keys + loc_keys)
    n = args.steps
    clocks = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    time.sleep(0.4)
    settle(step, 3)   # tensor-bound: the clocks under the 1 kW cap settle before anything is timed
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1) / n
    e0.record(stream)
    for _ in range(n):
        step_recompute()
    e1.record(stream)
    torch.cuda.synchronize()
    ms_recompute = e0.elapsed_time(e1) / n
    tpeak, tkind = tensor_peak(sustained=True)
    achieved = flops / (ms / 1e3) / 1e12
    units = w.batch * w.q_tokens
    # kernels per step of msa_attend_backward_saved: two RoPE passes (queries, local keys), then
    #   head_dim 128, 64- or 128-token blocks, G * Bq a multiple of 128: bwd_prep (dO . O and
    #     the saved log-sum-exp), bwd_index, bwd_dq_tc, bwd_dkdv_tc (msa_attend_backward adds
    #     the tcgen05 forward that recomputes O and the log-sum-exp);
    #   other blocks of a multiple of 64 tokens at head_dim 128: bwd_dq (mma.sync), to_bf16,
    #     bwd_index, bwd_dkdv_tc;
    #   anything else: bwd_dq and bwd_dkdv (mma.sync)
    G_ = w.n_q_heads // w.n_kv_heads
    if w.head_dim == 128 and w.route_block in (64, 128) and (G_ * w.route_block) % 128 == 0 and w.top_k <= 64:
        kernels, launches = "bwd_dq_tc_kernel + bwd_dkdv_tc_kernel (tcgen05; the forward's saved O and lse)", 6
    elif w.head_dim == 128 and w.route_block % 64 == 0:
        kernels, launches = "bwd_dq_kernel (mma.sync) + bwd_dkdv_tc_kernel (tcgen05)", 6
    else:
        kernels, launches = "bwd_dq_kernel + bwd_dkdv_kernel (mma.sync)", 4
    line = {
        "metric": "routed attention backward (the forward's O and log-sum-exp saved), query tokens/s", "value": units / (ms / 1e3), "unit": "tokens/s",
        "n_gpus": 1, "steps": n, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(base_config(w), parallelism="replicas x1"),
        "roofline": {"kernel": kernels, "bound": "tensor", "achieved": achieved,
                     "peak": tpeak, "peak_kind": tkind, "unit": "TFLOP/s", "frac": achieved / tpeak,
                     "algorithmic_flops_per_launch": flops},
        "recompute": {"ms_per_step": ms_recompute, "value": units / (ms_recompute / 1e3),
                      "note": "msa_attend_backward: the same gradients, recomputing the forward's O and lse"},
        "clocks": clk, "gpu_launches": launches * n,
    }
    print(json.dumps(line), flush=True)
    bank.close()


def run_build(args):
    """The offline bank build over a whole device bank, timed with CUDA events:
    reads the routing keys (2 d_r bytes per token per KV head) and reads and
    rewrites the keys (2 x 2 d bytes), writes K_r (small)."""
    import torch

    import synth
    from sparse_attention_routed_b200.runner import Bank
    from synth.device import bank_tensors

    w = synth.WORKLOADS[args.workload]
    K, V, R = bank_tensors(w)
    bank = Bank(K, V, w.doc_lens(), w.rope_base)
    stream = torch.cuda.current_stream()
    for _ in range(max(3, args.warmup)):
        bank.build(R)
    torch.cuda.synchronize()
    n = args.steps
    clocks = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    time.sleep(0.4)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        bank.build(R)  # RoPE turns the keys again each time: the same bytes and work
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1) / n
    tok = w.n_tokens * w.n_kv_heads
    nbytes = tok * (w.route_dim + 2 * w.head_dim) * 2 + w.n_kv_heads * bank.info["n_chunks"] * w.route_dim * (4 + 4)
    peak, kind = peaks()
    line = {
        "metric": "bank build HBM GB/s (pooling + Parallel RoPE, in place)", "value": nbytes / (ms / 1e3) / 1e9,
        "unit": "GB/s", "n_gpus": 1, "steps": n, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(base_config(w), bank_tokens=w.n_tokens),
        "roofline": {"kernel": "bank_build_kernel", "bound": "hbm", "achieved": nbytes / (ms / 1e3) / 1e9,
                     "peak": peak, "peak_kind": kind, "unit": "GB/s",
                     "frac": nbytes / (ms / 1e3) / 1e9 / peak, "algorithmic_bytes_per_launch": nbytes},
        "clocks": clk, "gpu_launches": n,
    }
    print(json.dumps(line), flush=True)
    bank.close()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.build_only:
        run_build(args)
    elif args.backward:
        run_backward(args)
    elif args.route_only:
        run_route_only(args)
    elif args.memory_parallel:
        run_memory_parallel(args)
    elif args.workload in ("ragged_planted", "bank_100m"):
        run_host_tier(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Benchmark of one Loki decode step at ctx 32k on B200.

Workload: Llama-3-8B-shaped GQA decode, batch 8, 32 query / 8 kv heads,
head dim 128, 32768 cached tokens per sequence, bf16 paged cache (16-token
blocks, shuffled block table), rank r = 32, k = 2048 plus the 64 most recent
tokens. Synthetic seeded inputs (rank_key_top_b200.synth).

One step = the whole hot path for one decode batch, one loki_decode_step
call: the append (rotate the current token's key by P and write it into slot
L-1 of every sequence) and the attention (query rotation, rank-r scoring,
top-k, exact attention over the kept tokens), the attention kernel launched
as a programmatic dependent of the append kernel. The L2 cache is flushed between
timed steps (a 256 MB write, then a read of it, so that L2 is cold and
holds no dirty lines), outside the timed events.

Prints one JSON line (rank 0). `--impl reference` times the reference oracle
(plain fp64 C) on the host cores instead. Under torchrun every rank runs its
own replica of the workload (independent batches, no collective on the data
path) and `value` is the aggregate over ranks.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "gqa32x8-d128-L32768-bf16"
METRIC = "sparse-attn decode steps/s & achieved HBM GB/s vs peak at ctx 32k, 1×B200"
UNIT = "steps/s"
FALLBACK_HBM_GBS = 6650.0
# the decode kernel's device code and its launch geometry (cluster size,
# shared-memory layout): the committed DRAM counters hold while these are unchanged
KERNEL_SOURCES = ["attn_core.cuh", "common.cuh", "sparse_decode.cuh", "sparse_launch.cuh"]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=30)
    ap.add_argument("--impl", choices=["loki", "reference"], default="loki")
    ap.add_argument("--profile", action="store_true",
                    help="only the timed device loop (for ncu): no e2e, dense, CPU baseline or clocks")
    ap.add_argument("--profile-dense", action="store_true",
                    help="with --profile: then run the dense-attention path steps + warmup times as well")
    ap.add_argument("--profile-rotate", action="store_true",
                    help="with --profile: then run the prompt prefill with rotation steps + warmup times as well")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="oracle time budget of the CPU baseline")
    ap.add_argument("--workload", default=WORKLOAD, help="named synthetic workload of the timed step")
    ap.add_argument("--r", type=int, default=None, help="override the workload's rank r")
    ap.add_argument("--k", type=int, default=None, help="override the workload's k")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the other workloads, the offload and the recall measurements")
    return ap.parse_args()


def workload_spec(args, synth, **extra):
    over = dict(extra)
    if args.r is not None:
        over["r"] = args.r
    if args.k is not None:
        over["k"] = args.k
    return synth.named_spec(args.workload, **over)


# ---------------------------------------------------------------------------
# Workload arithmetic (algorithmic bytes, per the roofline model)
# ---------------------------------------------------------------------------

def kept_rows(spec, b):
    """Tokens one (sequence b, kv head) pair attends to: its k (per sequence
    where the workload sets one) among the candidates, plus the window."""
    L = spec.seq_lens[b]
    w = min(spec.recent_window, L)
    kb = spec.k_per_seq[b] if spec.k_per_seq else spec.k
    return min(kb, L - w) + w


def algorithmic_bytes(spec):
    """Per decode launch: for each (sequence, kv head), L*r key elements for
    scoring plus 2*(k + W)*d key and value elements for the kept rows; plus
    the queries read and the fp32 outputs written."""
    es = 2 if spec.dtype == "bf16" else 4
    total = 0
    for b, L in enumerate(spec.seq_lens):
        total += spec.num_kv_heads * (L * spec.r + 2 * kept_rows(spec, b) * spec.head_dim) * es
    total += spec.batch * spec.num_q_heads * spec.head_dim * (es + 4)
    return total


def attended_tokens(spec):
    """Attended tokens of one step, counted per query head."""
    return sum(spec.num_q_heads * kept_rows(spec, b) for b in range(spec.batch))


def dense_bytes(spec):
    es = 2 if spec.dtype == "bf16" else 4
    total = sum(spec.num_kv_heads * 2 * L * spec.head_dim * es for L in spec.seq_lens)
    return total + spec.batch * spec.num_q_heads * spec.head_dim * (es + 4)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "rank_key_top_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic():
    """DRAM bytes per launch of the sparse kernel from the committed ncu
    summary, if it was taken on the current kernel sources."""
    path = os.path.join(ROOT, "profiles", "sparse_decode_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    if d.get("source_sha256") != kernel_source_hash():
        return None
    return d.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# Clock sampling during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_uuid):
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None
        self.uuid = device_uuid

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu=timestamp,{self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "100"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.reader = threading.Thread(target=self._read, daemon=True)
        self.reader.start()
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        if not self.proc:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((ts, float(parts[1]), float(parts[2]), parts[4:9]))
            except ValueError:
                continue
        inside = [r for r in rows if self.t0 is not None and self.t0 - 0.05 <= r[0] <= self.t1 + 0.05]
        use = inside if inside else rows[-3:]
        if not use:
            return None
        names = ["active_mask", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in use for i in range(1, 5) if r[3][i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": max(r[2] for r in use),
                "reasons": reasons, "samples": len(use), "samples_in_timed_region": len(inside)}


# ---------------------------------------------------------------------------
# CPU baseline: the oracle, on a bounded sample of the same workload
# ---------------------------------------------------------------------------

def cpu_baseline(spec, wl_pairs, budget_s, steps=None):
    """Times oracle.decode_batch on a sample of the workload's (sequence, kv
    head) pairs; returns steps/s = pairs/s / pairs per step."""
    import numpy as np
    import oracle
    from rank_key_top_b200 import synth
    pairs = sorted(wl_pairs)
    wl = synth.make_workload(spec, pairs=set(pairs))
    g = spec.group
    Kt = np.stack([wl.Kt[b, h].double().numpy() for b, h in pairs])
    V = np.stack([wl.V[b, h].double().numpy() for b, h in pairs])
    q = np.stack([wl.q[b, h * g:(h + 1) * g].double().numpy() for b, h in pairs])
    P = np.stack([wl.P[h].double().numpy() for _, h in pairs])
    L = [spec.seq_lens[b] for b, _ in pairs]
    kp = [spec.k_per_seq[b] if spec.k_per_seq else spec.k for b, _ in pairs]
    done, spent, reps = 0, 0.0, 0
    while (steps is None and spent < budget_s) or (steps is not None and reps < steps):
        t = time.perf_counter()
        oracle.decode_batch(Kt, V, q, P, L, spec.r, kp, W=spec.recent_window)
        spent += time.perf_counter() - t
        done += len(pairs)
        reps += 1
    per_step = spec.batch * spec.num_kv_heads
    return {"value": done / spent / per_step, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{len(pairs)} of the {per_step} (sequence, kv head) pairs of one decode step "
                      f"({spec.name}, r {spec.r}, k {spec.k}), decoded {reps} times by the fp64 oracle "
                      f"({spent:.1f} s); steps/s = pairs/s / {per_step}"}


def run_reference(args, spec, rank, world):
    """The reference arm: the oracle on the host cores, rank 0 only."""
    if rank != 0:
        return
    pairs = [(b, h) for b in range(2) for h in range(spec.num_kv_heads)]
    cpu_baseline(spec, pairs, 0, steps=max(1, args.warmup))
    t = time.perf_counter()
    cb = cpu_baseline(spec, pairs, 0, steps=args.steps)
    wall = time.perf_counter() - t
    line = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 / cb["value"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded; see rank_key_top_b200/synth.py)",
            "config": config_of(spec, "none (CPU)"), "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "wall_s": wall}
    print(json.dumps(line), flush=True)


def config_of(spec, l2):
    return {"workload": spec.name, "batch": spec.batch, "q_heads": spec.num_q_heads,
            "kv_heads": spec.num_kv_heads, "head_dim": spec.head_dim, "seq_len": spec.seq_lens[0],
            "r": spec.r, "k": spec.k, "recent_window": spec.recent_window, "index_dims": spec.r,
            "cache": "paged, 16-token blocks, shuffled table", "l2": l2, "parallelism": "replicas (independent batches per GPU)"}


# ---------------------------------------------------------------------------
# Secondary measurements (one GPU): the other workloads, the offloaded cache,
# kept-set recall of the alternative scorers
# ---------------------------------------------------------------------------

C5 = "gqa32x8-d128-L131072-bf16-outliers"
SWEEP = ([("single-head-d64-L1024-f32", None), ("mha32-d128-L4096-bf16", None),
          ("paged-b16-mha32-L4k-16k-bf16", None)] +
         [(C5, (r, k)) for r in (16, 32, 64) for k in (4096, 8192, 16384)])


def timed_median(launch, flush_l2, stream, n=20, warm=3):
    """Median device time (ms) of n launches, each after an L2 flush."""
    import torch
    for i in range(warm):
        launch(i)
    e0 = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    e1 = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for i in range(n):
        flush_l2()
        e0[i].record(stream)
        launch(i)
        e1[i].record(stream)
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in zip(e0, e1))


def config_sweep(loki, synth, dev, stream, flush_l2, peak, cpu_seconds):
    """Every other workload: decode launch time (eager, L2 flushed, median of
    20), steps/s, attended tokens/s, algorithmic bytes and roofline fraction,
    the dense path on the same cache, and the oracle on a bounded sample."""
    import dataclasses
    import torch
    rows = []
    names = []
    for name, _ in SWEEP:
        if name not in names:
            names.append(name)
    for name in names:
        spec = synth.named_spec(name)
        wl = synth.make_workload(spec)
        points = [rk for n, rk in SWEEP if n == name]
        index_dims = max(spec.r if rk is None else rk[0] for rk in points)
        cache = loki.Cache(wl.num_blocks, spec.num_kv_heads, spec.head_dim, synth.torch_dtype(spec.dtype), dev,
                           index_dims=index_dims)
        batch = loki.Batch(wl.block_table.to(dev), wl.seq_lens.to(dev), spec.max_seq_len)
        loki.loki_prefill_cache(cache, batch, wl.Kt.to(dev), wl.V.to(dev), stream=stream)
        q, P = wl.q.to(dev), wl.P.to(dev).contiguous()
        kps = wl.k_per_seq.to(dev) if wl.k_per_seq is not None else None
        out = torch.empty(spec.batch, spec.num_q_heads, spec.head_dim, device=dev)
        del wl
        ws = torch.empty(loki.loki_dense_workspace_bytes(cache, batch, spec.num_q_heads), dtype=torch.uint8,
                         device=dev)
        dense_ms = timed_median(lambda i: loki.loki_dense_attention(cache, batch, q, P, out, ws, stream=stream),
                                flush_l2, stream, n=10)
        for rk in points:
            sp = spec if rk is None else dataclasses.replace(spec, r=rk[0], k=rk[1])
            ms = timed_median(lambda i: loki.loki_decode_attention(
                cache, batch, q, P, sp.r, sp.k, out, k_per_seq=kps, recent_window=sp.recent_window,
                stream=stream), flush_l2, stream)
            alg = algorithmic_bytes(sp)
            achieved = alg / (ms / 1e3) / 1e9
            cb = cpu_baseline(sp, [(0, h) for h in range(min(2, sp.num_kv_heads))], cpu_seconds)
            rows.append({"workload": name, "r": sp.r, "k": "L_b/8 per sequence" if sp.k_per_seq else sp.k,
                         "recent_window": sp.recent_window, "launch_ms": ms, "steps_per_s": 1e3 / ms,
                         "attended_tokens_per_s": attended_tokens(sp) * 1e3 / ms,
                         "algorithmic_bytes_per_launch": alg, "achieved_gbs": achieved, "frac": achieved / peak,
                         "dense": {"ms": dense_ms, "steps_per_s": 1e3 / dense_ms,
                                   "achieved_gbs": dense_bytes(sp) / (dense_ms / 1e3) / 1e9},
                         "cpu_oracle_steps_per_s": cb["value"], "cpu_oracle_sample": cb["sample"]})
        del cache, batch, q, P, out, ws
        torch.cuda.empty_cache()
    assert loki.loki_device_error() == 0
    return rows


def offload_measurement(loki, spec, num_blocks, Kt_dev, V_dev, P, qs, batch, dev, stream, flush_l2):
    """The bench cache with every second block's key and value rows in pinned
    host memory: decode launch time and the bytes the decodes read over the
    host link (kept rows of offloaded blocks), before and after one pass of
    the planner that promotes the blocks the step's queries kept most."""
    import numpy as np
    import torch
    home = np.empty(num_blocks, np.int32)
    nd = nh = 0
    for b in range(num_blocks):
        if b % 2:
            home[b] = -(nh + 1)
            nh += 1
        else:
            home[b] = nd
            nd += 1
    off = loki.OffloadCache(num_blocks, spec.num_kv_heads, spec.head_dim, torch.bfloat16, home, nd + 1, nh, dev,
                            index_dims=spec.r)
    loki.loki_prefill_cache(off, batch, Kt_dev, V_dev, stream=stream)
    out = torch.empty(spec.batch, spec.num_q_heads, spec.head_dim, device=dev)
    row_bytes = 2 * spec.head_dim * 2   # one kept token: its key row and its value row

    def launch(i):
        loki.loki_decode_attention(off, batch, qs[i % len(qs)], P, spec.r, spec.k, out,
                                   recent_window=spec.recent_window, stream=stream)

    def host_bytes_per_step():
        off.touch.zero_()
        for i in range(len(qs)):
            launch(i)
        torch.cuda.synchronize()
        t = off.touch.cpu().numpy()[:num_blocks].astype(np.int64)
        return int(t[off.home.numpy() < 0].sum()) * row_bytes / len(qs), int(t.sum()) * row_bytes / len(qs)

    before_host, kept_bytes = host_bytes_per_step()
    ms_before = timed_median(launch, flush_l2, stream, n=10)
    host_bytes_per_step()                       # the counts the planner reads
    moves = loki.offload_rebalance(off, max_moves=num_blocks, stream=stream)
    torch.cuda.synchronize()
    after_host, _ = host_bytes_per_step()
    ms_after = timed_median(launch, flush_l2, stream, n=10)
    assert loki.loki_device_error() == 0
    res = {"offloaded_fraction": nh / num_blocks, "host_pages": nh, "device_pages": nd + 1,
           "kept_row_bytes_per_step": kept_bytes,
           "before_rebalance": {"launch_ms": ms_before, "steps_per_s": 1e3 / ms_before,
                                "host_link_bytes_per_step": before_host,
                                "host_link_gbs": before_host / (ms_before / 1e3) / 1e9},
           "after_rebalance": {"moves": len(moves), "launch_ms": ms_after, "steps_per_s": 1e3 / ms_after,
                               "host_link_bytes_per_step": after_host,
                               "host_link_gbs": after_host / (ms_after / 1e3) / 1e9},
           "note": "every second physical block's key/value rows in pinned host memory, read in place by the "
                   "decode (only kept rows cross the link); the planner then swaps the blocks the same 4 "
                   "queries kept most onto the device; eager launches, L2 flushed, median of 10"}
    del off
    torch.cuda.empty_cache()
    return res


def kept_set_recall(sel_a, sel_b):
    """Mean over pairs of |A & B| / |B| for two selected-index tensors."""
    a, b = sel_a.cpu().numpy(), sel_b.cpu().numpy()
    fr = []
    for ra, rb in zip(a.reshape(-1, a.shape[-1]), b.reshape(-1, b.shape[-1])):
        sb = set(rb[rb >= 0].tolist())
        fr.append(len(set(ra[ra >= 0].tolist()) & sb) / max(len(sb), 1))
    return float(sum(fr) / len(fr))


def saki_calibration(Q, K, r):
    """Offline calibration of the asymmetric score factors, done once per
    kv head before decoding (SAKI page, abstract): with the second moments
    S_q, S_k of calibration queries and keys, the rank-r truncated SVD
    U s V^T of S_q^1/2 S_k^1/2 gives A_q = S_q^-1/2 U sqrt(s) and
    A_k = S_k^-1/2 V sqrt(s). numpy on the host, like the PCA calibration of P."""
    import numpy as np

    def sym_power(S, e):
        w, vec = np.linalg.eigh(S)
        return (vec * np.maximum(w, 1e-12 * w.max()) ** e) @ vec.T
    Sq = Q.T @ Q / Q.shape[0]
    Sk = K.T @ K / K.shape[0]
    U, sv, Vt = np.linalg.svd(sym_power(Sq, 0.5) @ sym_power(Sk, 0.5))
    root = np.sqrt(sv[:r])
    return sym_power(Sq, -0.5) @ (U[:, :r] * root), sym_power(Sk, -0.5) @ (Vt[:r].T * root)


def saki_recall(loki, synth, spec, cache, mcache, batch, K_orig, Kt_dev, P, dev, top=64):
    """Top-64 recall at rank r of the kept sets that key PCA (the leading r
    dims of the bench cache) and the asymmetric factors (calibrated on 512
    queries and 4096 cached keys per kv head) give, against the exact top 64
    of the full-d scores (the leading scorer at r = d), for queries whose
    spectrum runs against the keys' (SAKI page, abstract: top-k recall of the
    asymmetric factors against PCA at the same rank)."""
    import numpy as np
    import torch
    g, Hkv, D, r = spec.group, spec.num_kv_heads, spec.head_dim, spec.r
    q = torch.empty(spec.batch, spec.num_q_heads, D, dtype=torch.float64)
    Aq, Ak = [], []
    for h in range(Hkv):
        Ph = P[h].double().cpu().numpy()
        keys = Kt_dev[0, h, :4096].double().cpu().numpy() @ Ph.T    # cached keys, original basis
        a_q, a_k = saki_calibration(synth.draw_anisotropic_queries(spec, h, 512, 0), keys, r)
        Aq.append(a_q)
        Ak.append(a_k)
        for b in range(spec.batch):
            q[b, h * g:(h + 1) * g] = torch.from_numpy(synth.draw_anisotropic_queries(spec, h, g, 1 + b))
    q = q.to(torch.bfloat16).to(dev)
    A_q = torch.from_numpy(np.stack(Aq)).float().to(dev).contiguous()
    A_k = torch.from_numpy(np.stack(Ak)).float().to(dev).contiguous()
    # the bench cache's key and value rows with a key index of their own, k A_k
    xs = torch.empty(loki.loki_index_bytes(cache.struct.num_blocks, Hkv, r, loki.LOKI_BF16), dtype=torch.uint8,
                     device=dev)
    view = loki.Cache.__new__(loki.Cache)
    view.k, view.v, view.x, view.dtype, view.index_dims = cache.k, cache.v, xs, torch.bfloat16, r
    view.struct = loki.loki_cache(cache.k.data_ptr(), cache.v.data_ptr(), xs.data_ptr(), cache.struct.num_blocks,
                                  Hkv, D, r, loki.LOKI_BF16)
    loki.loki_index_keys(view, batch, K_orig, A_k)
    out = torch.empty(spec.batch, spec.num_q_heads, D, device=dev)
    sels = {}
    for name in ("exact", "pca", "saki"):
        sels[name] = torch.empty(spec.batch, Hkv, top, dtype=torch.int32, device=dev)
    loki.loki_decode_attention(mcache, batch, q, P, D, top, out, selected_idx=sels["exact"])
    loki.loki_decode_attention(cache, batch, q, P, r, top, out, selected_idx=sels["pca"])
    loki.loki_decode_attention_asym(view, batch, q, P, A_q, r, top, out, selected_idx=sels["saki"])
    torch.cuda.synchronize()
    assert loki.loki_device_error() == 0
    return {"pca": kept_set_recall(sels["pca"], sels["exact"]), "saki": kept_set_recall(sels["saki"], sels["exact"]),
            "rank": r, "top": top,
            "note": "mean over the 64 (sequence, kv head) pairs of |kept & exact top-64| / 64; queries drawn "
                    "z diag(reversed key scales) U^T; factors from 512 such calibration queries and 4096 cached "
                    "keys per kv head; all three sets from the GPU (exact = leading scorer at r = d)"}


# ---------------------------------------------------------------------------
# The GPU arm
# ---------------------------------------------------------------------------

def main():
    args = parse_args()
    from rank_key_top_b200 import dist as rdist
    from rank_key_top_b200 import synth
    if args.impl == "reference":
        # rank 0 alone times the oracle on the host; other ranks exit at once
        if int(os.environ.get("RANK", "0")) == 0:
            run_reference(args, workload_spec(args, synth), 0, 1)
        return
    rank, world, local = rdist.init_from_env("nccl")
    barrier, max_over_ranks, finish = rdist.barrier, rdist.max_over_ranks, rdist.finish
    base = workload_spec(args, synth)
    spec = workload_spec(args, synth, seed=rdist.replica_seed(base.seed, rank))

    import torch
    from rank_key_top_b200 import loki
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)   # graphs cannot capture the legacy default stream
    torch.cuda.set_stream(stream)

    wl = synth.make_workload(spec)
    cache = loki.Cache(wl.num_blocks, spec.num_kv_heads, spec.head_dim, torch.bfloat16, dev, index_dims=spec.r)
    batch = loki.Batch(wl.block_table.to(dev), wl.seq_lens.to(dev), spec.max_seq_len)
    Kt_dev, V_dev = wl.Kt.to(dev), wl.V.to(dev)
    kps = wl.k_per_seq.to(dev) if wl.k_per_seq is not None else None
    loki.loki_prefill_cache(cache, batch, Kt_dev, V_dev)
    torch.cuda.synchronize()
    P = wl.P.to(dev).contiguous()
    pool = 4
    qs = [synth.draw_query_batch(spec, i).to(dev) for i in range(pool)]
    kvs = [synth.draw_new_tokens(spec, i) for i in range(pool)]
    ks = [k.to(dev) for k, _ in kvs]
    vs = [v.to(dev) for _, v in kvs]
    out = torch.empty(spec.batch, spec.num_q_heads, spec.head_dim, device=dev)
    ws = loki.decode_workspace(cache, batch, spec.num_q_heads, spec.k, spec.recent_window, dev)
    flush = torch.empty(64 * 2 ** 20, dtype=torch.float32, device=dev)  # 256 MB > L2
    flush_sum = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2():
        # write a buffer twice the L2, then read it back: the write evicts the
        # step's data, the read evicts the write's dirty lines, so the timed
        # step starts on a cold, clean L2 (no write-back of flush data inside it)
        flush.zero_()
        torch.sum(flush, dim=0, out=flush_sum)
    del wl
    torch.cuda.empty_cache()

    def rotate_setup():
        # the prompt's keys in the original basis (K = K~ P^T, P orthonormal) and a cache of their own
        K_orig = torch.einsum("bhtd,hed->bhte", Kt_dev.float(), P).to(torch.bfloat16).contiguous()
        rcache = loki.Cache(cache.struct.num_blocks, spec.num_kv_heads, spec.head_dim, torch.bfloat16, dev,
                            index_dims=spec.r)
        return K_orig, rcache

    def step(i, q=None, k=None, v=None):
        loki.loki_decode_step(cache, batch, ks[i % pool] if k is None else k, vs[i % pool] if v is None else v,
                              qs[i % pool] if q is None else q, P, spec.r, spec.k, out, k_per_seq=kps,
                              recent_window=spec.recent_window, workspace=ws, stream=stream)

    # warm-up
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    # each step (append + decode, no host work) is captured once per input
    # slot into a CUDA graph and replayed
    graphs = []
    for i in range(pool):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step(i)
        graphs.append(g)
    for i in range(args.warmup):
        graphs[i % pool].replay()
    torch.cuda.synchronize()

    K = args.steps
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    evm = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    sampler = None
    if not args.profile and rank == 0:
        uuid = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
        except Exception:
            pass
        sampler = ClockSampler(uuid)
        sampler.start()

    barrier(world)
    torch.cuda.synchronize()
    if sampler:
        sampler.mark("t0")
    wall0 = time.perf_counter()
    for i in range(K):
        flush_l2()
        ev0[i].record(stream)
        graphs[i % pool].replay()
        ev1[i].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    wall = time.perf_counter() - wall0
    if sampler:
        sampler.mark("t1")
    step_ms = sum(a.elapsed_time(b) for a, b in zip(ev0, ev1))
    # the decode kernel alone, eagerly launched, for its roofline
    for i in range(K):
        flush_l2()
        evm[i].record(stream)
        loki.loki_decode_attention(cache, batch, qs[i % pool], P, spec.r, spec.k, out, k_per_seq=kps,
                                   recent_window=spec.recent_window, workspace=ws, stream=stream)
        ev1[i].record(stream)
    torch.cuda.synchronize()
    decode_ms = sum(a.elapsed_time(b) for a, b in zip(evm, ev1))
    step_ms = max_over_ranks(step_ms, world)
    clocks = sampler.stop() if sampler else None
    assert loki.loki_device_error() == 0

    if args.profile:
        if args.profile_rotate:
            K_orig, rcache = rotate_setup()
            for i in range(args.warmup + K):
                flush_l2()
                loki.loki_prefill_rotate(rcache, batch, K_orig, V_dev, P, stream=stream)
            torch.cuda.synchronize()
            assert loki.loki_device_error() == 0
            del K_orig, rcache
        if args.profile_dense:
            ws = torch.empty(loki.loki_dense_workspace_bytes(cache, batch, spec.num_q_heads), dtype=torch.uint8,
                             device=dev)
            dout = torch.empty_like(out)
            for i in range(args.warmup + K):
                flush_l2()
                loki.loki_dense_attention(cache, batch, qs[i % pool], P, dout, ws, stream=stream)
            torch.cuda.synchronize()
            assert loki.loki_device_error() == 0
        if rank == 0:
            print(json.dumps({"profile_run": True, "ms_per_step": step_ms / K}), flush=True)
        finish(world)
        return

    # end to end through the public API: loki_decode_step_host takes the step's
    # inputs (q, k_new, v_new) and its output in pinned host memory, which its
    # kernels read and write in place over the host link, all on the stream;
    # one graph per input slot
    hq = [q.cpu().pin_memory() for q in qs]
    hk = [k.cpu().pin_memory() for k in ks]
    hv = [v.cpu().pin_memory() for v in vs]
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    staging = torch.empty(loki.loki_decode_step_host_bytes(cache, batch, spec.num_q_heads), dtype=torch.uint8,
                          device=dev)
    e0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    e1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    e2e_graphs = []
    for i in range(pool):
        loki.loki_decode_step_host(cache, batch, hk[i], hv[i], hq[i], P, spec.r, spec.k, hout, staging,
                                   k_per_seq=kps, recent_window=spec.recent_window, stream=stream)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            loki.loki_decode_step_host(cache, batch, hk[i], hv[i], hq[i], P, spec.r, spec.k, hout, staging,
                                       k_per_seq=kps, recent_window=spec.recent_window, stream=stream)
        e2e_graphs.append(g)
    for phase in ("warm", "timed"):
        n = args.warmup if phase == "warm" else K
        for i in range(n):
            flush_l2()
            if phase == "timed":
                e0[i].record(stream)
            e2e_graphs[i % pool].replay()
            if phase == "timed":
                e1[i].record(stream)
        torch.cuda.synchronize()
    e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(e0, e1)), world)
    h2d = sum(t.numel() * t.element_size() for t in (hq[0], hk[0], hv[0]))
    d2h = hout.numel() * hout.element_size()
    assert loki.loki_device_error() == 0

    # the GPU's own dense-attention kernel on the same cache, same conditions
    ws = torch.empty(loki.loki_dense_workspace_bytes(cache, batch, spec.num_q_heads), dtype=torch.uint8,
                     device=dev)
    dout = torch.empty_like(out)
    d0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    d1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    for i in range(args.warmup):
        loki.loki_dense_attention(cache, batch, qs[i % pool], P, dout, ws, stream=stream)
    for i in range(K):
        flush_l2()
        d0[i].record(stream)
        loki.loki_dense_attention(cache, batch, qs[i % pool], P, dout, ws, stream=stream)
        d1[i].record(stream)
    torch.cuda.synchronize()
    dense_ms = sum(a.elapsed_time(b) for a, b in zip(d0, d1)) / K

    # the prompt prefill with the rotation on the tensor cores, same conditions
    K_orig, rcache = rotate_setup()
    for i in range(3):
        loki.loki_prefill_rotate(rcache, batch, K_orig, V_dev, P, stream=stream)
    r0 = [torch.cuda.Event(enable_timing=True) for _ in range(10)]
    r1 = [torch.cuda.Event(enable_timing=True) for _ in range(10)]
    for i in range(10):
        flush_l2()
        r0[i].record(stream)
        loki.loki_prefill_rotate(rcache, batch, K_orig, V_dev, P, stream=stream)
        r1[i].record(stream)
    torch.cuda.synchronize()
    assert loki.loki_device_error() == 0
    rot_ms = statistics.median(a.elapsed_time(b) for a, b in zip(r0, r1))
    ntok = sum(spec.seq_lens) * spec.num_kv_heads
    rot_bytes = ntok * spec.head_dim * 2 * 4 + ntok * spec.r * 2   # K, V read; K~, V, index written
    del rcache

    # the magnitude scorer against the leading one, on a cache whose key index
    # holds every dim (the scorer chooses r single dims, or r / 16 of its d / 16
    # slabs, per pair)
    mcache = loki.Cache(cache.struct.num_blocks, spec.num_kv_heads, spec.head_dim, torch.bfloat16, dev,
                        index_dims=spec.head_dim)
    loki.loki_prefill_rotate(mcache, batch, K_orig, V_dev, P, stream=stream)
    mout = torch.empty_like(out)
    scorer_ms = {}
    width = spec.k + spec.recent_window
    kept = {}
    for name, scorer in (("magnitude", loki.LOKI_SCORER_MAGNITUDE), ("slabs", loki.LOKI_SCORER_MAGNITUDE_SLABS),
                         ("leading", loki.LOKI_SCORER_LEADING)):
        def mag_launch(i, sel=None):
            loki.loki_decode_attention_scored(mcache, batch, qs[i % pool], P, spec.r, spec.k, mout, scorer=scorer,
                                              recent_window=spec.recent_window, workspace=ws, stream=stream,
                                              selected_idx=sel)
        scorer_ms[name] = timed_median(mag_launch, flush_l2, stream, n=10)
        kept[name] = torch.empty(spec.batch, spec.num_kv_heads, width, dtype=torch.int32, device=dev)
        mag_launch(0, kept[name])
    torch.cuda.synchronize()
    assert loki.loki_device_error() == 0
    scorer_recall = {"slabs_vs_dims": kept_set_recall(kept["slabs"], kept["magnitude"]),
                     "leading_vs_dims": kept_set_recall(kept["leading"], kept["magnitude"])}

    # the asymmetric scorer (query factor A_q, here P's leading columns) on
    # the bench cache, same conditions
    Aq = P[:, :, :spec.r].contiguous()

    def asym_launch(i):
        loki.loki_decode_attention_asym(cache, batch, qs[i % pool], P, Aq, spec.r, spec.k, mout,
                                        recent_window=spec.recent_window, workspace=ws, stream=stream)
    asym_ms = timed_median(asym_launch, flush_l2, stream, n=10)
    assert loki.loki_device_error() == 0

    extras = {}
    if world == 1 and not args.no_sweep:
        extras["saki_recall_at_64"] = saki_recall(loki, synth, spec, cache, mcache, batch, K_orig, Kt_dev, P, dev)
    del mcache, K_orig
    torch.cuda.empty_cache()
    if world == 1 and not args.no_sweep:
        peak0, _ = measured_peaks()
        extras["offload"] = offload_measurement(loki, spec, cache.struct.num_blocks, Kt_dev, V_dev, P, qs, batch,
                                                dev, stream, flush_l2)
        extras["configs"] = config_sweep(loki, synth, dev, stream, flush_l2, peak0, min(args.cpu_seconds, 1.0))

    if rank != 0:
        finish(world)
        return
    peak, peak_kind = measured_peaks()
    alg = algorithmic_bytes(spec)
    dec_s = decode_ms / K / 1e3
    achieved = alg / dec_s / 1e9
    tokens = attended_tokens(spec)
    value = world * K / (step_ms / 1e3)
    cb = cpu_baseline(spec, [(b, h) for b in range(2) for h in range(spec.num_kv_heads)],
                      args.cpu_seconds) if world == 1 else None
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": step_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded; keys drawn in the PCA basis with sigma_j = j^-0.8, "
                                 "see rank_key_top_b200/synth.py)",
        "config": config_of(spec, "flushed between timed steps (256 MB write then 256 MB read, L2 left cold and "
                                  "clean, outside the timed events)"),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": recorded_traffic(),
                     "kernel": f"sparse_decode_kernel<bf16,{spec.head_dim},{spec.group}>",
                     "algorithmic_bytes_per_launch": alg, "peak_source": f"{peak_kind} hbm_gbs",
                     "launch_ms": decode_ms / K},
        "cpu_baseline": cb,
        "e2e": {"value": world * K / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "path": "loki_decode_step_host: q, k_new, v_new read from pinned host buffers and out written "
                        "to a pinned host buffer by the step's kernels (mapped, in place); one CUDA graph per "
                        "input slot"},
        "clocks": clocks,
        "gpu_launches": 2 * K,
        "step_launch": "CUDA graph per step: loki_decode_step (append kernel, then the decode kernel as its "
                       "programmatic dependent)",
        "attended_tokens_per_s": value * tokens,
        "prefill_rotate": {"ms": rot_ms, "tokens": ntok, "bytes": rot_bytes,
                           "achieved_gbs": rot_bytes / (rot_ms / 1e3) / 1e9,
                           "tflops": 2.0 * ntok * spec.head_dim ** 2 / (rot_ms / 1e3) / 1e12,
                           "kernel": "rotate_prefill_tc_kernel<128> (tcgen05)"},
        "magnitude_scorer": {"launch_ms": scorer_ms["magnitude"], "slabs_launch_ms": scorer_ms["slabs"],
                             "leading_launch_ms": scorer_ms["leading"], "index_dims": spec.head_dim,
                             "kept_set_recall": scorer_recall,
                             "note": "loki_decode_attention_scored on a cache whose key index holds all "
                                     f"{spec.head_dim} dims; r = {spec.r}: the r single dims of largest query "
                                     "magnitude (AQUA), the r/16 slabs with the most query energy, and the "
                                     "leading r dims, median of 10 L2-flushed launches each; kept_set_recall: "
                                     "mean over pairs of |kept set & per-dim kept set| / |per-dim kept set| for "
                                     "one query batch (the per-dim set is the one the GPU parity tests hold to "
                                     "the oracle's per-dimension selection)"},
        "asym_scorer": {"launch_ms": asym_ms, "recall_at_64": extras.get("saki_recall_at_64"),
                        "note": "loki_decode_attention_asym on the bench cache (index of the leading 32 dims, "
                                "A_q = the leading 32 columns of P), median of 10 L2-flushed launches"},
        "offload": extras.get("offload"),
        "configs": extras.get("configs"),
        "dense": {"ms_per_step": dense_ms, "steps_per_s": 1e3 / dense_ms,
                  "achieved_gbs": dense_bytes(spec) / (dense_ms / 1e3) / 1e9},
        "wall_s_timed_loop": wall,
    }
    print(json.dumps(line), flush=True)
    finish(world)


if __name__ == "__main__":
    main()

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
    return ap.parse_args()


# ---------------------------------------------------------------------------
# Workload arithmetic (algorithmic bytes, per the roofline model)
# ---------------------------------------------------------------------------

def algorithmic_bytes(spec):
    """Per decode launch: for each (sequence, kv head), L*r key elements for
    scoring plus 2*(k + W)*d key and value elements for the kept rows; plus
    the queries read and the fp32 outputs written."""
    es = 2 if spec.dtype == "bf16" else 4
    total = 0
    for L in spec.seq_lens:
        w = min(spec.recent_window, L)
        kept = min(spec.k, L - w) + w
        total += spec.num_kv_heads * (L * spec.r + 2 * kept * spec.head_dim) * es
    total += spec.batch * spec.num_q_heads * spec.head_dim * (es + 4)
    return total


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
    kp = [spec.k] * len(pairs)
    done, spent, reps = 0, 0.0, 0
    while (steps is None and spent < budget_s) or (steps is not None and reps < steps):
        t = time.perf_counter()
        oracle.decode_batch(Kt, V, q, P, L, spec.r, kp, W=spec.recent_window)
        spent += time.perf_counter() - t
        done += len(pairs)
        reps += 1
    per_step = spec.batch * spec.num_kv_heads
    return {"value": done / spent / per_step, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{len(pairs)} of the {per_step} (sequence, kv head) pairs of one decode step, "
                      f"decoded {reps} times by the fp64 oracle ({spent:.1f} s); steps/s = pairs/s / {per_step}"}


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
# The GPU arm
# ---------------------------------------------------------------------------

def main():
    args = parse_args()
    from rank_key_top_b200 import dist as rdist
    from rank_key_top_b200 import synth
    if args.impl == "reference":
        # rank 0 alone times the oracle on the host; other ranks exit at once
        if int(os.environ.get("RANK", "0")) == 0:
            run_reference(args, synth.named_spec(WORKLOAD), 0, 1)
        return
    rank, world, local = rdist.init_from_env("nccl")
    barrier, max_over_ranks, finish = rdist.barrier, rdist.max_over_ranks, rdist.finish
    base = synth.named_spec(WORKLOAD)
    spec = synth.named_spec(WORKLOAD, seed=rdist.replica_seed(base.seed, rank))

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
                              qs[i % pool] if q is None else q, P, spec.r, spec.k, out,
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
        loki.loki_decode_attention(cache, batch, qs[i % pool], P, spec.r, spec.k, out,
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

    # end to end through the public API: pinned host inputs in, output back
    # a step's inputs (q, k_new, v_new) travel as one pinned buffer and one copy
    nq, nk, nv = qs[0].numel(), ks[0].numel(), vs[0].numel()
    hin = [torch.cat([q.flatten(), k.flatten(), v.flatten()]).cpu().pin_memory() for q, k, v in zip(qs, ks, vs)]
    din = torch.empty(nq + nk + nv, dtype=qs[0].dtype, device=dev)
    dq = din[:nq].view(qs[0].shape)
    dk = din[nq:nq + nk].view(ks[0].shape)
    dv = din[nq + nk:].view(vs[0].shape)
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    e0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    e1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    e2e_graphs = []
    for i in range(pool):   # host copies in, the step, the output back: one graph per input slot
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            din.copy_(hin[i], non_blocking=True)
            step(i, dq, dk, dv)
            hout.copy_(out, non_blocking=True)
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
    h2d = din.numel() * din.element_size()
    d2h = out.numel() * out.element_size()

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
    # holds every dim (the scorer chooses r / 16 of its d / 16 slabs per pair)
    mcache = loki.Cache(cache.struct.num_blocks, spec.num_kv_heads, spec.head_dim, torch.bfloat16, dev,
                        index_dims=spec.head_dim)
    loki.loki_prefill_rotate(mcache, batch, K_orig, V_dev, P, stream=stream)
    del K_orig
    mout = torch.empty_like(out)
    scorer_ms = {}
    for name, scorer in (("magnitude", loki.LOKI_SCORER_MAGNITUDE), ("slabs", loki.LOKI_SCORER_MAGNITUDE_SLABS),
                         ("leading", loki.LOKI_SCORER_LEADING)):
        def mag_launch(i):
            loki.loki_decode_attention_scored(mcache, batch, qs[i % pool], P, spec.r, spec.k, mout, scorer=scorer,
                                              recent_window=spec.recent_window, workspace=ws, stream=stream)
        for i in range(3):
            mag_launch(i)
        m0 = [torch.cuda.Event(enable_timing=True) for _ in range(10)]
        m1 = [torch.cuda.Event(enable_timing=True) for _ in range(10)]
        for i in range(10):
            flush_l2()
            m0[i].record(stream)
            mag_launch(i)
            m1[i].record(stream)
        torch.cuda.synchronize()
        scorer_ms[name] = statistics.median(a.elapsed_time(b) for a, b in zip(m0, m1))
    assert loki.loki_device_error() == 0
    del mcache

    # the asymmetric scorer (query factor A_q, here P's leading columns) on
    # the bench cache, same conditions
    Aq = P[:, :, :spec.r].contiguous()

    def asym_launch(i):
        loki.loki_decode_attention_asym(cache, batch, qs[i % pool], P, Aq, spec.r, spec.k, mout,
                                        recent_window=spec.recent_window, workspace=ws, stream=stream)
    for i in range(3):
        asym_launch(i)
    a0 = [torch.cuda.Event(enable_timing=True) for _ in range(10)]
    a1 = [torch.cuda.Event(enable_timing=True) for _ in range(10)]
    for i in range(10):
        flush_l2()
        a0[i].record(stream)
        asym_launch(i)
        a1[i].record(stream)
    torch.cuda.synchronize()
    asym_ms = statistics.median(x.elapsed_time(y) for x, y in zip(a0, a1))
    assert loki.loki_device_error() == 0

    if rank != 0:
        finish(world)
        return
    peak, peak_kind = measured_peaks()
    alg = algorithmic_bytes(spec)
    dec_s = decode_ms / K / 1e3
    achieved = alg / dec_s / 1e9
    tokens = sum(spec.num_q_heads * (min(spec.k, L - min(spec.recent_window, L)) + min(spec.recent_window, L))
                 for L in spec.seq_lens)
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
                     "kernel": "sparse_decode_kernel<bf16,128,4>",
                     "algorithmic_bytes_per_launch": alg, "peak_source": f"{peak_kind} hbm_gbs",
                     "launch_ms": decode_ms / K},
        "cpu_baseline": cb,
        "e2e": {"value": world * K / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
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
                             "note": "loki_decode_attention_scored on a cache whose key index holds all "
                                     f"{spec.head_dim} dims; r = {spec.r}: the r single dims of largest query "
                                     "magnitude (AQUA), the r/16 slabs with the most query energy, and the "
                                     "leading r dims, median of 10 L2-flushed launches each"},
        "asym_scorer": {"launch_ms": asym_ms,
                        "note": "loki_decode_attention_asym on the bench cache (index of the leading 32 dims, "
                                "A_q = the leading 32 columns of P), median of 10 L2-flushed launches"},
        "dense": {"ms_per_step": dense_ms, "steps_per_s": 1e3 / dense_ms,
                  "achieved_gbs": dense_bytes(spec) / (dense_ms / 1e3) / 1e9},
        "wall_s_timed_loop": wall,
    }
    print(json.dumps(line), flush=True)
    finish(world)


if __name__ == "__main__":
    main()

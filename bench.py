#!/usr/bin/env python3
"""Decode-step benchmark of head-partitioned sparse attention on B200.

One step = one spa_decode call on one layer's buffers for the whole batch:
query prologue, index scoring, top-p selection, split-K attention over
sinks + window + selected rows, and the combine.  Inputs are seeded synthetic
tensors of the named workload (default: ctx128k, batch 4, 32/8 heads, 128K
context), resident in HBM before timing.  Several layer copies are cycled so
that each step reads cold data (the per-step working set exceeds L2 as well).

Prints one JSON line (rank 0).  ``--impl reference`` times the float64 CPU
oracle on the host cores instead (a bounded sample per step).

Multi-GPU: launched with torchrun, one process per GPU; every rank runs its own
batch (weak scaling, no collective in the data path); the time is the max over
ranks and ``value`` counts the layer-steps of all ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from head_partitioned_sparse_b200 import shard, synth  # noqa: E402

METRIC = "sparse decode-attention layer-steps/sec and achieved HBM GB/s at 128K ctx"
UNIT = "layer-steps/s"
CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--config", default="ctx128k", choices=synth.list_configs())
    ap.add_argument("--p", type=float, default=None, help="top-p threshold (default: the workload's)")
    ap.add_argument("--layers", type=int, default=2, help="layer copies cycled through")
    ap.add_argument("--split-rows", type=int, default=0)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-sweep", action="store_true", help="skip the per-p sweep")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-topk-sweep", action="store_true", help="skip the top-k selector measurements")
    ap.add_argument("--no-block-sweep", action="store_true", help="skip the block-granular selector measurements")
    ap.add_argument("--no-compact", action="store_true", help="skip the compact KV layout measurement")
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill measurement")
    ap.add_argument("--prefill-len", type=int, default=32768, help="prefill chunk length (from position 0)")
    ap.add_argument("--no-cp", action="store_true", help="skip the context-parallel measurement")
    ap.add_argument("--cp-ranks", type=int, default=4, help="ranks of the context-parallel measurement")
    ap.add_argument("--no-index-append", action="store_true", help="skip the index-append throughput leg")
    ap.add_argument("--no-configs", action="store_true", help="skip the other workloads' sub-records")
    ap.add_argument("--override", action="append", default=[], metavar="KEY=VALUE",
                    help="replace a workload field (e.g. B=1 for a small profiling case)")
    return ap.parse_args()


def overrides(args) -> dict:
    out = {}
    for kv in args.override:
        k, v = kv.split("=", 1)
        out[k] = type(synth.CONFIGS[args.config][k])(v) if k in synth.CONFIGS[args.config] else int(v)
    return out


def workload_desc(cfg: dict, name: str, p: float) -> str:
    return (f"{name}: batch {cfg['B']}, {cfg['Hq']}/{cfg['Hkv']} heads, head dim 128, context {cfg['L']}, "
            f"{cfg['dtype']}, {len(cfg['retrieval'])} retrieval KV heads, r=16 index, p={p:g}, "
            f"sinks {cfg['n_sink']}, window {cfg['window']}")


def config_dict(cfg: dict, name: str, p: float, world: int, n_layers: int) -> dict:
    """The ``config`` object of the JSON line, identical on both arms."""
    s_kv = 2 if cfg["dtype"] == "bf16" else 4
    layer_bytes = cfg["B"] * cfg["Hkv"] * cfg["L"] * (2 * 128 * s_kv + 32)
    return {"workload": workload_desc(cfg, name, p), "batch": cfg["B"], "seq_len": cfg["L"], "p": p,
            "storage": cfg["dtype"], "parallelism": f"dp{world}",
            "l2": f"inputs larger than L2: {n_layers} layer copies of {layer_bytes / 1e9:.2f} GB "
                  f"(K, V, index rows) cycled, one per step"}


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    def __init__(self, gpu_index: int):
        self.proc = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={CLOCK_FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", str(gpu_index)],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- profiles
def recorded_traffic(kernel_file: str, summary: str):
    """DRAM bytes per launch from a committed ncu summary, if the kernel source is unchanged."""
    path = os.path.join(ROOT, "profiles", summary)
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_sha = re.search(r"kernel_source_sha256:\s*([0-9a-f]{64})", text)
    m_b = re.search(r"dram_bytes_per_launch_full_workload:\s*([0-9.eE+]+)", text)
    if not (m_sha and m_b):
        return None
    src = os.path.join(ROOT, "head_partitioned_sparse_b200", "csrc", kernel_file)
    if hashlib.sha256(open(src, "rb").read()).hexdigest() != m_sha.group(1):
        return None
    return float(m_b.group(1))


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def measured_bf16_tflops():
    """Dense bf16 tensor peak: the burst figure (a kernel timed alone), else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        return float(json.load(open(path))["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


def prefill_flops(T: int, start: int, head_mask, G: int, n_sink: int, window: int) -> float:
    """Algorithmic flops of a prefill chunk: 4 * 128 per attended (query, key) pair
    (2 * 128 for q.k, 2 * 128 for p v), over every query head."""
    t = np.arange(start, start + T, dtype=np.float64)
    dense = (t + 1).sum()
    ns = np.minimum(n_sink, t + 1)
    w_lo = np.maximum(ns, t - window + 1)
    banded = (ns + (t + 1 - w_lo)).sum()
    n_ret = int(np.sum(np.asarray(head_mask) != 0))
    return 4.0 * 128 * G * (n_ret * dense + (len(head_mask) - n_ret) * banded)


# ----------------------------------------------------------------------------- helpers
def algorithmic_bytes(inp, counts: np.ndarray, s_kv: int):
    """Bytes a decode step must move: index rows of retrieval heads, sink/window K/V
    of every head, selected K/V rows, the query and the output."""
    idx = contig_rows = 0
    for b in range(inp.B):
        L = int(inp.seq_lens[b])
        n_s = min(inp.n_sink, L)
        w_lo = max(n_s, L - inp.window)
        contig = n_s + (L - w_lo)
        for g in range(inp.Hkv):
            contig_rows += contig
            if inp.head_mask[g]:
                idx += L * 32
    sel_rows = int(counts.sum())
    kv_row = 2 * 128 * s_kv
    q = inp.B * inp.Hq * 128 * s_kv
    out = inp.B * inp.Hq * 128 * 4
    return {"idx": idx, "contig_kv": contig_rows * kv_row, "selected_kv": sel_rows * kv_row, "q": q, "out": out,
            "contig_rows": contig_rows, "selected_rows": sel_rows,
            "total": idx + contig_rows * kv_row + sel_rows * kv_row + q + out}


def cpu_threads() -> int:
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max([i.get("num_threads", 1) for i in info] + [1])
    except Exception:
        return 1


def run_oracle_sample(inp, idx_bits, p, seqs):
    import oracle as O
    slices = [(b, g) for b in seqs for g in range(inp.Hkv)]
    t0 = time.perf_counter()
    O.decode_inputs(inp, idx_cache=idx_bits, p=p, slices=slices)
    return time.perf_counter() - t0


def selection_metrics(B, torch, h, q, idx, lens, inp, p, Lcap, dev, stream):
    """Realised sparsity, index mass captured and planted-key recall of one step's
    selection (the kept lists from spa_select).  Reported only: computed after timing,
    in float32 with torch (the index distribution restated for the report)."""
    sel = torch.full((inp.B, inp.Hkv, inp.Lmax), -1, dtype=torch.int32, device=dev)
    cnt = torch.zeros(inp.B * inp.Hkv, dtype=torch.int32, device=dev)
    B.spa_select(h, q, idx, inp.head_mask, lens, inp.B, Lcap, p, inp.n_sink, inp.window, sel, cnt, stream)
    B.spa_device_status(h, stream)
    cnt = cnt.cpu().numpy().reshape(inp.B, inp.Hkv)
    G = inp.G
    P_q = torch.from_numpy(inp.P_q).to(dev)
    qf = q.float()
    ret_tokens = ret_attended = all_attended = 0
    mass, recall_hit, recall_n = [], 0, 0
    for b in range(inp.B):
        L = int(inp.seq_lens[b])
        n_s = min(inp.n_sink, L)
        w_lo = max(n_s, L - inp.window)
        always = torch.zeros(L, dtype=torch.bool, device=dev)
        always[:n_s] = True
        always[w_lo:] = True
        for g in range(inp.Hkv):
            if not inp.head_mask[g]:
                all_attended += int(always.sum())
                continue
            keep = always.clone()
            lst = sel[b, g, :int(cnt[b, g])].long()
            keep[lst] = True
            heads = slice(g * G, (g + 1) * G)
            q_idx = torch.einsum("hrd,hd->hr", P_q[heads], qf[b, heads])              # [G][16]
            rows = idx[b, g, :L].view(torch.bfloat16).float()                     # bf16 bits -> values
            s = (rows @ q_idx.T) * inp.idx_scale                                   # [L][G]
            pi = torch.softmax(s, dim=0).mean(dim=1)
            mass.append(float(pi[keep].sum()))
            n_keep = int(keep.sum())
            ret_tokens += L
            ret_attended += n_keep
            all_attended += n_keep
            planted = inp.planted.get((b, g))
            if planted is not None and len(planted):
                pl = torch.from_numpy(np.asarray(planted)).to(dev)
                recall_hit += int(keep[pl].sum())
                recall_n += len(planted)
    total = int(sum(int(inp.seq_lens[b]) for b in range(inp.B))) * inp.Hkv
    return {"retrieval_sparsity": 1.0 - ret_attended / max(ret_tokens, 1),
            "overall_sparsity": 1.0 - all_attended / max(total, 1),
            "index_mass_captured": {"min": min(mass) if mass else None, "mean": float(np.mean(mass)) if mass else None},
            "planted_recall": recall_hit / recall_n if recall_n else None, "planted_keys": recall_n,
            "note": "sparsity: share of cached tokens not attended (retrieval heads; all heads); mass: the index "
                    "distribution's mass on each retrieval slice's attended set (sinks, window, kept); recall: "
                    "planted keys attended"}


def run_config(name, args, B, torch, dev, stream, rank, world, peak, timed, capture):
    """Headline-style measurement of another workload: graph-replayed steps over two layer
    copies, algorithmic bytes, achieved GB/s, and the selection metrics."""
    cfg = dict(synth.CONFIGS[name])
    p = float(np.float32(cfg["p"]))
    inp = synth.make_inputs(name, shard.rank_seed(args.seed, rank), draw_streaming_kpre=False)
    s_kv = 2 if inp.dtype == "bf16" else 4

    def up(a):
        if inp.dtype == "bf16":
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    P_q, P_k = torch.from_numpy(inp.P_q).to(dev), torch.from_numpy(inp.P_k).to(dev)
    h = B.spa_create(B.make_config(max_batch=inp.B, n_q_heads=inp.Hq, n_kv_heads=inp.Hkv, max_ctx=inp.Lmax,
                                   kv_dtype=B.SPA_BF16 if inp.dtype == "bf16" else B.SPA_F32, P_q=P_q, P_k=P_k,
                                   rope_theta=inp.rope_theta, idx_scale=inp.idx_scale))
    try:
        q = up(inp.q_pre)
        lens = torch.from_numpy(inp.seq_lens).to(dev)
        k0, v0 = up(inp.k_cache), up(inp.v_cache)
        kp = up(inp.k_pre)
        idx0 = torch.zeros((inp.B, inp.Hkv, inp.Lmax, 16), dtype=torch.int16, device=dev)
        B.spa_index_append(h, kp, torch.zeros(inp.B, dtype=torch.int64, device=dev), inp.B, inp.Lmax, idx0, stream)
        B.spa_device_status(h, stream)
        del kp
        layers = [(k0, v0, idx0), (k0.clone(), v0.clone(), idx0.clone())]
        out = torch.empty((inp.B, inp.Hq, 128), dtype=torch.float32, device=dev)
        cnt = torch.zeros(inp.B * inp.Hkv, dtype=torch.int32, device=dev)
        Lcap = int(inp.seq_lens.max())

        def step(i, st):
            k, v, ix = layers[i % 2]
            B.spa_decode(h, q, k, v, ix, inp.head_mask, lens, inp.B, Lcap, p, inp.n_sink, inp.window, out, None, st)
        step(0, stream)
        torch.cuda.synchronize(dev)
        graphs, err = [], None
        try:
            graphs = [capture(lambda st, j=j: step(j, st)) for j in range(2)]
        except Exception as e:
            err = repr(e)[:200]
        run = (lambda i: graphs[i % 2].replay()) if graphs else (lambda i: step(i, stream))
        for i in range(3):
            run(i)
        n = max(20, args.steps)
        ms, _ = timed(n, run)
        ms = shard.reduce_max(ms, dev) / n
        del graphs
        B.spa_decode(h, q, k0, v0, idx0, inp.head_mask, lens, inp.B, Lcap, p, inp.n_sink, inp.window, out, cnt,
                     stream)
        B.spa_device_status(h, stream)
        ab = algorithmic_bytes(inp, cnt.cpu().numpy(), s_kv)
        gbs = ab["total"] / (ms * 1e-3) / 1e9
        rec = {"workload": workload_desc(cfg, name, p), "ms_per_step": ms, "layer_steps_per_s": world * 1e3 / ms,
               "bytes_per_step": ab, "achieved_gbs": gbs, "frac_of_peak": gbs / peak, "steps": n,
               "timing": "CUDA graph replay, two layer copies cycled" if not err else f"eager ({err})"}
        rec.update(selection_metrics(B, torch, h, q, idx0, lens, inp, p, Lcap, dev, stream))
        return rec
    finally:
        B.spa_destroy(h)
        torch.cuda.synchronize(dev)
        torch.cuda.empty_cache()


# ----------------------------------------------------------------------------- reference arm
def main_reference(args):
    rank, _, world = shard.dist_env()
    if rank != 0:
        return 0
    import oracle as O
    cfg = dict(synth.CONFIGS[args.config])
    cfg.update(overrides(args))
    p = float(np.float32(args.p if args.p is not None else cfg["p"]))
    inp = synth.make_inputs(args.config, shard.rank_seed(args.seed, 0), overrides=overrides(args),
                            draw_streaming_kpre=False)
    ret = [g for g in range(inp.Hkv) if inp.head_mask[g]]
    idx = O.index_cache_for(inp, heads=ret)   # BLAS: fast setup, untimed
    # each step: the oracle's decode of a whole layer-step (every slice of the batch), or,
    # when K + W such steps would take more than about three minutes, of the first
    # n_seq sequences (the value is then scaled by B / n_seq; ms_per_step is measured)
    t_one = run_oracle_sample(inp, idx, p, list(range(inp.B)))
    n_seq = inp.B
    while n_seq > 1 and (args.steps + args.warmup) * t_one * n_seq / inp.B > 180.0:
        n_seq -= 1
    seqs = list(range(n_seq))
    for _ in range(max(0, args.warmup - 1)):
        run_oracle_sample(inp, idx, p, seqs)
    times = [run_oracle_sample(inp, idx, p, seqs) for _ in range(args.steps)]
    sec_per_step = float(np.mean(times))
    value = (n_seq / inp.B) / sec_per_step
    cores = cpu_threads()
    sample = (f"float64 NumPy oracle, a whole layer-step per step (all {inp.B}x{inp.Hkv} slices)" if n_seq == inp.B
              else f"float64 NumPy oracle, {n_seq} of {inp.B} sequences (all {inp.Hkv} KV heads) per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec_per_step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(cfg, args.config, p, world, args.layers),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- native arm
def main_native(args):
    import torch
    import torch.distributed as dist

    from head_partitioned_sparse_b200 import binding as B
    from head_partitioned_sparse_b200 import build as spa_build

    rank, local, world = shard.dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    if not os.path.exists(B.LIB_PATH):
        spa_build.build()
    B.load()

    cfg = dict(synth.CONFIGS[args.config])
    cfg.update(overrides(args))
    p = float(np.float32(args.p if args.p is not None else cfg["p"]))
    inp = synth.make_inputs(args.config, shard.rank_seed(args.seed, rank), overrides=overrides(args),
                            draw_streaming_kpre=False)
    s_kv = 2 if inp.dtype == "bf16" else 4

    def up(a):
        if inp.dtype == "bf16":
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    P_q = torch.from_numpy(inp.P_q).to(dev)
    P_k = torch.from_numpy(inp.P_k).to(dev)
    c = B.make_config(max_batch=inp.B, n_q_heads=inp.Hq, n_kv_heads=inp.Hkv, max_ctx=inp.Lmax,
                      kv_dtype=B.SPA_BF16 if inp.dtype == "bf16" else B.SPA_F32, P_q=P_q, P_k=P_k,
                      rope_theta=inp.rope_theta, idx_scale=inp.idx_scale, split_rows=args.split_rows)
    h = B.spa_create(c)
    stream = torch.cuda.current_stream(dev)
    q = up(inp.q_pre)
    lens = torch.from_numpy(inp.seq_lens).to(dev)
    head_mask = inp.head_mask

    # layer 0 from the generator; the index cache is built on the GPU by spa_index_append
    k0, v0 = up(inp.k_cache), up(inp.v_cache)
    kp = up(inp.k_pre)
    idx0 = torch.zeros((inp.B, inp.Hkv, inp.Lmax, 16), dtype=torch.int16, device=dev)
    zero = torch.zeros(inp.B, dtype=torch.int64, device=dev)
    B.spa_index_append(h, kp, zero, inp.B, inp.Lmax, idx0, stream)
    B.spa_device_status(h, stream)
    del kp
    layers = [(k0, v0, idx0)] + [(k0.clone(), v0.clone(), idx0.clone()) for _ in range(max(1, args.layers) - 1)]
    out = torch.empty((inp.B, inp.Hq, 128), dtype=torch.float32, device=dev)
    cnt = torch.zeros(inp.B * inp.Hkv, dtype=torch.int32, device=dev)
    Lcap = int(inp.seq_lens.max())

    def step(i, pp=p, st=stream):
        k, v, ix = layers[i % len(layers)]
        B.spa_decode(h, q, k, v, ix, head_mask, lens, inp.B, Lcap, pp, inp.n_sink, inp.window, out, None, st)

    def barrier():
        if world > 1:
            dist.barrier()

    def timed(n_steps, fn, profile_mask=0):
        torch.cuda.synchronize(dev)
        barrier()
        if profile_mask:
            B.spa_set_profiling(h, profile_mask)
        n0 = B.spa_launch_count(h)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(n_steps):
            fn(i)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        launches = B.spa_launch_count(h) - n0
        return e0.elapsed_time(e1), launches

    def capture(fn):
        """fn(st) captured in a CUDA graph on a side stream (thread-local capture mode, so
        other threads' CUDA calls, e.g. a process group's watchdog, stay legal)."""
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(device=dev)
        cap.wait_stream(stream)
        with torch.cuda.graph(g, stream=cap, capture_error_mode="thread_local"):
            fn(None)
        torch.cuda.synchronize(dev)
        return g

    class Stepper:
        """One step per call on layer copy i % layers, replayed from a CUDA graph per copy
        (eager launches if capture fails; the reason is reported)."""

        def __init__(self, fn):
            self.fn, self.graphs, self.error = fn, [], None
            n0 = B.spa_launch_count(h)
            fn(0, stream)                       # eager warm-up step, counts the launches
            torch.cuda.synchronize(dev)
            self.launches = B.spa_launch_count(h) - n0
            try:
                self.graphs = [capture(lambda st, j=j: fn(j, st)) for j in range(len(layers))]
            except Exception as e:
                self.graphs, self.error = [], repr(e)[:200]

        def __call__(self, i):
            if self.graphs:
                self.graphs[i % len(self.graphs)].replay()
            else:
                self.fn(i, stream)

        def time(self, n, warm=3):
            for i in range(warm):
                self(i)
            ms, _ = timed(n, self)
            return shard.reduce_max(ms, dev) / n

        def distribution(self, n):
            """Per-step device times (us) from events between consecutive steps."""
            torch.cuda.synchronize(dev)
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
            ev[0].record(stream)
            for i in range(n):
                self(i)
                ev[i + 1].record(stream)
            torch.cuda.synchronize(dev)
            return [1e3 * ev[i].elapsed_time(ev[i + 1]) for i in range(n)]

        def release(self):
            self.graphs = []

    clocks = ClockSampler(local) if rank == 0 else None
    main = Stepper(lambda i, st: step(i, st=st))
    for i in range(args.warmup):
        main(i)
    # headline: K steps replayed from the graphs, events only at both ends
    ms, _ = timed(args.steps, main)
    ms_max = shard.reduce_max(ms, dev)
    ms_per_step = ms_max / args.steps
    launches = main.launches * args.steps
    # per-step distribution (events between consecutive steps), at least 200 steps
    n_dist = max(200, args.steps)
    per_step = np.array(main.distribution(n_dist))
    dist_us = {"steps": n_dist, "median": float(np.median(per_step)), "p10": float(np.percentile(per_step, 10)),
               "p90": float(np.percentile(per_step, 90)), "min": float(per_step.min()),
               "max": float(per_step.max())}
    # per-kernel breakdown: a separate eager pass with events around every launch
    # (each event pair adds stream time; the attention kernel's roofline uses it)
    n_brk = max(20, args.steps)
    for i in range(3):
        step(i)
    timed(n_brk, step, profile_mask=(1 << B.SPA_K_COUNT) - 1)
    kern = {}
    for kid in range(B.SPA_K_COUNT):
        tot_k, n_k = B.spa_profile_read(h, kid)
        if n_k:
            kern[B.spa_kernel_name(kid)] = {"launches": n_k, "avg_us": 1e3 * tot_k / n_k}
    B.spa_set_profiling(h, 0)
    attend_us = kern.get("attend", {}).get("avg_us", float("nan"))

    # selected counts of this workload (identical every step)
    B.spa_decode(h, q, layers[0][0], layers[0][1], layers[0][2], head_mask, lens, inp.B, Lcap, p, inp.n_sink,
                 inp.window, out, cnt, stream)
    B.spa_device_status(h, stream)
    counts = cnt.cpu().numpy().reshape(inp.B, inp.Hkv)
    ab = algorithmic_bytes(inp, counts, s_kv)
    peak, peak_kind = measured_peaks()

    def record(ms_step, abx, stepper=None):
        gbs = abx["total"] / (ms_step * 1e-3) / 1e9
        r = {"ms_per_step": ms_step, "layer_steps_per_s": world * 1e3 / ms_step, "achieved_gbs": gbs,
             "frac_of_peak": gbs / peak, "selected_rows": abx["selected_rows"], "bytes_per_step": abx["total"]}
        if stepper is not None and stepper.error:
            r["graph_error"] = stepper.error
        return r

    # p sweep (same measurement, smaller step count)
    sweep = {}
    if not args.no_sweep and "p_sweep" in cfg:
        for pp in cfg["p_sweep"]:
            pq = float(np.float32(pp))
            sw = Stepper(lambda i, st, pq=pq: step(i, pq, st))
            msw = sw.time(max(20, args.steps))
            sw.release()
            B.spa_decode(h, q, layers[0][0], layers[0][1], layers[0][2], head_mask, lens, inp.B, Lcap, pq,
                         inp.n_sink, inp.window, out, cnt, stream)
            torch.cuda.synchronize(dev)
            sweep[f"{pp:g}"] = record(msw, algorithmic_bytes(inp, cnt.cpu().numpy(), s_kv), sw)

    # top-k selector variant (same measurement, smaller step count)
    topk_sweep = {}
    if not args.no_topk_sweep:
        for kk in (2048, 16384, 65536):
            def step_k(i, st, kk=kk):
                kc, vc, ixc = layers[i % len(layers)]
                B.spa_decode_topk(h, q, kc, vc, ixc, head_mask, lens, inp.B, Lcap, kk, inp.n_sink, inp.window,
                                  out, None, st)
            sk = Stepper(step_k)
            msk = sk.time(max(20, args.steps))
            sk.release()
            B.spa_decode_topk(h, q, layers[0][0], layers[0][1], layers[0][2], head_mask, lens, inp.B, Lcap, kk,
                              inp.n_sink, inp.window, out, cnt, stream)
            torch.cuda.synchronize(dev)
            topk_sweep[str(kk)] = record(msk, algorithmic_bytes(inp, cnt.cpu().numpy(), s_kv), sk)

    # block-granular top-p variant (64-token blocks; same measurement, smaller step count)
    block_sweep = {}
    if not args.no_block_sweep:
        for pp in (0.9, 0.99):
            pq = float(np.float32(pp))
            def step_b(i, st, pq=pq):
                kc, vc, ixc = layers[i % len(layers)]
                B.spa_decode_blocks(h, q, kc, vc, ixc, head_mask, lens, inp.B, Lcap, pq, inp.n_sink, inp.window,
                                    out, None, st)
            sb = Stepper(step_b)
            msb = sb.time(max(20, args.steps))
            sb.release()
            B.spa_decode_blocks(h, q, layers[0][0], layers[0][1], layers[0][2], head_mask, lens, inp.B, Lcap, pq,
                                inp.n_sink, inp.window, out, cnt, stream)
            torch.cuda.synchronize(dev)
            block_sweep[f"{pp:g}"] = record(msb, algorithmic_bytes(inp, cnt.cpu().numpy(), s_kv), sb)

    # compact KV layout: streaming heads keep only sinks + a ring-buffered window
    compact = None
    if not args.no_compact:
        ret = [g for g in range(inp.Hkv) if head_mask[g]]
        n_ret, n_str, ring = len(ret), inp.Hkv - len(ret), inp.n_sink + inp.window
        c_layers = []
        for (k, v, ix) in layers:
            kr = torch.empty((inp.B, max(n_ret, 1), inp.Lmax, 128), dtype=k.dtype, device=dev)
            vr = torch.empty_like(kr)
            ks = torch.empty((inp.B, max(n_str, 1), max(ring, 1), 128), dtype=k.dtype, device=dev)
            vs = torch.empty_like(ks)
            for b in range(inp.B):   # prefill each sequence into its slot through the library
                L_b = int(inp.seq_lens[b])
                B.spa_kv_append_compact(h, k[b:b + 1, :, :L_b].contiguous(), v[b:b + 1, :, :L_b].contiguous(),
                                        torch.zeros(1, dtype=torch.int64, device=dev), 1, L_b, head_mask,
                                        inp.n_sink, inp.window, kr[b], vr[b], ks[b], vs[b], stream)
            c_layers.append((kr, vr, ks, vs, ix[:, ret].contiguous()))
        B.spa_device_status(h, stream)

        def step_c(i, st):
            kr, vr, ks, vs, ixr = c_layers[i % len(c_layers)]
            B.spa_decode_compact(h, q, kr, vr, ks, vs, ixr, head_mask, lens, inp.B, Lcap, p, inp.n_sink,
                                 inp.window, out, None, st)
        sc = Stepper(step_c)
        msc = sc.time(max(20, args.steps))
        sc.release()
        row = 128 * s_kv * 2   # K + V bytes per position and head
        full_b = inp.B * inp.Hkv * inp.Lmax * row
        comp_b = inp.B * (n_ret * inp.Lmax + n_str * ring) * row
        compact = {"ms_per_step": msc, "layer_steps_per_s": world * 1e3 / msc,
                   "achieved_gbs": ab["total"] / (msc * 1e-3) / 1e9,
                   "kv_bytes_full_layout": full_b, "kv_bytes_compact": comp_b,
                   "kv_memory_ratio": full_b / comp_b}
        del c_layers

    # prefill of one sequence's first prefill_len positions (tensor cores; reported beside)
    prefill = None
    if not args.no_prefill and inp.dtype == "bf16":
        Tp = min(args.prefill_len, inp.Lmax)
        gq = torch.Generator(device=dev)
        gq.manual_seed(1234 + rank)
        q_chunk = torch.randn((1, inp.Hq, Tp, 128), generator=gq, device=dev).to(torch.bfloat16)
        out_p = torch.empty((1, inp.Hq, Tp, 128), dtype=torch.float32, device=dev)
        kc, vc = layers[0][0][0:1].contiguous(), layers[0][1][0:1].contiguous()
        zero1 = torch.zeros(1, dtype=torch.int64, device=dev)

        def step_p(i):
            B.spa_prefill(h, q_chunk, kc, vc, head_mask, zero1, 1, Tp, inp.n_sink, inp.window, out_p, stream)
        for i in range(3):
            step_p(i)
        B.spa_device_status(h, stream)
        n = 5
        msp, _ = timed(n, step_p)
        msp = shard.reduce_max(msp, dev) / n
        fl = prefill_flops(Tp, 0, head_mask, inp.G, inp.n_sink, inp.window)
        tpk, tpk_kind = measured_bf16_tflops()
        prefill = {"tokens": Tp, "ms": msp, "tokens_per_s": world * Tp / (msp * 1e-3),
                   "tflops": fl / (msp * 1e-3) / 1e12, "flops": fl, "peak_tflops": tpk, "peak_kind": tpk_kind,
                   "frac": fl / (msp * 1e-3) / 1e12 / tpk, "bound": "tensor",
                   "note": "one sequence from position 0: causal dense for retrieval heads, sinks + window "
                           "for streaming heads; bf16 inputs, float32 accumulation (tcgen05 MMA, TMEM accumulators)"}
        del q_chunk, out_p, kc, vc

    # context-parallel decode of the same step: the positions split over cp_ranks ranks,
    # emulated on this GPU (one handle and one cache shard per rank, the phases run rank
    # after rank, exchange buffers shared: no transfer is timed).  Reported: each rank's
    # kernel time per step (CUDA events around each of its launches), the whole emulated
    # step, the bytes each rank would all-gather, and agreement with the one-GPU step.
    cpar = None
    if not args.no_cp and inp.dtype == "bf16" and args.cp_ranks >= 1:
        from head_partitioned_sparse_b200 import context_parallel as cpm
        R = args.cp_ranks
        C = -(-inp.Lmax // R)          # rows per rank, rounded up to 64
        C = -(-C // 64) * 64
        k0_, v0_, ix0_ = layers[0]
        cp_handles, shards = [], []
        for r in range(R):
            cp_handles.append(B.spa_create(B.make_config(
                max_batch=inp.B, n_q_heads=inp.Hq, n_kv_heads=inp.Hkv, max_ctx=C, kv_dtype=B.SPA_BF16, P_q=P_q,
                P_k=P_k, rope_theta=inp.rope_theta, idx_scale=inp.idx_scale, split_rows=args.split_rows)))
            lo, hi = r * C, min((r + 1) * C, inp.Lmax)

            def sl(t):
                z = torch.zeros((inp.B, inp.Hkv, C) + tuple(t.shape[3:]), dtype=t.dtype, device=dev)
                if hi > lo:
                    z[:, :, :hi - lo] = t[:, :, lo:hi]
                return z
            shards.append({"k": sl(k0_), "v": sl(v0_), "idx": sl(ix0_)})
        out_cp = torch.empty_like(out)
        cp_bufs = cpm.alloc_exchange(B.spa_cp_exchange_sizes(cp_handles[0], inp.B, R, head_mask), dev)

        def step_cp(i, st=stream, ranks=None, combine=True, exchange=None):
            cpm.emulated_step(cp_handles, shards, q_pre=q, head_mask=head_mask, seq_lens=lens, Bsz=inp.B, p=p,
                              n_sink=inp.n_sink, window=inp.window, capacity=C, out=out_cp, bufs=cp_bufs,
                              max_seq_len=Lcap, stream=st, ranks=ranks, combine=combine, exchange=exchange)
        for i in range(3):
            step_cp(i)
        for hh in cp_handles:
            B.spa_device_status(hh, stream)
        n = max(10, args.steps // 10)
        ms_cp, _ = timed(n, step_cp)
        ms_cp = shard.reduce_max(ms_cp, dev) / n
        mask_cp = (1 << B.SPA_K_CP_SELECT) | (1 << B.SPA_K_ATTEND) | (1 << B.SPA_K_COMBINE)
        for hh in cp_handles:
            B.spa_set_profiling(hh, mask_cp)
        timed(n, step_cp)
        rank_us, sel_us, att_us = [], [], []
        for hh in cp_handles:
            ts, _ = B.spa_profile_read(hh, B.SPA_K_CP_SELECT)
            ta, _ = B.spa_profile_read(hh, B.SPA_K_ATTEND)
            sel_us.append(1e3 * ts / n)
            att_us.append(1e3 * ta / n)
            rank_us.append(1e3 * (ts + ta) / n)
        tc, _ = B.spa_profile_read(cp_handles[0], B.SPA_K_COMBINE)
        for hh in cp_handles:
            B.spa_set_profiling(hh, 0)
        B.spa_decode(h, q, k0_, v0_, ix0_, head_mask, lens, inp.B, Lcap, p, inp.n_sink, inp.window, out, None,
                     stream)
        step_cp(0)
        torch.cuda.synchronize(dev)
        # device time alone: each rank's launches (and the whole emulated step) captured
        # in a CUDA graph and replayed, so no host launch gap is timed
        def graph_of(fn):
            g = torch.cuda.CUDAGraph()
            cap = torch.cuda.Stream(device=dev)
            cap.wait_stream(stream)
            # thread-local capture: other threads' CUDA calls (a process group's watchdog
            # under torchrun) stay legal while this thread captures
            with torch.cuda.graph(g, stream=cap, capture_error_mode="thread_local"):
                fn()
            torch.cuda.synchronize(dev)
            return g

        def replay_us(g, reps):
            torch.cuda.synchronize(dev)
            a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                g.replay()
            z.record(stream)
            torch.cuda.synchronize(dev)
            return 1e3 * a.elapsed_time(z) / reps

        graph_step_us, graph_rank_us, graph_err, copy_us = None, [], None, None
        try:
            g_all = graph_of(lambda: step_cp(0, st=None))
            graph_step_us = replay_us(g_all, n)
            del g_all
            # one rank alone: the gathered buffers' other slots hold the full step's data;
            # the summed histograms get the full step's sums back after the phase that
            # adds into them (the all-reduce of a real step), and that copy's own time,
            # from a graph of the copies alone, is taken off the rank's time
            totals = {nm: cp_bufs[nm].clone() for nm in cpm.SUMMED}

            def restore(name):
                if name in totals:
                    cp_bufs[name].copy_(totals[name])
            g_c = graph_of(lambda: [restore(nm) for nm in cpm.SUMMED])
            copy_us = replay_us(g_c, n)
            del g_c
            for r in range(R):
                g_r = graph_of(lambda: step_cp(0, st=None, ranks=[r], combine=False, exchange=restore))
                graph_rank_us.append(replay_us(g_r, n) - copy_us)
                del g_r
            del totals
        except Exception as e:   # reported, not fatal: the step itself was timed above
            graph_err = repr(e)[:200]
        step_cp(0)
        torch.cuda.synchronize(dev)
        sizes = B.spa_cp_exchange_sizes(cp_handles[0], inp.B, R, head_mask)
        cpar = {"ranks": R, "rows_per_rank": C, "emulated_step_ms": ms_cp,
                "graph_step_us": graph_step_us, "graph_rank_us": graph_rank_us,
                "max_graph_rank_us": max(graph_rank_us) if graph_rank_us else None, "graph_error": graph_err,
                "rank_graph_sum_copy_us": copy_us,
                "rank_kernel_us": rank_us, "rank_select_us": sel_us, "rank_attend_us": att_us,
                "max_rank_kernel_us": max(rank_us), "combine_us": 1e3 * tc / n,
                "exchange_bytes_per_rank": int(sum(sz // (1 if nm in cpm.SUMMED else R)
                                                   for nm, sz in zip(cpm.BUFFERS, sizes))),
                "one_gpu_step_ms": ms_per_step,
                "max_abs_vs_one_gpu": float((out_cp - out).abs().max().item()),
                "note": "ranks emulated on one GPU one after another, exchanges not timed (buffers shared); "
                        "rank_*_us: CUDA events around each launch of a Python-driven step (host gaps "
                        "included); graph_*_us: the same launches replayed from a CUDA graph (device time; "
                        "graph_rank_us: one rank's launches alone, the summed histograms set to the full "
                        "step's sums after the phase that adds into them and that copy's time taken off); "
                        "exchange_bytes_per_rank: the rank's slot of each gathered buffer plus the whole of "
                        "each all-reduced one"}
        for hh in cp_handles:
            B.spa_destroy(hh)
        del shards, cp_bufs, out_cp

    # end to end through the public API: pinned host inputs in, result out, every step.
    # Every step copies its own inputs (query, new pre-RoPE key, positions, new K/V rows)
    # from pinned host memory and reads its output back.  The copies run on a copy
    # stream with double-buffered device buffers: step i+1's inputs load and step i-1's
    # output drains while step i computes (events order each copy against the kernels
    # that use its buffer).  The timed region ends when the last output is on the host.
    e2e = None
    if not args.no_e2e:
        pin = lambda t: t.cpu().pin_memory()
        t_last = Lcap - 1
        q_h = pin(q)
        kpre_new = torch.from_numpy(np.ascontiguousarray(inp.k_pre[:, :, t_last:t_last + 1]))
        kpre_h = (kpre_new.view(torch.int16) if inp.dtype == "bf16" else kpre_new).pin_memory()
        knew_h = pin(layers[0][0][:, :, t_last].contiguous())
        vnew_h = pin(layers[0][1][:, :, t_last].contiguous())
        pos_h = torch.full((inp.B,), t_last, dtype=torch.int64).pin_memory()
        out_h = [torch.empty((inp.B, inp.Hq, 128), dtype=torch.float32).pin_memory() for _ in range(2)]
        q_d = [torch.empty_like(q) for _ in range(2)]
        kpre_d = [torch.empty(kpre_h.shape, dtype=kpre_h.dtype, device=dev) for _ in range(2)]
        pos_d = [torch.empty(inp.B, dtype=torch.int64, device=dev) for _ in range(2)]
        out_d = [torch.empty_like(out) for _ in range(2)]
        cstream = torch.cuda.Stream(device=dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of the buffer set are on the device
        ev_used = [torch.cuda.Event() for _ in range(2)]   # the step using the buffer set has finished
        ev_out = [torch.cuda.Event() for _ in range(2)]    # its output has reached the host

        def load_inputs(i):
            j = i % 2
            k, v, _ = layers[i % len(layers)]
            with torch.cuda.stream(cstream):
                cstream.wait_event(ev_used[j])       # the step two back is done with this set
                q_d[j].copy_(q_h, non_blocking=True)
                kpre_d[j].copy_(kpre_h, non_blocking=True)
                pos_d[j].copy_(pos_h, non_blocking=True)
                k[:, :, t_last].copy_(knew_h, non_blocking=True)
                v[:, :, t_last].copy_(vnew_h, non_blocking=True)
                ev_in[j].record(cstream)

        def e2e_kernels(i, st):
            """The step's API calls: index rows of the new token, then the decode."""
            j = i % 2
            k, v, ix = layers[i % len(layers)]
            B.spa_index_append(h, kpre_d[j], pos_d[j], inp.B, 1, ix, st)
            B.spa_decode(h, q_d[j], k, v, ix, head_mask, lens, inp.B, Lcap, p, inp.n_sink, inp.window, out_d[j],
                         None, st)

        # the calls of each (buffer set, layer copy) pair captured once in a CUDA graph, as
        # a serving loop would replay them (eager calls if capture fails); both buffer
        # sets hold valid inputs before the eager warm-up calls
        e2e_graphs, e2e_graph_error = {}, None
        load_inputs(0)
        load_inputs(1)
        torch.cuda.synchronize(dev)
        for i in range(2):
            e2e_kernels(i, stream)
        torch.cuda.synchronize(dev)
        try:
            for i in range(2 * len(layers)):
                key = (i % 2, i % len(layers))
                if key not in e2e_graphs:
                    e2e_graphs[key] = capture(lambda st, i=i: e2e_kernels(i, st))
        except Exception as e:
            e2e_graphs, e2e_graph_error = {}, repr(e)[:200]

        def e2e_step(i):
            j = i % 2
            stream.wait_event(ev_in[j])
            stream.wait_event(ev_out[j])             # out_d[j] of two steps back has drained
            g = e2e_graphs.get((j, i % len(layers)))
            if g is not None:
                with torch.cuda.stream(stream):
                    g.replay()
            else:
                e2e_kernels(i, stream)
            ev_used[j].record(stream)
            with torch.cuda.stream(cstream):
                cstream.wait_event(ev_used[j])
                out_h[j].copy_(out_d[j], non_blocking=True)
                ev_out[j].record(cstream)
            load_inputs(i + 2)                        # two steps ahead (same buffer set)

        def e2e_run(n):
            cstream.wait_stream(stream)               # nothing before the timing start event
            load_inputs(0)
            load_inputs(1)
            for i in range(n):
                e2e_step(i)
            stream.wait_stream(cstream)               # the last outputs are on the host

        e2e_run(3)
        torch.cuda.synchronize(dev)
        mse, _ = timed(1, lambda _i: e2e_run(args.steps))
        mse = shard.reduce_max(mse, dev) / args.steps
        h2d = (q_h.numel() * q_h.element_size() + kpre_h.numel() * kpre_h.element_size() + pos_h.numel() * 8 +
               knew_h.numel() * knew_h.element_size() + vnew_h.numel() * vnew_h.element_size())
        d2h = out_h[0].numel() * 4
        e2e = {"value": world * 1e3 / mse, "unit": UNIT, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "ms_per_step": mse,
               "note": "copies on a second stream, double-buffered: step i+1's inputs load and step i-1's "
                       "output drains while step i computes; each step's spa_index_append + spa_decode calls "
                       "replayed from a CUDA graph captured from those calls"
                       + (f" (capture failed, eager calls: {e2e_graph_error})" if e2e_graph_error else "")}
    # selection metrics of the headline workload (reported, outside every timed region)
    sel_metrics = selection_metrics(B, torch, h, q, layers[0][2], lens, inp, p, Lcap, dev, stream)

    # index append throughput: the whole prefill of every head's index rows
    iapp = None
    if not args.no_index_append:
        kp = up(inp.k_pre)
        zero = torch.zeros(inp.B, dtype=torch.int64, device=dev)
        ix_t = torch.empty_like(layers[0][2])

        def step_ia(i, st):
            B.spa_index_append(h, kp, zero, inp.B, inp.Lmax, ix_t, st)
        sia = Stepper(step_ia)
        n = 10
        msi = sia.time(n)
        sia.release()
        B.spa_device_status(h, stream)
        rows = inp.B * inp.Hkv * inp.Lmax
        byts = rows * (128 * s_kv + 32)
        gbs = byts / (msi * 1e-3) / 1e9
        iapp = {"rows": rows, "ms": msi, "bytes": byts, "achieved_gbs": gbs, "frac_of_peak": gbs / peak,
                "peak": peak, "peak_kind": peak_kind, "bound": "hbm",
                "note": f"{inp.B}x{inp.Hkv} (sequence, KV head) slices x {inp.Lmax} positions: "
                        f"{128 * s_kv} B of pre-RoPE key read and 32 B of index row written per row"}
        del kp, ix_t

    # the other workloads, one sub-record each (a smaller step count)
    per_config = {}
    if not args.no_configs:
        for name in [c for c in ("llama3_8b_32k", "batch16_64k", "ctx1m") if c != args.config]:
            per_config[name] = run_config(name, args, B, torch, dev, stream, rank, world, peak, timed, capture)

    clk = clocks.stop() if clocks else None

    if rank == 0:
        att_bytes = (ab["contig_rows"] + ab["selected_rows"]) * 2 * 128 * s_kv
        achieved = att_bytes / (attend_us * 1e-6) / 1e9
        traffic = recorded_traffic("k_attend_mma.cu", "attend_ctx128k.md") if args.config == "ctx128k" else None
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            import oracle as O
            ret = [g for g in range(inp.Hkv) if inp.head_mask[g]]
            idx_o = O.index_cache_for(inp, heads=ret)   # untimed setup
            t_first = run_oracle_sample(inp, idx_o, p, list(range(inp.B)))
            reps = max(1, min(8, math.ceil(10.0 / max(t_first, 1e-3)))) - 1
            tot = t_first + sum(run_oracle_sample(inp, idx_o, p, list(range(inp.B))) for _ in range(reps))
            cpu = {"value": (reps + 1) / tot, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                   "sample": f"full layer-step (all {inp.B}x{inp.Hkv} slices) x{reps + 1} with the float64 "
                             f"NumPy oracle; index cache precomputed"}
        step_gbs = ab["total"] / (ms_per_step * 1e-3) / 1e9
        line = {
            "metric": METRIC, "value": world * 1e3 / ms_per_step, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": config_dict(cfg, args.config, p, world, len(layers)),
            "timing": ("each step replayed from a CUDA graph (one per layer copy); CUDA events on the launch "
                       "stream at both ends of the K timed steps" if main.graphs else
                       f"eager launches (graph capture failed: {main.error}); CUDA events at both ends"),
            "step_us_distribution": dist_us,
            "achieved_gbs": step_gbs,
            "frac_of_peak": step_gbs / peak,
            "bytes_per_step": ab,
            "selected_counts": counts.tolist(),
            "kernels_us": kern,
            "kernels_us_note": "separate eager pass with CUDA events around every launch; each pair adds stream time",
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic, "kernel": "attend",
                         "avg_us": attend_us, "bytes_per_launch": att_bytes, "peak_kind": peak_kind,
                         "step_achieved": step_gbs, "step_frac": step_gbs / peak,
                         "step_bytes": ab["total"], "step_us": ms_per_step * 1e3},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": int(launches),
            "clocks": clk,
            "p_sweep": sweep or None,
            "topk_sweep": topk_sweep or None,
            "block_sweep": block_sweep or None,
            "compact": compact,
            "prefill": prefill,
            "context_parallel": cpar,
            "selection": sel_metrics,
            "index_append": iapp,
            "configs": per_config or None,
        }
        print(json.dumps(line), flush=True)
    B.spa_destroy(h)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return main_reference(args)
    return main_native(args)


if __name__ == "__main__":
    sys.exit(main())

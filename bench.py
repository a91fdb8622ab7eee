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
    # each step: the oracle's decode of one sequence of the batch (all its KV heads);
    # a layer-step is B such samples.
    for i in range(args.warmup):
        run_oracle_sample(inp, idx, p, [i % inp.B])
    times = [run_oracle_sample(inp, idx, p, [i % inp.B]) for i in range(args.steps)]
    sec_per_layer_step = float(np.mean(times)) * inp.B
    value = 1.0 / sec_per_layer_step
    cores = cpu_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec_per_layer_step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(cfg, args.config, p), "batch": inp.B, "seq_len": inp.Lmax, "p": p},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"float64 NumPy oracle, one sequence (all {inp.Hkv} KV heads) per step, "
                                   f"x{inp.B} per layer-step"},
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

    def step(i, pp=p):
        k, v, ix = layers[i % len(layers)]
        B.spa_decode(h, q, k, v, ix, head_mask, lens, inp.B, Lcap, pp, inp.n_sink, inp.window, out, None, stream)

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

    clocks = ClockSampler(local) if rank == 0 else None
    for i in range(args.warmup):
        step(i)
    # headline: events only around the dominant kernel (attend), on the launch stream
    ms, launches = timed(args.steps, step, profile_mask=1 << B.SPA_K_ATTEND)
    tot, n = B.spa_profile_read(h, B.SPA_K_ATTEND)
    attend_us = 1e3 * tot / max(n, 1)
    B.spa_set_profiling(h, 0)
    ms_max = shard.reduce_max(ms, dev)
    ms_per_step = ms_max / args.steps
    # per-kernel breakdown: a separate pass with events around every launch (adds stream gaps)
    n_brk = max(10, args.steps // 4)
    timed(n_brk, step, profile_mask=(1 << B.SPA_K_COUNT) - 1)
    kern = {}
    for kid in range(B.SPA_K_COUNT):
        tot_k, n_k = B.spa_profile_read(h, kid)
        if n_k:
            kern[B.spa_kernel_name(kid)] = {"launches": n_k, "avg_us": 1e3 * tot_k / n_k}
    B.spa_set_profiling(h, 0)

    # selected counts of this workload (identical every step)
    B.spa_decode(h, q, layers[0][0], layers[0][1], layers[0][2], head_mask, lens, inp.B, Lcap, p, inp.n_sink,
                 inp.window, out, cnt, stream)
    B.spa_device_status(h, stream)
    counts = cnt.cpu().numpy().reshape(inp.B, inp.Hkv)
    ab = algorithmic_bytes(inp, counts, s_kv)

    # p sweep (same measurement, smaller step count)
    sweep = {}
    if not args.no_sweep and "p_sweep" in cfg:
        for pp in cfg["p_sweep"]:
            pq = float(np.float32(pp))
            for i in range(3):
                step(i, pq)
            n = max(10, args.steps // 4)
            msw, _ = timed(n, lambda i: step(i, pq))
            msw = shard.reduce_max(msw, dev) / n
            B.spa_decode(h, q, layers[0][0], layers[0][1], layers[0][2], head_mask, lens, inp.B, Lcap, pq,
                         inp.n_sink, inp.window, out, cnt, stream)
            torch.cuda.synchronize(dev)
            abw = algorithmic_bytes(inp, cnt.cpu().numpy(), s_kv)
            sweep[f"{pp:g}"] = {"ms_per_step": msw, "layer_steps_per_s": world * 1e3 / msw,
                                "achieved_gbs": abw["total"] / (msw * 1e-3) / 1e9,
                                "selected_rows": abw["selected_rows"]}

    # top-k selector variant (same measurement, smaller step count)
    topk_sweep = {}
    if not args.no_topk_sweep:
        for kk in (2048, 16384, 65536):
            def step_k(i, kk=kk):
                kc, vc, ixc = layers[i % len(layers)]
                B.spa_decode_topk(h, q, kc, vc, ixc, head_mask, lens, inp.B, Lcap, kk, inp.n_sink, inp.window,
                                  out, None, stream)
            for i in range(3):
                step_k(i)
            n = max(10, args.steps // 4)
            msk, _ = timed(n, step_k)
            msk = shard.reduce_max(msk, dev) / n
            B.spa_decode_topk(h, q, layers[0][0], layers[0][1], layers[0][2], head_mask, lens, inp.B, Lcap, kk,
                              inp.n_sink, inp.window, out, cnt, stream)
            torch.cuda.synchronize(dev)
            abk = algorithmic_bytes(inp, cnt.cpu().numpy(), s_kv)
            topk_sweep[str(kk)] = {"ms_per_step": msk, "layer_steps_per_s": world * 1e3 / msk,
                                   "achieved_gbs": abk["total"] / (msk * 1e-3) / 1e9,
                                   "selected_rows": abk["selected_rows"]}

    # block-granular top-p variant (64-token blocks; same measurement, smaller step count)
    block_sweep = {}
    if not args.no_block_sweep:
        for pp in (0.9, 0.99):
            pq = float(np.float32(pp))
            def step_b(i, pq=pq):
                kc, vc, ixc = layers[i % len(layers)]
                B.spa_decode_blocks(h, q, kc, vc, ixc, head_mask, lens, inp.B, Lcap, pq, inp.n_sink, inp.window,
                                    out, None, stream)
            for i in range(3):
                step_b(i)
            n = max(10, args.steps // 4)
            msb, _ = timed(n, step_b)
            msb = shard.reduce_max(msb, dev) / n
            B.spa_decode_blocks(h, q, layers[0][0], layers[0][1], layers[0][2], head_mask, lens, inp.B, Lcap, pq,
                                inp.n_sink, inp.window, out, cnt, stream)
            torch.cuda.synchronize(dev)
            abb = algorithmic_bytes(inp, cnt.cpu().numpy(), s_kv)
            block_sweep[f"{pp:g}"] = {"ms_per_step": msb, "layer_steps_per_s": world * 1e3 / msb,
                                      "achieved_gbs": abb["total"] / (msb * 1e-3) / 1e9,
                                      "selected_rows": abb["selected_rows"]}

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

        def step_c(i):
            kr, vr, ks, vs, ixr = c_layers[i % len(c_layers)]
            B.spa_decode_compact(h, q, kr, vr, ks, vs, ixr, head_mask, lens, inp.B, Lcap, p, inp.n_sink,
                                 inp.window, out, None, stream)
        for i in range(3):
            step_c(i)
        n = max(10, args.steps // 4)
        msc, _ = timed(n, step_c)
        msc = shard.reduce_max(msc, dev) / n
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
        cp_bufs = cpm.alloc_exchange(B.spa_cp_exchange_sizes(cp_handles[0], inp.B, R), dev)

        def step_cp(i, st=stream, ranks=None, combine=True):
            cpm.emulated_step(cp_handles, shards, q_pre=q, head_mask=head_mask, seq_lens=lens, Bsz=inp.B, p=p,
                              n_sink=inp.n_sink, window=inp.window, capacity=C, out=out_cp, bufs=cp_bufs,
                              max_seq_len=Lcap, stream=st, ranks=ranks, combine=combine)
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

        graph_step_us, graph_rank_us, graph_err = None, [], None
        try:
            g_all = graph_of(lambda: step_cp(0, st=None))
            graph_step_us = replay_us(g_all, n)
            del g_all
            for r in range(R):
                g_r = graph_of(lambda: step_cp(0, st=None, ranks=[r], combine=False))
                graph_rank_us.append(replay_us(g_r, n))
                del g_r
        except Exception as e:   # reported, not fatal: the step itself was timed above
            graph_err = repr(e)[:200]
        step_cp(0)
        torch.cuda.synchronize(dev)
        sizes = B.spa_cp_exchange_sizes(cp_handles[0], inp.B, R)
        cpar = {"ranks": R, "rows_per_rank": C, "emulated_step_ms": ms_cp,
                "graph_step_us": graph_step_us, "graph_rank_us": graph_rank_us,
                "max_graph_rank_us": max(graph_rank_us) if graph_rank_us else None, "graph_error": graph_err,
                "rank_kernel_us": rank_us, "rank_select_us": sel_us, "rank_attend_us": att_us,
                "max_rank_kernel_us": max(rank_us), "combine_us": 1e3 * tc / n,
                "exchange_bytes_per_rank": int(sum(sizes) // R),
                "one_gpu_step_ms": ms_per_step,
                "max_abs_vs_one_gpu": float((out_cp - out).abs().max().item()),
                "note": "ranks emulated on one GPU one after another, exchanges not timed (buffers shared); "
                        "rank_*_us: CUDA events around each launch of a Python-driven step (host gaps "
                        "included); graph_*_us: the same launches replayed from a CUDA graph (device time)"}
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

        def e2e_step(i):
            j = i % 2
            k, v, ix = layers[i % len(layers)]
            stream.wait_event(ev_in[j])
            stream.wait_event(ev_out[j])             # out_d[j] of two steps back has drained
            B.spa_index_append(h, kpre_d[j], pos_d[j], inp.B, 1, ix, stream)
            B.spa_decode(h, q_d[j], k, v, ix, head_mask, lens, inp.B, Lcap, p, inp.n_sink, inp.window, out_d[j],
                         None, stream)
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
                       "output drains while step i computes"}
    clk = clocks.stop() if clocks else None

    if rank == 0:
        peak, peak_kind = measured_peaks()
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
            "config": {"workload": workload_desc(cfg, args.config, p), "batch": inp.B, "seq_len": inp.Lmax,
                       "p": p, "storage": inp.dtype, "parallelism": f"dp{world}" if world > 1 else "single",
                       "l2": f"inputs larger than L2: {len(layers)} layer copies of "
                             f"{(layers[0][0].numel() * 2 * s_kv + layers[0][2].numel() * 2) / 1e9:.2f} GB "
                             f"cycled; {ab['total'] / 1e6:.0f} MB touched per step"},
            "achieved_gbs": step_gbs,
            "frac_of_peak": step_gbs / peak,
            "bytes_per_step": ab,
            "selected_counts": counts.tolist(),
            "kernels_us": kern,
            "kernels_us_note": "separate pass with CUDA events around every launch; each pair adds stream gaps",
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic, "kernel": "attend",
                         "avg_us": attend_us, "bytes_per_launch": att_bytes, "peak_kind": peak_kind},
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

"""Decode-attention benchmark over a CommVQ-compressed KV cache on B200.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--workload NAME]
                    [--path fused|naive]

One step is one commvq_attend_decode over the whole workload (all heads of one layer,
every cached position). With --path naive a step is the comparator the CommVQ review measures
against instead: commvq_decompress of the whole cache into dense 16-bit rows, then
commvq_dense_decode over them. The default workload is the LLaMA-3.1-8B-shaped 2-bit layer:
batch 1, 32 query / 8 KV heads, d = 128, T = 32768, R = 2, g = 8, Nc' = 256. Inputs are
seeded synthetic rows, codebooks fit on the GPU by the library's EM step, codes made by
the library's encoder. Under torchrun each rank runs its own replica (weak scaling; the
path has no exchange step); rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attention context-tokens/s and compressed-KV HBM GB/s vs B200 peak (1 GPU)"
UNIT = "context-tokens/s"
DEFAULT_WORKLOAD = "llama8b_2bit_T32768"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--algo", type=int, default=0)
    ap.add_argument("--splits", type=int, default=0)
    ap.add_argument("--path", default="fused", choices=["fused", "naive"],
                    help="fused: attention on the codes; naive: decompress the cache to dense "
                         "16-bit rows, then dense flash-decoding (the review's comparator)")
    ap.add_argument("--naive-dtype", default="bf16", choices=["bf16", "f16"])
    ap.add_argument("--unprepared", action="store_true",
                    help="rebuild the codebook images and RoPE tables in every step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-transfer", default="kernel", choices=["kernel", "copy"],
                    help="how the end-to-end step moves its inputs and output across the host link")
    ap.add_argument("--cpu-heads", type=int, default=32, help="query heads in the oracle sample")
    return ap.parse_args()


def workload(name):
    from decode_attention_commvq_b200 import synth
    for w in synth.WORKLOADS:
        if w.name == name:
            return w
    raise SystemExit(f"unknown workload {name}; known: {[w.name for w in synth.WORKLOADS]}")


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


KERNEL_SOURCES = {"attend_table_kernel": ("attend_table.cu",),
                  "attend_scores_kernel+attend_values_kernel": ("attend_mma.cu",),
                  "fast_attend_kernel": ("attend_fast.cu",),
                  "attend_scores_kernel+binv_*": ("attend_mma.cu", "binv.cu"),
                  "attend_generic_kernel": ("attend_generic.cu",),
                  "dense_decode_kernel": ("naive.cu",)}


def kernel_source_sha(kernel: str):
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "decode_attention_commvq_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload_name: str):
    """DRAM bytes per launch from a committed ncu summary, if taken on this exact source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel, {}).get(workload_name)
    if not e or e.get("source_sha") != kernel_source_sha(kernel):
        return None
    return float(e["dram_bytes_per_launch"])


def main_kernel(api, cfg, algo):
    """Name of the kernel(s) the main events bracket for this shape and algorithm, and the
    kernel launches of one step with prepared state."""
    run = algo
    if algo == api.ATTN_AUTO:
        g8 = cfg.g == 8 and cfg.n_codes <= 256
        mma_ok = g8 and cfg.R <= 2 and cfg.kv_heads in (1, 2, 4, 8) and \
            cfg.q_heads % cfg.kv_heads == 0 and cfg.q_heads // cfg.kv_heads <= 8
        run = api.ATTN_DECODE_MMA if mma_ok else (api.ATTN_TABLE if g8 and cfg.R <= 4 else api.ATTN_GENERIC)
    if run == api.ATTN_DECODE_MMA:
        fast = cfg.g == 8 and cfg.R <= 2 and cfg.n_codes <= 256 and cfg.kv_heads in (2, 4, 8) and \
            cfg.q_heads % cfg.kv_heads == 0 and cfg.q_heads // cfg.kv_heads <= 8
        if fast:
            return "fast_attend_kernel", 2                      # keys and values phases, merge
        return "attend_scores_kernel+attend_values_kernel", 3   # scores, values, merge
    if run == api.ATTN_GENERIC:
        return "attend_generic_kernel", 3                       # phasor tables, generic, merge
    return "attend_table_kernel", 2                             # table, merge


# ---------------------------------------------------------------------------------------
# clocks during the timed region

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index: int, bus_id: str | None):
        self.sel = bus_id if bus_id else str(device_index)
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.sel, f"--query-gpu=timestamp,{self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.flush()
        with open(self.f.name) as f:
            lines = [l.strip() for l in f if l.strip()]
        os.unlink(self.f.name)
        sm, mx, reasons = [], None, set()
        for l in lines:
            parts = [x.strip() for x in l.split(",")]
            if len(parts) < 8:
                continue
            try:
                s, m = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            sm.append(s)
            mx = m
            for name, val in zip(self.NAMES, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------------------
# multi-rank plumbing (replicas: no data-path collective)

def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time: one all-reduce (MAX) of a timing scalar."""
    if world <= 1:
        return float(ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, steps: int, units_per_step: int, ms_max: float) -> float:
    """Whole-job units per second: every rank processes units_per_step per step."""
    return world * steps * units_per_step / (ms_max / 1e3)


# ---------------------------------------------------------------------------------------
# our arm

def setup_inputs(w, dev, torch, api, fit):
    """Codebooks (GPU EM fit), encoded K/V cache, queries, offsets, all on the device."""
    from decode_attention_commvq_b200 import synth
    cfg = api.Config(d=w.d, g=w.g, R=w.R, n_codes=w.n_codes, q_heads=w.q_heads,
                     kv_heads=w.kv_heads, rope_base=w.rope_base)
    cbs = []
    for key in (True, False):
        if w.v_bits and not key:    # binary value code: C [n_bits, kv_heads * d]
            cbs.append(torch.from_numpy(synth.binary_value_codebook(w)).to(dev))
        elif w.codebook == "normal":
            cbs.append(torch.from_numpy(synth.normal_codebook(w, key)).to(dev))
        else:
            rows = torch.from_numpy(synth.fit_rows(w, key)).to(dev)
            cbs.append(fit.fit_codebook(rows, w.R, w.n_codes, w.em_iters,
                                        lambda r, N, key=key: synth.forgy_indices(w, key, r, N), g=w.g))
    kcb, vcb = cbs
    codes = []
    for key, cb in ((True, kcb), (False, vcb)):
        if w.v_bits and not key:    # seeded uniform bits (the value encoder is a learned network)
            codes.append(torch.from_numpy(synth.value_bits(w, int(w.lengths().sum()))).to(dev))
            continue
        parts = []
        L = w.lengths()
        for b in range(w.batch):
            x = torch.from_numpy(synth.kv_rows(w, key, int(L[b]), sub=b)).to(dev)
            parts.append(api.encode(cfg, x, cb))
            del x
        codes.append(torch.cat(parts, 0).contiguous())
    q_np = synth.queries(w)
    if w.q_dtype == "bf16":
        q = torch.from_numpy(q_np.view(np.int16)).to(dev).view(torch.bfloat16)
    else:
        q = torch.from_numpy(q_np.astype(np.float32)).to(dev)
    offs = torch.from_numpy(w.offsets()).to(dev)
    return cfg, kcb, vcb, codes[0], codes[1], q, offs


def run_ours(args, w, rank, world, dev):
    import torch
    import torch.distributed as dist
    from decode_attention_commvq_b200 import api, fit, synth

    torch.manual_seed(0)
    cfg, kcb, vcb, kc, vc, q, offs = setup_inputs(w, dev, torch, api, fit)
    L = w.lengths()
    total_T = int(L.sum())
    max_T = int(L.max())
    code_bytes = kc.numel() + vc.numel()
    props = torch.cuda.get_device_properties(dev)
    l2 = int(getattr(props, "L2_cache_size", 126 * 2 ** 20))
    n_copies = max(1, math.ceil(3 * l2 / code_bytes))
    kcs = [kc] + [kc.clone() for _ in range(n_copies - 1)]
    vcs = [vc] + [vc.clone() for _ in range(n_copies - 1)]
    # the binary code's C rotates with the codes, so that it is read from HBM like a layer's
    # parameters in a many-layer model
    cs = [vcb] + [vcb.clone() for _ in range(n_copies - 1)] if w.v_bits else None
    out = torch.empty((w.batch, w.q_heads, w.d), dtype=torch.float32, device=dev)
    lse = torch.empty((w.batch, w.q_heads), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    K, W = args.steps, args.warmup
    naive = args.path == "naive"
    binv = w.v_bits > 0
    if binv and (naive or args.algo not in (0, api.ATTN_DECODE_MMA)):
        raise SystemExit("the binary value code runs with the decode-and-rotate keys only")
    if binv:
        ws = torch.empty(api.attend_binv_workspace_bytes(cfg, w.v_bits, w.batch, max_T), dtype=torch.uint8,
                         device=dev)
        # the layer's key-side state (fp16 images, RoPE tables), once per layer
        api.attend_decode_binv(cfg, q, kc, vc, offs, max_T, kcb, vcb, out=out, lse=lse, workspace=ws,
                               stream=stream)
    elif naive:
        ndt = torch.bfloat16 if args.naive_dtype == "bf16" else torch.float16
        k_rows = torch.empty((total_T, w.kv_heads, w.d), dtype=ndt, device=dev)
        v_rows = torch.empty_like(k_rows)
        ws = torch.empty(api.decompress_workspace_bytes(cfg, max_T), dtype=torch.uint8, device=dev)
        ws_dense = torch.empty(api.dense_decode_workspace_bytes(cfg, w.batch, max_T, args.splits),
                               dtype=torch.uint8, device=dev)
    else:
        ws = api.attend_workspace(cfg, w.batch, max_T, dev, args.algo, args.splits)
        # the layer's codebook-dependent state (fp16 images, RoPE tables), once per layer
        api.attend_prepare(cfg, w.batch, max_T, kcb, vcb, ws, args.algo, args.splits, stream)
    prepared = not naive and not args.unprepared

    def attend(kc_i, vc_i, q_i, out_i, lse_i, events=None, prep=None, i=0):
        if binv:
            if events is not None:
                events[0].record(stream)
            api.attend_decode_binv(cfg, q_i, kc_i, vc_i, offs, max_T, kcb, cs[i % n_copies], out=out_i, lse=lse_i,
                                   workspace=ws, want_lse=lse_i is not None,
                                   prepared=prepared if prep is None else prep, stream=stream)
            if events is not None:
                events[1].record(stream)
        elif naive:
            api.decompress(cfg, kc_i, vc_i, offs, max_T, kcb, vcb, k_out=k_rows, v_out=v_rows,
                           workspace=ws, stream=stream)
            api.dense_decode(cfg, q_i, k_rows, v_rows, offs, max_T, out=out_i, lse=lse_i,
                             workspace=ws_dense, splits=args.splits, want_lse=lse_i is not None,
                             stream=stream, main_events=events)
        else:
            api.attend_decode(cfg, q_i, kc_i, vc_i, offs, max_T, kcb, vcb, out=out_i, lse=lse_i,
                              workspace=ws, algo=args.algo, splits=args.splits,
                              want_lse=lse_i is not None, stream=stream, main_events=events,
                              prepared=prepared if prep is None else prep)

    def step(i, events=None):
        attend(kcs[i % n_copies], vcs[i % n_copies], q, out, lse, events, i=i)

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K)]
    with torch.cuda.stream(stream):
        for a, b in evs:            # materialise the CUDA events before capture
            a.record(stream)
            b.record(stream)
        for i in range(W):
            step(i)
    torch.cuda.synchronize(dev)
    assert api.workspace_error(ws, stream) == 0

    # The timed graph holds only the steps: event nodes between kernels inside a graph cost
    # time of their own. The main-kernel times come from the same steps launched directly,
    # where the library records the events around its own launches.
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(K):
            step(W + i)
    with torch.cuda.stream(stream):
        graph.replay()               # one untimed replay (the graph's own upload)
    torch.cuda.synchronize(dev)

    bus = None
    try:
        bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
    except AttributeError:
        pass
    clocks = ClockSampler(dev.index or 0, bus)
    clocks.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):  # replay on the stream the events are recorded on
        t0.record(stream)
        graph.replay()
        t1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    # spread: the same graph replayed again, each replay timed on its own (not part of `value`)
    reps = []
    with torch.cuda.stream(stream):
        for _ in range(7):
            r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            r0.record(stream)
            graph.replay()
            r1.record(stream)
            reps.append((r0, r1))
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    rep_ms = np.array([a.elapsed_time(b) / K for a, b in reps])
    spread = {"replays": len(reps), "ms_per_step_median": float(np.median(rep_ms)),
              "ms_per_step_p10": float(np.percentile(rep_ms, 10)),
              "ms_per_step_p90": float(np.percentile(rep_ms, 90))}
    ms = t0.elapsed_time(t1)
    ms_max = max_over_ranks(ms, world, dev)
    with torch.cuda.stream(stream):
        for _ in range(3):   # keeps the GPU busy while the direct launches queue up behind it
            graph.replay()
        for i in range(K):
            step(W + i, evs[i])
    torch.cuda.synchronize(dev)
    kern_ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    del graph
    extra = {}
    if not naive:   # the same steps with the codebook-dependent state rebuilt every step
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2, stream=stream):
            for i in range(K):
                attend(kcs[i % n_copies], vcs[i % n_copies], q, out, lse, prep=False, i=i)
        with torch.cuda.stream(stream):
            g2.replay()
            torch.cuda.synchronize(dev)
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            g2.replay()
            a1.record(stream)
        torch.cuda.synchronize(dev)
        extra = {"prepared_state": {"reused_across_steps": prepared,
                                    "ms_per_step_rebuilding_it": a0.elapsed_time(a1) / K}}
        del g2
    if naive:   # the decompress half alone, for the breakdown
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2, stream=stream):
            for i in range(K):
                api.decompress(cfg, kcs[i % n_copies], vcs[i % n_copies], offs, max_T, kcb, vcb,
                               k_out=k_rows, v_out=v_rows, workspace=ws, stream=stream)
        with torch.cuda.stream(stream):
            g2.replay()
            torch.cuda.synchronize(dev)
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            g2.replay()
            a1.record(stream)
        torch.cuda.synchronize(dev)
        dec_ms = a0.elapsed_time(a1) / K
        del g2
        dense_bytes = 2 * k_rows.numel() * k_rows.element_size()
        extra = {"naive": {"rows_dtype": args.naive_dtype, "decompress_ms": dec_ms,
                           "decompress_gbs": (code_bytes + dense_bytes) / (dec_ms / 1e3) / 1e9,
                           "dense_kernel_ms": kern_ms,
                           "dense_rows_bytes": dense_bytes}}

    # ---- e2e: one decode step through the API with host buffers -----------------------
    e2e = run_e2e(args, w, cfg, kcb, vcb, kcs, vcs, offs, max_T, total_T, attend, stream, dev, torch,
                  api, synth, world, dist)

    value = job_throughput(world, K, total_T, ms_max)
    peak, peak_kind = measured_peaks()
    if naive:
        kname, launches_per_step = "dense_decode_kernel", 4   # decompress prep, decompress, dense, merge
        alg_bytes = 2 * k_rows.numel() * k_rows.element_size()
    else:
        if binv:   # scores, weights, bit-plane sums, merge and contraction with C, final division
            kname, launches_per_step = "attend_scores_kernel+binv_*", 5
        else:
            kname, launches_per_step = main_kernel(api, cfg, args.algo)
        if not prepared and (kname.startswith("attend_scores") or kname.startswith("fast_attend")):
            launches_per_step += 1   # the prep kernel
        alg_bytes = code_bytes + (vcb.numel() * vcb.element_size() if binv else 0)
    achieved = alg_bytes / (kern_ms / 1e3) / 1e9
    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms_max / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": dtype_label(w, naive, args, kname), "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "q_heads": w.q_heads, "kv_heads": w.kv_heads,
                   "d": w.d, "T": total_T, "R": w.R, "g": w.g, "n_codes": w.n_codes,
                   "q_dtype": w.q_dtype, "parallelism": f"replicas{world}",
                   **({"values": f"binary code, {w.v_bits} bits per position over the KV row, "
                                 f"C [{w.v_bits}, {w.kv_heads * w.d}] fp32"} if binv else {}),
                   "path": args.path, "algo": args.algo, "splits": args.splits,
                   "l2_defence": f"rotating {n_copies} cache copies{' and C' if binv else ''} "
                                 f"({n_copies * code_bytes / 2**20:.0f} MiB of codes "
                                 f">= 3x L2 {l2 / 2**20:.0f} MiB)",
                   "timing": "K steps in one CUDA graph, CUDA events on the launch stream; main-kernel "
                             "times from the same K steps launched directly, events recorded by the "
                             "library around its main kernels" + (" (here: around the whole call)" if binv else ""),
                   "codebook_state": ("fp16 codebook images and RoPE tables prepared once per layer "
                                      "(commvq_attend_prepare), reused by every step") if prepared
                   else "rebuilt inside every step"},
        "compressed_cache_gbs": code_bytes * K / (ms_max / 1e3) / 1e9 * 1.0 / world * world,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": f"{peak_kind} copy bandwidth",
                     "kernel": kname, "algorithmic_bytes_per_launch": alg_bytes,
                     "kernel_ms_mean": kern_ms,
                     "traffic": recorded_traffic(kname, w.name),
                     "traffic_source": "dram__bytes_read.sum + dram__bytes_write.sum per launch from a committed "
                                       "ncu capture (profiles/traffic.json: cold-cache replay of this exact kernel "
                                       "source, not measured in this run; null when the source changed since)"},
        "spread": spread,
        "e2e": e2e,
        "gpu_launches": launches_per_step * K,
        "clocks": clk,
    }
    result.update(extra)
    return result


def dtype_label(w, naive, args, kname):
    """The operand and accumulation types of the timed path."""
    if naive:
        return f"{args.naive_dtype} dense rows and operands, fp32 accumulate"
    if w.v_bits:
        return "keys: fp16 codebook entries, bf16/fp16 two-term operands; values: int8 digit MMAs (exact int32); fp32 accumulate"
    if kname == "fast_attend_kernel":
        return ("fp16 codebook entries; key rounds summed and rotated in fp32, fed as one fp16 operand "
                "(query fp16, saturating); softmax weights and value round sums fp16; fp32 accumulate")
    return ("fp16 codebook entries; keys rotated in fp32 and fed as two " +
            ("bf16" if w.q_dtype == "bf16" else "fp16") +
            " terms; softmax weights and values fp16; fp32 accumulate")


def run_e2e(args, w, cfg, kcb, vcb, kcs, vcs, offs, max_T, total_T, attend, stream, dev, torch, api,
            synth, world, dist):
    """Per step: one pinned host -> device copy of the step's inputs (the query, the new
    position's K and V rows, and for the binary value code its bits), encode of the new position
    into the cache (position T-1 of sequence 0; its K and V rows in one encode launch), decode
    attention, device -> host copy of the output."""
    K, W = args.steps, args.warmup
    n_copies = len(kcs)
    binv = w.v_bits > 0
    q_np = synth.queries(w).view(np.int16) if w.q_dtype == "bf16" else synth.queries(w).astype(np.float32)
    kv_new = np.stack([synth.kv_rows(w, True, 1, sub=1000, dtype="f16"),
                       synth.kv_rows(w, False, 1, sub=1000, dtype="f16")])   # [2, 1, Hkv, d]
    parts = [q_np, kv_new] + ([synth.value_bits(w, 1)] if binv else [])
    sizes = [int(x.nbytes) for x in parts]
    offsets = np.concatenate([[0], np.cumsum([(n + 255) // 256 * 256 for n in sizes])])   # 256-byte aligned
    stage_h = torch.zeros(int(offsets[-1]), dtype=torch.uint8).pin_memory()
    for x, o, n in zip(parts, offsets, sizes):
        stage_h[int(o):int(o) + n] = torch.from_numpy(np.ascontiguousarray(x).view(np.uint8).reshape(-1))
    stage_d = torch.empty_like(stage_h, device=dev)

    out_h = torch.empty((w.batch, w.q_heads, w.d), dtype=torch.float32).pin_memory()
    out_d = torch.empty((w.batch, w.q_heads, w.d), dtype=torch.float32, device=dev)
    # kernel: one commvq_copy_async kernel brings the step's inputs from the pinned host buffer
    # across the host link, and the merge kernel writes the output straight into the pinned host
    # output (both mapped at their host addresses under unified addressing); copy: copy-engine
    # transfers around the kernels
    mapped = (args.e2e_transfer == "kernel" and not binv and api.host_mapped(stage_h) and api.host_mapped(out_h))
    src = stage_d

    def view(k, dtype, shape):
        return src[int(offsets[k]):int(offsets[k]) + sizes[k]].view(dtype).view(shape)

    q_d = view(0, torch.bfloat16 if w.q_dtype == "bf16" else torch.float32, q_np.shape)
    kv_d = view(1, torch.float16, kv_new.shape)
    bits_d = view(2, torch.uint8, (1, w.v_bits // 8)) if binv else None
    last = int(w.offsets()[1]) - 1

    def step(i):
        kc, vc = kcs[i % n_copies], vcs[i % n_copies]
        if mapped:
            api.copy_async(stage_d, stage_h, stream=stream)
        else:
            stage_d.copy_(stage_h, non_blocking=True)
        if binv:   # the value encoder is a learned network: its bits arrive from the host
            vc[last:last + 1].copy_(bits_d, non_blocking=True)
            api.encode(cfg, kv_d[0], kcb, codes=kc[last:last + 1], stream=stream)
        else:      # the new key and value rows in one launch
            api.encode_kv(cfg, kv_d[0], kv_d[1], kcb, vcb, kc[last:last + 1], vc[last:last + 1], stream=stream)
        if mapped:
            attend(kc, vc, q_d, out_h, None, i=i)
        else:
            attend(kc, vc, q_d, out_d, None, i=i)
            out_h.copy_(out_d, non_blocking=True)

    with torch.cuda.stream(stream):
        for i in range(W):
            step(i)
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for i in range(K):
                step(W + i)
        graph.replay()
        torch.cuda.synchronize(dev)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        t0.record(stream)
        graph.replay()
        t1.record(stream)
        torch.cuda.synchronize(dev)
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    del graph
    return {"value": job_throughput(world, K, total_T, ms), "unit": UNIT,
            "h2d_bytes_per_step": int(stage_h.numel()),
            "d2h_bytes_per_step": int(out_h.numel() * out_h.element_size()),
            "ms_per_step": ms / K,
            "transfer": "kernel" if mapped else "copy",
            "note": ("q and the new position's K/V rows brought in from pinned host memory by one copy kernel "
                     "(commvq_copy_async, loads across the host link), the output written by the merge kernel "
                     "straight into pinned host memory" if mapped else
                     "one copy of q + the new position's K/V rows (+ value bits) in, output out (copy engine)") +
                    "; encode (K and V rows in one launch) + attend; one CUDA graph of K steps"}


# ---------------------------------------------------------------------------------------
# the encode + codebook-fit workload (not the headline line; measured for rows a1 and a8)

def run_encode_fit(args, w, rank, world, dev):
    """Step = encode all K and V rows of the workload (131072 tokens x 8 KV heads each) into
    2-bit codes. The codebooks come from the timed-once GPU fit (10 EM iterations per round
    on 65536 rows per tensor), reported beside the encode throughput."""
    import torch
    from decode_attention_commvq_b200 import api, fit, synth
    cfg = api.Config(d=w.d, g=w.g, R=w.R, n_codes=w.n_codes, q_heads=w.q_heads,
                     kv_heads=w.kv_heads, rope_base=w.rope_base)
    stream = torch.cuda.Stream(device=dev)
    K, W = args.steps, args.warmup
    # codebook fit (timed once per tensor, with events, after one untimed fit that loads the
    # kernels)
    fit_ms = {}
    cbs = []
    # warm-up at the full row count: loads the kernels and lets the caching allocator hold the
    # fit's buffers, so neither timed fit pays for a first cudaMalloc
    warm = torch.from_numpy(synth.fit_rows(w, True)).to(dev)
    fit.fit_codebook(warm, w.R, w.n_codes, 1, lambda r, N: synth.forgy_indices(w, True, r, N), g=w.g)
    del warm
    for key in (True, False):
        rows = torch.from_numpy(synth.fit_rows(w, key)).to(dev)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            cb = fit.fit_codebook(rows, w.R, w.n_codes, w.em_iters,
                                  lambda r, N, key=key: synth.forgy_indices(w, key, r, N), g=w.g)
            e1.record(stream)
        torch.cuda.synchronize(dev)
        fit_ms["K" if key else "V"] = e0.elapsed_time(e1)
        cbs.append(cb)
    xs = [torch.from_numpy(synth.encode_rows(w, key, w.encode_tokens)).to(dev) for key in (True, False)]
    codes = [torch.empty((w.encode_tokens, w.kv_heads, w.R, w.groups), dtype=torch.uint8, device=dev)
             for _ in range(2)]
    ties = torch.zeros(1, dtype=torch.int64, device=dev)

    def step():
        for x, cb, c in zip(xs, cbs, codes):
            api.encode(cfg, x, cb, codes=c, near_ties=ties, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(W):
            step()
    torch.cuda.synchronize(dev)
    props = torch.cuda.get_device_properties(dev)
    clocks = ClockSampler(dev.index or 0, None)
    clocks.start()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        t0.record(stream)
        for _ in range(K):
            step()
        t1.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    tokens = w.encode_tokens
    rows = 2 * tokens * w.kv_heads
    # algorithmic fp32 work: per (row, group) R * Nc' entries x (g subtracts + g fused multiply-adds)
    flop_instr = rows * w.groups * w.R * w.n_codes * 2 * w.g
    sm_mhz = (clk or {}).get("sm_mhz") or 1965.0
    peak_instr = props.multi_processor_count * 128 * sm_mhz * 1e6     # fp32 lanes x clock
    achieved = flop_instr / (ms / K / 1e3)
    return {
        "metric": "encode tokens/s (K and V, 2-bit) and EM fit time", "value": job_throughput(world, K, tokens, ms),
        "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": ms / K,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": w.name, "tokens": tokens, "kv_heads": w.kv_heads, "d": w.d, "R": w.R,
                   "g": w.g, "n_codes": w.n_codes, "em_rows": w.em_rows, "em_iters_per_round": w.em_iters,
                   "l2_defence": "inputs 512 MiB of fp16 rows per step (> 4x L2)"},
        "em_fit_ms": fit_ms,
        "near_ties_per_step": int(ties.item()) // max(1, K + W),
        "roofline": {"bound": "alu", "achieved": achieved / 1e12, "peak": peak_instr / 1e12,
                     "unit": "T fp32-instr/s", "frac": achieved / peak_instr,
                     "peak_kind": f"148 SMs x 128 fp32 lanes x {sm_mhz:.0f} MHz (median SM clock under load)",
                     "kernel": "encode_kernel", "traffic": None},
        "gpu_launches": 2 * K, "clocks": clk,
        "cpu_baseline": encode_cpu_baseline(w, cbs[0].cpu().numpy(), cbs[1].cpu().numpy()) if world == 1 else None,
    }


def encode_cpu_baseline(w, kcb, vcb, tokens=256):
    """The oracle encoder on a bounded sample: `tokens` positions x KV heads of K and of V."""
    from decode_attention_commvq_b200 import synth
    from oracle import oracle as O
    kx = synth.kv_rows(w, True, tokens, sub=0)
    vx = synth.kv_rows(w, False, tokens, sub=0)
    t0 = time.perf_counter()
    O.encode(kx, kcb)
    O.encode(vx, vcb)
    dt = time.perf_counter() - t0
    return {"value": tokens / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{tokens} positions x {w.kv_heads} KV heads of K and V ({2 * tokens * w.kv_heads} rows), "
                      f"single-threaded C oracle, {dt:.2f} s", "seconds": dt}


# ---------------------------------------------------------------------------------------
# the oracle (CPU baseline and the reference arm)

def oracle_sample(w, n_heads):
    """Inputs for timing the oracle on n_heads query heads (whole GQA groups) of the
    workload's first sequence: uniform codes and N(0,1) codebooks (the oracle's time does
    not depend on the values)."""
    from decode_attention_commvq_b200 import synth
    group = w.q_heads // w.kv_heads
    n_heads = max(group, min(w.q_heads, n_heads // group * group))
    n_kv = n_heads // group
    T = int(w.lengths()[0])
    ws = w.with_(kv_heads=n_kv, q_heads=n_heads, batch=1, ragged=None, seq_len=T)
    kc = synth.uniform_codes(ws, True, T)
    kcb = synth.normal_codebook(w, True)
    if w.v_bits:   # binary values: the bits of the whole KV row, C's columns of the sampled heads
        vc = synth.value_bits(w, T)
        vcb = np.ascontiguousarray(synth.binary_value_codebook(w)[:, :n_kv * w.d])
    else:
        vc = synth.uniform_codes(ws, False, T)
        vcb = synth.normal_codebook(w, False)
    q = synth.as_f32(synth.queries(w), w.q_dtype)[:1, :n_heads].astype(np.float64)
    return q, kc, vc, np.array([0, T]), kcb, vcb, n_heads, T


def time_oracle_step(w, sample, threads=1):
    from oracle import oracle as O
    q, kc, vc, offs, kcb, vcb, n_heads, T = sample
    t0 = time.perf_counter()
    if w.v_bits:
        O.attend_binv(q, kc, vc, offs, kcb, vcb, w.rope_base)
    else:
        O.attend_codes(q, kc, vc, offs, kcb, vcb, w.rope_base, threads=threads)
    dt = time.perf_counter() - t0
    tokens = T * n_heads / w.q_heads        # context tokens of the full step this sample covers
    return dt, tokens


def cpu_baseline(w, n_heads, min_seconds=10.0):
    """The oracle on a bounded sample: n_heads query heads of sequence 0, repeated until at least
    min_seconds of wall time have been spent, once single-threaded and once on every core this
    process may use (the oracle's threaded face: one KV head's query group per thread, the same
    single-threaded C calls). The multi-threaded figure is the line's baseline."""
    from oracle import oracle as O
    sample = oracle_sample(w, n_heads)

    def timed(threads):
        total_dt, total_tok, reps = 0.0, 0.0, 0
        while total_dt < min_seconds or reps == 0:
            dt, tokens = time_oracle_step(w, sample, threads)
            total_dt += dt
            total_tok += tokens
            reps += 1
        return total_tok / total_dt, total_dt, reps

    cores = O.host_threads()
    n_kv = sample[6] // (w.q_heads // w.kv_heads)
    threads = max(1, min(cores, n_kv))
    v1, dt1, r1 = timed(1)
    vn, dtn, rn = timed(threads)
    desc = f"{sample[6]} of {w.q_heads} query heads of sequence 0 (T={sample[7]}), C oracle in fp64"
    return {"value": vn, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{desc}, {threads} threads (one KV head's query group each), {rn} repetitions, {dtn:.1f} s",
            "seconds": dtn, "cpu": cpu_model(), "host_cores": cores,
            "single_thread": {"value": v1, "unit": UNIT, "cores": 1, "repetitions": r1, "seconds": dt1}}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for l in f:
                if l.startswith("model name"):
                    return l.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return None
    sample = oracle_sample(w, w.q_heads // w.kv_heads)
    for _ in range(args.warmup):
        time_oracle_step(w, sample)
    tot_t, tot_tok = 0.0, 0.0
    for _ in range(args.steps):
        dt, tok = time_oracle_step(w, sample)
        tot_t += dt
        tot_tok += tok
    value = tot_tok / tot_t
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": w.name, "batch": w.batch, "q_heads": w.q_heads,
                       "kv_heads": w.kv_heads, "d": w.d, "T": int(w.lengths().sum()), "R": w.R,
                       "g": w.g, "n_codes": w.n_codes},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": f"each step: {sample[6]} of {w.q_heads} query heads (one GQA "
                                       f"group) of sequence 0, T={sample[7]}; single-threaded C oracle"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    w = workload(args.workload)
    if args.impl == "reference":
        res = run_reference(args, w)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    try:
        if w.encode_tokens:
            res = run_encode_fit(args, w, rank, world, dev)
        else:
            res = run_ours(args, w, rank, world, dev)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline and not w.encode_tokens:
                res["cpu_baseline"] = cpu_baseline(w, args.cpu_heads)
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

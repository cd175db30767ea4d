"""Benchmark of the low-bit MLA decode step on B200.

One step = the whole hot path over one batch: quantize + pack + paged write of
the step's new tokens (mla_qcache_append), then the decode over the quantized
cache (mla_qdecode: split-KV decode kernel + combine). The BF16 comparison
decode (mla_decode_bf16) is timed as a separate leg on the same shapes.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload mtp]
  python bench.py --impl reference ...    # the CPU oracle, timed on host cores

Prints one JSON line on rank 0. Inputs are synthetic (seeded; see
bit_mla_kv_qdecode_b200/synth.py). L2 hygiene: every step reads a different
copy of the cache and queries, and the copies together exceed 3x the L2 size.
Multi-GPU runs (torchrun) are weak-scaling replicas: each rank decodes its own
batch of the same shape, with no collective on the data path.
"""
from __future__ import annotations

import argparse
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

METRIC = "KV tokens attended/sec·head-batch (head-tokens/s) and achieved HBM GB/s, 1 GPU"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def profiled_traffic(workload_name):
    """DRAM bytes per decode launch from the committed ncu capture (profiles/traffic.json), or None
    when the capture covers another workload or the kernel sources changed since it was taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    if rec.get("workload") != workload_name:
        return None
    h = hashlib.sha256()
    for rel in rec["source_files"]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    if h.hexdigest()[:16] != rec["source_sha256_16"]:
        return None
    return rec["dram_bytes_read_per_launch"] + rec["dram_bytes_write_per_launch"]


HYB_SINK = 64      # BF16 sink of the hybrid cache leg: one page
HYB_WINDOW = 128   # BF16 recent window: 128..191 tokens (history moves a page at a time)


def max_over_ranks(x, dist, device):
    """The largest of every rank's x: a multi-rank job ends when its slowest rank does."""
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank, world, ms):
    """Whole-job throughput: every rank runs the same workload (weak scaling), all within ms."""
    return units_per_rank * world / (ms * 1e-3)


def workload_stats(w, lens):
    """Head-tokens, KV tokens, algorithmic bytes and flops of one decode."""
    s_q, H = w.s_q, w.H
    vis = np.stack([np.maximum(lens.astype(np.int64) - s_q + 1 + i, 0) for i in range(s_q)], axis=1)
    head_tokens = int(vis.sum()) * H
    kv_tokens = int(lens.astype(np.int64).sum())
    bpt = (512 * w.bits_c // 8 + (512 // w.group_c) * 4 + 64 * w.bits_r // 8 + (64 // w.group_r) * 4)
    q_bytes = w.B * s_q * H * 576 * 2
    o_bytes = w.B * s_q * H * 512 * 2
    alg_bytes = kv_tokens * bpt + q_bytes + o_bytes
    alg_bytes_bf16 = kv_tokens * 1152 + q_bytes + o_bytes
    flops = 2 * head_tokens * (576 + 512)
    return dict(head_tokens=head_tokens, kv_tokens=kv_tokens, bytes_per_token=bpt, alg_bytes=alg_bytes,
                alg_bytes_bf16=alg_bytes_bf16, flops=flops, q_bytes=q_bytes, o_bytes=o_bytes)


def append_stats(w, ms):
    """Rate of the cache append of one step (B * n_new tokens) taking ms milliseconds: tokens/s and
    GB/s over its algorithmic bytes (bf16 tokens read, packed codes and metadata written)."""
    tokens = w.B * w.n_new
    bpt = (512 * w.bits_c // 8 + (512 // w.group_c) * 4 + 64 * w.bits_r // 8 + (64 // w.group_r) * 4)
    nbytes = tokens * (576 * 2 + bpt)
    return {"tokens": tokens, "ms": ms, "tokens_per_s": tokens / (ms * 1e-3), "gbs": nbytes / (ms * 1e-3) / 1e9,
            "bytes": nbytes}


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples over a region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not self.path:
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append(parts)
                except ValueError:
                    pass
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[5 + k].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def run_reference(args, w):
    """The CPU oracle as it stands, timed on this host's cores on a bounded sample."""
    from bit_mla_kv_qdecode_b200 import synth
    from oracle import attention, layout
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    lens = synth.seq_lens(w)
    table, num_pages = synth.block_table(w, lens)
    desc = layout.Desc(bits_c=w.bits_c, group_c=w.group_c, bits_r=w.bits_r, group_r=w.group_r)
    mag = synth.channel_magnitudes(w)
    qc_bits, qr_bits = synth.queries_bf16(w)
    qc, qr = synth.bf16_bits_to_f32(qc_bits), synth.bf16_bits_to_f32(qr_bits)
    hist = np.maximum(lens - w.n_new, 0)
    # sample: the first requests whose history fits a ~1.5 s packing budget per step
    budget_tokens = 300_000
    sample, tot = [], 0
    for b in range(w.B):
        if sample and tot + int(lens[b]) > budget_tokens:
            break
        sample.append(b)
        tot += int(lens[b])
    pool = np.zeros((num_pages, desc.page_bytes), dtype=np.uint8)
    new_tok = {}
    for b in sample:
        x = synth.bf16_bits_to_f32(synth.cache_tokens_bf16(w, b, int(lens[b]), mag))
        layout.append(desc, pool, table[b:b + 1], [0], x[None, :hist[b], :512], x[None, :hist[b], 512:])
        new_tok[b] = x[hist[b]:]
    sub = np.array(sample)
    st = workload_stats(w.scaled(B=len(sample)), lens[sub])

    def step():
        for b in sample:
            layout.append(desc, pool, table[b:b + 1], [hist[b]], new_tok[b][None, :, :512], new_tok[b][None, :, 512:])
        attention.qdecode(desc, pool, table, lens, qc, qr, w.scale, requests=sample)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / max(args.steps, 1)
    cores = _blas_threads()
    val = st["head_tokens"] / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "head-tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config(w, args.gpus, extra={"sample_requests": len(sample)}),
        "cpu_baseline": {"value": val, "unit": "head-tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{len(sample)} of {w.B} requests (all heads), append + decode per step"},
        "e2e": {"value": val, "unit": "head-tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def _config(w, n_gpus, extra=None):
    c = {"workload": f"{w.name}: B={w.B} H={w.H} s_q={w.s_q} T={w.t_lo}"
                     + (f"..{w.t_hi}" if w.t_hi != w.t_lo else "")
                     + f" INT{w.bits_c} g{w.group_c} content / INT{w.bits_r} g{w.group_r} rope,"
                     + (" paged 64-token pages" if w.paged else " contiguous"),
         "B": w.B, "H": w.H, "s_q": w.s_q, "d_c": 512, "d_r": 64, "page": 64,
         "n_new_per_step": w.n_new, "parallelism": f"replicas x{n_gpus}" if n_gpus > 1 else "1 GPU",
         "l2": "rotated cache+query copies > 3x L2"}
    if extra:
        c.update(extra)
    return c


def cpu_baseline_leg(w, seconds=12.0):
    """The oracle timed on a bounded sample (rank 0, N=1 only)."""
    from bit_mla_kv_qdecode_b200 import synth
    from oracle import attention, quant
    lens = synth.seq_lens(w)
    mag = synth.channel_magnitudes(w)
    qc_bits, qr_bits = synth.queries_bf16(w)
    qc, qr = synth.bf16_bits_to_f32(qc_bits), synth.bf16_bits_to_f32(qr_bits)
    head_tokens, done = 0, 0
    t_spent = 0.0
    tokens = {}
    for i in range(100 * w.B):  # cycle over the batch until about `seconds` of CPU work
        b = i % w.B
        if b not in tokens:
            tokens[b] = synth.bf16_bits_to_f32(synth.cache_tokens_bf16(w, b, int(lens[b]), mag))
        x = tokens[b]
        t0 = time.perf_counter()
        u, s, z = quant.quantize_groups(x[:, :512], w.bits_c, w.group_c)
        C = quant.dequantize_groups(u, s, z, w.group_c)
        u, s, z = quant.quantize_groups(x[:, 512:], w.bits_r, w.group_r)
        R = quant.dequantize_groups(u, s, z, w.group_r)
        rq_c, rq_r, L = attention.request_rows(qc[b], qr[b], int(lens[b]))
        attention.attend(rq_c, rq_r, C, R, w.scale, L)
        t_spent += time.perf_counter() - t0
        head_tokens += int(L.sum())
        done += 1
        if t_spent >= seconds:
            break
    return {"value": head_tokens / t_spent, "unit": "head-tokens/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"{done} request decodes (cycling over the {w.B} requests), all heads: quantize + "
                      f"dequantize the request's cache and attend in float64, {t_spent:.1f} s"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    # default: the largest workload that fits one GPU (B=128, H=128, s_q=2 causal,
    # ragged T in [1024, 32768], INT2/INT4, 2 tokens appended per request and step)
    ap.add_argument("--workload", default="mtp")
    ap.add_argument("--batch", type=int, default=0,
                    help="run the workload with this many requests instead (small cases for profiling)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-bf16", action="store_true")
    ap.add_argument("--no-hybrid", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    from bit_mla_kv_qdecode_b200 import synth
    w = synth.workload(args.workload)
    if args.batch > 0:
        w = w.scaled(B=args.batch)
    if args.impl == "reference":
        return run_reference(args, w)

    import torch
    import torch.distributed as dist

    from bit_mla_kv_qdecode_b200 import api

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()

    # ---- inputs (synthetic, seeded), resident in HBM ----
    lens = synth.seq_lens(w)
    table, num_pages = synth.block_table(w, lens)
    mag = synth.channel_magnitudes(w)
    hist = np.maximum(lens - w.n_new, 0).astype(np.int32)
    desc = api.make_desc(w.bits_c, w.group_c, w.bits_r, w.group_r, num_pages=num_pages)
    page_bytes = api.mla_qcache_page_bytes(desc)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    pool_bytes = num_pages * page_bytes
    R = max(3, math.ceil(3 * l2 / pool_bytes))

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)

    table_t = torch.from_numpy(table).to(dev)
    hist_t = torch.from_numpy(hist).to(dev)
    lens_t = torch.from_numpy(lens).to(dev)
    pool0 = api.new_qcache_pool(desc, device=dev)
    want_bf16 = (not args.no_bf16) and num_pages * 64 * 1152 * 3 < 60e9
    pool_b0 = api.new_bf16_pool(num_pages, device=dev) if want_bf16 else None
    new_c = np.zeros((w.B, w.n_new, 512), dtype=np.uint16)
    new_r = np.zeros((w.B, w.n_new, 64), dtype=np.uint16)
    # hybrid cache leg: a one-page BF16 sink, a BF16 window of HYB_WINDOW..+63
    # tokens, the history between them quantized (a page at a time)
    hyb_hist = np.maximum((lens.astype(np.int64) - HYB_SINK - HYB_WINDOW) // 64 * 64, 0)
    hyb_prot = []
    for b in range(w.B):
        toks = synth.cache_tokens_bf16(w, b, int(lens[b]), mag)
        if not args.no_hybrid:
            hyb_prot.append(np.concatenate([toks[:HYB_SINK], toks[HYB_SINK + hyb_hist[b]:]]))
        for t0 in range(0, int(lens[b]), 16384):
            part = toks[t0:t0 + 16384]
            lb = torch.tensor([t0], dtype=torch.int32, device=dev)
            c, r = to_dev(part[None, :, :512]), to_dev(part[None, :, 512:])
            api.mla_qcache_append(desc, pool0, table_t[b:b + 1], lb, c, r)
            if pool_b0 is not None:
                api.mla_bf16cache_append(pool_b0, table_t[b:b + 1], lb, c, r)
        new_c[b], new_r[b] = toks[hist[b]:, :512], toks[hist[b]:, 512:]
    qc_bits, qr_bits = synth.queries_bf16(w)
    pools = [pool0] + [pool0.clone() for _ in range(R - 1)]
    qcs = [to_dev(qc_bits) for _ in range(R)]
    qrs = [to_dev(qr_bits) for _ in range(R)]
    newc_t, newr_t = to_dev(new_c), to_dev(new_r)
    out = torch.empty((w.B, w.s_q, w.H, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.s_q, w.H), dtype=torch.float32, device=dev)
    max_len = int(lens.max())
    n_split = api.mla_decode_num_splits(w.B, w.s_q, w.H, max_len, w.num_splits)
    ws_bytes = api.mla_decode_workspace_bytes(w.B, w.s_q, w.H, max_len, w.num_splits)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    assert api.mla_get_device_status() == 0

    def step(k):
        # the step's append of its new tokens and the decode, in one C-ABI call
        # (the append runs inside the decode kernel where the tensor-core path applies)
        api.mla_qdecode_fused_append(desc, pools[k], table_t, lens_t, max_len, newc_t, newr_t, qcs[k], qrs[k],
                                     w.scale, out=out, lse=lse, num_splits=w.num_splits, workspace=ws, stream=stream)

    def step_separate(k, ev):
        # the same step as two calls: mla_qcache_append, then mla_qdecode
        ev[0].record(stream)
        api.mla_qcache_append(desc, pools[k], table_t, hist_t, newc_t, newr_t, stream=stream)
        ev[1].record(stream)
        api.mla_qdecode(desc, pools[k], table_t, lens_t, max_len, qcs[k], qrs[k], w.scale, out=out, lse=lse,
                        num_splits=w.num_splits, workspace=ws, stream=stream)
        ev[2].record(stream)

    for i in range(args.warmup):
        step(i % R)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    # no events between the timed steps: a record between two launches would
    # cut the programmatic (early) launch of the next decode kernel
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for i in range(args.steps):
            step(i % R)
        t_end.record(stream)
        torch.cuda.synchronize()
    ms_total = t_start.elapsed_time(t_end)
    if world > 1:
        ms_total = max_over_ranks(ms_total, dist, dev)
        dist.barrier()
    ms_step = ms_total / args.steps
    ms_decode = ms_step  # the step is one C-ABI call (decode kernel with the append fused in + combine)
    assert api.mla_get_device_status() == 0
    # the unfused step, for comparison (not the reported value)
    sep_steps = min(args.steps, 20)
    evs2 = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(sep_steps)]
    for i in range(args.warmup):
        step_separate(i % R, evs2[0])
    torch.cuda.synchronize()
    for i in range(sep_steps):
        step_separate(i % R, evs2[i])
    torch.cuda.synchronize()
    ms_append = statistics.mean(evs2[i][0].elapsed_time(evs2[i][1]) for i in range(sep_steps))
    ms_sep_decode = statistics.mean(evs2[i][1].elapsed_time(evs2[i][2]) for i in range(sep_steps))
    assert api.mla_get_device_status() == 0

    st = workload_stats(w, lens)
    value = job_rate(st["head_tokens"], world, ms_step)
    peaks, peak_src = load_peaks()
    flop_rate = st["flops"] / (ms_decode * 1e-3) / 1e12
    gbs = st["alg_bytes"] / (ms_decode * 1e-3) / 1e9
    # The timed region lasts well under the seconds-long loop behind the sustained
    # figure, so the burst bf16 peak is the denominator.
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    tensor_bound = st["flops"] / st["alg_bytes"] > ridge
    if tensor_bound:
        roof = {"bound": "tensor", "achieved": flop_rate, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": flop_rate / peaks["bf16_tflops"], "traffic": None,
                "peak_source": f"{peak_src} bf16_tflops (burst: the timed region is "
                               f"{ms_total:.0f} ms, not a seconds-long loop)"}
    else:
        roof = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / peaks["hbm_gbs"], "traffic": None, "peak_source": f"{peak_src} hbm_gbs"}
    roof["traffic"] = profiled_traffic(w.name)
    roof["kernel"] = ("mla_qdecode_fused_append (decode kernel with the step's append fused in + split-KV "
                      "combine, one C-ABI call)")
    roof["per_launch_ms"] = ms_decode
    roof["algorithmic"] = {"flops": st["flops"], "bytes": st["alg_bytes"]}

    # ---- BF16 comparison decode (separate leg, same shapes) ----
    bf16_leg = None
    if pool_b0 is not None:
        Rb = max(3, math.ceil(3 * l2 / (num_pages * 64 * 1152)))
        pools_b = [pool_b0] + [pool_b0.clone() for _ in range(Rb - 1)]
        for i in range(args.warmup):
            api.mla_decode_bf16(pools_b[i % Rb], table_t, lens_t, max_len, qcs[i % R], qrs[i % R], w.scale,
                                out=out, lse=lse, num_splits=w.num_splits, workspace=ws, stream=stream)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.steps):
            api.mla_decode_bf16(pools_b[i % Rb], table_t, lens_t, max_len, qcs[i % R], qrs[i % R], w.scale,
                                out=out, lse=lse, num_splits=w.num_splits, workspace=ws, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        ms_b = e0.elapsed_time(e1) / args.steps
        bf16_leg = {"ms_per_decode": ms_b, "head_tokens_per_s": st["head_tokens"] / (ms_b * 1e-3),
                    "alg_gbs": st["alg_bytes_bf16"] / (ms_b * 1e-3) / 1e9,
                    "qdecode_speedup": ms_b / ms_decode}
        del pools_b

    # ---- hybrid cache decode (same queries and keys; history = the pool's pages after the sink page) ----
    hybrid_leg = None
    if not args.no_hybrid:
        prot_lens = np.array([len(p) for p in hyb_prot], dtype=np.int32)
        pp = int((prot_lens.max() + 63) // 64)
        bpool_h = api.new_bf16_pool(w.B * pp, device=dev)
        ptab = torch.arange(w.B * pp, dtype=torch.int32, device=dev).view(w.B, pp)
        for b in range(w.B):
            pt = to_dev(hyb_prot[b][None])
            api.mla_bf16cache_append(bpool_h, ptab[b:b + 1], torch.zeros(1, dtype=torch.int32, device=dev),
                                     pt[..., :512].contiguous(), pt[..., 512:].contiguous())
        htab = table_t[:, HYB_SINK // 64:].contiguous()
        hl_t = torch.from_numpy(hyb_hist.astype(np.int32)).to(dev)
        pl_t = torch.from_numpy(prot_lens).to(dev)
        mh, mp = int(hyb_hist.max()), int(prot_lens.max())
        ws_h = torch.empty(max(api.mla_qdecode_hybrid_workspace_bytes(w.B, w.s_q, w.H, mh, mp), 1),
                           dtype=torch.uint8, device=dev)

        def hyb(k):
            api.mla_qdecode_hybrid(desc, pools[k], htab, hl_t, mh, bpool_h, ptab, pl_t, mp, qcs[k], qrs[k], w.scale,
                                   out=out, lse=lse, workspace=ws_h, stream=stream)

        for i in range(args.warmup):
            hyb(i % R)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.steps):
            hyb(i % R)
        e1.record(stream)
        torch.cuda.synchronize()
        assert api.mla_get_device_status() == 0
        ms_h = e0.elapsed_time(e1) / args.steps
        q_bytes = int(hyb_hist.sum()) * page_bytes // 64
        b_bytes = int(prot_lens.sum()) * 1152
        hybrid_leg = {"sink": HYB_SINK, "window": f"{HYB_WINDOW}..{HYB_WINDOW + 63}", "ms_per_decode": ms_h,
                      "head_tokens_per_s": st["head_tokens"] / (ms_h * 1e-3), "vs_qdecode_time": ms_h / ms_decode,
                      "cache_bytes": q_bytes + b_bytes,
                      "compression_vs_bf16": int(lens.astype(np.int64).sum()) * 1152 / (q_bytes + b_bytes)}

    # ---- the same step replayed from a CUDA graph (one graph launch per R steps) ----
    graph_leg = None
    try:
        def step_cur(k):  # launches on the current stream (the capture stream while capturing)
            api.mla_qdecode_fused_append(desc, pools[k], table_t, lens_t, max_len, newc_t, newr_t, qcs[k], qrs[k],
                                         w.scale, out=out, lse=lse, num_splits=w.num_splits, workspace=ws)
        cs = torch.cuda.Stream(device=dev)
        cs.wait_stream(stream)
        with torch.cuda.stream(cs):
            for k in range(R):
                step_cur(k)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cs, capture_error_mode="relaxed"):
            for k in range(R):
                step_cur(k)
        torch.cuda.synchronize()
        reps = max(1, args.steps // R)
        for _ in range(max(1, args.warmup // R)):
            graph.replay()
        torch.cuda.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record()
        for _ in range(reps):
            graph.replay()
        g1.record()
        torch.cuda.synchronize()
        ms_g = g0.elapsed_time(g1) / (reps * R)
        assert api.mla_get_device_status() == 0
        graph_leg = {"ms_per_step": ms_g, "head_tokens_per_s": job_rate(st["head_tokens"], 1, ms_g),
                     "steps_per_replay": R, "replays": reps}
        del graph
    except Exception as exc:  # capture unsupported here: report it, keep the other legs
        torch.cuda.synchronize()
        graph_leg = {"unavailable": f"{type(exc).__name__}: {exc}"[:200]}

    # ---- end to end through the C ABI with host buffers ----
    h_qc = torch.from_numpy(qc_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    h_qr = torch.from_numpy(qr_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    h_nc = torch.from_numpy(new_c.view(np.int16)).view(torch.bfloat16).pin_memory()
    h_nr = torch.from_numpy(new_r.view(np.int16)).view(torch.bfloat16).pin_memory()
    # Double-buffered: step k's uploads (on their own stream) overlap step k-1's
    # append + decode, and its read-back (another stream) overlaps step k+1's.
    # Every step still moves its inputs in and its output and lse out.
    hs, ds = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    slots = 2
    q_in = [(torch.empty_like(qcs[0]), torch.empty_like(qrs[0])) for _ in range(slots)]
    n_in = [(torch.empty_like(newc_t), torch.empty_like(newr_t)) for _ in range(slots)]
    outs = [torch.empty_like(out) for _ in range(slots)]
    lses = [torch.empty_like(lse) for _ in range(slots)]
    h_outs = [torch.empty(out.shape, dtype=torch.bfloat16).pin_memory() for _ in range(slots)]
    h_lses = [torch.empty(lse.shape, dtype=torch.float32).pin_memory() for _ in range(slots)]
    ev_in = [torch.cuda.Event() for _ in range(slots)]
    ev_out = [torch.cuda.Event() for _ in range(slots)]  # compute done: inputs free, outputs ready
    ev_done = [torch.cuda.Event() for _ in range(slots)]  # read-back done: outputs free
    for e in ev_out + ev_done:
        e.record(stream)

    def e2e_step(k):
        a = k % slots
        hs.wait_event(ev_out[a])
        with torch.cuda.stream(hs):
            q_in[a][0].copy_(h_qc, non_blocking=True)
            q_in[a][1].copy_(h_qr, non_blocking=True)
            n_in[a][0].copy_(h_nc, non_blocking=True)
            n_in[a][1].copy_(h_nr, non_blocking=True)
        ev_in[a].record(hs)
        stream.wait_event(ev_in[a])
        stream.wait_event(ev_done[a])
        api.mla_qdecode_fused_append(desc, pools[k % R], table_t, lens_t, max_len, n_in[a][0], n_in[a][1],
                                     q_in[a][0], q_in[a][1], w.scale, out=outs[a], lse=lses[a],
                                     num_splits=w.num_splits, workspace=ws, stream=stream)
        ev_out[a].record(stream)
        ds.wait_event(ev_out[a])
        with torch.cuda.stream(ds):
            h_outs[a].copy_(outs[a], non_blocking=True)
            h_lses[a].copy_(lses[a], non_blocking=True)
        ev_done[a].record(ds)

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    hs.wait_event(e0)
    ds.wait_event(e0)
    for i in range(args.steps):
        e2e_step(i)
    for e in ev_done:
        stream.wait_event(e)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = e0.elapsed_time(e1) / args.steps
    if world > 1:
        ms_e2e = max_over_ranks(ms_e2e, dist, dev)
    h2d = (h_qc.numel() + h_qr.numel() + h_nc.numel() + h_nr.numel()) * 2
    d2h = h_outs[0].numel() * 2 + h_lses[0].numel() * 4

    # a step is one decode launch (the append runs inside the tensor-core and the small-row
    # kernels), the combine for split plans, and, on the tensor-core path, one more
    # (single-block) kernel for a multi-wave split grid: its work list, units longest first
    # (the library's rule, restated here)
    rows = w.s_q * w.H
    units = w.B * n_split * ((rows + 127) // 128)
    chunk_pages = -(-((max_len + 63) // 64) // n_split)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    planned = rows > 16 and n_split > 1 and chunk_pages <= 128 and units > 2 * (sms // 2)
    launches_per_step = 1 + (1 if n_split > 1 else 0) + (1 if planned else 0)
    line = {
        "metric": METRIC, "value": value, "unit": "head-tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 hi+lo operand pairs, f32 accumulate", "data": "synthetic",
        "config": _config(w, world, extra={"num_splits": n_split, "pool_copies": R, "pool_mb": pool_bytes / 1e6}),
        "kv_tokens_per_s": job_rate(st["kv_tokens"], world, ms_step),
        "hbm": {"achieved_gbs": gbs, "peak_gbs": peaks["hbm_gbs"], "frac": gbs / peaks["hbm_gbs"],
                "note": "algorithmic bytes of one decode / decode-call time"},
        "legs_ms": {"fused_append_decode": ms_decode,
                    "separate": {"append": ms_append, "decode": ms_sep_decode, "sum": ms_append + ms_sep_decode}},
        "append": append_stats(w, ms_append),
        "roofline": roof,
        "e2e": {"value": job_rate(st["head_tokens"], world, ms_e2e), "unit": "head-tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e},
        "gpu_launches": launches_per_step * args.steps,
        "bf16_decode": bf16_leg,
        "hybrid_decode": hybrid_leg,
        "cuda_graph": graph_leg,
        "clocks": clk.summary(),
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_leg(w)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

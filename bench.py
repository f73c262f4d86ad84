"""Benchmark of the RainFusion2.0 block-sparse attention path on B200.

One step = one attention call of a video DiT layer at 720p (B=1 per GPU, 40
heads, d=128, latent 21x45x80 = 75,600 tokens, 64-token blocks, keep 20% of
key blocks per query block + first-frame sink): permute Q, K, V -> predict
the block mask -> block-sparse attention -> unpermute O, all through the C ABI.

Printed by rank 0 as one JSON line:
  value      effective TFLOP/s of kept-block attention work (sum over kept
             block pairs of 4*d*r_i*c_j) over the whole step, all ranks;
  e2e        the same metric with Q/K/V copied from pinned host memory and O
             copied back inside every timed step;
  roofline   the attention kernel against the measured dense bf16 peak
             (kept-block FLOPs only), timed with CUDA events in the timed region;
  stages     per-kernel ms, achieved GB/s or TFLOP/s and fraction of roofline;
  cpu_baseline  the fp64 oracle on a bounded sample of the same workload.

Multi-GPU (torchrun): each rank runs its own batch element (weak scaling, no
collective on the data path); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from image_dits_b200.workload import SWEEP_KEEPS, WORKLOADS, make_qkv  # noqa: E402

METRIC = "block-sparse attn ms/call + effective TFLOPS (kept blocks) at 75,600 tok, 80% sparse"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_desc(wl, per_gpu=True):
    return (f"{wl.name}: B={wl.batch}{'/GPU' if per_gpu else ' (one call over all GPUs)'}, {wl.heads} heads, d={wl.head_dim}, latent {wl.frames}x{wl.height}x"
            f"{wl.width}{f' + {wl.text_tokens} text' if wl.text_tokens else ''} ({wl.num_tokens:,} tokens), block 64, window {wl.win_t}x{wl.win_h}x{wl.win_w}, keep "
            f"{wl.keep:g} of key blocks (sparsity {1 - wl.keep:g}) + first-frame sink={'on' if wl.sink else 'off'}")


def kept_flops_from_mask(mask, wl) -> float:
    """Sum over kept (query block i, key block j) of 4*d*r_i*c_j (valid rows/cols)."""
    Tb, N, d = wl.num_blocks, wl.num_tokens, wl.head_dim
    last = N - 64 * (Tb - 1)
    rc = mask.row_count.to(torch.int64).view(-1, Tb)
    r = torch.full((Tb,), 64, dtype=torch.int64, device=rc.device)
    r[-1] = last
    # columns: every kept block has 64 valid keys except block Tb-1 (`last`);
    # block Tb-1 is kept in a row iff it is that row's last entry.
    rs = mask.row_start.to(torch.int64).view(-1, Tb)
    last_idx = mask.col_idx.to(torch.int64)[(rs + rc - 1).clamp(min=0)]
    has_last = (last_idx == Tb - 1) & (rc > 0)
    cols = rc * 64 - has_last.to(torch.int64) * (64 - last)
    return float((4 * d * (cols * r[None, :]).sum()).item())


# DRAM bytes (read + write) per (token, head) of one block_sparse_attn_kernel<128>
# launch: dram__bytes_read.sum + dram__bytes_write.sum of one ncu capture on the
# 720p shape with 8 heads (514.98 MB + 137.66 MB over 75,600 tokens x 8 heads), of
# the kernel as built at ATTN_TRAFFIC_BUILD.  The kernel's DRAM traffic is its
# compulsory Q/K/V reads and O writes (1,024 B per token-head; K/V re-reads hit L2),
# so it scales with the token-heads of the workload.  Re-measure whenever the
# kernel changes.
ATTN_DRAM_BYTES_PER_TOKEN_HEAD = (514.980864e6 + 137.662464e6) / (75600 * 8)
ATTN_TRAFFIC_BUILD = "02d6d5b"


def mask_bytes(wl, mask) -> float:
    """Algorithmic HBM bytes of mask prediction: Q and K read once + CSR written."""
    qk = 2 * wl.batch * wl.heads * wl.num_tokens * wl.head_dim * 2
    csr = 4 * (2 * mask.row_count.numel() + mask.kept_pairs())
    return float(qk + csr)


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.path = None
        try:
            props = torch.cuda.get_device_properties(device_index)
            uuid = str(props.uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            sel = []
        self.sel = sel
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            self.fh = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(["nvidia-smi", *sel, f"--query-gpu={self.Q}", "--format=csv,noheader",
                                          "-lms", "200"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        window = "timed region"
        if not rows:
            # The timed region was shorter than the sampler's start-up: one
            # query right after it, under the same residency.
            try:
                out = subprocess.run(["nvidia-smi", *self.sel, f"--query-gpu={self.Q}", "--format=csv,noheader"],
                                     capture_output=True, text=True, timeout=20).stdout
                rows = [[p.strip() for p in l.split(",")] for l in out.splitlines() if l.count(",") >= 8]
                window = "one sample right after the timed region (region shorter than the sampler start-up)"
            except Exception:
                rows = []
        if not rows:
            return None

        def num(s):
            try:
                return float(s.split()[0])
            except Exception:
                return float("nan")
        sm = [num(r[1]) for r in rows]
        mx = max(num(r[2]) for r in rows)
        power = [num(r[3]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[5 + k].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": reasons, "samples": len(rows),
                "power_w_max": max(power), "window": window}


def combine_over_ranks(ms_step, attn_ms, e2e_ms, flops, dist=None, device="cpu"):
    """Whole-job numbers: every time is the max over ranks, the work is the sum."""
    vals = torch.tensor([ms_step, attn_ms, e2e_ms, flops], dtype=torch.float64, device=device)
    if dist is not None:
        mx = vals.clone()
        dist.all_reduce(mx, op=dist.ReduceOp.MAX)
        sm = vals.clone()
        dist.all_reduce(sm, op=dist.ReduceOp.SUM)
        vals = torch.cat([mx[:3], sm[3:]])
    v = vals.cpu().tolist()
    return {"ms_step": v[0], "attn_ms": v[1], "e2e_ms": v[2], "flops": v[3]}


def rank_seed(rank: int) -> int:
    """Each rank runs its own batch element: independent seeded inputs."""
    return 1000 * rank


def cpu_info():
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except Exception:
        pass
    return model


def oracle_sample(wl, seed=0, n_query_blocks=32, budget_s=None):
    """The oracle as it stands on one head of the workload: permutation of Q,
    K, V, the full mask of that head, and attention for a sample of query
    blocks (one of them a sink block).  With budget_s, attention runs in
    chunks of n_query_blocks random query blocks until that many seconds have
    passed.  Returns (kept_flops, seconds, desc, stages): stages holds the
    wall time of each step for the head (attention for the sampled blocks,
    and extrapolated to all of the head's kept pairs)."""
    import oracle
    from image_dits_b200.workload import Workload
    one = Workload(wl.name, 1, 1, wl.head_dim, wl.frames, wl.height, wl.width, wl.win_t, wl.win_h, wl.win_w,
                   wl.keep, wl.sink, wl.rope, wl.text_tokens)
    q, k, v = make_qkv(one, "cpu", seed=seed)

    def bits(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)
    qb, kb, vb = bits(q), bits(k), bits(v)
    t0 = time.perf_counter()
    perm = oracle.permutation(wl.frames, wl.height, wl.width, wl.win_t, wl.win_h, wl.win_w, wl.sink, wl.text_tokens)
    qp, kp, vp = oracle.permute(qb, perm), oracle.permute(kb, perm), oracle.permute(vb, perm)
    t1 = time.perf_counter()
    mask, _, _ = oracle.predict_mask(qp, kp, wl.keep, wl.frames, wl.height, wl.width, wl.sink, wl.text_tokens)
    t2 = time.perf_counter()
    Tb = wl.num_blocks
    rng = np.random.default_rng(seed)
    s0 = oracle.sink_start(wl.frames, wl.height, wl.width, wl.sink, wl.text_tokens)
    upper = s0 if s0 > 0 else Tb
    order = [int(i) for i in rng.permutation(upper) if i != Tb - 1]
    N = wl.num_tokens
    blocks = []
    chunk = [Tb - 1] + order[:n_query_blocks - 1]
    pos = n_query_blocks - 1
    while chunk:
        items = np.array([(0, i) for i in chunk], dtype=np.int64)
        oracle.masked_attention(qp.reshape(1, N, -1), kp.reshape(1, N, -1), vp.reshape(1, N, -1),
                                mask.reshape(1, Tb, Tb), items)
        blocks += chunk
        if budget_s is None or time.perf_counter() - t0 >= budget_s or pos >= len(order):
            break
        chunk = order[pos:pos + n_query_blocks]
        pos += n_query_blocks
    t3 = time.perf_counter()
    oracle.unpermute(qp, perm)
    t4 = time.perf_counter()
    dt = t4 - t0
    last = N - 64 * (Tb - 1)

    def block_flops(i):
        r = 64 if i < Tb - 1 else last
        m = mask.reshape(Tb, Tb)[i]
        c = 64 * int(m.sum()) - (64 - last) * int(m[Tb - 1])
        return 4.0 * wl.head_dim * r * c
    flops = sum(block_flops(i) for i in blocks)
    head_flops = sum(block_flops(i) for i in range(Tb))
    stages = {"permute_qkv_s": t1 - t0, "predict_mask_s": t2 - t1, "attention_sample_s": t3 - t2,
              "attention_head_s_extrapolated": (t3 - t2) * head_flops / flops, "unpermute_s": t4 - t3}
    desc = (f"1 of {wl.heads} heads: permutation of Q/K/V, the head's full block mask, attention for "
            f"{len(blocks)} of {Tb} query blocks (1 sink block), unpermute")
    return flops, dt, desc, stages


def run_reference(args, wl, rank):
    """The oracle as the reference arm (CPU, bounded sample per step)."""
    if rank != 0:
        return
    import oracle
    oracle.build()
    for _ in range(args.warmup):
        oracle_sample(wl, n_query_blocks=2)
    times, flops = [], 0.0
    desc = ""
    for s in range(args.steps):
        f, dt, desc, _ = oracle_sample(wl, seed=s, n_query_blocks=32)
        times.append(dt)
        flops += f
    total = sum(times)
    value = flops / total / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(wl), "global_batch": 1, "seq_len": wl.num_tokens,
                   "parallelism": "none (CPU oracle)"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "cpu": cpu_info(), "sample": desc + " (per step)"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="video720p", choices=list(WORKLOADS))
    ap.add_argument("--keep", type=float, default=None)
    ap.add_argument("--heads", type=int, default=None,
                    help="override the workload's head count (smaller cases of the same shape, e.g. for ncu)")
    ap.add_argument("--tau", type=float, default=None,
                    help="CDF-threshold selection with this tau instead of the workload's top-n keep ratio")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-chunks", type=int, default=8, help="head chunks of the end-to-end pipeline")
    ap.add_argument("--sweep", action="store_true", help="also time the keep-ratio sweep (stderr)")
    ap.add_argument("--split", default="batch", choices=["batch", "heads"],
                    help="N > 1: one batch element per GPU (weak scaling), or one call's heads divided "
                         "among the GPUs (strong scaling); neither exchanges data")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    wl = WORKLOADS[args.workload]
    if args.keep is not None:
        wl = wl.with_keep(args.keep)
    if args.heads is not None:
        if args.heads < 1:
            raise SystemExit("--heads must be >= 1")
        wl = dataclasses.replace(wl, heads=args.heads, name=f"{wl.name}@heads{args.heads}")

    if args.impl == "reference":
        run_reference(args, wl, rank)
        return

    from image_dits_b200 import build as rf2_build
    from image_dits_b200 import rf2
    if rank == 0:
        rf2_build.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
        dist.barrier()
    rf2.lib()

    call = wl                                       # the workload one call computes (all ranks together)
    if args.split == "heads":
        # one call's inputs on every rank (same seed); this rank keeps heads [h0, h1)
        from image_dits_b200.shard import head_range
        h0, h1 = head_range(wl.heads, world, rank)
        q, k, v = (x[:, h0:h1].contiguous() for x in make_qkv(wl, dev, seed=rank_seed(0)))
        wl = dataclasses.replace(wl, heads=h1 - h0)
    else:
        q, k, v = make_qkv(wl, dev, seed=rank_seed(rank))
    g = rf2.geometry_of(wl)
    qp, kp, vp, op, o = (torch.empty_like(q) for _ in range(5))
    mask, ws = rf2.alloc_mask(g, 1.0 if args.tau is not None else wl.keep, dev)
    stream = torch.cuda.current_stream()

    # heads per (scores, select) launch pair, as the library groups them: as many
    # heads' scores as fit in 96 MiB, at most one score item (head, 128-row tile) per SM
    Tb_ = wl.num_blocks
    head_bytes = Tb_ * ((Tb_ + 3) // 4 * 4) * 4
    tiles = (Tb_ + 127) // 128
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    G = min(wl.batch * wl.heads, max(1, (96 << 20) // head_bytes), max(1, sms // tiles))
    score_groups = -(-wl.batch * wl.heads // G)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        rf2.permute_qk_pool(g, q, k, ws, qp, kp)
        if ev is not None:
            ev[1].record(stream)
        rf2.permute(g, v, vp)
        if ev is not None:
            ev[2].record(stream)
        if args.tau is not None:
            rf2.predict_mask_cdf_pooled(g, args.tau, mask, ws)
        else:
            rf2.predict_mask_pooled(g, wl.keep, mask, ws)
        if ev is not None:
            ev[3].record(stream)
        rf2.block_sparse_attn(g, qp, kp, vp, mask, op)
        if ev is not None:
            ev[4].record(stream)
        rf2.unpermute(g, op, o)
        if ev is not None:
            ev[5].record(stream)

    # permute+pool, permute V, (scores + select) per group of heads, attention, unpermute
    launches_per_step = 2 + 2 * score_groups + 2

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if rf2.device_status() != rf2.RF2_OK:
        raise RuntimeError("device status not ok after warm-up")
    flops = kept_flops_from_mask(mask, wl)
    kept_pairs = mask.kept_pairs()
    Tb = wl.num_blocks
    density = kept_pairs / (wl.batch * wl.heads * Tb * Tb)

    # Inputs smaller than twice the L2 (126 MB) would be timed warm: write a
    # 256 MB buffer before every timed step and time the steps one by one.
    resident = 4 * q.numel() * 2
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if resident < (252 << 20) else None
    sampler = ClockSampler(local_rank)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t_start.record(stream)
    for s in range(args.steps):
        if flush is not None:
            flush.fill_(s & 0xff)
        step(evs[s])
    t_end.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clocks = sampler.stop()
    if flush is None:
        total_ms = t_start.elapsed_time(t_end)
    else:
        total_ms = sum(e[0].elapsed_time(e[5]) for e in evs)
    stage_ms = {name: statistics.mean(e[a].elapsed_time(e[b]) for e in evs)
                for name, a, b in (("permute_qk_pool", 0, 1), ("permute_v", 1, 2), ("predict_mask_pooled", 2, 3),
                                   ("block_sparse_attn", 3, 4), ("unpermute", 4, 5))}
    if rf2.device_status() != rf2.RF2_OK:
        raise RuntimeError("device status not ok after timing")

    # ---- end to end through the public API with host buffers: rf2.HostPipeline
    # (head chunks; host-to-device copies, compute and device-to-host copies
    # of different chunks overlap).  Every step copies the step's inputs from
    # pinned host memory and reads the result back.
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
        ho = torch.empty_like(hq).pin_memory()
        pipe = rf2.HostPipeline(g, keep=None if args.tau is not None else wl.keep, tau=args.tau,
                                chunks=args.e2e_chunks)
        for _ in range(args.warmup):
            pipe.run(hq, hk, hv, ho)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(pipe.h2d)
        for _ in range(args.steps):
            pipe.run(hq, hk, hv, ho)
        e1.record(pipe.d2h)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        if rf2.device_status() != rf2.RF2_OK:
            raise RuntimeError("device status not ok after the end-to-end runs")
        e2e_ms = e0.elapsed_time(e1) / args.steps
        e2e = {"ms_per_step": e2e_ms, "h2d_bytes_per_step": 3 * q.numel() * 2, "d2h_bytes_per_step": o.numel() * 2,
               "chunks": len(pipe.parts)}
        del pipe

    # ---- max over ranks (times), sum over ranks (work)
    ms_step = total_ms / args.steps
    comb = combine_over_ranks(ms_step, stage_ms["block_sparse_attn"], e2e["ms_per_step"] if e2e else 0.0, flops,
                              dist, dev)
    ms_step_all, attn_ms_all, e2e_ms_all, flops_all = comb["ms_step"], comb["attn_ms"], comb["e2e_ms"], comb["flops"]

    peaks, peak_src = load_peaks()
    attn_tf = flops / (stage_ms["block_sparse_attn"] * 1e-3) / 1e12
    attn_peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    means = 2 * wl.batch * wl.heads * Tb * wl.head_dim * 4
    qkbytes = 2 * 2 * q.numel() * 2 + 2 * means        # read Q, K; write Qp, Kp and the hi/lo means
    vbytes = 2 * v.numel() * 2
    csr = 4 * (2 * mask.row_count.numel() + mask.kept_pairs())
    pbytes_mask = 2 * means + csr                       # read the means, write the CSR mask
    ubytes = 2 * o.numel() * 2
    hbm = peaks["hbm_gbs"]

    def gbs(b, ms):
        return b / (ms * 1e-3) / 1e9

    stages = {
        "permute_qk_pool": {"ms": stage_ms["permute_qk_pool"], "GB/s": gbs(qkbytes, stage_ms["permute_qk_pool"]),
                            "bytes": qkbytes, "frac": gbs(qkbytes, stage_ms["permute_qk_pool"]) / hbm,
                            "bound": "hbm"},
        "permute_v": {"ms": stage_ms["permute_v"], "GB/s": gbs(vbytes, stage_ms["permute_v"]), "bytes": vbytes,
                      "frac": gbs(vbytes, stage_ms["permute_v"]) / hbm, "bound": "hbm"},
        "predict_mask_pooled": {"ms": stage_ms["predict_mask_pooled"], "bytes": pbytes_mask,
                                "GB/s": gbs(pbytes_mask, stage_ms["predict_mask_pooled"]),
                                "note": "scores + top-n selection from the pooled means; the Q/K read of mask "
                                        "prediction is fused into permute_qk_pool"},
        "block_sparse_attn": {"ms": stage_ms["block_sparse_attn"], "TFLOP/s": attn_tf, "flops": flops,
                              "frac": attn_tf / attn_peak, "bound": "tensor"},
        "unpermute": {"ms": stage_ms["unpermute"], "GB/s": gbs(ubytes, stage_ms["unpermute"]), "bytes": ubytes,
                      "frac": gbs(ubytes, stage_ms["unpermute"]) / hbm, "bound": "hbm"},
    }

    line = {
        "metric": METRIC,
        "value": flops_all / (ms_step_all * 1e-3) / 1e12,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step_all,
        "attn_ms_per_call": attn_ms_all,
        "attn_tflops": flops_all / world / (attn_ms_all * 1e-3) / 1e12,
        "higher_is_better": True,
        "scaling": "strong" if args.split == "heads" else "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) + 0.5*smooth 3D field, 3D RoPE on Q/K, bf16)",
        "config": {"workload": workload_desc(call, args.split != "heads") if args.tau is None else
                   workload_desc(call, args.split != "heads").split(", keep")[0] + f", CDF-threshold selection tau={args.tau:g} + first-frame "
                   f"sink={'on' if wl.sink else 'off'}",
                   "global_batch": (call.batch if args.split == "heads" else world * wl.batch), "seq_len": wl.num_tokens,
                   "parallelism": (f"heads{world} (the call's {call.heads} heads divided among {world} GPUs, "
                                   f"{wl.heads} on rank 0; no collective)" if args.split == "heads"
                                   else f"dp{world} (independent batch element per GPU, no collective)"),
                   "kept_pairs_per_gpu": kept_pairs, "density": density,
                   "l2": (f"inputs larger than L2 ({q.numel() * 2 / 1e6:.0f} MB per tensor), no flush" if flush is None
                          else "256 MB buffer written before every timed step; steps timed one by one")},
        "roofline": {"bound": "tensor", "kernel": "block_sparse_attn", "achieved": attn_tf,
                     "peak": attn_peak, "unit": "TFLOP/s", "frac": attn_tf / attn_peak,
                     "peak_source": f"{peak_src} bf16_tflops_sustained (kernel timed inside a long step)",
                     "traffic": ATTN_DRAM_BYTES_PER_TOKEN_HEAD * wl.num_tokens * wl.batch * wl.heads,
                     "traffic_source": "dram__bytes_read.sum + dram__bytes_write.sum of one ncu capture of "
                                       "block_sparse_attn_kernel<128> on the 720p shape with 8 heads (build "
                                       f"{ATTN_TRAFFIC_BUILD}), scaled by token-heads"},
        "stages": stages,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if e2e:
        line["e2e"] = {"value": flops_all / (e2e_ms_all * 1e-3) / 1e12, "unit": "TFLOP/s",
                       "ms_per_step": e2e_ms_all, "h2d_bytes_per_step": e2e["h2d_bytes_per_step"],
                       "d2h_bytes_per_step": e2e["d2h_bytes_per_step"],
                       "api": f"rf2_attention_host (C ABI, through rf2.HostPipeline), {e2e['chunks']} head chunks, "
                              "copies overlapped with compute"}

    # mask prediction as one call on the permuted Q/K (Q and K read again), for its HBM roofline
    predict = ((lambda: rf2.predict_mask_cdf(g, qp, kp, args.tau, mask, ws)) if args.tau is not None
               else (lambda: rf2.predict_mask(g, qp, kp, wl.keep, mask, ws)))
    for _ in range(3):
        predict()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(5):
        predict()
    b.record(stream)
    torch.cuda.synchronize()
    ms_pm = a.elapsed_time(b) / 5
    mbytes = mask_bytes(wl, mask)
    stages["predict_mask_unfused"] = {"ms": ms_pm, "GB/s": gbs(mbytes, ms_pm), "bytes": mbytes,
                                      "frac": gbs(mbytes, ms_pm) / hbm, "bound": "hbm",
                                      "note": "rf2_predict_mask outside the step: reads Qp, Kp"}

    if args.sweep and rank == 0:
        sweep = []
        for keep in SWEEP_KEEPS:
            m2, ws2 = rf2.alloc_mask(g, keep, dev)
            for _ in range(3):
                rf2.predict_mask(g, qp, kp, keep, m2, ws2)
                rf2.block_sparse_attn(g, qp, kp, vp, m2, op)
            torch.cuda.synchronize()
            a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            reps = 5
            ms_mask = ms_attn = 0.0
            for _ in range(reps):
                a.record(stream)
                rf2.predict_mask(g, qp, kp, keep, m2, ws2)
                b.record(stream)
                rf2.block_sparse_attn(g, qp, kp, vp, m2, op)
                c.record(stream)
                torch.cuda.synchronize()
                ms_mask += a.elapsed_time(b) / reps
                ms_attn += b.elapsed_time(c) / reps
            f2 = kept_flops_from_mask(m2, wl)
            sweep.append({"keep": keep, "kept_pairs": m2.kept_pairs(),
                          "density": m2.kept_pairs() / (wl.heads * Tb * Tb), "mask_ms": ms_mask,
                          "mask_GB/s": gbs(mask_bytes(wl, m2), ms_mask), "attn_ms": ms_attn,
                          "attn_TFLOP/s": f2 / (ms_attn * 1e-3) / 1e12})
            del m2, ws2
        dense_ms = sweep[0]["attn_ms"]
        for r in sweep:
            r["speedup_vs_dense"] = dense_ms / r["attn_ms"]
        line["sweep"] = sweep

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        try:
            import oracle
            oracle.build()
            f, dt, desc, st = oracle_sample(wl, budget_s=12.0)
            heads = wl.batch * wl.heads
            full = heads * (st["permute_qkv_s"] + st["predict_mask_s"] + st["attention_head_s_extrapolated"]
                            + st["unpermute_s"])
            line["cpu_baseline"] = {"value": f / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                                    "kind": "oracle", "cpu": cpu_info(), "seconds": dt, "sample": desc,
                                    "stages_per_head_s": st,
                                    "full_call_s_extrapolated": full,
                                    "note": "full_call_s_extrapolated = heads x (permute + mask + attention over "
                                            "all of the head's kept pairs, extrapolated from the sample by kept "
                                            "FLOPs + unpermute)"}
        except Exception as exc:  # the baseline must not hide the GPU line
            line["cpu_baseline"] = {"value": None, "error": repr(exc)}

    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

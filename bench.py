"""Benchmark: last-scale block-sparse cross-scale attention on B200.

One step = the whole hot path for the Infinity-2B-like last scale (64x64
queries over the 10521-key prefix, B2 H16 D128, 128x128 blocks): the CSLA
block-list build followed by the block-sparse attention forward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line.  ``value`` is kept-block TFLOP/s of the whole job
(4 * n_q * n_k * D per kept block, valid elements only, summed over all ranks)
divided by the slowest rank's device time.  Multi-GPU runs (torchrun) give
every rank its own independent batch of the same size (weak scaling, no
collective on the data path).
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_cross_sparvar_b200 import inputs  # noqa: E402

WORKLOAD = dict(name="infinity2b_last_scale_64x64", sides=inputs.INFINITY_SIDES, q_scale=12,
                B=2, H=16, D=128, n_sink_scales=5, radius_prev=2, radius_own=4, block=128)
FLUSH_BYTES = 256 << 20
def e2e_chunks(B, H):
    """(b, h0, h1) head ranges of the end-to-end pipeline, in order.  Every copy
    costs about 4 us on top of its bytes, so the chunks are as large as a batch
    item allows, except towards the end, where they halve down to one head: only
    the last chunk's compute and copy back are not hidden behind input copies."""
    sizes, left = [], B * H
    tail = 1
    while left > 0:
        take = min(tail, left)
        sizes.append(take)
        left -= take
        if len(sizes) >= 2:
            tail *= 2
    sizes.reverse()  # large first, then 8, 4, 2, 1, 1 heads
    chunks, b_, h0 = [], 0, 0
    for n in sizes:
        while n > 0:  # a chunk does not span two batch items
            take = min(n, H - h0)
            chunks.append((b_, h0, h0 + take))
            n -= take
            h0 += take
            if h0 == H:
                b_, h0 = b_ + 1, 0
    return chunks


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return dict(bf16=p["bf16_tflops"], bf16_sustained=p["bf16_tflops_sustained"],
                    hbm=p["hbm_gbs"], source="measured")
    except Exception:
        return dict(bf16=1590.0, bf16_sustained=1400.0, hbm=6650.0, source="fallback")


ATTN_KERNEL = "attn_fwd_kernel<128, TOK=false, MULTI=false, ORD=true, FINE=false>"


def profiled_traffic():
    """DRAM bytes per launch of the attention kernel from the committed ncu data
    file, if it was taken on the current kernel source and instantiation (else None)."""
    import hashlib
    try:
        src = os.path.join(ROOT, "block_sparse_cross_sparvar_b200", "csrc", "attn_fwd_kernel.cuh")
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        with open(os.path.join(ROOT, "profiles", "attn_fwd_traffic.json")) as f:
            rec = json.load(f)
        if rec.get("kernel_source_sha256_16") == sha and rec.get("kernel") == ATTN_KERNEL:
            return int(rec["traffic_bytes_per_launch"])
    except Exception:
        pass
    return None


def workload_config(wl, cnt, idx, world):
    """The ``config`` object of the JSON line, identical for both arms: the
    workload, its shapes and the kept blocks of its CSLA lists."""
    sides, k, bq, D = wl["sides"], wl["q_scale"], wl["block"], wl["D"]
    off = inputs.token_offsets(sides)
    nq, L = off[k + 1] - off[k], off[k + 1]
    flops = kept_flops_from_lists(cnt, idx, nq, L, bq, bq, D) * wl["B"] * wl["H"]
    dense = 4 * nq * L * D * wl["B"] * wl["H"]
    return {"workload": wl["name"], "B": wl["B"], "H": wl["H"], "Lq": nq, "Lkv": L, "D": D,
            "block_q": bq, "block_kv": bq,
            "mask": f"csla sink<={wl['n_sink_scales']} r_prev={wl['radius_prev']} "
                    f"r_own={wl['radius_own']}",
            "kept_blocks": int(np.asarray(cnt).sum()), "total_blocks": int(idx.shape[0] * idx.shape[1]),
            "kept_flop_fraction": flops / dense,
            "kept_gflop_per_step_per_gpu": flops / 1e9,
            "l2": "256 MB flush write between timed steps",
            "parallelism": f"independent batch per GPU x{world}"}


def kept_flops_from_lists(cnt, idx, nq, L, bq, bk, D):
    total = 0
    for qb in range(cnt.shape[0]):
        nqr = min((qb + 1) * bq, nq) - qb * bq
        for kb in idx[qb, :cnt[qb]]:
            nkr = min((int(kb) + 1) * bk, L) - int(kb) * bk
            total += 4 * nqr * nkr * D
    return total


def start_clock_sampler(path):
    q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    try:
        f = open(path, "w")
        return subprocess.Popen(["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                 "-lms", "20"], stdout=f, stderr=subprocess.DEVNULL), f
    except Exception:
        return None, None


def stop_clock_sampler(proc, f, path, gpu_index, window="1 s of back-to-back steps + the timed region"):
    if proc is None:
        return None
    proc.terminate()
    try:
        proc.wait(timeout=5)
    except Exception:
        proc.kill()
    f.close()
    sm, mx, reasons = [], 0.0, set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for line in open(path):
        parts = [p.strip() for p in line.split(",")][1:]
        if len(parts) < 9 or parts[0] != str(gpu_index):
            continue
        try:
            sm.append(float(parts[1]))
            mx = max(mx, float(parts[2]))
        except ValueError:
            continue
        for n, v in zip(names, parts[5:9]):
            if v.lower() == "active":
                reasons.add(n)
    if not sm:
        return None
    return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "samples": len(sm),
            "reasons": sorted(reasons), "window": window}


def cpu_baseline(wl, budget_s=12.0, seed=0, d=None):
    """The fp64 oracle, as it stands, on a bounded sample of the workload:
    (batch, head) pairs one after another, query block by query block, until
    ``budget_s`` of CPU time has been spent."""
    from oracle import sparvar_oracle as orc
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = len(os.sched_getaffinity(0))
    sides, k, bq = wl["sides"], wl["q_scale"], wl["block"]
    if d is None:
        d = inputs.make_qkv(seed, wl["B"], wl["H"], sides, wl["D"], wl["n_sink_scales"])
    off = d["offsets"]
    t0 = time.perf_counter()
    flops, blocks, pairs = 0, 0, 0
    for b in range(wl["B"]):
        for h in range(wl["H"]):
            if time.perf_counter() - t0 >= budget_s:
                break
            q = d["qf"][b, h, off[k]:off[k + 1]].astype(np.float64)
            kk = d["kf"][b, h, :off[k + 1]].astype(np.float64)
            vv = d["vf"][b, h, :off[k + 1]].astype(np.float64)
            cnt, idx, blk = orc.build_csla_mask(sides, k, wl["n_sink_scales"], wl["radius_prev"],
                                                wl["radius_own"], bq, bq)
            nq, L = q.shape[0], kk.shape[0]
            pairs += 1
            for qb in range(blk.shape[0]):
                if time.perf_counter() - t0 >= budget_s:
                    break
                rows = np.arange(qb * bq, min((qb + 1) * bq, nq))
                orc.masked_attention_rows(rows, q, kk, vv, blk, bq, bq)
                sub = np.zeros_like(blk)
                sub[qb] = blk[qb]
                flops += orc.kept_flops(sub, nq, L, bq, bq, wl["D"])
                blocks += 1
    dt = time.perf_counter() - t0
    nqb = -(-(off[k + 1] - off[k]) // bq)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": int(threads), "kind": "oracle",
            "sample": f"{blocks} of {wl['B'] * wl['H'] * nqb} (batch, head, query block) units over "
                      f"{pairs} (batch, head) pairs, CSLA mask build included; numpy fp64, {dt:.1f} s",
            "seconds": dt}


def run_reference(args, wl, rank, world):
    if world > 1 and rank != 0:
        return
    from oracle import sparvar_oracle as orc
    per_step = []
    d = inputs.make_qkv(0, wl["B"], wl["H"], wl["sides"], wl["D"], wl["n_sink_scales"])
    cnt, idx, _ = orc.build_csla_mask(wl["sides"], wl["q_scale"], wl["n_sink_scales"],
                                      wl["radius_prev"], wl["radius_own"], wl["block"], wl["block"])
    budget = max(1.0, 90.0 / max(1, args.steps + args.warmup))
    for i in range(args.warmup + args.steps):
        res = cpu_baseline(wl, budget_s=budget, d=d)
        if i >= args.warmup:
            per_step.append(res)
    val = float(np.mean([r["value"] for r in per_step]))
    line = {"impl": "reference", "metric": "last-scale block-sparse attn ms and kept-block TFLOP/s "
            "(% of bf16 TC peak)", "value": val, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": float(np.mean([r["seconds"] for r in per_step]) * 1e3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(wl, cnt, idx, world),
            "cpu_baseline": {k: per_step[-1][k] for k in ("kind", "cores", "sample")} | {"value": val,
                                                                                      "unit": "TFLOP/s"},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--extra", action="store_true",
                    help="after the main line, print one line per further workload (CS4A full pass, "
                         "Infinity-8B radius sweep, density sweep)")
    ap.add_argument("--soak-s", type=float, default=1.0,
                    help="seconds of untimed back-to-back steps while the clock sampler starts")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    wl = WORKLOAD

    if args.impl == "reference":
        run_reference(args, wl, rank, world)
        return

    import torch
    import torch.distributed as dist
    from block_sparse_cross_sparvar_b200 import ops

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    sides, k, D, B, H, bq = wl["sides"], wl["q_scale"], wl["D"], wl["B"], wl["H"], wl["block"]
    d = inputs.make_qkv(rank, B, H, sides, D, wl["n_sink_scales"])
    off = d["offsets"]
    nq, L = off[k + 1] - off[k], off[k + 1]
    to_host = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)  # noqa: E731
    hq = to_host(d["q"][:, :, off[k]:off[k + 1]]).pin_memory()
    hk = to_host(d["k"]).pin_memory()
    hv = to_host(d["v"]).pin_memory()
    del d
    q, kk, vv = hq.to(dev), hk.to(dev), hv.to(dev)
    o = torch.empty_like(q)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    # the lists and, from the builder's last CTA, the order of the query tiles for the
    # persistent attention kernel (longest list first within each wave of SM-count tiles)
    assert bq == 128
    done = torch.zeros(1, dtype=torch.int32, device=dev)
    order = torch.empty(B * H * ((nq + bq - 1) // bq), dtype=torch.int32, device=dev)

    def build():
        return ops.sparvar_build_csla_mask_ordered(sides, k, wl["n_sink_scales"], wl["radius_prev"],
                                                   wl["radius_own"], B, H, device=dev, done=done,
                                                   out=order)

    def step(qq, kk_, vv_, out):
        cnt, idx, order_ = build()
        ops.sparvar_block_sparse_attn_fwd(qq, kk_, vv_, cnt, idx, bq, bq, out=out, dev_status=status,
                                          tile_order=order_)
        return cnt, idx

    cnt, idx = step(q, kk, vv, o)
    torch.cuda.synchronize()
    cnt_h, idx_h = cnt.cpu().numpy(), idx.cpu().numpy()
    flops_step = kept_flops_from_lists(cnt_h, idx_h, nq, L, bq, bq, D) * B * H

    for _ in range(args.warmup):
        step(q, kk, vv, o)
    torch.cuda.synchronize()

    # the step (list build, then attention) replayed from one CUDA graph, as a generation
    # loop would run it: its device time then holds no gap for the host-side
    # preparation of a launch (tensor maps, argument checks).  The attention and the
    # build are also captured on their own, for their separate times.
    g_step, g_attn, g_build = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step):
        cnt_g, idx_g, order_g = build()
        ops.sparvar_block_sparse_attn_fwd(q, kk, vv, cnt_g, idx_g, bq, bq, out=o, dev_status=status,
                                          tile_order=order_g)
    with torch.cuda.graph(g_attn):
        ops.sparvar_block_sparse_attn_fwd(q, kk, vv, cnt_g, idx_g, bq, bq, out=o, dev_status=status,
                                          tile_order=order_g)
    with torch.cuda.graph(g_build):
        build()
    for _ in range(args.warmup):
        g_step.replay()
        g_attn.replay()
        g_build.replay()
    torch.cuda.synchronize()

    # raw nvidia-smi samples; the JSON line carries their summary
    clocks_dir = os.environ.get("SPARVAR_CLOCKS_DIR", "/tmp")
    clocks_path = os.path.join(clocks_dir, f"sparvar_clocks_rank{rank}.csv")
    sampler, sf = start_clock_sampler(clocks_path) if rank == 0 else (None, None)
    t_soak = time.perf_counter()
    while time.perf_counter() - t_soak < args.soak_s:  # same load as the timed steps, untimed
        for _ in range(20):
            flush.fill_(0)
            g_step.replay()
        torch.cuda.synchronize()

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    def timed(graph):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        for i in range(args.steps):
            flush.fill_(i)  # evict inputs from the 126 MB L2 between steps (not timed)
            ev[i][0].record()
            graph.replay()
            ev[i][1].record()
        torch.cuda.synchronize()
        return [a.elapsed_time(b_) for a, b_ in ev]

    step_ms = timed(g_step)
    attn_ms = timed(g_attn)  # the same attention alone, for the roofline
    mask_ms = timed(g_build)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = stop_clock_sampler(sampler, sf, clocks_path, torch.cuda.current_device()) if rank == 0 else None
    # the same steps launched directly through the bindings, for comparison
    direct_ms = []
    for i in range(5):
        flush.fill_(i)
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        d0.record()
        step(q, kk, vv, o)
        d1.record()
        torch.cuda.synchronize()
        direct_ms.append(d0.elapsed_time(d1))
    if not torch.equal(cnt_g, cnt) or not torch.equal(idx_g, idx):
        raise SystemExit("the replayed list build differs from the direct one")
    del g_step, g_attn, g_build

    # end to end through the public API: pinned host inputs -> device -> result -> host.
    # The heads are processed in chunks on three streams: the host-to-device copy of
    # chunk c + 1 runs while chunk c is computed and chunk c - 1 is copied back, so
    # the step approaches the time of the input copy alone.
    ho = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    chunks = e2e_chunks(B, H)
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    s_cmp = torch.cuda.current_stream(dev)
    e2e_ms, copy_ms = [], []

    def e2e_step():
        cnt_e, idx_e, _ = ops.sparvar_build_csla_mask(sides, k, wl["n_sink_scales"], wl["radius_prev"],
                                                      wl["radius_own"], bq, bq, device=dev)
        done_in, done_cmp = [], []
        for b_, h0, h1 in chunks:
            sl = (slice(b_, b_ + 1), slice(h0, h1))
            with torch.cuda.stream(s_in):
                q[sl].copy_(hq[sl], non_blocking=True)
                kk[sl].copy_(hk[sl], non_blocking=True)
                vv[sl].copy_(hv[sl], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(s_in)
                done_in.append(ev)
        for (b_, h0, h1), ev in zip(chunks, done_in):
            sl = (slice(b_, b_ + 1), slice(h0, h1))
            s_cmp.wait_event(ev)
            ops.sparvar_block_sparse_attn_fwd(q[sl], kk[sl], vv[sl], cnt_e, idx_e, bq, bq, out=o[sl],
                                              dev_status=status)
            evc = torch.cuda.Event()
            evc.record(s_cmp)
            done_cmp.append(evc)
        for (b_, h0, h1), evc in zip(chunks, done_cmp):
            sl = (slice(b_, b_ + 1), slice(h0, h1))
            s_out.wait_event(evc)
            with torch.cuda.stream(s_out):
                ho[sl].copy_(o[sl], non_blocking=True)
        s_cmp.wait_stream(s_out)

    for i in range(max(3, min(args.steps, 10)) + 1):
        flush.fill_(i)
        torch.cuda.synchronize()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s_in.wait_stream(s_cmp)
        s0.record(s_cmp)
        s_in.wait_event(s0)
        e2e_step()
        s1.record(s_cmp)
        torch.cuda.synchronize()
        if i > 0:  # the first pass warms the streams up
            e2e_ms.append(s0.elapsed_time(s1))
    # the input copy alone, for reference
    for i in range(3):
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record()
        q.copy_(hq, non_blocking=True)
        kk.copy_(hk, non_blocking=True)
        vv.copy_(hv, non_blocking=True)
        c1.record()
        torch.cuda.synchronize()
        copy_ms.append(c0.elapsed_time(c1))
    if status.item() != 0:
        raise SystemExit(f"device status {status.item()} after the bench")

    t_step = float(np.mean(step_ms))
    t_attn = float(np.mean(attn_ms))
    t_e2e = float(np.mean(e2e_ms))
    from block_sparse_cross_sparvar_b200 import multi
    t_step, t_attn, t_e2e = multi.max_over_ranks([t_step, t_attn, t_e2e], dev)
    (total_flops,) = multi.sum_over_ranks([float(flops_step)], dev)
    pk = peaks()
    if rank == 0:
        achieved = flops_step / (t_attn * 1e-3) / 1e12
        peak = pk["bf16_sustained"] if args.soak_s > 0 else pk["bf16"]
        line = {
            "metric": "last-scale block-sparse attn ms and kept-block TFLOP/s (% of bf16 TC peak)",
            "value": total_flops / (t_step * 1e-3) / 1e12,
            "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t_step,
            "attn_ms": t_attn, "mask_build_ms": float(np.mean(mask_ms)),
            "launch": "each step (list build, then attention) replayed from one CUDA graph; "
                      "attention and build also timed alone from graphs of their own",
            "ms_per_step_direct_launch": float(np.median(direct_ms)),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": workload_config(wl, cnt_h, idx_h, world),
            "tile_order": "longest list first within each wave of the persistent kernel, "
                          "written by the list builder (natural order in the e2e chunks)",
            # the timed launches follow a soak of back-to-back steps under the power cap,
            # so they run at sustained clocks: the sustained GEMM figure is the peak they
            # compare with (the burst one when there is no soak); both fractions are given
            "roofline": {"bound": "tensor", "kernel": ATTN_KERNEL,
                         "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak,
                         "frac_of_burst": achieved / pk["bf16"],
                         "frac_of_sustained": achieved / pk["bf16_sustained"],
                         "peak_note": f"{pk['source']} bf16 dense "
                                      f"{'sustained' if args.soak_s > 0 else 'burst'} peak "
                                      f"(burst {pk['bf16']}, sustained {pk['bf16_sustained']}); "
                                      f"the timed steps follow a {args.soak_s:g} s soak",
                         "traffic": profiled_traffic(),
                         "traffic_note": "ncu dram bytes read+write per launch of this kernel source; "
                                         "null when the source changed since the capture"},
            "e2e": {"value": total_flops / (t_e2e * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "ms_per_step": t_e2e, "input_copy_alone_ms": float(np.median(copy_ms)),
                    "pipeline": f"{len(chunks)} chunks of "
                                f"{'/'.join(str(h1 - h0) for _, h0, h1 in chunks)} heads: copy in, "
                                "compute and copy out on three streams",
                    "h2d_bytes_per_step": int(hq.numel() * 2 + hk.numel() * 2 + hv.numel() * 2),
                    "d2h_bytes_per_step": int(ho.numel() * 2)},
            # the library's kernels in the timed regions: K steps (list build + attention),
            # then K attention launches and K list builds timed alone
            "gpu_launches": 4 * args.steps,
            "clocks": clocks,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = {kk_: v for kk_, v in cpu_baseline(wl).items() if kk_ != "seconds"}
        print(json.dumps(line), flush=True)
        if args.extra and world == 1:
            from block_sparse_cross_sparvar_b200 import workloads
            del q, kk, vv, o, hq, hk, hv
            torch.cuda.empty_cache()
            for fn in (workloads.cs4a_full_pass, workloads.cs4a_topk_2d_pass, workloads.cs4a_fused_pass,
                       workloads.decision_fused_vs_separate, workloads.csla_radius_sweep,
                       workloads.csla_granularity_sweep, workloads.density_sweep, workloads.ocache_scales):
                # SM clocks and throttle reasons over the whole run of the workload
                xs, xf = start_clock_sampler(clocks_path)
                rec = fn(dev)
                rec["clocks"] = stop_clock_sampler(xs, xf, clocks_path, torch.cuda.current_device(),
                                                   window="the whole workload, warm-up included")
                print(json.dumps({"extra": rec}), flush=True)
                torch.cuda.empty_cache()
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

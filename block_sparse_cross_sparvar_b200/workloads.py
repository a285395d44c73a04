"""GPU runs of the Infinity-shaped workloads beyond the headline last scale.

* ``cs4a_full_pass``: all 13 scales of one generation step with CS4A: scales
  1-10 dense (the 32x32 scale also yields the row LSE), the decision on the
  32x32 scale (pooled mass >= 0.95), and the mapped lists for 40x40, 48x48 and
  64x64; ``cs4a_topk_2d_pass`` the same with the Top-K rule (ratio 0.2), the
  scale-aware 2-D mapping and the output cache; ``cs4a_fused_pass`` the Top-K /
  2-D pass with the scales in two multi-problem launches.
* ``csla_radius_sweep``: the Infinity-8B-like last two scales (B2 H32) with the
  CSLA locality radius of earlier scales at 1, 2 and 4.
* ``csla_granularity_sweep``: the last scale under CSLA with 128x128 blocks,
  64x64 blocks and the token mask inside 128x128 tiles.
* ``density_sweep``: the last scale with random block lists at fixed densities
  (sink block always kept), with the full key prefix and with the 40x40 and
  48x48 scales skipped from the prefix; each also with the query tiles taken
  longest list first.
* ``ocache_scales``: the CS4A output cache alone, from the 32x32 decision scale
  to the 40x40, 48x48 and 64x64 scales, against the HBM bytes it must move.

Every step runs in the library's kernels; torch only provides memory, streams
and events.
"""
from __future__ import annotations

import numpy as np
import torch

from . import inputs, ops

FLUSH_BYTES = 256 << 20


def _dev(bits, device):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def _dense_lists(nqb, nkb, device):
    cnt = torch.full((nqb,), nkb, dtype=torch.int32, device=device)
    idx = torch.arange(nkb, dtype=torch.int32, device=device).repeat(nqb, 1).contiguous()
    return cnt, idx


def kept_flops(cnt, idx, nq, L, block, D):
    """4 * n_q * n_k * D over kept blocks (host copy of the lists)."""
    cnt = cnt.cpu().numpy()
    idx = idx.cpu().numpy()
    lead = cnt.shape[:-1]
    cnt2 = cnt.reshape(-1, cnt.shape[-1])
    idx2 = idx.reshape(-1, idx.shape[-2], idx.shape[-1])
    total = 0
    for r in range(cnt2.shape[0]):
        for qb in range(cnt2.shape[1]):
            nqr = min((qb + 1) * block, nq) - qb * block
            for kb in idx2[r, qb, :cnt2[r, qb]]:
                total += 4 * nqr * (min((int(kb) + 1) * block, L) - int(kb) * block) * D
    return total, int(np.prod(lead)) if lead else 1


def time_ms(fn, reps, device, warmup=3, sleep_ahead=False):
    """Median device time of fn over reps runs, a 256 MB L2 flush before each.
    sleep_ahead: a GPU sleep is queued after the flush, so that the host has
    queued the start event, fn's launches and the end event before the GPU
    reaches them (for calls shorter than their own host-side launch cost)."""
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.int32, device=device)
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize(device)
    out = []
    for i in range(reps):
        flush.fill_(i)
        if sleep_ahead:
            torch.cuda._sleep(400_000)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize(device)
        out.append(a.elapsed_time(b))
    return float(np.median(out))


def cs4a_fused_pass(device, reps=10, seed=0, B=2, H=16, D=128, topk_ratio=0.2, decision_scale=9):
    """The 13-scale pass in two attention launches: scales 1-10 (dense, with the
    decision scale's LSE) as one multi-problem launch, then the decision (Top-K),
    the 2-D mapping and scales 11-13 as a second multi-problem launch."""
    sides = inputs.INFINITY_SIDES
    d = inputs.make_qkv(seed, B, H, sides, D, 5)
    off = d["offsets"]
    q_all, k_all, v_all = _dev(d["q"], device), _dev(d["k"], device), _dev(d["v"], device)
    del d
    n_scales = len(sides)
    out = torch.zeros_like(q_all)
    dense = []
    for s in range(decision_scale + 1):
        cnt, idx = _dense_lists(-(-(off[s + 1] - off[s]) // 128), -(-off[s + 1] // 128), device)
        dense.append((off[s], off[s + 1] - off[s], off[s + 1], cnt, idx))
    state = {}

    def run():
        _, lse = ops.sparvar_block_sparse_attn_fwd_multi(q_all, k_all, v_all, dense, out=out,
                                                         return_lse=True)
        dec = decision_scale
        dc, di, _ = ops.sparvar_decide_blocks(
            q_all[:, :, off[dec]:off[dec + 1]], k_all[:, :, :off[dec + 1]], 0.95,
            lse=lse[:, :, off[dec]:off[dec + 1]].contiguous(), topk_ratio=topk_ratio)
        late = []
        for s in range(dec + 1, n_scales):
            mc, mi, _ = ops.sparvar_map_indices_2d(dc, di, sides, dec, s, 128, 128, off[5])
            state[s] = (mc, mi)
            late.append((off[s], off[s + 1] - off[s], off[s + 1], mc, mi))
        ops.sparvar_block_sparse_attn_fwd_multi(q_all, k_all, v_all, late, out=out)

    ms = time_ms(run, reps, device)
    flops = 0
    per_scale = {}
    for s in range(n_scales):
        nq, L = off[s + 1] - off[s], off[s + 1]
        f = 4 * nq * L * D * B * H if s <= decision_scale else kept_flops(*state[s], nq, L, 128, D)[0]
        per_scale[f"{sides[s]}x{sides[s]}"] = {"gflop": f / 1e9, "density": f / (4 * nq * L * D * B * H)}
        flops += f
    return {"workload": "cs4a_13_scales_two_launches_2d_mapping", "B": B, "H": H, "D": D,
            "selection": f"topk {topk_ratio}", "ms": ms, "gflop": flops / 1e9,
            "tflops": flops / (ms * 1e-3) / 1e12, "scales": per_scale}


def cs4a_topk_2d_pass(device, reps=10, seed=0):
    """The 13-scale pass with the Top-K rule (ratio 0.2), the 2-D mapping and the
    output cache (the decision scale's sparse output and the corrections add work
    that the GFLOP count below does not include)."""
    return cs4a_full_pass(device, reps, seed, topk_ratio=0.2, mapping="2d", ocache=True)


def cs4a_full_pass(device, reps=10, seed=0, B=2, H=16, D=128, tau=0.95, decision_scale=9,
                   topk_ratio=0.0, mapping="1d", ocache=False, fused_decision=True):
    sides = inputs.INFINITY_SIDES
    d = inputs.make_qkv(seed, B, H, sides, D, 5)
    off = d["offsets"]
    q_all, k_all, v_all = _dev(d["q"], device), _dev(d["k"], device), _dev(d["v"], device)
    del d
    n_scales = len(sides)
    outs = [torch.empty(B, H, off[s + 1] - off[s], D, dtype=torch.bfloat16, device=device)
            for s in range(n_scales)]
    dense = [_dense_lists(-(-(off[s + 1] - off[s]) // 128), -(-off[s + 1] // 128), device)
             for s in range(decision_scale + 1)]
    state = {}

    def run():
        for s in range(decision_scale + 1):
            q = q_all[:, :, off[s]:off[s + 1]]
            k = k_all[:, :, :off[s + 1]]
            v = v_all[:, :, :off[s + 1]]
            cnt, idx = dense[s]
            if s == decision_scale and fused_decision:
                _, _, dc, di, _ = ops.sparvar_decision_attn_fwd(q, k, v, tau, topk_ratio=topk_ratio,
                                                                out=outs[s])
                state["dec"] = (dc, di)
                if ocache:
                    state["o_sparse"] = ops.sparvar_block_sparse_attn_fwd(q, k, v, dc, di)
            elif s == decision_scale:
                _, lse = ops.sparvar_block_sparse_attn_fwd(q, k, v, cnt, idx, out=outs[s], return_lse=True)
                dc, di, _ = ops.sparvar_decide_blocks(q, k, tau, lse=lse, topk_ratio=topk_ratio)
                state["dec"] = (dc, di)
                if ocache:
                    state["o_sparse"] = ops.sparvar_block_sparse_attn_fwd(q, k, v, dc, di)
            else:
                ops.sparvar_block_sparse_attn_fwd(q, k, v, cnt, idx, out=outs[s])
        dc, di = state["dec"]
        src_nq, src_lkv = off[decision_scale + 1] - off[decision_scale], off[decision_scale + 1]
        for s in range(decision_scale + 1, n_scales):
            nq, L = off[s + 1] - off[s], off[s + 1]
            if mapping == "2d":
                mc, mi, _ = ops.sparvar_map_indices_2d(dc, di, sides, decision_scale, s, 128, 128,
                                                       off[5])
            else:
                mc, mi, _ = ops.sparvar_map_indices(dc, di, src_nq, src_lkv, nq, L, 128, 128, off[5])
            state[s] = (mc, mi)
            ops.sparvar_block_sparse_attn_fwd(q_all[:, :, off[s]:off[s + 1]], k_all[:, :, :L],
                                              v_all[:, :, :L], mc, mi, out=outs[s])
            if ocache:
                ops.sparvar_ocache_apply(outs[s], outs[decision_scale], state["o_sparse"],
                                         sides[decision_scale], sides[s], out=outs[s])

    ms = time_ms(run, reps, device)
    flops = 0
    per_scale = {}
    for s in range(n_scales):
        nq, L = off[s + 1] - off[s], off[s + 1]
        if s <= decision_scale:
            f = 4 * nq * L * D * B * H
        else:
            f, _ = kept_flops(*state[s], nq, L, 128, D)
        per_scale[f"{sides[s]}x{sides[s]}"] = {"gflop": f / 1e9,
                                                "density": f / (4 * nq * L * D * B * H)}
        flops += f
    rule = (f"topk {topk_ratio}" if topk_ratio > 0 else f"mass {tau}") + (" + ocache" if ocache else "")
    rule += ", fused decision" if fused_decision else ", decision after the dense pass"
    return {"workload": f"cs4a_full_pass_13_scales_{mapping}_mapping", "B": B, "H": H, "D": D,
            "selection": rule,
            "ms": ms, "gflop": flops / 1e9, "tflops": flops / (ms * 1e-3) / 1e12,
            "scales": per_scale}


def decision_fused_vs_separate(device, reps=20, seed=0, B=2, H=16, D=128, decision_scale=9):
    """The decision scale (32x32 over its 2521-key prefix): dense attention with the
    decision fused in (one launch) against dense attention followed by the
    stand-alone decision kernel (two launches, QK^T recomputed), for the mass
    rule and the Top-K rule."""
    sides = inputs.INFINITY_SIDES
    d = inputs.make_qkv(seed, B, H, sides, D, 5)
    off = d["offsets"]
    s = decision_scale
    q = _dev(d["q"][:, :, off[s]:off[s + 1]], device)
    k = _dev(d["k"][:, :, :off[s + 1]], device)
    v = _dev(d["v"][:, :, :off[s + 1]], device)
    del d
    nq, L = off[s + 1] - off[s], off[s + 1]
    cnt, idx = _dense_lists(-(-nq // 128), -(-L // 128), device)
    out = torch.empty_like(q)
    dense = 4 * nq * L * D * B * H
    res = []
    for tau, ratio in ((0.95, 0.0), (0.0, 0.2)):
        def separate():
            _, lse = ops.sparvar_block_sparse_attn_fwd(q, k, v, cnt, idx, out=out, return_lse=True)
            ops.sparvar_decide_blocks(q, k, tau, lse=lse, topk_ratio=ratio)

        ms_sep = time_ms(separate, reps, device)
        ms_fused = time_ms(lambda: ops.sparvar_decision_attn_fwd(q, k, v, tau, topk_ratio=ratio,
                                                                 out=out), reps, device)
        res.append({"selection": f"topk {ratio}" if ratio > 0 else f"mass {tau}",
                    "fused_ms": ms_fused, "separate_ms": ms_sep,
                    "dense_tflops_fused": dense / (ms_fused * 1e-3) / 1e12})
    return {"workload": "cs4a_decision_scale_32x32", "B": B, "H": H, "D": D, "runs": res}


def csla_radius_sweep(device, reps=10, seed=0, B=2, H=32, D=128, radii=(1, 2, 4)):
    sides = inputs.INFINITY_SIDES
    d = inputs.make_qkv(seed, B, H, sides, D, 5)
    off = d["offsets"]
    q_all, k_all, v_all = _dev(d["q"], device), _dev(d["k"], device), _dev(d["v"], device)
    del d
    res = []
    for s in (11, 12):
        nq, L = off[s + 1] - off[s], off[s + 1]
        q = q_all[:, :, off[s]:off[s + 1]]
        out = torch.empty_like(q)
        for r in radii:
            cnt, idx, _ = ops.sparvar_build_csla_mask(sides, s, 5, r, 4, 128, 128, device=device)
            ms = time_ms(lambda: ops.sparvar_block_sparse_attn_fwd(q, k_all[:, :, :L], v_all[:, :, :L],
                                                                   cnt, idx, out=out), reps, device)
            f, _ = kept_flops(cnt, idx, nq, L, 128, D)
            f *= B * H
            res.append({"scale": f"{sides[s]}x{sides[s]}", "radius_prev": r, "radius_own": 4,
                        "density": f / (4 * nq * L * D * B * H), "ms": ms,
                        "tflops": f / (ms * 1e-3) / 1e12})
    return {"workload": "infinity8b_last_two_scales_csla_radius_sweep", "B": B, "H": H, "D": D,
            "runs": res}


def csla_granularity_sweep(device, reps=10, seed=0, B=2, H=16, D=128):
    """The Infinity-2B last scale under CSLA at three granularities: 128x128
    blocks, 64x64 blocks (coarsened to 128x128 tiles with masks inside the call,
    the coarsening timed with it), and the token mask applied inside the 128x128
    tiles.  ``tflops`` counts the kept blocks' work at the run's own block size;
    for the token mask it counts the executed tiles' work (fewer token pairs are
    kept than the tiles hold)."""
    sides = inputs.INFINITY_SIDES
    s = len(sides) - 1
    d = inputs.make_qkv(seed, B, H, sides, D, 5)
    off = d["offsets"]
    nq, L = off[s + 1] - off[s], off[s + 1]
    q = _dev(d["q"][:, :, off[s]:off[s + 1]], device)
    k = _dev(d["k"][:, :, :L], device)
    v = _dev(d["v"][:, :, :L], device)
    del d
    out = torch.empty_like(q)
    dense = 4 * nq * L * D * B * H
    res = []
    for block in (128, 64):
        cnt, idx, _ = ops.sparvar_build_csla_mask(sides, s, 5, 2, 4, block, block, device=device)
        f, _ = kept_flops(cnt, idx, nq, L, block, D)
        f *= B * H
        if block == 128:
            ms = time_ms(lambda: ops.sparvar_block_sparse_attn_fwd(q, k, v, cnt, idx, out=out), reps,
                         device)
            res.append({"granularity": "block128", "density": f / dense, "ms": ms,
                        "tflops": f / (ms * 1e-3) / 1e12})
            continue
        # 64x64 lists: coarsened to 128x128 tiles with per-tile masks inside the
        # allocation-free call (no allocation in the timed region; the coarsening
        # kernel is timed with the attention); the executed tiles' work is reported too
        ms = time_ms(lambda: ops.sparvar_block_sparse_attn_fwd_static(q, k, v, cnt, idx, block,
                                                                      out=out), reps, device)
        t_cnt, t_idx, _ = ops.sparvar_coarsen_lists(cnt, idx, B, H, nq, L, block)
        ft, _ = kept_flops(t_cnt.reshape(-1), t_idx.reshape(-1, t_idx.shape[-1]), nq, L, 128, D)
        ft *= B * H
        res.append({"granularity": "block64", "density": f / dense, "ms": ms,
                    "tflops": f / (ms * 1e-3) / 1e12, "tile_density": ft / dense,
                    "tile_tflops": ft / (ms * 1e-3) / 1e12,
                    "note": "coarsening kernel included, no allocation in the timed region"})
    cnt, idx, _ = ops.sparvar_build_csla_mask(sides, s, 5, 2, 4, 128, 128, device=device)
    f, _ = kept_flops(cnt, idx, nq, L, 128, D)
    f *= B * H
    ms = time_ms(lambda: ops.sparvar_csla_token_attn_fwd(q, k, v, sides, s, 5, 2, 4, cnt, idx, out=out),
                 reps, device)
    res.append({"granularity": "token mask inside 128x128 tiles", "tile_density": f / dense, "ms": ms,
                "tile_tflops": f / (ms * 1e-3) / 1e12})
    return {"workload": "infinity2b_last_scale_csla_granularity", "B": B, "H": H, "D": D,
            "mask": "csla sink<=5 r_prev=2 r_own=4", "runs": res}


def density_sweep(device, reps=10, seed=0, B=2, H=16, D=128, densities=(0.05, 0.1, 0.2, 0.35, 0.5, 1.0)):
    sides = inputs.INFINITY_SIDES
    d = inputs.make_qkv(seed, B, H, sides, D, 5)
    off = d["offsets"]
    rng = d["rng"]
    q = _dev(d["q"][:, :, off[12]:off[13]], device)
    prefixes = {"full_10521": np.arange(off[13]),
                "skip_40_48_6617": np.concatenate([np.arange(off[10]), np.arange(off[12], off[13])]),
                "skip_7225": np.arange(7225)}
    res = []
    for name, keys in prefixes.items():
        k = _dev(np.ascontiguousarray(d["k"][:, :, keys]), device)
        v = _dev(np.ascontiguousarray(d["v"][:, :, keys]), device)
        L = keys.size
        nqb, nkb = 32, -(-L // 128)
        out = torch.empty_like(q)
        for dens in densities:
            keep = inputs.bernoulli_keep(rng, (B, H, nqb, nkb), dens)
            keep[..., 0] = True
            cnt = torch.from_numpy(keep.sum(-1).astype(np.int32)).to(device)
            idx_np = np.full((B, H, nqb, nkb), -1, np.int32)
            for bb in range(B):
                for hh in range(H):
                    for qb in range(nqb):
                        kept = np.nonzero(keep[bb, hh, qb])[0]
                        idx_np[bb, hh, qb, :kept.size] = kept
            idx = torch.from_numpy(idx_np).to(device)
            ms = time_ms(lambda: ops.sparvar_block_sparse_attn_fwd(q, k, v, cnt, idx, out=out), reps, device)
            # the same lists with the query tiles taken longest list first; the order is
            # built inside the timed call
            order = torch.empty(B * H * nqb, dtype=torch.int32, device=device)
            ms_lpt = time_ms(lambda: ops.sparvar_block_sparse_attn_fwd(
                q, k, v, cnt, idx, out=out,
                tile_order=ops.sparvar_tile_order(cnt, B, H, 4096, out=order)), reps, device)
            f, _ = kept_flops(cnt, idx, 4096, L, 128, D)
            res.append({"prefix": name, "Lkv": L, "target_density": dens,
                        "density": f / (4 * 4096 * L * D * B * H), "ms": ms,
                        "tflops": f / (ms * 1e-3) / 1e12, "ms_longest_first": ms_lpt,
                        "tflops_longest_first": f / (ms_lpt * 1e-3) / 1e12})
    return {"workload": "last_scale_density_sweep", "B": B, "H": H, "D": D, "runs": res}


def ocache_scales(device, reps=20, seed=0, B=2, H=16, D=128, s_src=32, targets=(40, 48, 64)):
    """The output cache alone (out of place), L2 flushed between runs, timed
    behind a GPU sleep (the call is shorter than its host-side cost).  Its bytes:
    the target output read and the corrected output written once, the decision
    scale's dense and sparse outputs read once (their re-reads by neighbouring
    target tokens come from L2)."""
    g = torch.Generator(device=device).manual_seed(seed)
    rnd = lambda n: torch.randn(B, H, n, D, generator=g, device=device).to(torch.bfloat16)  # noqa: E731
    o_d, o_s = rnd(s_src * s_src), rnd(s_src * s_src)
    res = []
    for t in targets:
        o_t = rnd(t * t)
        out = torch.empty_like(o_t)
        ms = time_ms(lambda: ops.sparvar_ocache_apply(o_t, o_d, o_s, s_src, t, out=out), reps, device,
                     sleep_ahead=True)
        nbytes = 2 * B * H * D * (2 * t * t + 2 * s_src * s_src)
        res.append({"s_src": s_src, "s_dst": t, "ms": ms, "bytes": nbytes, "gbs": nbytes / (ms * 1e-3) / 1e9})
    return {"workload": "cs4a_output_cache", "B": B, "H": H, "D": D, "runs": res}

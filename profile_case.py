"""Fixed launches of one kernel for profiling (ncu) on a workload of the bench.

    python profile_case.py [--kernel attn|attn_natural|decision|mass|csla|ocache] [--launches N]

attn:     Infinity-2B-like last scale (B2 H16, 4096 queries x 10521 keys, D128),
          CSLA lists, block-sparse attention forward with the query tiles in the
          list builder's order (as the bench's step); attn_natural: the same in
          natural tile order.  About 240 MB on the device (inputs larger than the
          126 MB L2).
decision: the CS4A decision scale (B2 H16, 1024 x 2521, D128): dense attention
          with the pooled mass and selection fused in.
mass:     the stand-alone decision kernel on the same scale.
csla:     the CSLA list build for the 64x64 scale, with the tile order.
ocache:   the output cache from the 32x32 decision scale to the 64x64 scale.
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

from block_sparse_cross_sparvar_b200 import inputs, ops  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--kernel", default="attn", choices=["attn", "attn_natural", "decision", "mass", "csla", "ocache"])
    ap.add_argument("--launches", type=int, default=3)
    args = ap.parse_args()
    sides = inputs.INFINITY_SIDES
    d = inputs.make_qkv(0, 2, 16, sides, 128, 5)
    off = d["offsets"]
    dev = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()  # noqa: E731
    if args.kernel in ("attn", "attn_natural", "csla"):
        q = dev(d["q"][:, :, off[12]:off[13]])
        k, v = dev(d["k"]), dev(d["v"])
        done = torch.zeros(1, dtype=torch.int32, device="cuda")
        cnt, idx, order = ops.sparvar_build_csla_mask_ordered(sides, 12, 5, 2, 4, 2, 16, done=done)
        if args.kernel == "attn_natural":
            order = None
        out = torch.empty_like(q)
        for _ in range(args.launches):
            if args.kernel == "csla":
                ops.sparvar_build_csla_mask_ordered(sides, 12, 5, 2, 4, 2, 16, done=done)
            else:
                ops.sparvar_block_sparse_attn_fwd(q, k, v, cnt, idx, out=out, tile_order=order)
    elif args.kernel in ("decision", "mass"):
        q = dev(d["q"][:, :, off[9]:off[10]])
        k = dev(d["k"][:, :, :off[10]])
        v = dev(d["v"][:, :, :off[10]])
        for _ in range(args.launches):
            if args.kernel == "decision":
                ops.sparvar_decision_attn_fwd(q, k, v, 0.95)
            else:
                ops.sparvar_decide_blocks(q, k, 0.95)
    else:
        o_t = dev(d["q"][:, :, off[12]:off[13]])
        o_d = dev(d["k"][:, :, off[9]:off[10]])
        o_s = dev(d["v"][:, :, off[9]:off[10]])
        out = torch.empty_like(o_t)
        for _ in range(args.launches):
            ops.sparvar_ocache_apply(o_t, o_d, o_s, 32, 64, out=out)
    torch.cuda.synchronize()
    print("profile_case done:", args.kernel, args.launches)


if __name__ == "__main__":
    main()

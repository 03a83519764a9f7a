"""Run one GEMM form a few times on seeded inputs: a small, self-contained case
for profilers (e.g. ncu) and quick timing.

    python -m moe_grouped_gemm_tcgen05_b200.profile_case dense --m 4096 --n 7168 --k 16384 --iters 3 [--cta-group 2]
    python -m moe_grouped_gemm_tcgen05_b200.profile_case dense ... --acc-f32     # D = C + A.B^T, fp32, in place
    python -m moe_grouped_gemm_tcgen05_b200.profile_case dense ... --sfb-per-row # one weight scale row per row of B
    python -m moe_grouped_gemm_tcgen05_b200.profile_case masked --groups 32 --max-m 256 --expected-m 96 --n 4096 --k 7168
    python -m moe_grouped_gemm_tcgen05_b200.profile_case contiguous --groups 8 --n 4096 --k 7168

Prints the median device time per call (CUDA events) to stderr.
"""

from __future__ import annotations

import argparse
import statistics
import sys

import numpy as np
import torch

import moe_grouped_gemm_tcgen05_b200 as dg
from moe_grouped_gemm_tcgen05_b200 import workloads as W


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("form", choices=["dense", "masked", "contiguous"])
    ap.add_argument("--m", type=int, default=4096)
    ap.add_argument("--n", type=int, default=7168)
    ap.add_argument("--k", type=int, default=16384)
    ap.add_argument("--groups", type=int, default=32)
    ap.add_argument("--max-m", type=int, default=256)
    ap.add_argument("--expected-m", type=int, default=96)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--block-n", type=int, default=0)
    ap.add_argument("--cta-group", type=int, default=0, help="dense only: 1 = single CTAs, 2 = CTA pairs")
    ap.add_argument("--acc-f32", action="store_true", help="dense only: D = C + A.B^T in fp32, accumulated in place")
    ap.add_argument("--sfb-per-row", action="store_true", help="dense only: B scaled per row (1x128 blocks)")
    args = ap.parse_args(argv)

    torch.cuda.set_device(0)
    dg.init()
    dg.set_block_n(args.block_n)
    dg.set_cta_group(args.cta_group)
    if args.form == "dense":
        p = W.dense_t(args.m, args.n, args.k, seed=1001)
        sfa, sfb = dg.pack_ue8m0(p["sfa_f32"]), dg.pack_ue8m0(p["sfb_f32"])
        d = torch.empty((args.m, args.n), dtype=torch.bfloat16, device="cuda")
        call = lambda: dg.fp8_gemm_nt(p["a"], sfa, p["b"], sfb, d)
        if args.acc_f32:
            d32 = torch.zeros((args.m, args.n), dtype=torch.float32, device="cuda")
            call = lambda: dg.fp8_gemm_nt_acc(p["a"], sfa, p["b"], sfb, d32, c=d32)
        elif args.sfb_per_row:
            sfb_rows = sfb.repeat_interleave(128, dim=0)[: args.n].contiguous()
            call = lambda: dg.fp8_gemm_nt_sfb_gran(p["a"], sfa, p["b"], sfb_rows, d, 1)
    elif args.form == "masked":
        mm = W.masked_m_uniform(W.rng_for(1003), G=args.groups, expected=args.expected_m)
        mm = np.minimum(mm, args.max_m)
        p = W.masked_t(mm, args.max_m, args.n, args.k, seed=1003)
        sfa, sfb = dg.pack_ue8m0(p["sfa_f32"]), dg.pack_ue8m0(p["sfb_f32"])
        d = torch.empty((args.groups, args.max_m, args.n), dtype=torch.bfloat16, device="cuda")
        call = lambda: dg.m_grouped_fp8_gemm_nt_masked(p["a"], sfa, p["b"], sfb, d, p["masked_m"])
    else:
        counts = W.contiguous_counts(G=args.groups)
        p = W.contiguous_t(counts, args.n, args.k, seed=1002)
        sfa, sfb = dg.pack_ue8m0(p["sfa_f32"]), dg.pack_ue8m0(p["sfb_f32"])
        d = torch.empty((p["M_total"], args.n), dtype=torch.bfloat16, device="cuda")
        call = lambda: dg.m_grouped_fp8_gemm_nt_contiguous(p["a"], sfa, p["b"], sfb, d, p["m_indices"])
    torch.cuda.synchronize()
    times = []
    for _ in range(args.iters):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        call()
        e.record()
        torch.cuda.synchronize()
        times.append(s.elapsed_time(e) * 1e3)
    err = dg.device_error()
    print(f"{args.form}: median {statistics.median(times):.1f} us over {args.iters} calls; device status {err}",
          file=sys.stderr)
    return 1 if err else 0


if __name__ == "__main__":
    sys.exit(main())

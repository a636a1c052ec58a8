"""Run a few eager launches of one workload, for profilers.

    python -m dense_fp8_gemm_b200.run_case --workload attn32b --tokens 16 --repeat 3
    python -m dense_fp8_gemm_b200.run_case --workload chain36b --tokens 16 --repeat 2
    python -m dense_fp8_gemm_b200.run_case --shape 51200x5120 --dense-frac 0.25 --tokens 16 --repeat 3
    python -m dense_fp8_gemm_b200.run_case --shape 5120x25600 --scattered --tokens 8192 --repeat 1
    python -m dense_fp8_gemm_b200.run_case --shape 25600x5120 --output-split --tokens 16 --repeat 1

`attn32b` issues, per repeat, the two launches of one decoder layer's attention
projections: q, k and v grouped on one input, then o_proj. `chain36b` issues
the four launches of one layer of the 36B-class stack (q/k/v grouped, o_proj,
gate+up, down), its weights drawn on the GPU as the benchmark draws them. `--shape NxK` runs a
single GEMM: with `--scattered` its dense columns are a seeded random set
(SpenseGPT+, so each call gathers X into the packed column order first); with
`--output-split` its 2:4 rows and its dense rows (a seeded random set) are
packed as two weights (spense_pack_rows) that share one launch. Every launch
goes through the C ABI; inputs are seeded synthetic tensors (see synth.py).
"""
from __future__ import annotations

import argparse
import sys

import numpy as np
import torch

from . import spense, synth, workloads


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default=None, choices=[None, "attn32b", "chain36b"])
    ap.add_argument("--shape", default=None, help="NxK for a single GEMM")
    ap.add_argument("--dense-frac", type=float, default=0.25)
    ap.add_argument("--tokens", type=int, default=16)
    ap.add_argument("--repeat", type=int, default=3)
    ap.add_argument("--scattered", action="store_true", help="SpenseGPT+ dense column set (seeded)")
    ap.add_argument("--output-split", action="store_true", help="2:4 rows and dense rows packed apart")
    args = ap.parse_args(argv)
    dev = torch.device("cuda")
    M = args.tokens

    def packed(wl, i):
        w = workloads.make_weight(wl, i, args.dense_frac)
        return spense.pack(torch.from_numpy(w.W).to(dev), torch.from_numpy(w.s_w).to(dev), Kd=w.Kd,
                           dense_idx=w.dense_idx)

    launches = []
    if args.shape is not None:
        N, K = (int(v) for v in args.shape.lower().split("x"))
        W, s_w = synth.quantize_rows(synth.normal(1, 2, (N, K), 0.02))
        Wd, sd = torch.from_numpy(W).to(dev), torch.from_numpy(s_w).to(dev)
        Kd = workloads.dense_count(K, args.dense_frac)
        rng = np.random.default_rng(5)
        if args.output_split:
            nd = int(round(args.dense_frac * N / 8)) * 8
            dense_rows = np.sort(rng.choice(N, nd, replace=False))
            sparse_rows = np.setdiff1d(np.arange(N), dense_rows)
            grp = [spense.pack(Wd, sd, Kd=0, rows=sparse_rows), spense.pack(Wd, sd, Kd=K, rows=dense_rows)]
        elif args.scattered:
            grp = [spense.pack(Wd, sd, dense_idx=np.sort(rng.choice(K, Kd, replace=False)))]
        else:
            grp = [spense.pack(Wd, sd, Kd=Kd)]
        X, s_x = synth.quantize_rows(synth.normal(1, 3, (M, K), 1.0))
        launches.append((grp, torch.from_numpy(X).to(dev), torch.from_numpy(s_x).to(dev)))
    elif args.workload == "chain36b":
        wl = workloads.CHAIN36B

        def packed_dev(i):
            _, N, K = wl.shapes[i]
            q, sc = synth.device_fp8_rows(wl.seed, workloads.weight_id(i, 0), (N, K), wl.w_std, dev)
            return spense.pack(q, sc, Kd=workloads.dense_count(K, args.dense_frac))

        for grp_idx in ((0, 1, 2), (3,), (4,), (5,)):
            X, s_x = workloads.make_activations(wl, grp_idx[0], M)
            launches.append(([packed_dev(i) for i in grp_idx], torch.from_numpy(X).to(dev),
                             torch.from_numpy(s_x).to(dev)))
    else:
        wl = workloads.ATTN32B
        qkv = [packed(wl, i) for i in range(3)]
        o = [packed(wl, 3)]
        for grp, i in ((qkv, 0), (o, 3)):
            X, s_x = workloads.make_activations(wl, i, M)
            launches.append((grp, torch.from_numpy(X).to(dev), torch.from_numpy(s_x).to(dev)))
    outs = [[torch.empty((M, pw.N), dtype=torch.bfloat16, device=dev) for pw in grp] for grp, _, _ in launches]
    ws = spense.new_workspace(max(spense.grouped_workspace_size(grp, M) for grp, _, _ in launches))
    for _ in range(args.repeat):
        for (grp, X, s_x), Ys in zip(launches, outs):
            spense.gemm_grouped(grp, X, s_x, Ys, ws)
    torch.cuda.synchronize()
    status = spense.workspace_status(ws)
    print(f"ran {args.repeat} x {len(launches)} launches, status {status:#x}")
    return 0 if status == 0 else 1


if __name__ == "__main__":
    sys.exit(main())

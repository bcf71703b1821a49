"""Run one kernel case a fixed number of times, for profiling under ncu.

    python -m binary_weight_gemm_b200.profile_case decode --m 16 --reps 40 [--static]
    python -m binary_weight_gemm_b200.profile_case prefill --reps 6
    python -m binary_weight_gemm_b200.profile_case dbf --m 512 --reps 6
    python -m binary_weight_gemm_b200.profile_case dbf --m 1 --reps 20 --static [--path stack]
    python -m binary_weight_gemm_b200.profile_case stack --m 1 --blocks 8 --reps 5 [--dataflow]
    python -m binary_weight_gemm_b200.profile_case stack --m 1 --chain 128 --reps 5 --path i8

The workloads are the benchmark's: OneBit 4096 x 4096 decode at M tokens, OneBit
prefill X 2048 x 4096 -> 11008, DBF K = N = 4096 with r = 2048, and the layer stack:
one ob_linear_stack over `blocks` 7B-shaped blocks (q, k, v, o 4096 -> 4096; gate, up
4096 -> 11008; down 11008 -> 4096), or with --chain C over C chained 1024 -> 1024
layers (one barrier group each: the per-group cost with little work in it).  Weights
come from the library's own pack and SVID of the seeded W.  Several distinct weight /
input sets rotate so that their total exceeds the 126 MB L2 (DRAM counters then count
real traffic), while the device holds a few hundred MB at most; every stack layer has
its own copy of the weights.  Prints one JSON
line with the mean time per call measured with CUDA events (not meaningful under
a profiler).
"""
from __future__ import annotations

import argparse
import json

import numpy as np
import torch

from . import ops, synth

L2_BYTES = 126 * 2**20


def _sets_for(bytes_per_set: int) -> int:
    return max(2, -(-3 * L2_BYTES // (2 * bytes_per_set)))  # about 1.5x L2 in total


def _bf16(x_bits: np.ndarray, dev) -> torch.Tensor:
    return torch.from_numpy(x_bits.view(np.int16)).to(dev).view(torch.bfloat16)


def main(argv=None) -> None:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("case", choices=("decode", "prefill", "dbf", "stack"))
    ap.add_argument("--m", type=int, default=None, help="tokens (decode default 16, dbf default 512, stack 1)")
    ap.add_argument("--reps", type=int, default=6)
    ap.add_argument("--blocks", type=int, default=8, help="stack: 7B-shaped blocks")
    ap.add_argument("--chain", type=int, default=0, help="stack: chained 1024 -> 1024 layers instead")
    ap.add_argument("--path", choices=("auto", "mma", "i8", "stack"), default="auto",
                    help="stack / decode / dbf: kernel form (AUTO, the bf16 warp MMA, the int8 form; dbf also "
                         "'stack': both products in one persistent launch)")
    ap.add_argument("--dataflow", action="store_true",
                    help="stack: the workspace of ob_linear_stack_workspace_size (tagged outputs, no grid barriers)")
    ap.add_argument("--static", action="store_true",
                    help="decode / dbf: OR OB_FLAG_STATIC_WEIGHTS into the path (as the benchmark's decode calls do)")
    args = ap.parse_args(argv)
    dev = torch.device("cuda", 0)
    torch.cuda.init()
    path = {"auto": ops.OB_PATH_AUTO, "mma": ops.OB_PATH_MMA_DECODE, "i8": ops.OB_PATH_I8,
            "stack": ops.OB_PATH_STACK}[args.path]
    lin_path = path | (ops.OB_FLAG_STATIC_WEIGHTS if args.static else 0)

    if args.case in ("decode", "prefill"):
        M, N, K = (args.m or 16, 4096, 4096) if args.case == "decode" else (args.m or 2048, 11008, 4096)
        seed = 1 if args.case == "decode" else 2
        W = torch.from_numpy(synth.weights(seed, N, K)).to(dev)
        P0 = ops.ob_pack_signs(W)
        a0, b0, _, _, _ = ops.ob_svid_rank1(W)
        del W
        per_set = N * K // 8 + 2 * M * K + 2 * M * N
        n_sets = _sets_for(per_set)
        X0 = _bf16(synth.activations(seed, M, K)[0], dev)
        sets = [(X0.clone(), P0.clone(), a0.clone(), b0.clone(), torch.empty((M, N), dtype=torch.bfloat16, device=dev))
                for _ in range(n_sets)]

        def call(i):
            X, P, a, b, Y = sets[i % n_sets]
            ops.ob_linear(X, P, a, b, out=Y, path=lin_path)
    elif args.case == "stack":
        M = args.m or 1
        if args.chain:
            shapes = [(f"l{i}", 1024, 1024) for i in range(args.chain)]
        else:
            shapes = [(n, K, N) for _ in range(args.blocks)
                      for n, K, N in (("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
                                      ("gate", 4096, 11008), ("up", 4096, 11008), ("down", 11008, 4096))]
        base = {}
        for _, K, N in shapes:
            if (K, N) not in base:
                W = torch.from_numpy(synth.weights(7 + K % 97 + N % 89, N, K)).to(dev)
                a0, b0, _, _, _ = ops.ob_svid_rank1(W)
                base[(K, N)] = (ops.ob_pack_signs(W), a0, b0)
                del W
        X0 = _bf16(synth.activations(7, M, shapes[0][1])[0], dev)
        spec, out, x = [], {}, X0
        for i, (name, K, N) in enumerate(shapes):
            P, a0, b0 = (t.clone() for t in base[(K, N)])
            Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            src = {"q": x, "k": x, "v": x, "o": out.get("q"), "gate": out.get("o"), "up": out.get("o"),
                   "down": out.get("gate")}.get(name, x)
            spec.append((src, P, a0, b0, Y, i > 0 and name not in ("k", "v", "up")))
            out[name] = Y
            if name in ("down",) or args.chain:
                x = Y
        desc = {"layers": len(spec), "blocks": 0 if args.chain else args.blocks}
        nws = ops.ob_linear_stack_workspace_size(spec, M) if args.dataflow else ops.ob_stack_workspace_size()
        ws = torch.zeros(nws, dtype=torch.uint8, device=dev)
        desc["dataflow"] = nws > ops.ob_stack_workspace_size()
        n_sets = 1

        def call(i):
            ops.ob_linear_stack(spec, M, workspace=ws, path=path)
    else:
        M, N, K, r = args.m or 512, 4096, 4096, 2048
        f = synth.dbf_factors(3, N, r, K)
        SAp = ops.ob_pack_signs(torch.from_numpy(f["S_A"].astype(np.float32)).to(dev))
        SBp = ops.ob_pack_signs(torch.from_numpy(f["S_B"].astype(np.float32)).to(dev))
        a, mvec, b = (torch.from_numpy(f[k]).to(dev) for k in ("a", "m", "b"))
        per_set = (r * K + N * r) // 8 + 2 * M * K + 2 * M * N
        n_sets = _sets_for(per_set)
        X0 = _bf16(synth.activations(3, M, K)[0], dev)
        ws = torch.empty(max(ops.dbf_workspace_size(M, r), 16), dtype=torch.uint8, device=dev)
        sets = [(X0.clone(), SBp.clone(), SAp.clone(), torch.empty((M, N), dtype=torch.bfloat16, device=dev))
                for _ in range(n_sets)]

        def call(i):
            X, SBq, SAq, Y = sets[i % n_sets]
            ops.dbf_linear(X, SBq, mvec, SAq, a, b, out=Y, workspace=ws, path=lin_path)

    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.reps):
        call(i)
    e1.record()
    torch.cuda.synchronize()
    assert ops.ob_last_device_error() == 0
    if args.case != "stack":
        desc = {"N": N, "K": K}
    print(json.dumps({"case": args.case, "M": M, **desc, "path": args.path, "static": args.static, "reps": args.reps,
                      "sets": n_sets,
                      "us_per_call": e0.elapsed_time(e1) * 1e3 / args.reps}))


if __name__ == "__main__":
    main()

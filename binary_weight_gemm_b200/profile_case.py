"""Run one kernel case a fixed number of times, for profiling under ncu.

    python -m binary_weight_gemm_b200.profile_case decode --m 16 --reps 40
    python -m binary_weight_gemm_b200.profile_case prefill --reps 6
    python -m binary_weight_gemm_b200.profile_case dbf --m 512 --reps 6

The workloads are the benchmark's: OneBit 4096 x 4096 decode at M tokens, OneBit
prefill X 2048 x 4096 -> 11008, DBF K = N = 4096 with r = 2048.  Weights come from
the library's own pack and SVID of the seeded W.  Several distinct weight / input
sets rotate so that their total exceeds the 126 MB L2 (DRAM counters then count
real traffic), while the device holds a few hundred MB at most.  Prints one JSON
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
    ap.add_argument("case", choices=("decode", "prefill", "dbf"))
    ap.add_argument("--m", type=int, default=None, help="tokens (decode default 16, dbf default 512)")
    ap.add_argument("--reps", type=int, default=6)
    args = ap.parse_args(argv)
    dev = torch.device("cuda", 0)
    torch.cuda.init()

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
            ops.ob_linear(X, P, a, b, out=Y)
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
            ops.dbf_linear(X, SBq, mvec, SAq, a, b, out=Y, workspace=ws)

    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.reps):
        call(i)
    e1.record()
    torch.cuda.synchronize()
    assert ops.ob_last_device_error() == 0
    print(json.dumps({"case": args.case, "M": M, "N": N, "K": K, "reps": args.reps, "sets": n_sets,
                      "us_per_call": e0.elapsed_time(e1) * 1e3 / args.reps}))


if __name__ == "__main__":
    main()

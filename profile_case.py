"""Run one W4A16 GEMM case repeatedly, for a profiler to capture (ncu, CUDA events).

    python profile_case.py decode  [--layer 2] [--m 1] [--iters 12]
    python profile_case.py prefill [--layer 0] [--m 4096] [--iters 6]
    python profile_case.py chain   [--m 1] [--blocks 4] [--iters 3]
    python profile_case.py fp4     [--layer 2] [--m 1] [--iters 12] [--fmt nvfp4]

decode:  one projection of the Llama-7B-shaped stack (layers 0..3 = qkv 4096x12288,
         o 4096x4096, gate_up 4096x22016, down 11008x4096), fp16 activations with s_inv,
         asymmetric INT4 g128; eight weight copies are rotated so the 126 MB L2 cannot
         hold the codes between launches.
prefill: one 8B-shaped layer (0 = up 4096x14336, 1 = down 14336x4096), bf16
         activations already scaled, asymmetric INT4 g128.
chain:   the decode step's projections as one layer sequence (w4a16_gemm_chain): --blocks
         blocks of qkv -> o -> gate_up -> down, each fed from the previous output, one
         weight copy per block (4 blocks = 430 MB of packed weights, above L2).
fp4:     one 7B projection with NVFP4 or MXFP4 weights (w4a16_fp4_gemm), fp16
         activations, eight rotated weight copies.

Inputs are the seeded synthetic workloads of bit_weight_only_w4_b200.workloads, quantised
on the GPU by w4_quantize_pack.  Nothing is checked here (the tests do that); the case only
launches the library's kernels.
"""
import argparse

import numpy as np


def _bits(torch, a, dt):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(dt).cuda()


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("kind", choices=["decode", "prefill", "chain", "fp4"])
    ap.add_argument("--fmt", default="nvfp4", choices=["nvfp4", "mxfp4"])
    ap.add_argument("--blocks", type=int, default=4)
    ap.add_argument("--layer", type=int, default=None)
    ap.add_argument("--m", type=int, default=None)
    ap.add_argument("--iters", type=int, default=None)
    args = ap.parse_args(argv)

    import torch
    import bit_weight_only_w4_b200 as w4
    from bit_weight_only_w4_b200 import workloads

    if args.kind == "decode":
        layer = 2 if args.layer is None else args.layer
        M = 1 if args.m is None else args.m
        iters = 12 if args.iters is None else args.iters
        li = workloads.make_layer(workloads.workload(2), layer, M=M)
        qw, sc, zr = w4.w4_quantize_pack(_bits(torch, li.W.view(np.uint16), torch.float16),
                                         torch.from_numpy(li.s).cuda(), 128)
        copies = [(qw, sc, zr)] + [(qw.clone(), sc.clone(), zr.clone()) for _ in range(7)]
        X = _bits(torch, li.X, torch.float16)
        s_inv = torch.from_numpy(li.s_inv).cuda()
        Y = torch.empty(M, li.N, dtype=torch.float16, device="cuda")
        for i in range(iters):
            q, s, z = copies[i % len(copies)]
            w4.w4a16_gemm(X, q, s, z, 128, s_inv=s_inv, Y=Y)
    elif args.kind == "fp4":
        layer = 2 if args.layer is None else args.layer
        M = 1 if args.m is None else args.m
        iters = 12 if args.iters is None else args.iters
        li = workloads.make_layer(workloads.workload(2), layer, M=M)
        qw, bs, ts = w4.w4_fp4_quantize_pack(_bits(torch, li.W.view(np.uint16), torch.float16), args.fmt)
        copies = [(qw, bs)] + [(qw.clone(), bs.clone()) for _ in range(7)]
        X = _bits(torch, li.X, torch.float16)
        Y = torch.empty(M, li.N, dtype=torch.float16, device="cuda")
        for i in range(iters):
            q, b = copies[i % len(copies)]
            w4.w4a16_fp4_gemm(X, q, b, ts, args.fmt, Y=Y)
    elif args.kind == "chain":
        import os
        import sys
        sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
        import bench
        layer = "all"
        M = 1 if args.m is None else args.m
        iters = 3 if args.iters is None else args.iters
        _, projs, _ = bench.prepare_weights(w4, torch, n_layers=args.blocks)
        layers, _, _ = bench.chain_layers(w4, torch, projs, M, n_blocks=args.blocks)
        for _ in range(iters):
            w4.w4a16_gemm_chain(layers)
    else:
        layer = 0 if args.layer is None else args.layer
        M = 4096 if args.m is None else args.m
        iters = 6 if args.iters is None else args.iters
        li = workloads.make_layer(workloads.workload(4), layer, M=M)
        qw, sc, zr = w4.w4_quantize_pack(_bits(torch, li.W.view(np.uint16), torch.float16),
                                         torch.from_numpy(li.s).cuda(), 128)
        X = _bits(torch, li.X, torch.bfloat16)
        Y = torch.empty(M, li.N, dtype=torch.bfloat16, device="cuda")
        for _ in range(iters):
            w4.w4a16_gemm(X, qw, sc, zr, 128, Y=Y)
    torch.cuda.synchronize()
    w4.w4_check_device_error()
    print(f"ok {args.kind} layer {layer} M={M} x{iters}")


if __name__ == "__main__":
    main()

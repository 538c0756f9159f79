"""Run the fused producer kernels a few times, for profilers.

    python -m fp8_w8a8_dynamic_b200.run_producer --kind silu --M 2048 --reps 2

Builds nothing (the library must be built).  Draws seeded inputs with the
workload recipe: for `rmsnorm`, X [M, 4096] and a gain near 1; for `silu`,
the packed gate_up output [M, 2 x 12288].  Makes `reps` calls of
mfp8_rmsnorm_quantize or mfp8_silu_mul_quantize (codes and scales only) on
the current stream, synchronises, checks the device status word and prints
one line.  A profiler such as Nsight Compute captures the kernels of those
calls by name.
"""
import argparse


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--kind", choices=("rmsnorm", "silu"), default="silu")
    ap.add_argument("--M", type=int, default=2048)
    ap.add_argument("--reps", type=int, default=2)
    ap.add_argument("--seed", type=int, default=1)
    args = ap.parse_args()

    import torch
    from fp8_w8a8_dynamic_b200 import mfp8
    from fp8_w8a8_dynamic_b200 import workloads as W

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    M = args.M
    if args.kind == "rmsnorm":
        x = W.make_x(M, W.HIDDEN, seed=args.seed, kind="rowscale", device=dev)
        g = (1.0 + 0.1 * torch.randn(W.HIDDEN, device=dev)).to(torch.bfloat16)
        for _ in range(args.reps):
            mfp8.rmsnorm_quantize(x, g, 1e-6, want_y=False)
    else:
        gu = W.make_x(M, 2 * W.INTERMEDIATE, seed=args.seed, kind="rowscale", device=dev)
        for _ in range(args.reps):
            mfp8.silu_mul_quantize(gu, want_y=False)
    torch.cuda.synchronize()
    st = mfp8.device_status()
    if st != mfp8.OK:
        raise mfp8.Mfp8Error(st, "run_producer")
    print(f"run_producer {args.kind} M={M} reps={args.reps}: ok")


if __name__ == "__main__":
    main()

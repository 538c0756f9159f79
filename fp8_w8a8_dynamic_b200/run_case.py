"""Run one FP8_DYNAMIC Linear shape a few times, for profilers.

    python -m fp8_w8a8_dynamic_b200.run_case --M 8 --N 12288 --K 4096 --path auto --reps 3

Builds nothing (the library must be built), draws seeded synthetic inputs
with the workload recipe, quantizes the weights once, then makes `reps`
calls of mfp8_linear_ex (or, with --gemm-only, of mfp8_gemm on activations
quantized beforehand) on the current stream, synchronises, checks the
device status word and prints one line.  A profiler such as Nsight Compute
captures the kernels of those calls by name.
"""
import argparse

PATHS = {"auto": 0, "tiled": 1, "splitk": 2, "pair": 3, "fused": 4}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--M", type=int, required=True)
    ap.add_argument("--N", type=int, required=True)
    ap.add_argument("--K", type=int, required=True)
    ap.add_argument("--path", choices=sorted(PATHS), default="auto")
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--gemm-only", action="store_true")
    ap.add_argument("--static-weights", action="store_true")
    ap.add_argument("--seed", type=int, default=1)
    args = ap.parse_args()

    import torch
    from fp8_w8a8_dynamic_b200 import mfp8
    from fp8_w8a8_dynamic_b200 import workloads as W

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    M, N, K = args.M, args.N, args.K
    x = W.make_x(M, K, seed=args.seed, kind="rowscale" if M > 64 else "normal", device=dev)
    W8, sw = mfp8.quantize_weight(W.make_w(N, K, seed=args.seed, device=dev))
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    path = PATHS[args.path]
    flags = mfp8.FLAG_STATIC_WEIGHTS if args.static_weights else 0
    h = torch.cuda.current_stream().cuda_stream
    if args.gemm_only:
        x8, xs = mfp8.quantize_act(x)
        ws = torch.zeros((max(16, mfp8.mfp8_gemm_workspace_bytes(M, N, K)),), dtype=torch.uint8, device=dev)
        torch.cuda.synchronize()
        for _ in range(args.reps):
            st = mfp8.mfp8_gemm(x8.data_ptr(), xs.data_ptr(), M, K, W8.data_ptr(), sw.data_ptr(), N, y.data_ptr(),
                                ws.data_ptr(), ws.numel(), path, h)
            if st != mfp8.OK:
                raise mfp8.Mfp8Error(st, "mfp8_gemm")
    else:
        ws = mfp8.workspace_for(M, N, K, dev)
        torch.cuda.synchronize()
        for _ in range(args.reps):
            st = mfp8.mfp8_linear_ex(x.data_ptr(), M, K, W8.data_ptr(), sw.data_ptr(), N, y.data_ptr(),
                                     ws.data_ptr(), ws.numel(), path, flags, None, None, h)
            if st != mfp8.OK:
                raise mfp8.Mfp8Error(st, "mfp8_linear_ex")
    torch.cuda.synchronize()
    st = mfp8.device_status()
    if st != mfp8.OK:
        raise mfp8.Mfp8Error(st, "device status")
    chosen = path if path != 0 else mfp8.mfp8_choose_path(M, N, K)
    print(f"run_case M={M} N={N} K={K} path={chosen} ({mfp8.KERNEL_OF_PATH[chosen]}) reps={args.reps} ok")


if __name__ == "__main__":
    main()

"""Run the KV-cache kernels on one tensor a few times, for profilers.

    python -m fp8_w8a8_dynamic_b200.run_kv --cache int8 --T 16384 --H 8 --D 128 --reps 2

Builds nothing (the library must be built).  Draws one seeded K or V tensor
[T, H, D] with the workload recipe, then makes `reps` rounds of quantize and
read-back calls on the current stream: for the INT8 cache, mfp8_kv8_quantize
of the history (the positions mfp8_kv8_history_tokens gives for T) and
mfp8_kv8_read of history and bf16 tail; for the FP8 cache, mfp8_kv_quantize
and mfp8_kv_dequantize of all T positions.  Synchronises, checks the device
status word and prints one line.  A profiler such as Nsight Compute captures
the kernels of those calls by name.
"""
import argparse


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--cache", choices=("int8", "fp8"), default="int8")
    ap.add_argument("--T", type=int, default=16384)
    ap.add_argument("--H", type=int, default=8)
    ap.add_argument("--D", type=int, default=128)
    ap.add_argument("--reps", type=int, default=2)
    ap.add_argument("--seed", type=int, default=1)
    args = ap.parse_args()

    import torch
    from fp8_w8a8_dynamic_b200 import mfp8
    from fp8_w8a8_dynamic_b200 import workloads as W

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    T, H, D = args.T, args.H, args.D
    kv = W.make_kv(T, H, D, seed=args.seed, device=dev)
    for _ in range(args.reps):
        if args.cache == "int8":
            tq = mfp8.mfp8_kv8_history_tokens(T)
            codes, scale, zero = mfp8.kv8_quantize(kv[:tq])
            out = mfp8.kv8_read(codes, scale, zero, kv[tq:])
        else:
            codes, scales = mfp8.kv_quantize(kv)
            out = mfp8.kv_dequantize(codes, scales)
    torch.cuda.synchronize()
    st = mfp8.device_status()
    if st != mfp8.OK:
        raise mfp8.Mfp8Error(st, "run_kv")
    print(f"run_kv {args.cache} T={T} H={H} D={D} reps={args.reps}: ok, out {tuple(out.shape)}")


if __name__ == "__main__":
    main()

"""Phase timeline of the one-kernel decode Linear inside the decode step.

    python -m fp8_w8a8_dynamic_b200.phase_trace

Builds an instrumented copy of the library under _build/trace/ (the product
sources are not changed): every CTA of gemm_stream_kernel records
%globaltimer at the boundaries of its phases into a device buffer.  Then it
runs the decode step (q/k/v/o/gate/up/down at M = 1, 4, 8, three weight sets,
one CUDA graph), replays it, reads the records and prints a markdown table:
per Linear, the median over its CTAs of each phase, and the time from the
previous Linear's last record to this one's dependency release.  The
timer's resolution on B200 is about 0.26 us.
"""
import ctypes
import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
OUT = os.path.join(PKG, "_build", "trace")
LIB = os.path.join(OUT, "libmfp8_trace.so")

# Stamp slots (slot 0: kind << 32 | block, 14: the launch's Y pointer, 15: grid << 32 | N).
SLOTS = {1: "start", 2: "setup", 3: "dependency released", 4: "X slice + absmax", 5: "scale known",
         7: "all codes written", 8: "MMAs start", 9: "MMAs issued", 10: "accumulator complete",
         11: "partials received", 12: "producer done"}

TRACE_H = r'''
#pragma once
#include <cstdint>
namespace mfp8 {
constexpr int kTrRecs = 16384, kTrSlots = 16;
__device__ unsigned long long g_tr[kTrRecs][kTrSlots];
__device__ unsigned int g_tr_n;
__device__ __forceinline__ unsigned long long tr_now() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
}
#define TR_DECL __shared__ unsigned int tr_rec_;
#define TR_OPEN(kind, N_, P_) if (threadIdx.x == 0) { \
    unsigned int r_ = atomicAdd(&::mfp8::g_tr_n, 1u); \
    tr_rec_ = r_ < ::mfp8::kTrRecs ? r_ : ::mfp8::kTrRecs - 1; \
    ::mfp8::g_tr[tr_rec_][0] = ((unsigned long long)(kind) << 32) | blockIdx.x; \
    ::mfp8::g_tr[tr_rec_][1] = ::mfp8::tr_now(); \
    ::mfp8::g_tr[tr_rec_][14] = (unsigned long long)(P_); \
    ::mfp8::g_tr[tr_rec_][15] = ((unsigned long long)gridDim.x << 32) | (unsigned)(N_); }
#define TR(slot) { ::mfp8::g_tr[tr_rec_][slot] = ::mfp8::tr_now(); }
'''

# (anchor line in gemm_stream.cuh, stamp to insert, before/after)
STREAM_STAMPS = [
    ("#include \"quant.cuh\"", "#include \"trace.cuh\"", "after"),
    ("    const int CV = TPR > 64 ? TPR : 64;", "    TR_DECL\n    TR_OPEN(1, N, args.Y)\n    __syncthreads();", "after"),
    ("    const uint32_t tmem_base = *tmem_holder;", "    if (threadIdx.x == 0) TR(2)", "after"),
    ("        // X may be the previous kernel's output.\n        grid_dependency_wait();", "        if (t == 0) TR(3)",
     "after"),
    ("        if (real && (j & 31) == 0) atomicMax(amax_loc + m, amax);\n        named_bar_sync(1, kQuantThreads);",
     "        if (t == 0) TR(4)", "after"),
    ("        if (have_scale) {\n            if (real) {", "        if (t == 0) TR(5)", "before"),
    ("        named_bar_sync(1, kQuantThreads);  // sa_sm complete", "        if (t == 0) TR(7)", "after"),
    ("                if (c == 0 && T > 0 && !mbar_wait(tcopy_bar, 0, abort_flag)) { ok = false; break; }",
     "                if (c == 0) TR(8)", "after"),
    ("            if (ok) {\n                mma_commit(tfull_bar);", "            TR(9)", "before"),
    ("        const bool have_acc = have_scale && mbar_wait(tfull_bar, 0, abort_flag);", "        if (t == 0) TR(10)",
     "after"),
    ("            const bool have_partials = mbar_wait(rbar, 0, abort_flag);", "            if (t == 0) TR(11)", "after"),
    ("    tc_fence_before();\n    __syncthreads();\n    if (warp == 1) {\n        tc_fence_after();\n"
     "        tmem_dealloc(tmem_base, tmem_cols(args.g.tm_blocks));", "    if (threadIdx.x == 0) TR(12)", "before"),
]

READERS = r'''
extern "C" __attribute__((visibility("default"))) int mfp8_trace_clear(void) {
    unsigned int z = 0;
    static unsigned long long zeros[64 * 16];
    cudaMemcpyToSymbol(mfp8::g_tr_n, &z, sizeof z);
    for (int i = 0; i < mfp8::kTrRecs; i += 64)
        cudaMemcpyToSymbol(mfp8::g_tr, zeros, sizeof zeros, sizeof(unsigned long long) * 16 * i);
    return cudaDeviceSynchronize();
}
extern "C" __attribute__((visibility("default"))) int mfp8_trace_read(void* out, unsigned int* n) {
    cudaMemcpyFromSymbol(n, mfp8::g_tr_n, sizeof(unsigned int));
    return cudaMemcpyFromSymbol(out, mfp8::g_tr, sizeof(unsigned long long) * 16 * mfp8::kTrRecs);
}
'''


def _insert(text, anchor, stamp, where):
    if anchor not in text:
        raise RuntimeError(f"anchor not found: {anchor[:60]!r}")
    return text.replace(anchor, anchor + "\n" + stamp if where == "after" else stamp + "\n" + anchor, 1)


def build() -> str:
    """The instrumented copy of the library; returns the path of the .so."""
    shutil.rmtree(OUT, ignore_errors=True)
    os.makedirs(os.path.join(OUT, "csrc"))
    os.makedirs(os.path.join(OUT, "include"))
    shutil.copy(os.path.join(ROOT, "include", "mfp8.h"), os.path.join(OUT, "include", "mfp8.h"))
    for f in os.listdir(os.path.join(PKG, "csrc")):
        with open(os.path.join(PKG, "csrc", f)) as fh:
            text = fh.read().replace("../../include/mfp8.h", "../include/mfp8.h")
        if f == "gemm_stream.cuh":
            for anchor, stamp, where in STREAM_STAMPS:
                text = _insert(text, anchor, stamp, where)
        if f == "mfp8.cu":
            text += READERS
        with open(os.path.join(OUT, "csrc", f), "w") as fh:
            fh.write(text)
    with open(os.path.join(OUT, "csrc", "trace.cuh"), "w") as fh:
        fh.write(TRACE_H)
    from . import build as B
    subprocess.run([B.nvcc(), *B.NVCC_FLAGS, os.path.join(OUT, "csrc", "mfp8.cu"), "-o", LIB], check=True)
    return LIB


def _launches(recs):
    """Records grouped by launch (kernel kind, Y pointer, grid and N), in
    order of their first start."""
    groups = {}
    for i, r in enumerate(recs):
        groups.setdefault((int(r[0]) >> 32, int(r[14]), int(r[15])), []).append(i)
    return sorted(groups.values(), key=lambda ix: min(recs[j][1] for j in ix))


def table(recs, names):
    import numpy as np
    recs = np.asarray(recs, dtype=np.int64)
    rows = ["| Linear | previous end -> dependency released | X slice + absmax | cluster exchange and scale | "
            "scale -> all codes | codes -> MMAs issued | MMAs issued -> partials received | launch period |",
            "|---|---|---|---|---|---|---|---|"]
    prev_end = None
    for li, ix in enumerate(_launches(recs)):
        r = recs[ix]
        med = lambda s: float(np.median(r[:, s][r[:, s] > 0]))
        end = max(max(v for v in row[1:13] if v > 0) for row in r)
        cells = [med(3) - prev_end if prev_end else None, med(4) - med(3), med(5) - med(4), med(7) - med(5),
                 med(9) - med(7), med(11) - med(9), end - prev_end if prev_end else None]
        name = names[li] if li < len(names) else f"launch {li}"
        rows.append(f"| {name} | " + " | ".join("—" if c is None else f"{c / 1e3:.2f}" for c in cells) + " |")
        prev_end = end
    return "\n".join(rows)


def main():
    import numpy as np
    import torch
    from . import mfp8
    from . import workloads as W
    build()
    mfp8.LIB_PATH = LIB
    L = mfp8.lib()
    L.mfp8_trace_read.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    Ms = (1, 4, 8)
    calls = []
    for si, M in enumerate(Ms):
        for i, lin in enumerate(W.LAYER_LINEARS):
            x = W.make_x(M, lin.K, seed=1, stream=M * 16 + i, device=dev)
            w8, sw = mfp8.quantize_weight(W.make_w(lin.N, lin.K, seed=1, stream=100 * si + i, device=dev))
            y = torch.empty((M, lin.N), dtype=torch.bfloat16, device=dev)
            ws = mfp8.workspace_for(M, lin.N, lin.K, dev)
            calls.append((x, w8, sw, y, ws, M, lin))
    torch.cuda.synchronize()

    def step(h):
        for x, w8, sw, y, ws, M, lin in calls:
            st = mfp8.mfp8_linear_ex(x.data_ptr(), M, lin.K, w8.data_ptr(), sw.data_ptr(), lin.N, y.data_ptr(),
                                     ws.data_ptr(), ws.numel(), mfp8.PATH_AUTO, mfp8.FLAG_STATIC_WEIGHTS, None, None,
                                     h)
            if st != mfp8.OK:
                raise mfp8.Mfp8Error(st, "mfp8_linear_ex")

    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        step(s.cuda_stream)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step(torch.cuda.current_stream().cuda_stream)
    for _ in range(5):
        g.replay()
    torch.cuda.synchronize()
    L.mfp8_trace_clear()
    g.replay()
    torch.cuda.synchronize()
    buf = np.zeros((16384, 16), dtype=np.uint64)
    n = ctypes.c_uint(0)
    L.mfp8_trace_read(buf.ctypes.data, ctypes.byref(n))
    if mfp8.device_status() != mfp8.OK:
        raise RuntimeError("device status")
    names = [f"{lin.name} M={M}" for (_, _, _, _, _, M, lin) in calls]
    print(table(buf[:n.value].astype(np.int64), names))


if __name__ == "__main__":
    main()

"""Benchmark of the FP8_DYNAMIC Linear on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one decode pass through the seven projections of one language
layer (q, k, v, o, gate, up, down) at M = 1, 4 and 8 tokens: 21 FP8_DYNAMIC
Linears, each quantizing its activations per token and running the FP8 GEMM.
The three M values use three separate weight sets, so a step streams 579 MB
of e4m3 weights (more than the 126 MB L2) and no step hits L2 for weights.

Headline: weight-read GB/s = (N*K + 4N) bytes summed over the step / step
time, from CUDA-graph replays with inputs resident in HBM.  The same line
carries the end-to-end figure through the C ABI with host buffers, the
roofline of the dominant kernel, the prefill (M = 2048) TFLOPS with its
tensor roofline, the one-time weight quantization, and the CPU oracle timed
on a bounded sample as a baseline.

Multi-GPU (torchrun): every rank runs its own independent decode batch
(data parallel, no collective on the data path); value = all ranks' bytes /
the slowest rank's time.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

DECODE_MS = (1, 4, 8)
PREFILL_M = 2048


def load_traffic(kernel, bytes_per_launch):
    """DRAM bytes per launch of `kernel`: the ratio of DRAM traffic to
    algorithmic bytes from the committed one-kernel ncu captures
    (profiles/roofline_traffic.json) times this run's algorithmic bytes per
    launch, or None."""
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "profiles", "roofline_traffic.json")
    try:
        with open(path) as f:
            ratio = json.load(f).get(kernel, {}).get("dram_over_algorithmic")
    except (OSError, ValueError):
        return None
    return None if ratio is None else round(ratio * bytes_per_launch)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# --------------------------------------------------------------- clocks --

class ClockSampler:
    """nvidia-smi clock and throttle-reason samples while the timed region runs."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        mhz, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(mhz)}


# Clock-event reasons that rule a timed region out (power capping is kept
# and reported).
DISQUALIFYING_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


def clocks_disqualify(summary, floor=0.85):
    """True when a timed region's clock record rules its number out: a
    hardware or thermal slowdown was active, or the median SM clock sat below
    `floor` of its maximum with no reason active (a clock lock)."""
    reasons = summary.get("reasons") or []
    if any(r in reasons for r in DISQUALIFYING_REASONS):
        return True
    mhz, mx = summary.get("sm_mhz"), summary.get("sm_max_mhz")
    return bool(mhz and mx and not reasons and mhz < floor * mx)


# ------------------------------------------------------------- workload --

class Layer:
    """One layer's seven projections: BF16 activations per M, FP8 weights."""

    def __init__(self, torch, mfp8, W, seed, weight_sets, Ms, device, x_kind, lins=None):
        self.lins = W.LAYER_LINEARS if lins is None else lins
        self.Ms = Ms
        self.x = {}
        self.y = {}
        self.ws = {}
        # All of a step's activations are views of one buffer, and all of its
        # outputs of another, so that a step's inputs and results move between
        # host and device in one copy each (every view starts 16-byte aligned:
        # M*K and M*N are multiples of 8).
        keys = [(M, i, lin) for M in Ms for i, lin in enumerate(self.lins)]
        self.x_flat = torch.empty((sum(M * lin.K for M, _, lin in keys),), dtype=torch.bfloat16, device=device)
        self.y_flat = torch.empty((sum(M * lin.N for M, _, lin in keys),), dtype=torch.bfloat16, device=device)
        ox = oy = 0
        for M, i, lin in keys:
            self.x[(M, i)] = self.x_flat[ox:ox + M * lin.K].view(M, lin.K)
            self.x[(M, i)].copy_(W.make_x(M, lin.K, seed=seed, stream=M * 16 + i, kind=x_kind, device=device))
            self.y[(M, i)] = self.y_flat[oy:oy + M * lin.N].view(M, lin.N)
            self.ws[(M, i)] = mfp8.workspace_for(M, lin.N, lin.K, device)
            ox += M * lin.K
            oy += M * lin.N
        # weights: one BF16 draw per projection, quantized into `weight_sets` copies
        self.w8 = [[None] * len(self.lins) for _ in range(weight_sets)]
        self.sw = [[None] * len(self.lins) for _ in range(weight_sets)]
        self.wq_time_ms = 0.0
        self.wq_bytes = 0
        for i, lin in enumerate(self.lins):
            for s in range(weight_sets):
                w = W.make_w(lin.N, lin.K, seed=seed, stream=100 * s + i, device=device)
                w8 = torch.empty((lin.N, lin.K), dtype=torch.uint8, device=device)
                sw = torch.empty((lin.N,), dtype=torch.float32, device=device)
                h = torch.cuda.current_stream().cuda_stream
                # once untimed (the first launch of a kernel loads it), then timed
                st = mfp8.mfp8_quantize_weight(w.data_ptr(), lin.N, lin.K, w8.data_ptr(), sw.data_ptr(), h)
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()  # the kernel alone: outputs allocated before
                st = st or mfp8.mfp8_quantize_weight(w.data_ptr(), lin.N, lin.K, w8.data_ptr(), sw.data_ptr(), h)
                e1.record()
                torch.cuda.synchronize()
                if st != mfp8.OK:
                    raise mfp8.Mfp8Error(st, "mfp8_quantize_weight")
                self.w8[s][i], self.sw[s][i] = w8, sw
                self.wq_time_ms += e0.elapsed_time(e1)
                self.wq_bytes += lin.N * lin.K * 3 + lin.N * 4
                del w
        self.weight_sets = weight_sets

    def weight_set(self, mi):
        return mi % self.weight_sets

    def io_buffers(self, torch, k):
        """Activation and output buffers of buffer set k (0: the ones built
        above; k > 0: copies with the same layout, made on first use)."""
        if not hasattr(self, "_io"):
            self._io = [(self.x_flat, self.y_flat)]
        while len(self._io) <= k:
            self._io.append((self.x_flat.clone(), torch.empty_like(self.y_flat)))
        return self._io[k]

    def step(self, mfp8, stream, bufset=0):
        """One C-ABI call per Linear; the argument lists are built once (the
        buffers do not move), so a step costs the host only the calls.
        `bufset` selects the activation/output buffers (see io_buffers)."""
        if getattr(self, "_calls", None) is None:
            self._calls = {}
        if bufset not in self._calls:
            xb, yb = self._io[bufset] if bufset else (self.x_flat, self.y_flat)
            dx = (xb.data_ptr() - self.x_flat.data_ptr())
            dy = (yb.data_ptr() - self.y_flat.data_ptr())
            calls = []
            for mi, M in enumerate(self.Ms):
                s = self.weight_set(mi)
                for i, lin in enumerate(self.lins):
                    ws = self.ws[(M, i)]
                    calls.append((self.x[(M, i)].data_ptr() + dx, M, lin.K, self.w8[s][i].data_ptr(),
                                  self.sw[s][i].data_ptr(), lin.N, self.y[(M, i)].data_ptr() + dy, ws.data_ptr(),
                                  ws.numel(), mfp8.PATH_AUTO, mfp8.FLAG_STATIC_WEIGHTS, None, None))
            self._calls[bufset] = calls
        fn = mfp8.lib().mfp8_linear_ex
        for a in self._calls[bufset]:
            st = fn(*a, stream)
            if st != mfp8.OK:
                raise mfp8.Mfp8Error(st, "mfp8_linear_ex")

    def weight_bytes_per_step(self):
        return sum(lin.N * lin.K + 4 * lin.N for lin in self.lins) * len(self.Ms)

    def flops_per_step(self):
        return sum(2 * M * lin.N * lin.K for M in self.Ms for lin in self.lins)

    def launches_per_step(self, mfp8):
        """Library kernels one step launches: one per Linear on the
        one-kernel decode path, a quantize pass and a GEMM otherwise."""
        return sum(1 if mfp8.mfp8_choose_path(M, lin.N, lin.K) == mfp8.PATH_FUSED else 2
                   for M in self.Ms for lin in self.lins)


def time_graph(torch, fn, steps, warmup, dist_ctx):
    """Capture fn() in a CUDA graph; time `steps` replays after `warmup`."""
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        fn(stream.cuda_stream)  # populate lazy state outside capture
    torch.cuda.current_stream().wait_stream(stream)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn(torch.cuda.current_stream().cuda_stream)
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    if dist_ctx is not None:
        dist_ctx.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    del g
    if dist_ctx is None:
        return ms
    dist_ctx.barrier()
    return dist_ctx.max(ms)


def kernel_times(torch, mfp8, layer, steps, warmup):
    """Average launch duration of the step's GEMM kernel (and of the quantize
    kernel where it is a launch of its own) over the step's Linears.  Each is
    a CUDA graph of that kernel's launches alone, one per Linear with nothing
    between them, timed with CUDA events around `steps` replays on the
    launching stream; the average includes the gaps between graph nodes, so
    it is an upper bound on a launch's own time.  Where every Linear takes
    the one-kernel decode path (quantization on chip), the graph of the
    step's launches is that kernel's graph.  The GEMMs run on codes
    quantized once before the timing (mfp8_gemm); no kernel keeps anything in
    a workspace."""
    keys = [(mi, M, i, lin) for mi, M in enumerate(layer.Ms) for i, lin in enumerate(layer.lins)]
    paths = sorted({mfp8.mfp8_choose_path(M, lin.N, lin.K) for (mi, M, i, lin) in keys})
    n = len(keys)
    out = dict(launches=steps * n, kernel="+".join(mfp8.KERNEL_OF_PATH[p] for p in paths),
               gemm_bytes=sum(lin.N * lin.K + 4 * lin.N + 2 * M * lin.K + 2 * M * lin.N
                              for (mi, M, i, lin) in keys) / n,
               gemm_flops=sum(2 * M * lin.N * lin.K for (mi, M, i, lin) in keys) / n,
               quant_us=None, quant_bytes=None)
    if paths == [mfp8.PATH_FUSED]:
        out["gemm_us"] = time_graph(torch, lambda h: layer.step(mfp8, h), steps, warmup, None) * 1e3 / (steps * n)
        return out

    x8 = {(M, i): mfp8.quantize_act(layer.x[(M, i)]) for (mi, M, i, lin) in keys}
    gws_of = {(M, i): torch.zeros((max(16, mfp8.mfp8_gemm_workspace_bytes(M, lin.N, lin.K)),), dtype=torch.uint8,
                                  device=layer.x[(M, i)].device) for (mi, M, i, lin) in keys}
    torch.cuda.synchronize()

    def gemms(h):
        for (mi, M, i, lin) in keys:
            s = layer.weight_set(mi)
            q8, qs = x8[(M, i)]
            gws = gws_of[(M, i)]
            st = mfp8.mfp8_gemm(q8.data_ptr(), qs.data_ptr(), M, lin.K, layer.w8[s][i].data_ptr(),
                                layer.sw[s][i].data_ptr(), lin.N, layer.y[(M, i)].data_ptr(),
                                gws.data_ptr(), gws.numel(), mfp8.PATH_AUTO, h)
            if st != mfp8.OK:
                raise mfp8.Mfp8Error(st, "mfp8_gemm")

    def quants(h):
        for (mi, M, i, lin) in keys:
            q8, qs = x8[(M, i)]
            st = mfp8.mfp8_quantize_act(layer.x[(M, i)].data_ptr(), M, lin.K, q8.data_ptr(), qs.data_ptr(), h)
            if st != mfp8.OK:
                raise mfp8.Mfp8Error(st, "mfp8_quantize_act")

    out["gemm_us"] = time_graph(torch, gemms, steps, warmup, None) * 1e3 / (steps * n)
    out["quant_us"] = time_graph(torch, quants, steps, warmup, None) * 1e3 / (steps * n)
    out["gemm_bytes"] = sum(lin.N * lin.K + 4 * lin.N + M * lin.K + 4 * M + 2 * M * lin.N
                            for (mi, M, i, lin) in keys) / n
    out["quant_bytes"] = sum(3 * M * lin.K + 4 * M for (mi, M, i, lin) in keys) / n
    return out


def layer_prefill_fused(torch, mfp8, W, device, steps, warmup, dist_ctx):
    """One layer's seven Linears at M = 2048 (seed 2) in the model's
    dataflow, with the activation quantization fused into the producers:
    RMSNorm + quantize for the packed qkv_proj, a
    quantize pass for o (its input comes from attention, outside this
    library), RMSNorm + quantize for the packed gate_up_proj (one GEMM writing
    [gate | up]), and SiLU(gate) * up + quantize on that output for down.  TFLOP/s of the seven GEMMs
    over the whole sequence (producers and quantize included)."""
    M, H, I = 2048, W.HIDDEN, W.INTERMEDIATE
    lins = {l.name: l for l in W.LAYER_LINEARS}
    w = {}
    for i, name in enumerate(("o_proj", "down_proj")):
        l = lins[name]
        w[name] = mfp8.quantize_weight(W.make_w(l.N, l.K, seed=2, stream=3 + 3 * i, device=device))
    # q/k/v as the packed qkv_proj
    wq = torch.cat([W.make_w(lins[n].N, H, seed=2, stream=i, device=device)
                    for i, n in enumerate(("q_proj", "k_proj", "v_proj"))])
    w["qkv_proj"] = mfp8.quantize_weight(wq)
    del wq
    # gate and up as the packed gate_up_proj: one GEMM writes [gate | up]
    wg = torch.cat([W.make_w(I, H, seed=2, stream=4, device=device), W.make_w(I, H, seed=2, stream=5, device=device)])
    w["gate_up_proj"] = mfp8.quantize_weight(wg)
    del wg
    lins = dict(lins, qkv_proj=W.PACKED_LAYER_LINEARS[0], gate_up_proj=W.PACKED_LAYER_LINEARS[2])
    h_attn = W.make_x(M, H, seed=2, stream=1, kind="rowscale", device=device)   # RMSNorm input (residual stream)
    h_mlp = W.make_x(M, H, seed=2, stream=2, kind="rowscale", device=device)
    attn = W.make_x(M, H, seed=2, stream=3, kind="rowscale", device=device)     # attention output, o_proj input
    g1 = (1.0 + 0.1 * torch.randn(H, device=device)).to(torch.bfloat16)
    g2 = (1.0 + 0.1 * torch.randn(H, device=device)).to(torch.bfloat16)
    c_h, s_h = torch.empty((M, H), dtype=torch.uint8, device=device), torch.empty((M,), dtype=torch.float32, device=device)
    c_i, s_i = torch.empty((M, I), dtype=torch.uint8, device=device), torch.empty((M,), dtype=torch.float32, device=device)
    y = {n: torch.empty((M, lins[n].N), dtype=torch.bfloat16, device=device) for n in w}
    gu = y["gate_up_proj"]  # gate | up
    gws = torch.zeros((max(16, max(mfp8.mfp8_gemm_workspace_bytes(M, lins[n].N, lins[n].K) for n in w)),),
                      dtype=torch.uint8, device=device)
    torch.cuda.synchronize()

    def gemm(codes, scales, name, out, h):
        l = lins[name]
        st = mfp8.mfp8_gemm(codes.data_ptr(), scales.data_ptr(), M, l.K, w[name][0].data_ptr(), w[name][1].data_ptr(),
                            l.N, out.data_ptr(), gws.data_ptr(), gws.numel(), mfp8.PATH_AUTO, h)
        if st != mfp8.OK:
            raise mfp8.Mfp8Error(st, "mfp8_gemm")

    def check(st, what):
        if st != mfp8.OK:
            raise mfp8.Mfp8Error(st, what)

    def layer(h):
        check(mfp8.mfp8_rmsnorm_quantize(h_attn.data_ptr(), g1.data_ptr(), 1e-6, M, H, None, c_h.data_ptr(),
                                         s_h.data_ptr(), h), "mfp8_rmsnorm_quantize")
        gemm(c_h, s_h, "qkv_proj", y["qkv_proj"], h)
        check(mfp8.mfp8_quantize_act(attn.data_ptr(), M, H, c_h.data_ptr(), s_h.data_ptr(), h), "mfp8_quantize_act")
        gemm(c_h, s_h, "o_proj", y["o_proj"], h)
        check(mfp8.mfp8_rmsnorm_quantize(h_mlp.data_ptr(), g2.data_ptr(), 1e-6, M, H, None, c_h.data_ptr(),
                                         s_h.data_ptr(), h), "mfp8_rmsnorm_quantize")
        gemm(c_h, s_h, "gate_up_proj", gu, h)
        check(mfp8.mfp8_silu_mul_quantize(gu.data_ptr(), M, I, None, c_i.data_ptr(), s_i.data_ptr(), h),
              "mfp8_silu_mul_quantize")
        gemm(c_i, s_i, "down_proj", y["down_proj"], h)

    n = max(5, steps // 2)
    ms = time_graph(torch, layer, n, warmup, dist_ctx) / n
    flops = sum(2 * M * l.N * l.K for l in W.LAYER_LINEARS)
    assert mfp8.device_status() == mfp8.OK
    return {"workload": "one layer's 7 Linears at M=2048 (seed 2) in the model's dataflow, packed as the README's "
                        "qkv_proj and gate_up_proj: RMSNorm+quantize for each packed projection, a quantize pass for "
                        "o, SiLU(gate)*up+quantize on the gate_up output for down",
            "value": round(flops / (ms * 1e-3) / 1e12 * dist_ctx.world, 1), "unit": "TFLOP/s",
            "ms_per_layer": round(ms, 4), "launches_per_layer": 8}


def q_proj_m16(torch, mfp8, W, device, steps, warmup, dist_ctx, peaks):
    """The single q_proj-shaped Linear at M = 16 (seed 0): 4096 -> 4096,
    16.8 MB of e4m3 weights.  One weight set fits in L2, so the graph cycles
    through 16 copies of it (268 MB, more than twice the 126 MB L2): every
    call reads its weights from HBM.  Weight-read GB/s and the average
    launch time of the one-kernel decode Linear."""
    lin, M, copies = W.LAYER_LINEARS[0], 16, 16
    x = W.make_x(M, lin.K, seed=0, stream=M, device=device)
    w8, sw = mfp8.quantize_weight(W.make_w(lin.N, lin.K, seed=0, stream=lin.N, device=device))
    w8s = [w8] + [w8.clone() for _ in range(copies - 1)]
    y = torch.empty((M, lin.N), dtype=torch.bfloat16, device=device)
    ws = mfp8.workspace_for(M, lin.N, lin.K, device)
    torch.cuda.synchronize()
    calls = [(x.data_ptr(), M, lin.K, c.data_ptr(), sw.data_ptr(), lin.N, y.data_ptr(), ws.data_ptr(), ws.numel(),
              mfp8.PATH_AUTO, mfp8.FLAG_STATIC_WEIGHTS, None, None) for c in w8s]

    def fn(h):
        for a in calls:
            st = mfp8.lib().mfp8_linear_ex(*a, h)
            if st != mfp8.OK:
                raise mfp8.Mfp8Error(st, "mfp8_linear_ex")

    ms = time_graph(torch, fn, steps, warmup, dist_ctx)
    assert mfp8.device_status() == mfp8.OK
    us = ms * 1e3 / (steps * copies)
    wb = lin.N * lin.K + 4 * lin.N
    gbs = wb / (us * 1e-6) / 1e9
    return {"workload": "q_proj 4096->4096 at M=16, X ~N(0,1) + 0.1% x50 outliers, W ~N(0,0.02), seed 0; "
                        f"{copies} rotated weight copies ({copies * wb / 1e6:.0f} MB, > 2x L2)",
            "value": round(gbs * dist_ctx.world, 1), "unit": "GB/s", "avg_launch_us": round(us, 3),
            "kernel": mfp8.KERNEL_OF_PATH[mfp8.mfp8_choose_path(M, lin.N, lin.K)],
            "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4), "all_bytes_per_launch": wb + 2 * M * lin.K + 2 * M * lin.N}


def kv_cache_line(torch, mfp8, W, device, steps, warmup, peaks):
    """The FP8 e4m3 KV cache (the README's SGLang --kv-cache-dtype fp8_e4m3):
    quantize and dequantize K and V of T = 16384 tokens (the long video
    context), 8 KV heads x 128, one scale per (token, head).  Four buffer sets
    (4 x 96 MB, more than L2) are cycled so every call reads from HBM.
    GB/s of algorithmic bytes: quantize 2 + 1 bytes per value + 4 per row,
    dequantize 1 + 2 per value + 4 per row."""
    T, H, D, sets = 16384, 8, 128, 4
    kv = [W.make_x(T * H, D, seed=5, stream=i, kind="rowscale", device=device).view(T, H, D) for i in range(2 * sets)]
    q = [torch.empty((T, H, D), dtype=torch.uint8, device=device) for _ in kv]
    sc = [torch.empty((T, H), dtype=torch.float32, device=device) for _ in kv]
    out = [torch.empty((T, H, D), dtype=torch.bfloat16, device=device) for _ in kv]
    torch.cuda.synchronize()

    def quant(h):
        for a, b, c in zip(kv, q, sc):
            st = mfp8.mfp8_kv_quantize(a.data_ptr(), T, H, D, b.data_ptr(), c.data_ptr(), h)
            if st != mfp8.OK:
                raise mfp8.Mfp8Error(st, "mfp8_kv_quantize")

    def dequant(h):
        for b, c, o in zip(q, sc, out):
            st = mfp8.mfp8_kv_dequantize(b.data_ptr(), c.data_ptr(), T, H, D, o.data_ptr(), h)
            if st != mfp8.OK:
                raise mfp8.Mfp8Error(st, "mfp8_kv_dequantize")

    n = len(kv)
    res = {"workload": "K and V of T=16384 tokens x 8 KV heads x 128 (long video context), one scale per "
                       "(token, head); 4 buffer sets cycled (> L2)"}
    for name, fn, per in (("quantize", quant, 3), ("dequantize", dequant, 3)):
        ms = time_graph(torch, fn, steps, warmup, None)
        us = ms * 1e3 / (steps * n)
        nbytes = T * H * D * per + T * H * 4
        gbs = nbytes / (us * 1e-6) / 1e9
        res[name] = {"GB/s": round(gbs, 1), "avg_launch_us": round(us, 3), "bytes_per_launch": nbytes,
                     "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4)}
    assert mfp8.device_status() == mfp8.OK
    del kv, q, sc, out
    torch.cuda.empty_cache()
    return res


def kv8_cache_line(torch, mfp8, W, device, steps, warmup, peaks):
    """The INT8 KV cache (the README's KV8 section: hqq backend, nbits 8,
    group 64 along the tokens, residual 128): a cache of T = 16384 positions,
    8 KV heads x 128, holds 16256 positions quantized and the latest 128 in
    bf16.  Timed: quantizing the 16256-position history (a prefill filling the
    cache) and reading the whole cache back (dequantize + the bf16 tail).
    Eight tensors (K and V of four layers, 8 x 32 MB, more than L2) and
    eight outputs are cycled.  GB/s of algorithmic bytes: quantize 2 + 1 bytes per value + 8 per
    group and column, read 1 + 2 per history value + 8 per group and column +
    2 + 2 per tail value."""
    T, H, D, n = 16384, 8, 128, 8
    Tq = mfp8.mfp8_kv8_history_tokens(T)
    Tr, C = T - Tq, H * D
    kv = [W.make_kv(T, H, D, seed=8, stream=i, device=device) for i in range(n)]
    q = [torch.empty((Tq, H, D), dtype=torch.uint8, device=device) for _ in kv]
    sc = [torch.empty((Tq // 64, H, D), dtype=torch.float32, device=device) for _ in kv]
    zp = [torch.empty((Tq // 64, H, D), dtype=torch.float32, device=device) for _ in kv]
    out = [torch.empty((T, H, D), dtype=torch.bfloat16, device=device) for _ in range(n)]
    torch.cuda.synchronize()

    def quant(h):
        for a, b, c, z in zip(kv, q, sc, zp):
            st = mfp8.mfp8_kv8_quantize(a.data_ptr(), Tq, H, D, b.data_ptr(), c.data_ptr(), z.data_ptr(), h)
            if st != mfp8.OK:
                raise mfp8.Mfp8Error(st, "mfp8_kv8_quantize")

    def read(h):
        for i, (a, b, c, z) in enumerate(zip(kv, q, sc, zp)):
            st = mfp8.mfp8_kv8_read(b.data_ptr(), c.data_ptr(), z.data_ptr(), Tq, a[Tq:].data_ptr(), Tr, H, D,
                                    out[i].data_ptr(), h)
            if st != mfp8.OK:
                raise mfp8.Mfp8Error(st, "mfp8_kv8_read")

    res = {"workload": f"K and V of a cache of T={T} positions x 8 KV heads x 128 (long video context): "
                       f"{Tq} positions quantized in groups of 64 tokens, the latest {Tr} in bf16; 8 tensors "
                       "cycled (> L2)"}
    fits = (Tq // 64) * C * 8
    for name, fn, nbytes in (("quantize", quant, Tq * C * 3 + fits),
                             ("read", read, Tq * C * 3 + fits + Tr * C * 4)):
        ms = time_graph(torch, fn, steps, warmup, None)
        us = ms * 1e3 / (steps * n)
        gbs = nbytes / (us * 1e-6) / 1e9
        res[name] = {"GB/s": round(gbs, 1), "avg_launch_us": round(us, 3), "bytes_per_launch": nbytes,
                     "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4)}
    assert mfp8.device_status() == mfp8.OK
    del kv, q, sc, zp, out
    torch.cuda.empty_cache()
    return res


def producers_line(torch, mfp8, W, device, steps, warmup, peaks):
    """The activation quantization fused into its producers at the prefill
    size M = 2048: RMSNorm + quantize (hidden 4096; reads the bf16 rows and
    the gain, writes codes and scales only) and SiLU(gate) * up + quantize on
    the packed gate_up output (I = 12288).  Buffer sets are cycled past L2.
    GB/s of algorithmic bytes."""
    M, H, I = 2048, 4096, 12288
    res = {"workload": "prefill M=2048: RMSNorm+quantize (4096) and SiLU(gate)*up+quantize on the packed gate_up "
                       "output (2 x 12288); codes and scales written, no bf16 copy"}
    g = (1.0 + 0.1 * torch.randn(H, device=device)).to(torch.bfloat16)
    xs = [W.make_x(M, H, seed=6, stream=i, kind="rowscale", device=device) for i in range(10)]
    gus = [W.make_x(M, 2 * I, seed=7, stream=i, kind="rowscale", device=device) for i in range(3)]
    cq = torch.empty((M, I), dtype=torch.uint8, device=device)
    cs = torch.empty((M,), dtype=torch.float32, device=device)
    torch.cuda.synchronize()

    def norm(h):
        for x in xs:
            st = mfp8.mfp8_rmsnorm_quantize(x.data_ptr(), g.data_ptr(), 1e-6, M, H, None, cq.data_ptr(),
                                            cs.data_ptr(), h)
            if st != mfp8.OK:
                raise mfp8.Mfp8Error(st, "mfp8_rmsnorm_quantize")

    def silu(h):
        for gu in gus:
            st = mfp8.mfp8_silu_mul_quantize(gu.data_ptr(), M, I, None, cq.data_ptr(), cs.data_ptr(), h)
            if st != mfp8.OK:
                raise mfp8.Mfp8Error(st, "mfp8_silu_mul_quantize")

    for name, fn, n, nbytes in (("rmsnorm_quantize", norm, len(xs), 3 * M * H + 2 * H + 4 * M),
                                ("silu_mul_quantize", silu, len(gus), 5 * M * I + 4 * M)):
        ms = time_graph(torch, fn, steps, warmup, None)
        us = ms * 1e3 / (steps * n)
        gbs = nbytes / (us * 1e-6) / 1e9
        res[name] = {"GB/s": round(gbs, 1), "avg_launch_us": round(us, 3), "bytes_per_launch": nbytes,
                     "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4)}
    assert mfp8.device_status() == mfp8.OK
    del xs, gus
    torch.cuda.empty_cache()
    return res


def fp8_ceiling_tflops(torch, device, n=8192, reps=10):
    """The box's dense e4m3 GEMM ceiling, as a denominator only: cuBLASLt
    through torch._scaled_mm on n x n x n, bf16 out, best of `reps` launches
    timed alone with CUDA events after warm-up."""
    g = torch.Generator(device=device).manual_seed(0)
    a = torch.randn(n, n, device=device, generator=g).to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device=device, generator=g).to(torch.float8_e4m3fn).t()  # column-major operand
    one = torch.ones((), device=device, dtype=torch.float32)
    for _ in range(3):
        torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    best = None
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        e1.record()
        torch.cuda.synchronize()
        t = e0.elapsed_time(e1)
        best = t if best is None else min(best, t)
    del a, b
    torch.cuda.empty_cache()
    return 2.0 * n ** 3 / (best * 1e-3) / 1e12


def stack_sweep(torch, mfp8, W, device, steps, warmup, dist_ctx, Ms=None):
    """The 252-Linear stack (36 self-attention layers x 7 projections, weight
    std jittered per layer, seed 4) swept at M in {1, 16, 128, 1024, 8192}
    (or the M values in `Ms`): one CUDA graph per M runs the 252 Linears in
    order.  One X buffer per (M, K) and one Y buffer per (M, N) are reused
    across layers.  Weight-read GB/s for M <= 128, TFLOP/s (quantize
    included) above."""
    seed = 4
    jitter = W.layer_std_jitter(seed, len(W.SELF_LAYERS))
    weights = []
    for li in range(len(W.SELF_LAYERS)):
        for i, lin in enumerate(W.LAYER_LINEARS):
            w = W.make_w(lin.N, lin.K, seed=seed, stream=100 * li + i, std=0.02 * jitter[li], device=device)
            weights.append((lin, *mfp8.quantize_weight(w)))
            del w
    torch.cuda.synchronize()
    wbytes = sum(lin.N * lin.K + 4 * lin.N for lin, _, _ in weights)
    out = {"workload": "252-Linear stack (36 self-attention layers x 7, ~7 GB of e4m3 weights, per-layer std "
                       "jitter +-20%), seed 4", "weight_bytes": wbytes,
           "rates": "per GPU (under torchrun every rank sweeps the same stack)", "by_M": {}}
    for M in (Ms or W.WORKLOADS[4]["Ms"]):
        xs = {K: W.make_x(M, K, seed=seed, stream=K, device=device) for K in {lin.K for lin, _, _ in weights}}
        ys = {N: torch.empty((M, N), dtype=torch.bfloat16, device=device) for N in {lin.N for lin, _, _ in weights}}
        ws = torch.zeros((max(16, max(mfp8.mfp8_linear_workspace_bytes(M, lin.N, lin.K) for lin, _, _ in weights)),),
                         dtype=torch.uint8, device=device)

        def sweep(h):
            for lin, w8, sw in weights:
                st = mfp8.mfp8_linear_ex(xs[lin.K].data_ptr(), M, lin.K, w8.data_ptr(), sw.data_ptr(), lin.N,
                                         ys[lin.N].data_ptr(), ws.data_ptr(), ws.numel(), mfp8.PATH_AUTO,
                                         mfp8.FLAG_STATIC_WEIGHTS, None, None, h)
                if st != mfp8.OK:
                    raise mfp8.Mfp8Error(st, "mfp8_linear_ex")

        n = max(2, steps // 10) if M >= 1024 else steps
        ms = time_graph(torch, sweep, n, warmup, dist_ctx) / n
        flops = sum(2 * M * lin.N * lin.K for lin, _, _ in weights)
        out["by_M"][str(M)] = {"ms_per_sweep": round(ms, 4),
                               "weight_GB/s": round(wbytes / (ms * 1e-3) / 1e9, 1),
                               "TFLOP/s": round(flops / (ms * 1e-3) / 1e12, 1)}
        del xs, ys, ws
        torch.cuda.empty_cache()
    assert mfp8.device_status() == mfp8.OK
    del weights
    torch.cuda.empty_cache()
    return out


def e2e_time(torch, mfp8, layer, steps, warmup, dist_ctx):
    """Through the C ABI with host buffers.  Every step copies its own
    activations from pinned host memory (one copy: they are one buffer),
    runs the 21 Linears with one C-ABI call each and copies all its outputs
    back to pinned host memory (one copy).  Steps are independent batches,
    so the copies run on their own streams, double-buffered: step i+1's
    activations go up and step i-1's outputs come down while step i
    computes.  The time runs from the first copy to the last output on the
    host."""
    nbuf = 2
    bufs = [layer.io_buffers(torch, k) for k in range(nbuf)]
    host_x = [layer.x_flat.cpu().pin_memory() for _ in range(nbuf)]
    host_y = [torch.empty(layer.y_flat.shape, dtype=layer.y_flat.dtype).pin_memory() for _ in range(nbuf)]
    h2d = host_x[0].numel() * host_x[0].element_size()
    d2h = host_y[0].numel() * host_y[0].element_size()
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    up_done = [ev() for _ in range(nbuf)]
    comp_done = [ev() for _ in range(nbuf)]
    down_done = [ev() for _ in range(nbuf)]
    started = [False] * nbuf

    def upload(i):
        b = i % nbuf
        with torch.cuda.stream(up):
            if started[b]:
                up.wait_event(comp_done[b])    # step i - nbuf has read this buffer
            bufs[b][0].copy_(host_x[b], non_blocking=True)
            up_done[b].record(up)

    def run(n):
        upload(0)
        for i in range(n):
            b = i % nbuf
            if i + 1 < n:
                upload(i + 1)
            comp.wait_event(up_done[b])
            if started[b]:
                comp.wait_event(down_done[b])  # step i - nbuf's outputs are on the host
            layer.step(mfp8, comp.cuda_stream, bufset=b)
            comp_done[b].record(comp)
            started[b] = True
            with torch.cuda.stream(down):
                down.wait_event(comp_done[b])
                host_y[b].copy_(bufs[b][1], non_blocking=True)
                down_done[b].record(down)
        torch.cuda.synchronize()

    run(warmup)
    dist_ctx.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    run(steps)
    ms = (time.perf_counter() - t0) * 1e3
    # Every buffer set computed the same batch: its outputs on the host must
    # equal the graph-timed step's.
    ref = layer.y_flat.cpu().view(torch.int16)
    assert all(torch.equal(hy.view(torch.int16), ref) for hy in host_y), "e2e outputs differ"
    dist_ctx.barrier()
    return dist_ctx.max(ms), h2d, d2h


# ----------------------------------------------------------- CPU oracle --

def oracle_decode_sample(budget_s=12.0):
    """The CPU oracle on decode steps of the same workload (BF16 inputs drawn
    on the CPU with the same recipe), until about `budget_s` seconds:
    per-token quantization of X and the exact contraction, per Linear.
    Weights are quantized once, outside the timing (one-time, offline).
    Returns (weight-read GB/s, threads, sample description)."""
    import numpy as np
    import torch
    import oracle
    from fp8_w8a8_dynamic_b200 import workloads as W

    def bits(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    lins = W.LAYER_LINEARS
    wq = []
    for i, lin in enumerate(lins):
        w8, sw = oracle.quantize_rows(bits(W.make_w(lin.N, lin.K, seed=1, stream=i, device="cpu")))
        wq.append((w8, sw))
    xs = {(M, i): bits(W.make_x(M, lin.K, seed=1, stream=M * 16 + i, device="cpu"))
          for M in DECODE_MS for i, lin in enumerate(lins)}
    done_bytes, elapsed, n_lin = 0, 0.0, 0
    while elapsed < budget_s:
        for M in DECODE_MS:
            for i, lin in enumerate(lins):
                t0 = time.perf_counter()
                x8, sa = oracle.quantize_rows(xs[(M, i)])
                oracle.linear_ref(x8, sa, wq[i][0], wq[i][1], want_abs=False)
                elapsed += time.perf_counter() - t0
                done_bytes += lin.N * lin.K + 4 * lin.N
                n_lin += 1
    return done_bytes / elapsed / 1e9, oracle.num_threads(), \
        f"{n_lin} Linears of the decode step (M in {{1,4,8}}, q/k/v/o/gate/up/down), {elapsed:.1f} s of CPU time"


# ---------------------------------------------------------------- dist --

class DistCtx:
    """One process per GPU: rank bookkeeping, the barrier around the timed
    region and the max over ranks of a timing.  Nothing on the data path
    goes through it; each rank's batch is its own."""

    def __init__(self, torch, backend=None):
        self.torch = torch
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
        self.dev = torch.device("cuda", self.local_rank) if self.backend == "nccl" else torch.device("cpu")
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            kw = {}
            if self.backend == "nccl":
                torch.cuda.set_device(self.local_rank)
                kw["device_id"] = self.dev
            dist.init_process_group(self.backend, timeout=datetime.timedelta(seconds=120), **kw)
            self.dist = dist

    def barrier(self):
        if self.world > 1:
            self.dist.barrier()

    def max(self, v):
        if self.world == 1:
            return v
        t = self.torch.tensor([v], dtype=self.torch.float64, device=self.dev)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.world > 1:
            self.dist.destroy_process_group()


def rank_seed(base, rank):
    """Seed of a rank's independent batch: every rank draws its own inputs."""
    return base + 1000 * rank


def job_throughput(units_per_rank, world, max_ms):
    """Whole-job rate: the units all ranks processed / the slowest rank's
    time (ms), per second."""
    return units_per_rank * world / (max_ms * 1e-3)


def run_reference(args):
    """The reference arm: the CPU oracle, as it stands, on the decode workload."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world > 1 and rank != 0:
        return
    per_step = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    vals = []
    for i in range(args.warmup + args.steps):
        gbs, cores, sample = oracle_decode_sample(budget_s=per_step)
        if i >= args.warmup:
            vals.append(gbs)
    v = statistics.median(vals)
    out = {
        "impl": "reference", "metric": "FP8-dynamic Linear weight-read GB/s (decode, M in {1,4,8})",
        "value": round(v, 4), "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": decode_config(),
        "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out))


def decode_config():
    return {"workload": "decode: q/k/v/o/gate/up/down of one layer (hidden 4096, 32 Q / 8 KV heads, "
                        "MLP 12288) at M in {1,4,8}, X ~N(0,1) + 0.1% x50 outliers, W ~N(0,0.02), seed 1",
            "linears_per_step": 21, "weight_sets": 3, "l2": "inputs larger than L2: 579 MB of distinct e4m3 "
            "weights per step (126 MB L2)", "graph": True}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-packed", action="store_true")
    ap.add_argument("--no-stack", action="store_true")
    ap.add_argument("--stack-m", default=None, help="comma-separated M values for the stack sweep")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
        return

    import torch
    from fp8_w8a8_dynamic_b200 import build as B
    from fp8_w8a8_dynamic_b200 import mfp8
    from fp8_w8a8_dynamic_b200 import workloads as W

    ctx = DistCtx(torch)
    device = torch.device("cuda", ctx.local_rank)
    torch.cuda.set_device(device)
    B.build()
    peaks = load_peaks()

    # ---- decode (headline) ----
    layer = Layer(torch, mfp8, W, seed=rank_seed(1, ctx.rank), weight_sets=3, Ms=DECODE_MS, device=device,
                  x_kind="normal")
    wbytes = layer.weight_bytes_per_step()

    def timed_decode():
        with ClockSampler(ctx.local_rank) as clocks:
            t = time_graph(torch, lambda h: layer.step(mfp8, h), args.steps, args.warmup, ctx)
        return t, clocks.summary()

    ms, clk = timed_decode()
    # A region that saw a slowdown or a clock lock is measured once more.  The
    # decision is the max over ranks, so that every rank takes the same
    # barriers.
    if ctx.max(1.0 if clocks_disqualify(clk) else 0.0) > 0:
        first = clk
        ms, clk = timed_decode()
        clk["remeasured_after"] = {"sm_mhz": first["sm_mhz"], "reasons": first["reasons"]}
    assert mfp8.device_status() == mfp8.OK
    step_ms = ms / args.steps
    value = job_throughput(wbytes * args.steps, ctx.world, ms) / 1e9

    kt = kernel_times(torch, mfp8, layer, steps=max(5, min(args.steps, 20)), warmup=args.warmup)
    gemm_gbs = kt["gemm_bytes"] / (kt["gemm_us"] * 1e-6) / 1e9
    if kt["quant_us"] is None:
        quant = "fused into " + kt["kernel"]
    else:
        quant = {"GB/s": round(kt["quant_bytes"] / (kt["quant_us"] * 1e-6) / 1e9, 1),
                 "avg_launch_us": round(kt["quant_us"], 3)}
    launches = layer.launches_per_step(mfp8) * args.steps

    # The same step with q/k/v and gate/up packed (4 launches per M): the
    # same weights, outputs and arithmetic, fewer dependent launches.
    packed = None
    if not args.no_packed:
        pk_layer = Layer(torch, mfp8, W, seed=rank_seed(1, ctx.rank), weight_sets=3, Ms=DECODE_MS, device=device,
                         x_kind="normal", lins=W.PACKED_LAYER_LINEARS)
        assert pk_layer.weight_bytes_per_step() == wbytes
        pms = time_graph(torch, lambda h: pk_layer.step(mfp8, h), args.steps, args.warmup, ctx)
        assert mfp8.device_status() == mfp8.OK
        packed = {"workload": "the same decode step with q/k/v packed into qkv_proj (N=6144) and gate/up into "
                              "gate_up_proj (N=24576): 12 launches per step",
                  "value": round(job_throughput(wbytes * args.steps, ctx.world, pms) / 1e9, 1), "unit": "GB/s",
                  "ms_per_step": round(pms / args.steps, 5),
                  "frac_of_hbm": round(wbytes * args.steps / (pms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                  "launches_per_step": pk_layer.launches_per_step(mfp8)}
        del pk_layer
        torch.cuda.empty_cache()

    e2e_steps = max(10, args.steps // 2)
    e2e_ms, h2d, d2h = e2e_time(torch, mfp8, layer, e2e_steps, 3, ctx)
    e2e_val = job_throughput(wbytes * e2e_steps, ctx.world, e2e_ms) / 1e9
    wq = {"GB/s": round(layer.wq_bytes / (layer.wq_time_ms * 1e-3) / 1e9, 1),
          "bytes": layer.wq_bytes, "ms": round(layer.wq_time_ms, 3),
          "frac_of_hbm": round(layer.wq_bytes / (layer.wq_time_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}
    del layer
    torch.cuda.empty_cache()

    # ---- prefill M = 2048 (the TFLOPS half of the metric) ----
    prefill = None
    if not args.no_prefill:
        pl = Layer(torch, mfp8, W, seed=rank_seed(2, ctx.rank), weight_sets=1, Ms=(PREFILL_M,), device=device,
                   x_kind="rowscale")
        psteps = max(5, args.steps // 2)
        pms = time_graph(torch, lambda h: pl.step(mfp8, h), psteps, args.warmup, ctx)
        tflops = job_throughput(pl.flops_per_step() * psteps, ctx.world, pms) / 1e12
        pk = kernel_times(torch, mfp8, pl, steps=5, warmup=args.warmup)
        g_tf = pk["gemm_flops"] / (pk["gemm_us"] * 1e-6) / 1e12
        fp8_peak = 2.0 * peaks["bf16_tflops"]
        fp8_ceiling = fp8_ceiling_tflops(torch, device)
        prefill = {"metric": "FP8-dynamic Linear TFLOPS (M=2048, 7 Linears, quantize included)",
                   "value": round(tflops, 1), "unit": "TFLOP/s", "ms_per_step": round(pms / psteps, 4),
                   "frac_of_fp8_peak": round(tflops / ctx.world / fp8_peak, 4),
                   "fp8_ceiling": {"value": round(fp8_ceiling, 1), "unit": "TFLOP/s",
                                   "how": "cuBLASLt e4m3 8192^3 via torch._scaled_mm, bf16 out, best of 10, "
                                          "timed alone in this run (a denominator only)",
                                   "frac_end_to_end": round(tflops / ctx.world / fp8_ceiling, 4),
                                   "frac_gemms": round(g_tf / fp8_ceiling, 4)},
                   "roofline": {"bound": "tensor", "achieved": round(g_tf, 1), "peak": round(fp8_peak, 1),
                                "unit": "TFLOP/s", "frac": round(g_tf / fp8_peak, 4),
                                # DRAM bytes per launch of the pair kernel, which runs 5 of
                                # the 7 Linears and 96% of the FLOPs
                                "traffic": load_traffic("gemm_pair_kernel", pk["gemm_bytes"])
                                if "gemm_pair_kernel" in pk["kernel"] else None,
                                "kernel": pk["kernel"], "avg_launch_us": round(pk["gemm_us"], 3),
                                "peak_source": f"{peaks['source']} bf16 x 2 (fp8/bf16 nominal ratio)"}}
        del pl
        torch.cuda.empty_cache()

    fused_layer = None
    if not args.no_prefill:
        fused_layer = layer_prefill_fused(torch, mfp8, W, device, args.steps, args.warmup, ctx)
        fused_layer["frac_of_fp8_ceiling"] = round(fused_layer["value"] / ctx.world / prefill["fp8_ceiling"]["value"], 4)
        torch.cuda.empty_cache()

    # Long video-context prefill: gate/up/down at M = 16384 (seed 3).
    video = None
    if not args.no_prefill:
        vl = Layer(torch, mfp8, W, seed=rank_seed(3, ctx.rank), weight_sets=1, Ms=(16384,), device=device,
                   x_kind="rowscale", lins=W.MLP_LINEARS)
        vsteps = max(3, args.steps // 10)
        vms = time_graph(torch, lambda h: vl.step(mfp8, h), vsteps, args.warmup, ctx)
        assert mfp8.device_status() == mfp8.OK
        video = {"workload": "long video-context prefill: gate/up 4096->12288 and down 12288->4096 at M=16384, "
                             "X as the prefill workload, seed 3",
                 "value": round(job_throughput(vl.flops_per_step() * vsteps, ctx.world, vms) / 1e12, 1),
                 "unit": "TFLOP/s", "ms_per_step": round(vms / vsteps, 4),
                 "frac_of_fp8_peak": round(vl.flops_per_step() * vsteps / (vms * 1e-3) / 1e12
                                           / (2.0 * peaks["bf16_tflops"]), 4)}
        del vl
        torch.cuda.empty_cache()

    # The single q_proj Linear at M = 16 (seed 0), weights rotated past L2.
    config0 = q_proj_m16(torch, mfp8, W, device, max(5, args.steps), args.warmup, ctx, peaks)
    torch.cuda.empty_cache()
    kv_cache = kv_cache_line(torch, mfp8, W, device, max(5, min(args.steps, 20)), args.warmup, peaks)
    kv8_cache = kv8_cache_line(torch, mfp8, W, device, max(5, min(args.steps, 20)), args.warmup, peaks)
    producers = producers_line(torch, mfp8, W, device, max(5, min(args.steps, 20)), args.warmup, peaks)

    stack = None
    if not args.no_stack:
        stack_ms = tuple(int(v) for v in args.stack_m.split(",")) if args.stack_m else None
        stack = stack_sweep(torch, mfp8, W, device, max(3, min(args.steps, 10)), args.warmup, ctx, stack_ms)

    cpu = None
    if ctx.rank == 0 and ctx.world == 1 and not args.no_cpu_baseline:
        gbs, cores, sample = oracle_decode_sample(budget_s=12.0)
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample}

    out = {
        "metric": "FP8-dynamic Linear weight-read GB/s (decode, M in {1,4,8})",
        "value": round(value, 1), "unit": "GB/s", "n_gpus": ctx.world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(step_ms, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 x e4m3 -> f32 -> bf16",
        "data": "synthetic", "config": decode_config(),
        "frac_of_hbm": round(value / ctx.world / peaks["hbm_gbs"], 4),
        "roofline": {"bound": "hbm", "achieved": round(gemm_gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(gemm_gbs / peaks["hbm_gbs"], 4), "traffic": load_traffic(kt["kernel"], kt["gemm_bytes"]),
                     "kernel": kt["kernel"], "launches_timed": kt["launches"],
                     "avg_launch_us": round(kt["gemm_us"], 3),
                     "bytes_per_launch": round(kt["gemm_bytes"]),
                     "peak_source": peaks["source"]},
        "quantize_act": quant,
        "weight_quant": wq,
        "packed": packed,
        "e2e": {"value": round(e2e_val, 1), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps, "copies": "double-buffered on copy streams (step i+1 up, step i-1 down, "
                                              "during step i); host wall clock"},
        "gpu_launches": launches,
        "clocks": clk,
        "q_proj_m16": config0,
        "kv_cache_fp8": kv_cache,
        "kv_cache_int8": kv8_cache,
        "fused_producers": producers,
        "prefill": prefill,
        "layer_prefill_fused_producers": fused_layer,
        "long_video": video,
        "stack": stack,
        "cpu_baseline": cpu,
    }
    if ctx.rank == 0:
        print(json.dumps(out))
    ctx.close()



if __name__ == "__main__":
    main()

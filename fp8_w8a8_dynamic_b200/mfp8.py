"""Python binding of the C ABI in include/mfp8.h.

The ``mfp8_*`` functions here have the C names and arguments (integer device
pointers, sizes, a cudaStream_t as an integer) and only marshal arguments.
The torch helpers below them allocate outputs with torch and pass pointers;
every step of the computation runs in the CUDA kernels of libmfp8.so.  There
is no CPU fallback: without the built library every call raises.
"""
import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmfp8.so")

OK = 0
ERR_INVALID_ARG = 1
ERR_MISALIGNED = 2
ERR_UNSUPPORTED_SHAPE = 3
ERR_WORKSPACE = 4
ERR_CUDA = 5
ERR_TIMEOUT = 6
ERR_DEVICE = 7

PATH_AUTO = 0
PATH_TILED = 1
PATH_SPLITK = 2
PATH_PAIR = 3
PATH_FUSED = 4

FLAG_STATIC_WEIGHTS = 1


class Mfp8Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {mfp8_status_string(status)} (status {status})")


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing "
                               "(python -m fp8_w8a8_dynamic_b200.build)")
        L = ctypes.CDLL(LIB_PATH)
        P, i64, sz, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
        sig = {
            "mfp8_quantize_weight": (i32, [P, i64, i64, P, P, P]),
            "mfp8_quantize_act": (i32, [P, i64, i64, P, P, P]),
            "mfp8_linear_workspace_bytes": (sz, [i64, i64, i64]),
            "mfp8_linear": (i32, [P, i64, i64, P, P, i64, P, P, sz, P]),
            "mfp8_linear_ex": (i32, [P, i64, i64, P, P, i64, P, P, sz, i32, i32, P, P, P]),
            "mfp8_linear_noalloc": (i32, [P, i64, i64, P, P, i64, P, P]),
            "mfp8_choose_path": (i32, [i64, i64, i64]),
            "mfp8_gemm_workspace_bytes": (sz, [i64, i64, i64]),
            "mfp8_gemm": (i32, [P, P, i64, i64, P, P, i64, P, P, sz, i32, P]),
            "mfp8_rmsnorm_quantize": (i32, [P, P, ctypes.c_float, i64, i64, P, P, P, P]),
            "mfp8_silu_mul_quantize": (i32, [P, i64, i64, P, P, P, P]),
            "mfp8_kv_quantize": (i32, [P, i64, i64, i64, P, P, P]),
            "mfp8_kv_dequantize": (i32, [P, P, i64, i64, i64, P, P]),
            "mfp8_kv8_quantize": (i32, [P, i64, i64, i64, P, P, P, P]),
            "mfp8_kv8_read": (i32, [P, P, P, i64, P, i64, i64, i64, P, P]),
            "mfp8_kv8_history_tokens": (i64, [i64]),
            "mfp8_debug_kv8_code_check": (i32, [P, i64, ctypes.c_uint32, P]),
            "mfp8_e4m3_encode_f32": (i32, [P, i64, P, P]),
            "mfp8_debug_quantize_check": (i32, [P, P]),
            "mfp8_debug_bounded_wait": (i32, [i64, P]),
            "mfp8_get_device_status": (i32, [P]),
            "mfp8_status_string": (ctypes.c_char_p, [i32]),
            "mfp8_version": (i32, []),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


# ---------------------------------------------------------------- C names --

def mfp8_quantize_weight(W_bf16, N, K, W_fp8, w_scale, stream=0):
    return lib().mfp8_quantize_weight(W_bf16, N, K, W_fp8, w_scale, stream)


def mfp8_quantize_act(X_bf16, M, K, X_fp8, x_scale, stream=0):
    return lib().mfp8_quantize_act(X_bf16, M, K, X_fp8, x_scale, stream)


def mfp8_linear_workspace_bytes(M, N, K):
    return lib().mfp8_linear_workspace_bytes(M, N, K)


def mfp8_linear(X_bf16, M, K, W_fp8, w_scale, N, Y_bf16, workspace, workspace_bytes, stream=0):
    return lib().mfp8_linear(X_bf16, M, K, W_fp8, w_scale, N, Y_bf16, workspace, workspace_bytes, stream)


def mfp8_linear_ex(X_bf16, M, K, W_fp8, w_scale, N, Y_bf16, workspace, workspace_bytes, path, flags,
                   X_fp8_out, x_scale_out, stream=0):
    return lib().mfp8_linear_ex(X_bf16, M, K, W_fp8, w_scale, N, Y_bf16, workspace, workspace_bytes,
                                path, flags, X_fp8_out, x_scale_out, stream)


def mfp8_linear_noalloc(X_bf16, M, K, W_fp8, w_scale, N, Y_bf16, stream=0):
    return lib().mfp8_linear_noalloc(X_bf16, M, K, W_fp8, w_scale, N, Y_bf16, stream)


STATIC_WORKSPACE_BYTES = 16 << 20  # MFP8_STATIC_WORKSPACE_BYTES


def mfp8_choose_path(M, N, K):
    return lib().mfp8_choose_path(M, N, K)


KERNEL_OF_PATH = {PATH_TILED: "gemm_tiled_kernel", PATH_SPLITK: "gemm_cluster_kernel",
                  PATH_PAIR: "gemm_pair_kernel", PATH_FUSED: "gemm_stream_kernel"}


def mfp8_gemm_workspace_bytes(M, N, K):
    return lib().mfp8_gemm_workspace_bytes(M, N, K)


def mfp8_gemm(X_fp8, x_scale, M, K, W_fp8, w_scale, N, Y_bf16, workspace, workspace_bytes, path=PATH_AUTO,
              stream=0):
    return lib().mfp8_gemm(X_fp8, x_scale, M, K, W_fp8, w_scale, N, Y_bf16, workspace, workspace_bytes, path,
                           stream)


def mfp8_rmsnorm_quantize(X_bf16, gamma_bf16, eps, M, K, Y_bf16, X_fp8, x_scale, stream=0):
    return lib().mfp8_rmsnorm_quantize(X_bf16, gamma_bf16, eps, M, K, Y_bf16, X_fp8, x_scale, stream)


def mfp8_silu_mul_quantize(GU_bf16, M, I, Y_bf16, X_fp8, x_scale, stream=0):
    return lib().mfp8_silu_mul_quantize(GU_bf16, M, I, Y_bf16, X_fp8, x_scale, stream)


def mfp8_kv_quantize(KV_bf16, T, H, D, KV_fp8, kv_scale, stream=0):
    return lib().mfp8_kv_quantize(KV_bf16, T, H, D, KV_fp8, kv_scale, stream)


def mfp8_kv_dequantize(KV_fp8, kv_scale, T, H, D, KV_bf16, stream=0):
    return lib().mfp8_kv_dequantize(KV_fp8, kv_scale, T, H, D, KV_bf16, stream)


def mfp8_kv8_quantize(KV_bf16, T, H, D, KV_u8, kv_scale, kv_zero, stream=0):
    return lib().mfp8_kv8_quantize(KV_bf16, T, H, D, KV_u8, kv_scale, kv_zero, stream)


def mfp8_kv8_read(KV_u8, kv_scale, kv_zero, Tq, tail_bf16, Tr, H, D, out_bf16, stream=0):
    return lib().mfp8_kv8_read(KV_u8, kv_scale, kv_zero, Tq, tail_bf16, Tr, H, D, out_bf16, stream)


def mfp8_kv8_history_tokens(T):
    return lib().mfp8_kv8_history_tokens(T)


def mfp8_debug_kv8_code_check(out, n_scale_pairs, seed, stream=0):
    return lib().mfp8_debug_kv8_code_check(out, n_scale_pairs, seed, stream)


def mfp8_e4m3_encode_f32(inp, n, out, stream=0):
    return lib().mfp8_e4m3_encode_f32(inp, n, out, stream)


def mfp8_debug_quantize_check(out, stream=0):
    return lib().mfp8_debug_quantize_check(out, stream)


def mfp8_debug_bounded_wait(timeout_us, stream=0):
    return lib().mfp8_debug_bounded_wait(timeout_us, stream)


def mfp8_get_device_status(stream=0):
    return lib().mfp8_get_device_status(stream)


def mfp8_status_string(status):
    return lib().mfp8_status_string(int(status)).decode()


def mfp8_version():
    return lib().mfp8_version()


# ---------------------------------------------------------- torch helpers --

def _check(status, where):
    if status != OK:
        raise Mfp8Error(status, where)


def _stream_handle(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _ptr(t):
    return t.data_ptr() if t is not None else None


def quantize_weight(W, stream=None):
    """W: bf16 [N, K] CUDA tensor -> (W_fp8 uint8 [N, K], w_scale fp32 [N])."""
    import torch
    N, K = W.shape
    W8 = torch.empty((N, K), dtype=torch.uint8, device=W.device)
    sw = torch.empty((N,), dtype=torch.float32, device=W.device)
    _check(mfp8_quantize_weight(_ptr(W), N, K, _ptr(W8), _ptr(sw), _stream_handle(stream)),
           "mfp8_quantize_weight")
    return W8, sw


def quantize_act(X, stream=None):
    """X: bf16 [M, K] CUDA tensor -> (X_fp8 uint8 [M, K], x_scale fp32 [M])."""
    import torch
    M, K = X.shape
    X8 = torch.empty((M, K), dtype=torch.uint8, device=X.device)
    sa = torch.empty((M,), dtype=torch.float32, device=X.device)
    _check(mfp8_quantize_act(_ptr(X), M, K, _ptr(X8), _ptr(sa), _stream_handle(stream)),
           "mfp8_quantize_act")
    return X8, sa


def workspace_for(M, N, K, device):
    """A workspace for mfp8_linear at these sizes: room for the activation
    codes and scales of the quantize pass (none below 17 tokens, where one
    kernel quantizes on chip).  The kernels need no particular contents; it
    is zero-filled only so that a fresh buffer is deterministic."""
    import torch
    nbytes = mfp8_linear_workspace_bytes(M, N, K)
    return torch.zeros((max(nbytes, 16),), dtype=torch.uint8, device=device)


def linear(X, W8, w_scale, out=None, workspace=None, path=PATH_AUTO, x8_out=None, xs_out=None,
           flags=0, stream=None):
    """Y = FP8_DYNAMIC Linear(X) with pre-quantized weights.  X bf16 [M, K]."""
    import torch
    M, K = X.shape
    N = W8.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    if workspace is None:
        workspace = workspace_for(M, N, K, X.device)
    ws_bytes = workspace.numel() if workspace is not None else 0
    _check(mfp8_linear_ex(_ptr(X), M, K, _ptr(W8), _ptr(w_scale), N, _ptr(out), _ptr(workspace),
                          ws_bytes, path, flags, _ptr(x8_out), _ptr(xs_out), _stream_handle(stream)),
           "mfp8_linear_ex")
    return out


def gemm(X8, x_scale, W8, w_scale, out=None, path=PATH_AUTO, workspace=None, stream=None):
    """The contraction alone on pre-quantized activations."""
    import torch
    M, K = X8.shape
    N = W8.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=X8.device)
    if workspace is None:
        workspace = torch.zeros((max(mfp8_gemm_workspace_bytes(M, N, K), 16),), dtype=torch.uint8,
                                device=X8.device)
    _check(mfp8_gemm(_ptr(X8), _ptr(x_scale), M, K, _ptr(W8), _ptr(w_scale), N, _ptr(out), _ptr(workspace),
                     workspace.numel(), path, _stream_handle(stream)), "mfp8_gemm")
    return out


def rmsnorm_quantize(X, gamma, eps, want_y=True, stream=None):
    """X bf16 [M, K], gamma bf16 [K] -> (y bf16 [M, K] or None, codes uint8 [M, K], scales fp32 [M])."""
    import torch
    M, K = X.shape
    y = torch.empty((M, K), dtype=torch.bfloat16, device=X.device) if want_y else None
    codes = torch.empty((M, K), dtype=torch.uint8, device=X.device)
    scales = torch.empty((M,), dtype=torch.float32, device=X.device)
    _check(mfp8_rmsnorm_quantize(_ptr(X), _ptr(gamma), float(eps), M, K, _ptr(y), _ptr(codes), _ptr(scales),
                                 _stream_handle(stream)), "mfp8_rmsnorm_quantize")
    return y, codes, scales


def silu_mul_quantize(GU, want_y=True, stream=None):
    """GU bf16 [M, 2I] (gate | up) -> (y bf16 [M, I] or None, codes uint8 [M, I], scales fp32 [M])."""
    import torch
    M, I2 = GU.shape
    I = I2 // 2
    y = torch.empty((M, I), dtype=torch.bfloat16, device=GU.device) if want_y else None
    codes = torch.empty((M, I), dtype=torch.uint8, device=GU.device)
    scales = torch.empty((M,), dtype=torch.float32, device=GU.device)
    _check(mfp8_silu_mul_quantize(_ptr(GU), M, I, _ptr(y), _ptr(codes), _ptr(scales), _stream_handle(stream)),
           "mfp8_silu_mul_quantize")
    return y, codes, scales


def kv_quantize(KV, stream=None):
    """KV: bf16 [T, H, D] CUDA tensor -> (codes uint8 [T, H, D], scales fp32 [T, H])."""
    import torch
    T, H, D = KV.shape
    codes = torch.empty((T, H, D), dtype=torch.uint8, device=KV.device)
    scales = torch.empty((T, H), dtype=torch.float32, device=KV.device)
    _check(mfp8_kv_quantize(_ptr(KV), T, H, D, _ptr(codes), _ptr(scales), _stream_handle(stream)),
           "mfp8_kv_quantize")
    return codes, scales


def kv_dequantize(codes, scales, stream=None):
    """codes uint8 [T, H, D], scales fp32 [T, H] -> bf16 [T, H, D]."""
    import torch
    T, H, D = codes.shape
    out = torch.empty((T, H, D), dtype=torch.bfloat16, device=codes.device)
    _check(mfp8_kv_dequantize(_ptr(codes), _ptr(scales), T, H, D, _ptr(out), _stream_handle(stream)),
           "mfp8_kv_dequantize")
    return out


def kv8_quantize(KV, stream=None):
    """KV: bf16 [T, H, D] CUDA tensor, T % 64 == 0 -> (codes uint8 [T, H, D],
    scale fp32 [T/64, H, D], zero fp32 [T/64, H, D])."""
    import torch
    T, H, D = KV.shape
    codes = torch.empty((T, H, D), dtype=torch.uint8, device=KV.device)
    scale = torch.empty((T // 64, H, D), dtype=torch.float32, device=KV.device)
    zero = torch.empty((T // 64, H, D), dtype=torch.float32, device=KV.device)
    _check(mfp8_kv8_quantize(_ptr(KV), T, H, D, _ptr(codes), _ptr(scale), _ptr(zero), _stream_handle(stream)),
           "mfp8_kv8_quantize")
    return codes, scale, zero


def kv8_read(codes, scale, zero, tail, out=None, stream=None):
    """History (codes [Tq, H, D], scale and zero [Tq/64, H, D]) and bf16 tail
    [Tr, H, D] -> bf16 [Tq + Tr, H, D]: the history dequantized, then the
    tail."""
    import torch
    Tq, H, D = codes.shape
    Tr = tail.shape[0]
    if out is None:
        out = torch.empty((Tq + Tr, H, D), dtype=torch.bfloat16, device=codes.device)
    _check(mfp8_kv8_read(_ptr(codes), _ptr(scale), _ptr(zero), Tq, _ptr(tail), Tr, H, D, _ptr(out),
                         _stream_handle(stream)), "mfp8_kv8_read")
    return out


class Kv8Cache:
    """One K or V tensor of a layer held as the INT8 cache: a history of
    whole 64-token groups (codes, scale, zero) and the bf16 tail of the
    latest positions.  Buffers are allocated once for `capacity` positions.
    ``append`` stages the old tail and the new positions in one bf16 buffer,
    quantizes the positions that mfp8_kv8_history_tokens moves into the
    history (mfp8_kv8_quantize, written in place after the existing groups)
    and keeps the rest as the tail; ``read`` returns every position as bf16
    (mfp8_kv8_read).  Work is queued on the current torch stream."""

    def __init__(self, capacity, H, D, device):
        import torch
        groups = (capacity + 63) // 64
        self.capacity, self.H, self.D = capacity, H, D
        self.codes = torch.empty((groups * 64, H, D), dtype=torch.uint8, device=device)
        self.scale = torch.empty((groups, H, D), dtype=torch.float32, device=device)
        self.zero = torch.empty((groups, H, D), dtype=torch.float32, device=device)
        self.tail = torch.empty((0, H, D), dtype=torch.bfloat16, device=device)
        self.T = 0

    @property
    def Tq(self):
        return mfp8_kv8_history_tokens(self.T)

    def append(self, kv):
        import torch
        n = kv.shape[0]
        if kv.shape[1:] != (self.H, self.D) or kv.dtype != torch.bfloat16:
            raise ValueError("Kv8Cache.append: expected bf16 [n, H, D]")
        if self.T + n > self.capacity:
            raise ValueError("Kv8Cache.append: capacity exceeded")
        tq, tq2 = self.Tq, mfp8_kv8_history_tokens(self.T + n)
        staged = torch.cat([self.tail, kv]) if self.tail.shape[0] else kv.contiguous()
        f = tq2 - tq
        if f:
            g = tq // 64
            _check(mfp8_kv8_quantize(_ptr(staged), f, self.H, self.D, _ptr(self.codes[tq]), _ptr(self.scale[g]),
                                     _ptr(self.zero[g]), _stream_handle(None)), "mfp8_kv8_quantize")
        self.tail = staged[f:].clone()
        self.T += n

    def read(self, out=None):
        tq = self.Tq
        return kv8_read(self.codes[:tq], self.scale[:tq // 64], self.zero[:tq // 64], self.tail, out=out)


def e4m3_encode(values, stream=None):
    """fp32 CUDA tensor -> uint8 codes from the device's conversion."""
    import torch
    out = torch.empty(values.shape, dtype=torch.uint8, device=values.device)
    _check(mfp8_e4m3_encode_f32(_ptr(values), values.numel(), _ptr(out), _stream_handle(stream)),
           "mfp8_e4m3_encode_f32")
    return out


def device_status(stream=None):
    return mfp8_get_device_status(_stream_handle(stream))

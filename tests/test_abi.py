"""The C ABI library: it builds, loads without a GPU, exports every symbol the
header declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

from fp8_w8a8_dynamic_b200 import build as B
from fp8_w8a8_dynamic_b200 import mfp8

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "mfp8.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return mfp8.lib()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MFP8_API\s+[\w\s\*]+?\b(mfp8_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for required in ("mfp8_quantize_weight", "mfp8_quantize_act", "mfp8_linear",
                     "mfp8_linear_workspace_bytes", "mfp8_get_device_status", "mfp8_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    raw = ctypes.CDLL(mfp8.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(raw, name), f"{name} declared in mfp8.h but not exported"


def test_static_workspace_size_matches_header():
    text = open(HEADER).read()
    m = re.search(r"#define MFP8_STATIC_WORKSPACE_BYTES \((\d+)u << (\d+)\)", text)
    assert m and int(m.group(1)) << int(m.group(2)) == mfp8.STATIC_WORKSPACE_BYTES


def test_library_does_not_need_libcuda():
    # The driver is reached through cudaGetDriverEntryPoint at run time.
    out = os.popen(f"ldd {mfp8.LIB_PATH}").read()
    assert "libcuda.so" not in out and "libtorch" not in out


def test_status_strings_and_version(lib):
    for code in range(8):
        assert mfp8.mfp8_status_string(code)
    assert "unknown" in mfp8.mfp8_status_string(99)
    assert mfp8.mfp8_version() >= 100


def test_workspace_bytes(lib):
    # X8 [M, K] and s_a [M] of the quantize pass, each rounded up to 256 bytes
    assert mfp8.mfp8_linear_workspace_bytes(300, 4096, 4096) == 300 * 4096 + 1280
    assert mfp8.mfp8_linear_workspace_bytes(16, 4096, 4096) == 65536 + 256
    assert mfp8.mfp8_linear_workspace_bytes(3, 8, 48) == 256 + 256
    assert mfp8.mfp8_gemm_workspace_bytes(16, 4096, 4096) == 0
    assert mfp8.mfp8_gemm_workspace_bytes(300, 4096, 4096) == 0
    # the AUTO choice: the one-kernel path up to 16 tokens, the cluster
    # split-K kernel to 128, 128-row tiles for mid M, pairs above
    assert mfp8.mfp8_choose_path(8, 12288, 4096) == mfp8.PATH_FUSED
    assert mfp8.mfp8_choose_path(16, 4096, 12288) == mfp8.PATH_FUSED
    assert mfp8.mfp8_choose_path(17, 4096, 4096) == mfp8.PATH_SPLITK
    assert mfp8.mfp8_choose_path(112, 4096, 4096) == mfp8.PATH_SPLITK
    assert mfp8.mfp8_choose_path(128, 4096, 4096) == mfp8.PATH_SPLITK
    assert mfp8.mfp8_choose_path(129, 4096, 4096) == mfp8.PATH_TILED
    assert mfp8.mfp8_choose_path(200, 4096, 4096) == mfp8.PATH_TILED
    assert mfp8.mfp8_choose_path(2048, 4096, 4096) == mfp8.PATH_PAIR
    assert mfp8.mfp8_choose_path(0, 4096, 4096) == mfp8.PATH_AUTO
    assert mfp8.mfp8_linear_workspace_bytes(0, 8, 48) == 0
    assert mfp8.mfp8_linear_workspace_bytes(4, 8, -1) == 0


FAKE = 1 << 20  # a 16-byte-aligned non-null address; never dereferenced


def test_argument_errors_are_reported_before_any_launch(lib):
    q = mfp8.mfp8_quantize_act
    assert q(FAKE, 4, 0, FAKE * 2, FAKE * 3, None) == mfp8.ERR_UNSUPPORTED_SHAPE  # K == 0
    assert q(FAKE, 4, 40, FAKE * 2, FAKE * 3, None) == mfp8.ERR_UNSUPPORTED_SHAPE  # K % 16
    assert q(FAKE, -1, 64, FAKE * 2, FAKE * 3, None) == mfp8.ERR_INVALID_ARG
    assert q(None, 4, 64, FAKE * 2, FAKE * 3, None) == mfp8.ERR_INVALID_ARG
    assert q(FAKE + 8, 4, 64, FAKE * 2, FAKE * 3, None) == mfp8.ERR_MISALIGNED
    assert q(FAKE, 4, 64, FAKE + 16, FAKE * 3, None) == mfp8.ERR_INVALID_ARG  # output overlaps input
    assert q(FAKE, 0, 64, None, None, None) == mfp8.OK  # empty: nothing to do
    w = mfp8.mfp8_quantize_weight
    assert w(FAKE, 8, 24, FAKE * 2, FAKE * 3, None) == mfp8.ERR_UNSUPPORTED_SHAPE
    rq, sq = mfp8.mfp8_rmsnorm_quantize, mfp8.mfp8_silu_mul_quantize
    assert rq(FAKE, FAKE * 5, 1e-6, 4, 40, None, FAKE * 2, FAKE * 3, None) == mfp8.ERR_UNSUPPORTED_SHAPE  # K % 16
    assert rq(FAKE, FAKE * 5, 1e-6, 4, 32768, None, FAKE * 2, FAKE * 3, None) == mfp8.ERR_UNSUPPORTED_SHAPE
    assert rq(FAKE, FAKE * 5, -1.0, 4, 64, None, FAKE * 2, FAKE * 3, None) == mfp8.ERR_INVALID_ARG  # eps
    assert rq(FAKE, None, 1e-6, 4, 64, None, FAKE * 2, FAKE * 3, None) == mfp8.ERR_INVALID_ARG  # no gain
    assert rq(FAKE, FAKE * 5 + 2, 1e-6, 4, 64, None, FAKE * 2, FAKE * 3, None) == mfp8.ERR_MISALIGNED
    assert rq(FAKE, FAKE * 5, 1e-6, 4, 64, FAKE + 16, FAKE * 2, FAKE * 3, None) == mfp8.ERR_INVALID_ARG
    assert rq(FAKE, FAKE * 5, 1e-6, 0, 64, None, FAKE * 2, FAKE * 3, None) == mfp8.OK
    assert sq(FAKE, 4, 40, None, FAKE * 2, FAKE * 3, None) == mfp8.ERR_UNSUPPORTED_SHAPE
    assert sq(FAKE, -1, 64, None, FAKE * 2, FAKE * 3, None) == mfp8.ERR_INVALID_ARG
    assert sq(FAKE, 4, 64, None, FAKE + 32, FAKE * 3, None) == mfp8.ERR_INVALID_ARG  # codes overlap input
    assert sq(FAKE + 4, 4, 64, None, FAKE * 2, FAKE * 3, None) == mfp8.ERR_MISALIGNED
    assert sq(FAKE, 0, 64, None, FAKE * 2, FAKE * 3, None) == mfp8.OK
    kq, kd = mfp8.mfp8_kv_quantize, mfp8.mfp8_kv_dequantize
    assert kq(FAKE, 2, 8, 40, FAKE * 2, FAKE * 3, None) == mfp8.ERR_UNSUPPORTED_SHAPE  # D % 16
    assert kq(FAKE, 2, 0, 128, FAKE * 2, FAKE * 3, None) == mfp8.ERR_UNSUPPORTED_SHAPE  # no heads
    assert kq(FAKE, -1, 8, 128, FAKE * 2, FAKE * 3, None) == mfp8.ERR_INVALID_ARG
    assert kq(FAKE + 8, 2, 8, 128, FAKE * 2, FAKE * 3, None) == mfp8.ERR_MISALIGNED
    assert kq(FAKE, 2, 8, 128, FAKE + 64, FAKE * 3, None) == mfp8.ERR_INVALID_ARG  # codes overlap input
    assert kq(FAKE, 0, 8, 128, None, None, None) == mfp8.OK
    assert kd(FAKE, FAKE * 2, 2, 8, 40, FAKE * 3, None) == mfp8.ERR_UNSUPPORTED_SHAPE
    assert kd(None, FAKE * 2, 2, 8, 128, FAKE * 3, None) == mfp8.ERR_INVALID_ARG
    assert kd(FAKE, FAKE * 2 + 4, 2, 8, 128, FAKE * 3, None) == mfp8.ERR_MISALIGNED
    assert kd(FAKE, FAKE * 2, 2, 8, 128, FAKE + 16, None) == mfp8.ERR_INVALID_ARG  # output overlaps codes
    assert kd(FAKE, FAKE * 2, 0, 8, 128, FAKE * 3, None) == mfp8.OK
    q8, r8 = mfp8.mfp8_kv8_quantize, mfp8.mfp8_kv8_read
    assert q8(FAKE, 100, 8, 128, FAKE * 2, FAKE * 3, FAKE * 4, None) == mfp8.ERR_UNSUPPORTED_SHAPE  # T % 64
    assert q8(FAKE, 64, 8, 40, FAKE * 2, FAKE * 3, FAKE * 4, None) == mfp8.ERR_UNSUPPORTED_SHAPE  # D % 16
    assert q8(FAKE, -64, 8, 128, FAKE * 2, FAKE * 3, FAKE * 4, None) == mfp8.ERR_INVALID_ARG
    assert q8(FAKE, 64, 8, 128, FAKE * 2, None, FAKE * 4, None) == mfp8.ERR_INVALID_ARG
    assert q8(FAKE, 64, 8, 128, FAKE * 2, FAKE * 3 + 4, FAKE * 4, None) == mfp8.ERR_MISALIGNED
    assert q8(FAKE, 64, 8, 128, FAKE + 256, FAKE * 3, FAKE * 4, None) == mfp8.ERR_INVALID_ARG  # codes overlap input
    assert q8(FAKE, 64, 8, 128, FAKE * 2, FAKE * 3, FAKE * 3 + 16, None) == mfp8.ERR_INVALID_ARG  # zero overlaps scale
    assert q8(FAKE, 0, 8, 128, None, None, None, None) == mfp8.OK
    assert r8(FAKE, FAKE * 2, FAKE * 3, 100, FAKE * 4, 5, 8, 128, FAKE * 5, None) == mfp8.ERR_UNSUPPORTED_SHAPE
    assert r8(FAKE, FAKE * 2, FAKE * 3, 64, None, 5, 8, 128, FAKE * 5, None) == mfp8.ERR_INVALID_ARG  # no tail
    assert r8(FAKE, FAKE * 2, FAKE * 3, 64, FAKE * 4, 5, 8, 128, None, None) == mfp8.ERR_INVALID_ARG
    assert r8(FAKE, FAKE * 2, FAKE * 3, 64, FAKE * 4 + 2, 5, 8, 128, FAKE * 5, None) == mfp8.ERR_MISALIGNED
    assert r8(FAKE, FAKE * 2, FAKE * 3, 64, FAKE * 4, 5, 8, 128, FAKE + 64, None) == mfp8.ERR_INVALID_ARG  # overlap
    assert r8(None, None, None, 0, None, 0, 8, 128, None, None) == mfp8.OK
    assert [mfp8.mfp8_kv8_history_tokens(t) for t in (-1, 0, 127, 128, 191, 192, 255, 256, 1000)] == \
        [-1, 0, 0, 0, 0, 64, 64, 128, 832]

    L = mfp8.mfp8_linear_ex
    args = dict(X=FAKE, M=4, K=64, W=FAKE * 2, sw=FAKE * 3, N=64, Y=FAKE * 4, ws=FAKE * 5, wsb=1 << 16)

    def call(**kw):
        a = {**args, **kw}
        return L(a["X"], a["M"], a["K"], a["W"], a["sw"], a["N"], a["Y"], a["ws"], a["wsb"],
                 kw.get("path", 0), kw.get("flags", 0), kw.get("x8", None), kw.get("xs", None), None)

    assert call(N=12, wsb=100) == mfp8.ERR_WORKSPACE  # N % 8 != 0 takes a padded scratch in the workspace
    assert call(N=12, path=mfp8.PATH_FUSED, ws=None) == mfp8.ERR_WORKSPACE  # even on the fused path
    assert mfp8.mfp8_linear_workspace_bytes(4, 12, 64) > mfp8.mfp8_linear_workspace_bytes(4, 16, 64)
    assert mfp8.mfp8_gemm_workspace_bytes(4, 16, 64) == 0 and mfp8.mfp8_gemm_workspace_bytes(4, 13, 64) > 0
    assert call(N=0) == mfp8.ERR_UNSUPPORTED_SHAPE
    assert call(K=8) == mfp8.ERR_UNSUPPORTED_SHAPE
    assert call(W=None) == mfp8.ERR_INVALID_ARG
    assert call(Y=FAKE * 4 + 4) == mfp8.ERR_MISALIGNED
    assert call(M=65, ws=None) == mfp8.ERR_WORKSPACE  # quantize pass needs the workspace
    assert call(M=65, wsb=100) == mfp8.ERR_WORKSPACE
    assert call(M=4, path=mfp8.PATH_TILED, ws=None) == mfp8.ERR_WORKSPACE
    assert call(flags=2) == mfp8.ERR_INVALID_ARG
    assert call(path=7) == mfp8.ERR_INVALID_ARG
    assert call(path=5) == mfp8.ERR_INVALID_ARG
    assert call(path=mfp8.PATH_FUSED, M=17) == mfp8.ERR_UNSUPPORTED_SHAPE
    assert call(ws=None, path=mfp8.PATH_SPLITK) == mfp8.ERR_WORKSPACE  # the quantize pass's codes
    assert call(path=mfp8.PATH_SPLITK, M=257) == mfp8.ERR_UNSUPPORTED_SHAPE
    assert call(x8=FAKE * 6) == mfp8.ERR_INVALID_ARG  # codes without scales
    assert call(Y=FAKE + 64) == mfp8.ERR_INVALID_ARG  # Y overlaps X
    assert call(M=0) == mfp8.OK
    NA = mfp8.mfp8_linear_noalloc
    assert NA(FAKE, 4, 40, FAKE * 2, FAKE * 3, 12, FAKE * 4, None) == mfp8.ERR_UNSUPPORTED_SHAPE  # K % 16
    assert NA(FAKE, 0, 64, FAKE * 2, FAKE * 3, 64, FAKE * 4, None) == mfp8.OK
    # more than the library's fixed scratch: codes alone are 4096 * 8192 bytes
    assert NA(FAKE, 4096, 8192, FAKE * 2, FAKE * 3, 64, FAKE * 4, None) == mfp8.ERR_WORKSPACE
    G = mfp8.mfp8_gemm
    assert G(None, FAKE, 4, 64, FAKE * 2, FAKE * 3, 64, FAKE * 4, None, 0, 0, None) == mfp8.ERR_INVALID_ARG
    assert G(FAKE, FAKE * 9 + 4, 4, 64, FAKE * 2, FAKE * 3, 64, FAKE * 4, None, 0, 0, None) == mfp8.ERR_MISALIGNED
    assert G(FAKE, FAKE * 9, 257, 64, FAKE * 2, FAKE * 3, 64, FAKE * 4, None, 0, mfp8.PATH_SPLITK,
             None) == mfp8.ERR_UNSUPPORTED_SHAPE  # split-K kernel: M <= 256
    assert G(FAKE, FAKE * 9, 4, 64, FAKE * 2, FAKE * 3, 64, FAKE * 4, None, 0, mfp8.PATH_FUSED, None) == mfp8.ERR_INVALID_ARG
    assert mfp8.mfp8_e4m3_encode_f32(FAKE, -1, FAKE * 2, None) == mfp8.ERR_INVALID_ARG
    assert mfp8.mfp8_debug_bounded_wait(0, None) == mfp8.ERR_INVALID_ARG
    assert mfp8.mfp8_debug_bounded_wait(10 ** 6, None) == mfp8.ERR_INVALID_ARG


def test_binding_raises_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(mfp8, "_lib", None)
    monkeypatch.setattr(mfp8, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="not built"):
        mfp8.lib()


C_PROGRAM = r"""
#include <stdio.h>
#include "mfp8.h"

int main(void) {
    /* every entry point is a plain C function */
    typedef void (*fn_t)(void);
    fn_t fns[] = {%s};
    size_t n = sizeof fns / sizeof fns[0];
    for (size_t i = 0; i < n; ++i)
        if (!fns[i]) return 10;
    if (mfp8_version() < 100) return 11;
    if (mfp8_linear_workspace_bytes(300, 4096, 4096) != (size_t)300 * 4096 + 1280) return 12;
    if (mfp8_choose_path(8, 4096, 4096) != MFP8_PATH_FUSED) return 13;
    /* argument errors come back before any device work */
    if (mfp8_linear(NULL, 4, 64, NULL, NULL, 64, NULL, NULL, 0, NULL) != MFP8_ERR_INVALID_ARG) return 14;
    if (mfp8_linear_noalloc((void*)4096, 4, 40, (void*)8192, (float*)12288, 12, (void*)16384, NULL)
        != MFP8_ERR_UNSUPPORTED_SHAPE) return 15;
    printf("%%s\n", mfp8_status_string(MFP8_ERR_MISALIGNED));
    return 0;
}
"""


def test_header_is_plain_c_and_links(lib, tmp_path):
    """A C99 program (no C++, no CUDA headers) includes mfp8.h, takes the
    address of every declared entry point, links against libmfp8.so and gets
    the host-side answers and argument errors without a GPU."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_mfp8.c"
    src.write_text(C_PROGRAM % ", ".join(f"(fn_t){n}" for n in declared_symbols()))
    exe = tmp_path / "use_mfp8"
    libdir = os.path.dirname(mfp8.LIB_PATH)
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.dirname(HEADER), str(src), "-o", str(exe),
                    "-L", libdir, "-l:libmfp8.so", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out
    assert out.stdout.strip() == mfp8.mfp8_status_string(mfp8.ERR_MISALIGNED)

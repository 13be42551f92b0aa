"""C-ABI checks that need no GPU: the library builds and loads, exports every function that
include/fp4mx.h declares, and rejects bad arguments synchronously (before any CUDA call), so
these run on a machine without a device.  The pointers below are never dereferenced: every call
fails validation first."""
import ctypes
import os
import re

import pytest

import block_scaled_fp4_amax_b200 as fp4
from block_scaled_fp4_amax_b200 import build as fp4build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "fp4mx.h")


@pytest.fixture(scope="module")
def L():
    fp4build.build()
    return fp4.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    # the identifier right before the parameter list: the return type may be several words
    names = re.findall(r"^FP4_API\s+[^(;]*[\s*]([a-z_][a-z0-9_]*)\s*\(", src, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "while")))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert set(names) == set(fp4.EXPORTS), names
    for n in names:
        assert hasattr(L, n), n


def test_status_strings_and_workspace(L):
    assert L.fp4_status_str(0) == b"FP4_OK"
    assert b"EINVAL" in L.fp4_status_str(1)
    assert L.fp4_workspace_size(fp4.OP_NVFP4_QUANTIZE, 8192, 8192) >= 4
    assert L.fp4_workspace_size(fp4.OP_BLOCK_GEMM, 8192, 8192) >= 4
    assert L.fp4_workspace_size(fp4.OP_MX_QUANTIZE, 8192, 8192) == 0
    assert L.fp4_gemm_status_word() == 0
    # the GEMM wait limit: default 2 s, returned by the next call that sets it
    old = L.fp4_set_gemm_wait_limit(12345)
    assert old == 2000000000 and L.fp4_set_gemm_wait_limit(old) == 12345


FAKE = ctypes.c_void_p(0x10000)  # aligned, never dereferenced


def _mx(L, **kw):
    a = dict(x=FAKE, dtype=1, rows=128, cols=256, block=32, policy=0, round=0, seed=0, layout=0,
             q=FAKE, s=FAKE, c=None)
    a.update(kw)
    return L.mx_quantize(a["x"], a["dtype"], a["rows"], a["cols"], a["block"], a["policy"], a["round"],
                         a["seed"], a["layout"], a["q"], a["s"], a["c"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(block=16), 1),                 # MXFP4 block must be 32: no block-size inference
    (dict(block=24), 1),
    (dict(cols=48), 1),                  # incomplete block
    (dict(cols=0), 1),
    (dict(rows=-1), 1),
    (dict(dtype=7), 1),
    (dict(policy=5), 1),
    (dict(round=9), 1),
    (dict(layout=4), 1),
    (dict(layout=1, rows=100), 1),       # tiled scales need rows % 128 == 0
    (dict(layout=1, cols=96), 1),        # ... and (cols/32) % 4 == 0
    (dict(x=None), 1),
    (dict(q=None), 1),
    (dict(x=ctypes.c_void_p(0x10004)), 1),  # misaligned input
])
def test_mx_quantize_rejects(L, kw, status):
    assert _mx(L, **kw) == status
    assert L.fp4_last_error()


def test_nvfp4_rejects(L):
    # block 32 for NVFP4, no workspace without a global scale, MXFP4-only policy irrelevant
    assert L.nvfp4_quantize(FAKE, 1, 128, 256, 32, 0, 0, 0, 0, None, None, FAKE, FAKE, None, FAKE, 256, None) == 1
    assert L.nvfp4_quantize(FAKE, 1, 128, 256, 16, 0, 0, 0, 0, None, None, FAKE, FAKE, None, None, 0, None) == 1
    assert L.nvfp4_quantize(FAKE, 1, 128, 200, 16, 0, 0, 0, 0, None, None, FAKE, FAKE, None, FAKE, 256, None) == 1
    assert L.nvfp4_quantize(FAKE, 1, 128, 256, 16, 0, 0, 0, 0, None, None, FAKE, FAKE, None, FAKE, 8, None) == 1


def test_if4_rejects(L):
    # IF4 is round-to-nearest NVFP4 only (also in the rotation path); block modes beyond IF4
    assert L.nvfp4_quantize(FAKE, 1, 128, 256, 16, 1, 2, 0, 0, FAKE, None, FAKE, FAKE, None, None, 0, None) == 2
    assert L.nvfp4_quantize(FAKE, 1, 128, 256, 16, 0, 3, 0, 0, FAKE, None, FAKE, FAKE, None, None, 0, None) == 1
    assert L.fwht_quantize(FAKE, 1, 4, 8192, None, 1, 16, 1, 2, 0, 0, FAKE, None, None, FAKE, FAKE, None, FAKE, 256, None) == 2
    assert L.fwht_quantize(FAKE, 1, 4, 8192, None, 0, 32, 0, 2, 0, 0, FAKE, None, None, FAKE, FAKE, None, FAKE, 256, None) == 2
    assert L.fwht_quantize(FAKE, 1, 4, 8192, None, 1, 16, 0, 3, 0, 0, FAKE, None, None, FAKE, FAKE, None, FAKE, 256, None) == 1
    # IF4 GEMM: the fp16 operands need fp4_workspace_size(FP4_OP_BLOCK_GEMM_IF4, M + N, K) bytes, both
    # global scales, and the FP4 GEMM's shape rules
    need = L.fp4_workspace_size(6, 128 + 256, 256)
    assert need == 512 + 2 * (128 + 256) * 256
    assert L.fp4_block_gemm(2, 128, 256, 256, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 256, FAKE, 256, None) == 1
    assert L.fp4_block_gemm(2, 128, 256, 256, FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, 256, FAKE, need, None) == 1
    assert L.fp4_block_gemm(2, 128, 256, 192, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 256, FAKE, need, None) == 2
    # the stored-rotation workspace: the amax word, padding and the fp32 rotation
    assert L.fp4_workspace_size(5, 64, 8192) == 512 + 64 * 8192 * 4 and L.fp4_workspace_size(2, 64, 8192) == 256
    # IF4 dequantisation: block 16 and a global scale
    assert L.fp4_dequantize(FAKE, FAKE, 2, 32, 0, FAKE, 128, 256, 0, FAKE, None) == 1
    assert L.fp4_dequantize(FAKE, FAKE, 2, 16, 0, None, 128, 256, 0, FAKE, None) == 1


def test_e4m3_route_rejects(L):
    # expansion: cols % 32, NULL, misalignment; FP8 GEMM: shape rules, ldc, workspace
    assert L.fp4_to_e4m3(FAKE, 4, 48, FAKE, None) == 1
    assert L.fp4_to_e4m3(None, 4, 64, FAKE, None) == 1
    assert L.fp4_to_e4m3(FAKE, 4, 64, ctypes.c_void_p(0x10008), None) == 1
    assert L.fp4_to_e4m3(FAKE, 0, 64, FAKE, None) == 0  # empty: nothing launched
    g = L.fp4_block_gemm_e4m3
    assert g(100, 256, 128, FAKE, FAKE, FAKE, FAKE, FAKE, 256, FAKE, 256, None) == 2  # M % 128
    assert g(128, 128, 128, FAKE, FAKE, FAKE, FAKE, FAKE, 256, FAKE, 256, None) == 2  # N % 256
    assert g(128, 256, 96, FAKE, FAKE, FAKE, FAKE, FAKE, 256, FAKE, 256, None) == 2   # K % 128
    assert g(128, 256, 128, FAKE, FAKE, FAKE, FAKE, FAKE, 100, FAKE, 256, None) == 1  # ldc < N
    assert g(128, 256, 128, FAKE, FAKE, FAKE, FAKE, FAKE, 256, None, 0, None) == 1    # workspace
    assert g(128, 256, 128, None, FAKE, FAKE, FAKE, FAKE, 256, FAKE, 256, None) == 1  # NULL A


def test_fwht_rejects(L):
    # d not a power of two / out of range, MXFP4 with four-over-six, block mismatch
    assert L.fwht_quantize(FAKE, 1, 4, 3000, None, 1, 16, 0, 0, 0, 0, FAKE, None, None, FAKE, FAKE, None, FAKE, 256, None) == 1
    assert L.fwht_quantize(FAKE, 1, 4, 512, None, 1, 16, 0, 0, 0, 0, FAKE, None, None, FAKE, FAKE, None, FAKE, 256, None) == 1
    assert L.fwht_quantize(FAKE, 1, 4, 32768, None, 1, 16, 0, 0, 0, 0, FAKE, None, None, FAKE, FAKE, None, FAKE, 256, None) == 1
    assert L.fwht_quantize(FAKE, 1, 4, 8192, None, 0, 32, 0, 1, 0, 0, None, None, None, FAKE, FAKE, None, None, 0, None) == 2
    assert L.fwht_quantize(FAKE, 1, 4, 8192, None, 0, 16, 0, 0, 0, 0, None, None, None, FAKE, FAKE, None, None, 0, None) == 1
    assert L.fwht_quantize(FAKE, 1, 4, 8192, None, 5, 16, 0, 0, 0, 0, None, None, None, FAKE, FAKE, None, None, 0, None) == 1


def test_swiglu_fwht_rejects(L):
    # fp32 inputs (bf16 only), a NULL or misaligned up projection, and the rotation's own checks
    assert L.swiglu_fwht_quantize(FAKE, FAKE, 0, 4, 8192, None, 1, 16, 0, 0, 0, 0, FAKE, None, None, FAKE, FAKE, None,
                                  FAKE, 256, None) == 2
    assert L.swiglu_fwht_quantize(FAKE, None, 1, 4, 8192, None, 1, 16, 0, 0, 0, 0, FAKE, None, None, FAKE, FAKE, None,
                                  FAKE, 256, None) == 1
    assert L.swiglu_fwht_quantize(FAKE, ctypes.c_void_p(0x10010), 1, 4, 8192, None, 1, 16, 0, 0, 0, 0, FAKE, None, None, FAKE, FAKE,
                                  None, FAKE, 256, None) == 1
    assert L.swiglu_fwht_quantize(FAKE, FAKE, 1, 4, 3000, None, 1, 16, 0, 0, 0, 0, FAKE, None, None, FAKE, FAKE, None,
                                  FAKE, 256, None) == 1


def test_dequant_rejects(L):
    assert L.fp4_dequantize(FAKE, FAKE, 1, 32, 0, FAKE, 128, 256, 0, FAKE, None) == 1  # block mismatch
    assert L.fp4_dequantize(FAKE, FAKE, 1, 16, 0, None, 128, 256, 0, FAKE, None) == 1  # NVFP4 needs s_g
    assert L.fp4_dequantize(FAKE, FAKE, 0, 32, 0, None, 128, 80, 0, FAKE, None) == 1   # ragged block
    assert L.fp4_dequantize(FAKE, FAKE, 0, 32, 0, None, 128, 256, 3, FAKE, None) == 1  # out dtype


def test_gemm_rejects(L):
    g = L.fp4_block_gemm
    assert g(1, 100, 256, 256, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 256, FAKE, 256, None) == 2  # M % 128
    assert g(1, 128, 200, 256, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 256, FAKE, 256, None) == 2  # N % 256
    assert g(1, 128, 256, 200, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 256, FAKE, 256, None) == 2  # K % 256
    assert g(1, 128, 256, 256, FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, 256, FAKE, 256, None) == 1  # no Ag
    assert g(1, 128, 256, 256, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 100, FAKE, 256, None) == 1  # ldc < N
    assert g(1, 128, 256, 256, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 256, None, 0, None) == 1    # workspace
    assert g(3, 128, 256, 256, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 256, FAKE, 256, None) == 1  # format


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(fp4, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(fp4, "_lib", None)
    with pytest.raises(ImportError):
        fp4.lib()


def test_header_is_plain_c_and_links_from_c(L, tmp_path):
    """include/fp4mx.h is a C header: a C99 program includes it, links libfp4mx.so and gets the
    synchronous argument checks without a GPU."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_fp4mx.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "fp4mx.h"
int main(void) {
  if (strcmp(fp4_status_str(FP4_OK), "FP4_OK") != 0) return 1;
  if (fp4_workspace_size(FP4_OP_NVFP4_QUANTIZE, 8192, 8192) < 4) return 2;
  /* block 16 is not MXFP4's block: rejected before any CUDA call */
  if (mx_quantize((const void*)0x10000, FP4_BF16, 128, 256, 16, FP4_MX_OCP_FLOOR, FP4_RNE, 0,
                  FP4_SCALES_ROWMAJOR, (unsigned char*)0x10000, (unsigned char*)0x10000, 0, 0) != FP4_EINVAL)
    return 3;
  if (fp4_block_gemm_e4m3(100, 256, 128, 0, 0, 0, 0, 0, 256, 0, 0, 0) != FP4_EUNSUPPORTED) return 4;
  printf("ok %s\n", fp4_last_error());
  return 0;
}
''')
    exe = tmp_path / "use_fp4mx"
    libdir = os.path.dirname(fp4.LIB_PATH)
    subprocess.check_call([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe),
                           "-L", libdir, "-lfp4mx", "-Wl,-rpath," + libdir])
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, (out.returncode, out.stdout, out.stderr)
    assert out.stdout.startswith("ok ")

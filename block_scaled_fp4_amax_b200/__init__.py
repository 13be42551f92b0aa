"""block_scaled_fp4_amax_b200 — Python binding of libfp4mx.so (block-scaled FP4 microscaling on B200).

Argument marshalling only: every function here checks tensor devices/dtypes/shapes, allocates the
outputs with torch (device memory is torch's job) and calls the C ABI declared in
``include/fp4mx.h`` on torch's current CUDA stream.  All arithmetic runs in the CUDA kernels of
libfp4mx.so; there is no CPU path.  If the shared library is missing or was built for nothing this
process can load, the first call raises.

    from block_scaled_fp4_amax_b200 import mx_quantize, nvfp4_quantize, fwht_quantize, \
        swiglu_fwht_quantize, fp4_dequantize, fp4_block_gemm, fp4_to_e4m3, fp4_block_gemm_e4m3

NVFP4 block modes: nvfp4_quantize / fwht_quantize take four_six=True (four over six) or if4=True
(IF4: E2M1 or INT4 per block, flagged in scale bit 7; read back with fp4_dequantize(fmt=IF4)).
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp4mx.so")

# enums of include/fp4mx.h
F32, BF16 = 0, 1
MXFP4, NVFP4, IF4 = 0, 1, 2          # fp4_format
NV_PLAIN, NV_FOUR_SIX, NV_IF4 = 0, 1, 2  # fp4_nv_mode
RNE, STOCHASTIC = 0, 1
OCP_FLOOR, NOSAT_CEIL = 0, 1
ROWMAJOR, MMA_TILED = 0, 1
(OP_MX_QUANTIZE, OP_NVFP4_QUANTIZE, OP_FWHT_QUANTIZE, OP_DEQUANTIZE, OP_BLOCK_GEMM, OP_FWHT_QUANTIZE_STORED,
 OP_BLOCK_GEMM_IF4) = range(7)
STATUS = {0: "FP4_OK", 1: "FP4_EINVAL", 2: "FP4_EUNSUPPORTED", 3: "FP4_ECUDA"}

# Every symbol include/fp4mx.h declares.
EXPORTS = ("mx_quantize", "nvfp4_quantize", "fwht_quantize", "swiglu_fwht_quantize", "fp4_dequantize", "fp4_block_gemm",
           "fp4_workspace_size", "fp4_gemm_status_word", "fp4_status_str", "fp4_last_error",
           "nvfp4_quantize_noalloc", "fp4_to_e4m3", "fp4_block_gemm_e4m3", "fp4_set_gemm_wait_limit")


class Fp4Error(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{STATUS.get(status, status)}: {detail}")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load libfp4mx.so and declare its C signatures (raises if it is not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m block_scaled_fp4_amax_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, LG, ULL, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_long, ctypes.c_ulonglong, ctypes.c_size_t
    L.mx_quantize.argtypes = [P, I, LG, LG, I, I, I, ULL, I, P, P, P, P]
    L.nvfp4_quantize.argtypes = [P, I, LG, LG, I, I, I, ULL, I, P, P, P, P, P, P, SZ, P]
    L.fwht_quantize.argtypes = [P, I, LG, LG, P, I, I, I, I, ULL, I, P, P, P, P, P, P, P, SZ, P]
    L.swiglu_fwht_quantize.argtypes = [P, P, I, LG, LG, P, I, I, I, I, ULL, I, P, P, P, P, P, P, P, SZ, P]
    L.fp4_dequantize.argtypes = [P, P, I, I, I, P, LG, LG, I, P, P]
    L.fp4_block_gemm.argtypes = [I, I, I, I, P, P, P, P, P, P, P, LG, P, SZ, P]
    L.fp4_to_e4m3.argtypes = [P, LG, LG, P, P]
    L.fp4_block_gemm_e4m3.argtypes = [I, I, I, P, P, P, P, P, LG, P, SZ, P]
    L.nvfp4_quantize_noalloc.argtypes = [P, I, LG, LG, I, I, I, ULL, I, P, P, P, P, P, P]
    L.nvfp4_quantize_noalloc.restype = I
    L.fp4_workspace_size.argtypes = [I, LG, LG]
    L.fp4_workspace_size.restype = SZ
    L.fp4_gemm_status_word.argtypes = []
    L.fp4_gemm_status_word.restype = SZ
    L.fp4_status_str.argtypes = [I]
    L.fp4_status_str.restype = ctypes.c_char_p
    L.fp4_last_error.argtypes = []
    L.fp4_last_error.restype = ctypes.c_char_p
    L.fp4_set_gemm_wait_limit.argtypes = [ULL]
    L.fp4_set_gemm_wait_limit.restype = ULL
    for name in ("mx_quantize", "nvfp4_quantize", "fwht_quantize", "swiglu_fwht_quantize", "fp4_dequantize",
                 "fp4_block_gemm", "fp4_to_e4m3", "fp4_block_gemm_e4m3"):
        getattr(L, name).restype = I
    _lib = L
    return L


def _check(status: int):
    if status != 0:
        raise Fp4Error(status, lib().fp4_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"input dtype must be float32 or bfloat16, got {t.dtype}")


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def workspace_size(op: int, rows: int = 0, cols: int = 0) -> int:
    return int(lib().fp4_workspace_size(op, rows, cols))


def _workspace(op, device, rows=0, cols=0):
    n = workspace_size(op, rows, cols)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def _alloc_outputs(rows, cols, block, device):
    q = torch.empty((rows, cols // 2), dtype=torch.uint8, device=device)
    s = torch.empty((rows * cols // block,), dtype=torch.uint8, device=device)
    c = torch.empty(4, dtype=torch.int64, device=device)  # zeroed by the library on its stream
    return q, s, c


def _outputs(out, rows, cols, block, device, with_scale):
    """The quantisers' outputs: the caller's `out` (checked: contiguous, on `device`, the sizes the
    call writes) or new tensors.  Returns (q, scales, s_g or None, counts)."""
    if out is None:
        q, s, c = _alloc_outputs(rows, cols, block, device)
        g = torch.empty(1, dtype=torch.float32, device=device) if with_scale else None
        return q, s, g, c
    q, s, g, c = out
    want = [(q, rows * cols // 2, torch.uint8), (s, rows * cols // block, torch.uint8), (c, 4, torch.int64)]
    if with_scale:
        want.append((g, 1, torch.float32))
    for t, n, dt in want:
        if t is None or t.device != device or t.dtype != dt or t.numel() != n or not t.is_contiguous():
            raise ValueError(f"out: expected a contiguous {dt} tensor of {n} elements on {device}")
    return q, s, (g if with_scale else None), c


def mx_quantize(x: torch.Tensor, policy: int = OCP_FLOOR, round: int = RNE, seed: int = 0,
                layout: int = ROWMAJOR, block: int = 32, stream=None, out=None):
    """MXFP4: returns (q uint8 [rows, cols/2], scales uint8 [rows*cols/32] in `layout`,
    counts int64[4] on device: underflow, saturation, nonfinite, blocks_four).  `out` = (q, scales,
    None, counts) preallocated by the caller (else allocated here)."""
    _need_cuda(x)
    rows, cols = x.shape
    q, s, _, c = _outputs(out, rows, cols, 32, x.device, False)
    _check(lib().mx_quantize(_ptr(x), _dtype_code(x), rows, cols, block, policy, round, seed, layout,
                             _ptr(q), _ptr(s), _ptr(c), _stream(stream)))
    return q, s, c


def _nv_mode(four_six: bool, if4: bool) -> int:
    if four_six and if4:
        raise ValueError("four_six and if4 are exclusive block modes")
    return NV_IF4 if if4 else (NV_FOUR_SIX if four_six else NV_PLAIN)


def nvfp4_quantize(x: torch.Tensor, round: int = RNE, four_six: bool = False, seed: int = 0,
                   layout: int = ROWMAJOR, global_in: torch.Tensor | None = None, block: int = 16,
                   stream=None, workspace: torch.Tensor | None = None, if4: bool = False, out=None):
    """NVFP4 (with `if4`, IF4: E2M1 or INT4 per block, flagged in scale bit 7): returns
    (q, scales, s_g float32[1] on device, counts); `out` = those four preallocated by the caller."""
    _need_cuda(x, global_in)
    rows, cols = x.shape
    q, s, g, c = _outputs(out, rows, cols, 16, x.device, True)
    ws = workspace if workspace is not None else _workspace(OP_NVFP4_QUANTIZE, x.device, rows, cols)
    _check(lib().nvfp4_quantize(_ptr(x), _dtype_code(x), rows, cols, block, round, _nv_mode(four_six, if4), seed,
                                layout, _ptr(global_in), _ptr(g), _ptr(q), _ptr(s), _ptr(c), _ptr(ws),
                                ws.numel(), _stream(stream)))
    return q, s, g, c


def nvfp4_quantize_noalloc(x: torch.Tensor, round: int = RNE, four_six: bool = False, seed: int = 0,
                           layout: int = ROWMAJOR, global_in: torch.Tensor | None = None, block: int = 16,
                           stream=None, if4: bool = False, out=None):
    """nvfp4_quantize for callers that cannot hand the library a device workspace: the amax pass's
    per-CTA partial maxima live in a fixed area of the library's own device memory.  Calls that
    overlap on the GPU share that area and must be serialised.  `out` = (q, scales, s_g, counts)
    preallocated by the caller (else allocated here).  Returns (q, scales, s_g, counts)."""
    _need_cuda(x, global_in)
    rows, cols = x.shape
    if out is None:
        q, s, c = _alloc_outputs(rows, cols, 16, x.device)
        g = torch.empty(1, dtype=torch.float32, device=x.device)
    else:
        q, s, g, c = out
        _need_cuda(q, s, g, c)
    _check(lib().nvfp4_quantize_noalloc(_ptr(x), _dtype_code(x), rows, cols, block, round, _nv_mode(four_six, if4),
                                        seed, layout, _ptr(global_in), _ptr(g), _ptr(q), _ptr(s), _ptr(c),
                                        _stream(stream)))
    return q, s, g, c


def _fwht_op(fmt, global_in, want_rotated):
    """The workspace to allocate by default: room for the fp32 rotation when a two-pass NVFP4 call
    would otherwise rotate twice (a requested rotated_out serves that purpose itself)."""
    if fmt == NVFP4 and global_in is None and not want_rotated:
        return OP_FWHT_QUANTIZE_STORED
    return OP_FWHT_QUANTIZE


def fwht_quantize(x: torch.Tensor, fmt: int = NVFP4, round: int = RNE, four_six: bool = False, seed: int = 0,
                  layout: int = ROWMAJOR, global_in: torch.Tensor | None = None, want_rotated: bool = False,
                  block: int | None = None, stream=None, workspace: torch.Tensor | None = None,
                  signs: torch.Tensor | None = None, if4: bool = False, out=None):
    """Walsh-Hadamard rotation of each row fused with the quantiser of `fmt`; with `signs` (device
    int32/uint32 [d/32], bit i negates channel i first) the randomised rotation c*H*D; with `if4`
    (NVFP4, round to nearest) IF4 blocks.  `out` = (q, scales, s_g or None, counts) preallocated.
    Returns (q, scales, s_g (NVFP4; None for MXFP4), counts, rotated fp32 or None)."""
    _need_cuda(x, global_in, signs)
    rows, d = x.shape
    B = block if block is not None else (32 if fmt == MXFP4 else 16)
    q, s, g, c = _outputs(out, rows, d, 16 if fmt == NVFP4 else 32, x.device, fmt == NVFP4)
    rot = torch.empty((rows, d), dtype=torch.float32, device=x.device) if want_rotated else None
    ws = workspace if workspace is not None else _workspace(_fwht_op(fmt, global_in, want_rotated), x.device, rows, d)
    if signs is not None and (signs.numel() != d // 32 or signs.element_size() != 4):
        raise ValueError("signs must hold d/32 32-bit words")
    _check(lib().fwht_quantize(_ptr(x), _dtype_code(x), rows, d, _ptr(signs), fmt, B, round, _nv_mode(four_six, if4), seed,
                               layout, _ptr(global_in), _ptr(g), _ptr(rot), _ptr(q), _ptr(s), _ptr(c),
                               _ptr(ws), ws.numel(), _stream(stream)))
    return q, s, g, c, rot


def swiglu_fwht_quantize(g: torch.Tensor, u: torch.Tensor, fmt: int = NVFP4, round: int = RNE,
                         four_six: bool = False, seed: int = 0, layout: int = ROWMAJOR,
                         global_in: torch.Tensor | None = None, want_rotated: bool = False,
                         block: int | None = None, stream=None, workspace: torch.Tensor | None = None,
                         signs: torch.Tensor | None = None, if4: bool = False, out=None):
    """fl(SiLU(g) * u) in fp32 (never stored), rotated (randomised with `signs`) and quantised to `fmt`
    (IF4 blocks with `if4`).  `out` = (q, scales, s_g or None, counts) preallocated.
    g, u: bf16 [rows, d].  Returns (q, scales, s_g (NVFP4; None for MXFP4), counts, rotated fp32 or None)."""
    _need_cuda(g, u, global_in, signs)
    if g.shape != u.shape:
        raise ValueError("g and u must have the same shape")
    rows, d = g.shape
    B = block if block is not None else (32 if fmt == MXFP4 else 16)
    q, s, gs, c = _outputs(out, rows, d, 16 if fmt == NVFP4 else 32, g.device, fmt == NVFP4)
    rot = torch.empty((rows, d), dtype=torch.float32, device=g.device) if want_rotated else None
    ws = workspace if workspace is not None else _workspace(_fwht_op(fmt, global_in, want_rotated), g.device, rows, d)
    if signs is not None and (signs.numel() != d // 32 or signs.element_size() != 4):
        raise ValueError("signs must hold d/32 32-bit words")
    _check(lib().swiglu_fwht_quantize(_ptr(g), _ptr(u), _dtype_code(g), rows, d, _ptr(signs), fmt, B, round,
                                      _nv_mode(four_six, if4), seed, layout, _ptr(global_in), _ptr(gs), _ptr(rot),
                                      _ptr(q), _ptr(s), _ptr(c), _ptr(ws), ws.numel(), _stream(stream)))
    return q, s, gs, c, rot


def fp4_dequantize(q: torch.Tensor, scales: torch.Tensor, fmt: int, global_scale: torch.Tensor | None = None,
                   layout: int = ROWMAJOR, out_dtype: torch.dtype = torch.float32, block: int | None = None,
                   stream=None, out: torch.Tensor | None = None):
    """x_hat [rows, 2*q.shape[1]] in out_dtype (or in `out`, whose dtype then decides)."""
    _need_cuda(q, scales, global_scale, out)
    rows, half = q.shape
    B = block if block is not None else (32 if fmt == MXFP4 else 16)
    if out is None:
        out = torch.empty((rows, 2 * half), dtype=out_dtype, device=q.device)
    elif out.shape != (rows, 2 * half) or not out.is_contiguous():
        raise ValueError("out must be a contiguous [rows, 2 * q.shape[1]] tensor")
    _check(lib().fp4_dequantize(_ptr(q), _ptr(scales), fmt, B, layout, _ptr(global_scale), rows, 2 * half,
                                _dtype_code(out), _ptr(out), _stream(stream)))
    return out


def fp4_block_gemm(fmt: int, Aq: torch.Tensor, As: torch.Tensor, Bq: torch.Tensor, Bs: torch.Tensor,
                   Ag: torch.Tensor | None = None, Bg: torch.Tensor | None = None, out: torch.Tensor | None = None,
                   stream=None, workspace: torch.Tensor | None = None):
    """C = alpha * A @ B^T in bf16 from packed operands with MMA-tiled scales (IF4: through fp16
    expansions held in the workspace).  Returns (C, workspace); workspace[0:4] holds the kernel
    status word (0 = ok)."""
    _need_cuda(Aq, As, Bq, Bs, Ag, Bg)
    M, K = Aq.shape[0], Aq.shape[1] * 2
    N = Bq.shape[0]
    if Bq.shape[1] * 2 != K:
        raise ValueError("A and B disagree on K")
    C = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=Aq.device)
    if workspace is not None:
        ws = workspace
    elif fmt == IF4:
        ws = _workspace(OP_BLOCK_GEMM_IF4, Aq.device, M + N, K)
    else:
        ws = _workspace(OP_BLOCK_GEMM, Aq.device, M, N)
    _check(lib().fp4_block_gemm(fmt, M, N, K, _ptr(Aq), _ptr(As), _ptr(Ag), _ptr(Bq), _ptr(Bs), _ptr(Bg),
                                _ptr(C), C.stride(0), _ptr(ws), ws.numel(), _stream(stream)))
    return C, ws


def set_gemm_wait_limit(ns: int) -> int:
    """Limit (ns) of each pipeline wait in GEMM launches made from now on; returns the previous one
    (default 2 s).  A tiny limit makes the kernel give up early and report it in its status word."""
    return int(lib().fp4_set_gemm_wait_limit(ns))


def fp4_to_e4m3(q: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """E4M3 bytes (value * 2^-6 of every nibble) of packed E2M1 q [rows, cols/2] -> uint8 [rows, cols]."""
    _need_cuda(q)
    rows, half = q.shape
    o = out if out is not None else torch.empty((rows, 2 * half), dtype=torch.uint8, device=q.device)
    _check(lib().fp4_to_e4m3(_ptr(q), rows, 2 * half, _ptr(o), _stream(stream)))
    return o


def fp4_block_gemm_e4m3(A8: torch.Tensor, As: torch.Tensor, B8: torch.Tensor, Bs: torch.Tensor,
                        out: torch.Tensor | None = None, stream=None, workspace: torch.Tensor | None = None):
    """MXFP4 GEMM on the FP8 tensor-core path from E4M3 expansions (fp4_to_e4m3) and MMA-tiled E8M0
    scales.  Returns (C bf16 [M, N], workspace); workspace[0:4] holds the kernel status word."""
    _need_cuda(A8, As, B8, Bs)
    M, K = A8.shape
    N = B8.shape[0]
    if B8.shape[1] != K:
        raise ValueError("A and B disagree on K")
    C = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=A8.device)
    ws = workspace if workspace is not None else _workspace(OP_BLOCK_GEMM, A8.device, M, N)
    _check(lib().fp4_block_gemm_e4m3(M, N, K, _ptr(A8), _ptr(As), _ptr(B8), _ptr(Bs), _ptr(C), C.stride(0),
                                     _ptr(ws), ws.numel(), _stream(stream)))
    return C, ws

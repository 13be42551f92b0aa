"""CPU oracle for block-scaled 4-bit microscaling.

TEST INFRASTRUCTURE: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA library.  The arithmetic
lives in ``fp4_oracle.c`` (plain C, fp32 steps written out, encoders by lattice enumeration);
this module only builds it, marshals numpy arrays and adds the fp64 GEMM reference and the
tensor-core scale layout.

Sources: "Sub-4-Bit Microscaling (NVFP4, MXFP4 & Walsh-Hadamard Rotation)" §1-§3; "MXFP4
Quantization: Audit the 4.25-Bit Blocks"; metrale ``hardware::exec`` docs; podcast "Adaptive
Block-Scaled Data Types for FP4 Training"; Salmon et al., SC'11 (Philox).

Parity status: every function is pinned by a test in ``tests/test_oracle_*.py`` except the
NVFP4-vs-MXFP4 "~2.4x lower block MSE" figure, which is reported as context only (parity
unpinned: the page gives no data distribution).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

MXFP4, NVFP4, IF4 = 0, 1, 2
RNE, STOCHASTIC = 0, 1
OCP_FLOOR, NOSAT_CEIL = 0, 1


def build(force: bool = False) -> str:
    """Compile fp4_oracle.c into liboracle.so (gcc, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
               "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


class _Counts(ctypes.Structure):
    _fields_ = [("underflow", ctypes.c_uint64), ("saturation", ctypes.c_uint64),
                ("nonfinite", ctypes.c_uint64), ("blocks_four", ctypes.c_uint64)]

    def as_dict(self):
        return {k: int(getattr(self, k)) for k, _ in self._fields_}


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = configure(ctypes.CDLL(build()))
    return _lib


def configure(L: ctypes.CDLL) -> ctypes.CDLL:
    """Declare the C signatures on a loaded copy of the oracle library."""
    P = ctypes.c_void_p
    L.ora_e2m1_value.restype = ctypes.c_double
    L.ora_e2m1_value.argtypes = [ctypes.c_int]
    L.ora_e2m1_encode_rne.restype = ctypes.c_int
    L.ora_e2m1_encode_rne.argtypes = [ctypes.c_float]
    L.ora_e2m1_encode_sr.restype = ctypes.c_int
    L.ora_e2m1_encode_sr.argtypes = [ctypes.c_float, ctypes.c_uint32]
    L.ora_int4_value.restype = ctypes.c_double
    L.ora_int4_value.argtypes = [ctypes.c_int]
    L.ora_int4_encode_rne.restype = ctypes.c_int
    L.ora_int4_encode_rne.argtypes = [ctypes.c_float]
    L.ora_e4m3_value.restype = ctypes.c_double
    L.ora_e4m3_value.argtypes = [ctypes.c_int]
    L.ora_e4m3_encode_rne_satfinite.restype = ctypes.c_int
    L.ora_e4m3_encode_rne_satfinite.argtypes = [ctypes.c_float]
    L.ora_f32_to_bf16_rne.restype = ctypes.c_uint16
    L.ora_f32_to_bf16_rne.argtypes = [ctypes.c_float]
    L.ora_philox4x32_10.restype = None
    L.ora_philox4x32_10.argtypes = [P, P, P]
    L.ora_sr_word.restype = ctypes.c_uint32
    L.ora_sr_word.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
    L.ora_mx_exponent.restype = ctypes.c_int
    L.ora_mx_exponent.argtypes = [ctypes.c_float, ctypes.c_int]
    L.ora_mx_encode_block.restype = None
    L.ora_mx_encode_block.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_uint64,
                                      ctypes.c_uint64, P, P]
    L.ora_mx_quantize.restype = None
    L.ora_mx_quantize.argtypes = [P, ctypes.c_long, ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                  ctypes.c_uint64, P, P, P]
    L.ora_mx_quantize_at.restype = None
    L.ora_mx_quantize_at.argtypes = [P, ctypes.c_long, ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_uint64, ctypes.c_uint64, P, P, P, P]
    L.ora_nvfp4_global_scale.restype = ctypes.c_float
    L.ora_nvfp4_global_scale.argtypes = [ctypes.c_float, ctypes.c_int]
    L.ora_nvfp4_quantize.restype = None
    L.ora_nvfp4_quantize.argtypes = [P, ctypes.c_long, ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_uint64, P, P, P, P, P]
    L.ora_nvfp4_quantize_spec.restype = None
    L.ora_nvfp4_quantize_spec.argtypes = [P, ctypes.c_long, ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_uint64, P, P, P, P, P, P]
    L.ora_block_nonfinite.restype = ctypes.c_int
    L.ora_block_nonfinite.argtypes = [P, ctypes.c_int]
    L.ora_dequantize.restype = None
    L.ora_dequantize.argtypes = [P, P, ctypes.c_int, ctypes.c_long, ctypes.c_long, ctypes.c_float, P]
    L.ora_dequantize_f64.restype = None
    L.ora_dequantize_f64.argtypes = [P, P, ctypes.c_int, ctypes.c_long, ctypes.c_long, ctypes.c_float, P]
    L.ora_e2m1_to_e4m3.restype = None
    L.ora_e2m1_to_e4m3.argtypes = [P, ctypes.c_long, ctypes.c_long, P]
    L.ora_fwht_norm_const.restype = ctypes.c_float
    L.ora_fwht_norm_const.argtypes = [ctypes.c_long]
    L.ora_fwht_rows.restype = None
    L.ora_fwht_rows.argtypes = [P, ctypes.c_long, ctypes.c_long, P]
    L.ora_rht_rows.restype = None
    L.ora_rht_rows.argtypes = [P, ctypes.c_long, ctypes.c_long, P, P]
    L.ora_exp_cw.restype = ctypes.c_float
    L.ora_exp_cw.argtypes = [ctypes.c_float]
    L.ora_silu_mul_rows.restype = None
    L.ora_silu_mul_rows.argtypes = [P, P, ctypes.c_long, P]
    return L


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f32(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    return x


# ----------------------------------------------------------------------------------------------
# Scalars and tables

def e2m1_value(code: int) -> float:
    return lib().ora_e2m1_value(int(code))


def e2m1_encode_rne(y: float) -> int:
    return lib().ora_e2m1_encode_rne(float(y))


def e2m1_encode_sr(y: float, r: int) -> int:
    return lib().ora_e2m1_encode_sr(float(y), int(r))


def int4_value(code: int) -> float:
    """Value of a sign-magnitude INT4 nibble of IF4 (-7..7, bit 3 the sign)."""
    return lib().ora_int4_value(int(code))


def int4_encode_rne(y: float) -> int:
    """IF4's INT4 nibble for a value already divided by the integer step."""
    return lib().ora_int4_encode_rne(float(y))


def e4m3_value(code: int) -> float:
    return lib().ora_e4m3_value(int(code))


def e4m3_encode(u: float) -> int:
    return lib().ora_e4m3_encode_rne_satfinite(float(u))


def f32_to_bf16_bits(f: float) -> int:
    return lib().ora_f32_to_bf16_rne(float(f))


def philox4x32_10(counter, key):
    c = np.ascontiguousarray(counter, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    out = np.zeros(4, dtype=np.uint32)
    lib().ora_philox4x32_10(_p(c), _p(k), _p(out))
    return out


def sr_word(seed: int, idx: int) -> int:
    return lib().ora_sr_word(int(seed), int(idx))


def mx_exponent(amax: float, policy: int = OCP_FLOOR) -> int:
    return lib().ora_mx_exponent(float(amax), int(policy))


def nvfp4_global_scale(amax_t: float, four_six: bool = False) -> float:
    return lib().ora_nvfp4_global_scale(float(amax_t), int(bool(four_six)))


def fwht_norm_const(d: int) -> float:
    return lib().ora_fwht_norm_const(int(d))


# ----------------------------------------------------------------------------------------------
# Tensor operations (numpy in, numpy out)

def mx_encode_block(x, e: int, round: int = RNE, seed: int = 0, idx0: int = 0):
    """Manual-exponent MXFP4 encode of one block (unpacked codes) + counters."""
    x = _f32(x)
    codes = np.zeros(x.size, dtype=np.uint8)
    c = _Counts()
    lib().ora_mx_encode_block(_p(x), x.size, int(e), int(round), int(seed), int(idx0), _p(codes),
                              ctypes.byref(c))
    return codes, c.as_dict()


def mx_quantize(x, policy: int = OCP_FLOOR, round: int = RNE, seed: int = 0, spec: bool = False):
    """MXFP4 quantise a [rows, cols] array. Returns (q [rows, cols/2] u8, scales [rows, cols/32] u8,
    counts), and with `spec` also the bool [rows, cols/32] mask of blocks whose outputs are defined
    (False for a rejected block, one holding Inf or NaN: its codes and scale are left open)."""
    return mx_quantize_rows_at(x, 0, policy=policy, round=round, seed=seed, spec=spec)


def mx_quantize_rows_at(x, idx_base: int, policy: int = OCP_FLOOR, round: int = RNE, seed: int = 0,
                        spec: bool = False):
    """mx_quantize of rows that start at flat element index `idx_base` of a larger tensor (the
    random words of stochastic rounding follow the flat index)."""
    x = _f32(x)
    rows, cols = x.shape
    assert cols % 32 == 0
    q = np.zeros((rows, cols // 2), dtype=np.uint8)
    s = np.zeros((rows, cols // 32), dtype=np.uint8)
    m = np.zeros((rows, cols // 32), dtype=np.uint8)
    c = _Counts()
    lib().ora_mx_quantize_at(_p(x), rows, cols, int(policy), int(round), int(seed), int(idx_base), _p(q), _p(s),
                             ctypes.byref(c), _p(m))
    return (q, s, c.as_dict(), m.astype(bool)) if spec else (q, s, c.as_dict())


def nvfp4_quantize(x, round: int = RNE, four_six: bool = False, seed: int = 0, global_in=None, if4: bool = False,
                   spec: bool = False):
    """NVFP4 quantise (with `if4`, IF4: each block E2M1 or INT4, the choice in scale bit 7).
    Returns (q, scales [rows, cols/16], s_g, counts), and with `spec` also the bool [rows, cols/16]
    mask of blocks whose outputs are defined (see ora_nvfp4_quantize_spec)."""
    assert not (four_six and if4)
    mode = 2 if if4 else int(bool(four_six))
    x = _f32(x)
    rows, cols = x.shape
    assert cols % 16 == 0
    q = np.zeros((rows, cols // 2), dtype=np.uint8)
    s = np.zeros((rows, cols // 16), dtype=np.uint8)
    gin = None if global_in is None else np.array([global_in], dtype=np.float32)
    gout = np.zeros(1, dtype=np.float32)
    m = np.zeros((rows, cols // 16), dtype=np.uint8)
    c = _Counts()
    lib().ora_nvfp4_quantize_spec(_p(x), rows, cols, int(round), mode, int(seed),
                                  None if gin is None else _p(gin), _p(gout), _p(q), _p(s), ctypes.byref(c), _p(m))
    out = (q, s, float(gout[0]), c.as_dict())
    return out + (m.astype(bool),) if spec else out


def dequantize(q, scales, fmt: int, s_g: float = 1.0) -> np.ndarray:
    """fp32 reconstruction fl(fl(v*d)*s_g) (NVFP4) / v*2^e (MXFP4); IF4 blocks flagged INT4 in
    scale bit 7 give fl(fl(k*d)*fl(s_g*fl(6/7)))."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, half = q.shape
    out = np.zeros((rows, half * 2), dtype=np.float32)
    lib().ora_dequantize(_p(q), _p(scales), int(fmt), rows, half * 2, float(s_g), _p(out))
    return out


def dequantize_f64(q, scales, fmt: int, s_g: float = 1.0) -> np.ndarray:
    """Exact fp64 reconstruction v*d*s_g (MXFP4 v*2^e; IF4 INT4 blocks k*d*s_g*6/7)."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, half = q.shape
    out = np.zeros((rows, half * 2), dtype=np.float64)
    lib().ora_dequantize_f64(_p(q), _p(scales), int(fmt), rows, half * 2, float(s_g), _p(out))
    return out


def e2m1_to_e4m3(q) -> np.ndarray:
    """E4M3 byte of value * 2^-6 for every nibble of q [rows, cols/2] -> uint8 [rows, cols]."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    rows, half = q.shape
    out = np.zeros((rows, 2 * half), dtype=np.uint8)
    lib().ora_e2m1_to_e4m3(_p(q), rows, 2 * half, _p(out))
    return out


def fwht(x, signs=None) -> np.ndarray:
    """Normalised Walsh-Hadamard rotation of every row (fixed butterfly order, fp32).  With `signs`
    (uint32 [d/32], bit i negates channel i first) it is the randomised rotation c * H * D."""
    x = _f32(x)
    rows, d = x.shape
    y = np.zeros_like(x)
    if signs is None:
        lib().ora_fwht_rows(_p(x), rows, d, _p(y))
    else:
        sg = np.ascontiguousarray(signs, dtype=np.uint32)
        assert sg.size == d // 32
        lib().ora_rht_rows(_p(x), rows, d, sg.ctypes.data_as(ctypes.c_void_p), _p(y))
    return y


def exp_cw(x: float) -> float:
    """The written-out fp32 exponential used by the SwiGLU activation (Cody-Waite reduction,
    degree-6 Taylor polynomial)."""
    return float(lib().ora_exp_cw(float(np.float32(x))))


def silu_mul(g, u) -> np.ndarray:
    """a = fl(SiLU(g) * u) elementwise in fp32, SiLU(g) = g * fl(1 / fl(1 + exp(-g)))."""
    g, u = _f32(g), _f32(u)
    assert g.shape == u.shape
    a = np.zeros_like(g)
    lib().ora_silu_mul_rows(_p(g), _p(u), g.size, _p(a))
    return a


def swiglu_fwht_quantize(g, u, fmt: int = NVFP4, round: int = RNE, four_six: bool = False, seed: int = 0,
                         global_in=None, signs=None, if4: bool = False, spec: bool = False):
    """SiLU(g) * u in fp32 (no storage rounding), then the rotation and quantiser of fwht_quantize."""
    return fwht_quantize(silu_mul(g, u), fmt=fmt, round=round, four_six=four_six, seed=seed,
                         global_in=global_in, signs=signs, if4=if4, spec=spec)


def fwht_quantize(x, fmt: int = NVFP4, round: int = RNE, four_six: bool = False, seed: int = 0,
                  global_in=None, signs=None, if4: bool = False, spec: bool = False):
    """Rotation (randomised with `signs`) followed by the quantiser of `fmt` on the rotated fp32
    tensor.  Returns (y, q, s, s_g, counts) and, with `spec`, the defined-block mask."""
    y = fwht(x, signs)
    if fmt == NVFP4:
        r = nvfp4_quantize(y, round=round, four_six=four_six, seed=seed, global_in=global_in, if4=if4, spec=spec)
        return (y,) + r
    r = mx_quantize(y, policy=OCP_FLOOR, round=round, seed=seed, spec=spec)
    return (y,) + r[:2] + (1.0,) + r[2:]


def bf16_bits(x) -> np.ndarray:
    """Vector RNE fp32 -> bf16 bit patterns (uint16) through the C definition."""
    x = _f32(x).ravel()
    f = lib().ora_f32_to_bf16_rne
    return np.array([f(float(v)) for v in x], dtype=np.uint16)


# ----------------------------------------------------------------------------------------------
# Tensor-core scale layout (the sm_100 block-scaled MMA's 128 x 4 scale tile, 512 bytes each,
# tiles ordered with the block-column group fastest):
#   off(r, j) = ((r // 128) * (nb // 4) + j // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + j % 4

def scales_to_mma_tiled(scales: np.ndarray) -> np.ndarray:
    rows, nb = scales.shape
    assert rows % 128 == 0 and nb % 4 == 0
    r = np.arange(rows)[:, None]
    j = np.arange(nb)[None, :]
    off = ((r // 128) * (nb // 4) + j // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + j % 4
    out = np.zeros(rows * nb, dtype=np.uint8)
    out[off.ravel()] = scales.ravel()
    return out


def scales_from_mma_tiled(tiled: np.ndarray, rows: int, nb: int) -> np.ndarray:
    r = np.arange(rows)[:, None]
    j = np.arange(nb)[None, :]
    off = ((r // 128) * (nb // 4) + j // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + j % 4
    return np.asarray(tiled).ravel()[off]


# ----------------------------------------------------------------------------------------------
# Block-scaled GEMM reference ("Sub-4-Bit Microscaling" §2: W4A4 on the block-scaled MMA).
# Both operands are dequantised exactly in fp64; C64 = A_hat @ B_hat^T by a library fp64 matmul,
# S = |A_hat| @ |B_hat|^T (the sum of |a*b| that bounds the accepted error).

def gemm_f64(Aq, As, Ag, Bq, Bs, Bg, fmt: int, rows=None, cols=None):
    """Returns (C64, S) for the selected rows of A and rows of B (all when None)."""
    if rows is not None:
        Aq, As = np.asarray(Aq)[rows], np.asarray(As)[rows]
    if cols is not None:
        Bq, Bs = np.asarray(Bq)[cols], np.asarray(Bs)[cols]
    a = dequantize_f64(Aq, As, fmt, 1.0 if fmt == MXFP4 else Ag)
    b = dequantize_f64(Bq, Bs, fmt, 1.0 if fmt == MXFP4 else Bg)
    return a @ b.T, np.abs(a) @ np.abs(b).T

"""GPU parity of the IF4 GEMM (podcast "Adaptive Block-Scaled Data Types for FP4 Training", IF4
segment): blocks flagged INT4 (scale byte bit 7) hold integers on a step six sevenths of the E2M1
unit, so a mixed block pair carries 6/7 and an INT4 pair 36/49.  The library expands both operands
to fp16 (E2M1 blocks exact, INT4 blocks rounded once to fp16) and runs the kind::f16 tensor-core
GEMM; the reference is the oracle's exact fp64 product with the exact factor 6/7.

Bars: the benchmark spec's |C - C64| <= 1e-3 * sum |a b| on quantised data; on single-product operands
|C - C64| <= (2^-8 + 2^-10 + 2^-16) |C64| (bf16 output rounding plus the fp16 rounding of two INT4
elements), and bit-exact bf16(C64) wherever neither block is INT4.
"""
import numpy as np
import pytest
import torch

import block_scaled_fp4_amax_b200 as fp4
import oracle as O
from block_scaled_fp4_amax_b200 import synth
from tests.test_gpu_gemm import bf16_of, check, npy, status_ok, structured_operands

pytestmark = pytest.mark.gpu


def if4_structured(M, N, K, seed):
    """Single-product operands (tests/test_gpu_gemm.py) with each block's INT4 flag drawn at random."""
    Aq, sa, Bq, sb = structured_operands(M, N, K, fp4.NVFP4, seed)
    rng = np.random.default_rng(seed + 1)
    sa = sa | (rng.integers(0, 2, sa.shape) << 7).astype(np.uint8)
    sb = sb | (rng.integers(0, 2, sb.shape) << 7).astype(np.uint8)
    return Aq, sa, Bq, sb


@pytest.mark.parametrize("M", [256, 3968])
def test_if4_gemm_structured(cuda, M):
    """K = 8192; N = 4096 at M = 3968 gives 496 tiles of 128 x 256 over 148 CTAs."""
    N, K = (256, 8192) if M == 256 else (4096, 8192)
    Aq, sa, Bq, sb = if4_structured(M, N, K, seed=M)
    ga, gb = 0.75, 1.25
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(cuda)
    C, ws = fp4.fp4_block_gemm(fp4.IF4, dev(Aq), dev(O.scales_to_mma_tiled(sa)), dev(Bq),
                               dev(O.scales_to_mma_tiled(sb)), torch.tensor([ga], device=cuda),
                               torch.tensor([gb], device=cuda))
    assert status_ok(ws)
    C64, S = O.gemm_f64(Aq, sa, ga, Bq, sb, gb, O.IF4)
    assert np.all(C64 != 0) and np.allclose(np.abs(C64), S, rtol=1e-15, atol=0)
    got = npy(C.float()).astype(np.float64)
    rel = np.abs(got - C64) / np.abs(C64)
    assert rel.max() <= 2.0 ** -8 + 2.0 ** -10 + 2.0 ** -16, float(rel.max())
    # which block pair each output used: group g = (m + n) mod 32, position 8 ((g - m) mod 32) + (g mod 8)
    m = np.arange(M)[:, None]
    n = np.arange(N)[None, :]
    g = (m + n) % 32
    blk = (g * 256 + 8 * ((g - m) % 32) + (g % 8)) // 16
    fp_pair = ((sa[m, blk] & 0x80) == 0) & ((sb[n, blk] & 0x80) == 0)
    assert fp_pair.any() and (~fp_pair).any()
    assert np.array_equal(got[fp_pair], bf16_of(C64)[fp_pair])


@pytest.mark.parametrize("shape", [(128, 256, 256), (256, 512, 1024), (384, 256, 2560), (2048, 2048, 8192)])
@pytest.mark.parametrize("data", ["normal", "outliers"])
def test_if4_gemm_quantised_operands(cuda, shape, data):
    """IF4 operands from the GPU quantiser (checked against the oracle elsewhere), reference from the
    oracle's own IF4 quantisation of the same inputs."""
    M, N, K = shape
    if data == "normal":
        a, b = synth.gemm_operand(M, K, 1), synth.gemm_operand(N, K, 2)
    else:
        a, b = synth.nv_outliers(M, K, seed=5), synth.nv_outliers(N, K, seed=6)
    qa, sa, ga, _ = fp4.nvfp4_quantize(a.to(cuda), if4=True, layout=fp4.MMA_TILED)
    qb, sb, gb, _ = fp4.nvfp4_quantize(b.to(cuda), if4=True, layout=fp4.MMA_TILED)
    C, ws = fp4.fp4_block_gemm(fp4.IF4, qa, sa, qb, sb, ga, gb)
    assert status_ok(ws)
    qao, sao, gao, ca = O.nvfp4_quantize(synth.as_f32_numpy(a), if4=True)
    qbo, sbo, gbo, cb = O.nvfp4_quantize(synth.as_f32_numpy(b), if4=True)
    assert ca["blocks_four"] > 0 and cb["blocks_four"] > 0  # both operands hold INT4 blocks
    C64, S = O.gemm_f64(qao, sao, gao, qbo, sbo, gbo, O.IF4)
    check(C, C64, S)


def test_if4_gemm_without_int4_blocks_matches_nvfp4(cuda):
    """An NVFP4 operand is an IF4 operand with no INT4 block: the IF4 route then sums the same exact
    products as the block-scaled FP4 GEMM, in another order, so the two agree to one bf16 step plus
    an fp32 accumulation term (2^-16 of sum |a b|, computed from the GPU's own dequantisation)."""
    M, N, K = 256, 512, 1024
    A = fp4.nvfp4_quantize(synth.gemm_operand(M, K, 7).to(cuda), layout=fp4.MMA_TILED)
    B = fp4.nvfp4_quantize(synth.gemm_operand(N, K, 8).to(cuda), layout=fp4.MMA_TILED)
    C4, ws = fp4.fp4_block_gemm(fp4.NVFP4, A[0], A[1], B[0], B[1], A[2], B[2])
    assert status_ok(ws)
    C16, ws = fp4.fp4_block_gemm(fp4.IF4, A[0], A[1], B[0], B[1], A[2], B[2])
    assert status_ok(ws)
    Ad = fp4.fp4_dequantize(A[0], A[1], fp4.NVFP4, A[2], layout=fp4.MMA_TILED).double()
    Bd = fp4.fp4_dequantize(B[0], B[1], fp4.NVFP4, B[2], layout=fp4.MMA_TILED).double()
    S = Ad.abs() @ Bd.abs().T
    d = (C4.double() - C16.double()).abs()
    assert torch.all(d <= 2.0 ** -7 * C4.double().abs() + 2.0 ** -16 * S)


def test_if4_gemm_argument_errors(cuda):
    A = fp4.nvfp4_quantize(synth.gemm_operand(128, 256, 9).to(cuda), if4=True, layout=fp4.MMA_TILED)
    B = fp4.nvfp4_quantize(synth.gemm_operand(256, 256, 10).to(cuda), if4=True, layout=fp4.MMA_TILED)
    small = torch.empty(256, dtype=torch.uint8, device=cuda)
    with pytest.raises(fp4.Fp4Error):
        fp4.fp4_block_gemm(fp4.IF4, A[0], A[1], B[0], B[1], A[2], B[2], workspace=small)  # too small
    with pytest.raises(fp4.Fp4Error):
        fp4.fp4_block_gemm(fp4.IF4, A[0], A[1], B[0], B[1])                               # no global scales

"""GPU parity of the FP8 tensor-core route for MXFP4 operands (metrale `hardware::exec`: FP4
operands run exactly on the FP8 MMA after the E2M1 -> E4M3 conversion): the expansion kernel bit-exact
against the oracle's E4M3 encode of value * 2^-6, and the kind::mxf8f6f4 GEMM against the same fp64
reference as the FP4 GEMM (|C - C64| <= 1e-3 * sum |ab|, plus 2^-8 |C64| on small shapes for the bf16
output rounding) and against the FP4 GEMM itself.
"""
import numpy as np
import pytest
import torch

import block_scaled_fp4_amax_b200 as fp4
import oracle as O
from block_scaled_fp4_amax_b200 import synth
from tests.test_gpu_gemm import (check, check_sampled, npy, packed_from_codes, status_ok, structured_operands,
                                  structured_reference)

pytestmark = pytest.mark.gpu


def mx_operand(x_cpu, cuda):
    q, s, _ = fp4.mx_quantize(x_cpu.to(cuda), layout=fp4.MMA_TILED)
    return q, s


def gemm_e4m3(A, B):
    (Aq, As), (Bq, Bs) = A, B
    C, ws = fp4.fp4_block_gemm_e4m3(fp4.fp4_to_e4m3(Aq), As, fp4.fp4_to_e4m3(Bq), Bs)
    assert status_ok(ws)
    return C


def test_expansion_bit_exact(cuda):
    rng = np.random.default_rng(50)
    q = rng.integers(0, 256, size=(96, 512), dtype=np.uint8)         # every nibble pair, 1024 columns
    assert np.array_equal(npy(fp4.fp4_to_e4m3(torch.from_numpy(q).to(cuda))), O.e2m1_to_e4m3(q))
    x = synth.swiglu_act(64, 2048, seed=5)
    qg, _, _ = fp4.mx_quantize(x.to(cuda))
    assert np.array_equal(npy(fp4.fp4_to_e4m3(qg)), O.e2m1_to_e4m3(npy(qg)))
    # 7 rows x 32 columns: 112 packed bytes, a ragged multiple of 16 bytes
    q7 = rng.integers(0, 256, size=(7, 16), dtype=np.uint8)
    assert np.array_equal(npy(fp4.fp4_to_e4m3(torch.from_numpy(q7).to(cuda))), O.e2m1_to_e4m3(q7))


@pytest.mark.parametrize("mn", [(128, 256), (512, 768)])
def test_gemm_e4m3_one_hot_structure(cuda, mn):
    """One nonzero per row of A and of B, distinct E8M0 scales: C is exact, which pins the byte
    order of the expansion, the K order in the swizzled tile and the scale byte chosen per MMA."""
    M, N = mn
    K = 512
    nb = K // 32
    km = (np.arange(M) * 7 + 3) % K
    kn = (np.arange(N) * 5 + 1) % K
    ca = np.zeros((M, K), np.uint8)
    ca[np.arange(M), km] = 2
    cb = np.zeros((N, K), np.uint8)
    cb[np.arange(N), kn] = 2
    rng = np.random.default_rng(0)
    sa = rng.integers(120, 134, size=(M, nb)).astype(np.uint8)
    sb = rng.integers(120, 134, size=(N, nb)).astype(np.uint8)
    A = (torch.from_numpy(packed_from_codes(ca)).to(cuda), torch.from_numpy(O.scales_to_mma_tiled(sa)).to(cuda))
    B = (torch.from_numpy(packed_from_codes(cb)).to(cuda), torch.from_numpy(O.scales_to_mma_tiled(sb)).to(cuda))
    C = gemm_e4m3(A, B)
    C64, _ = O.gemm_f64(packed_from_codes(ca), sa, 1.0, packed_from_codes(cb), sb, 1.0, O.MXFP4)
    assert np.count_nonzero(C64) > 0
    assert np.array_equal(npy(C.float()).astype(np.float64), C64)


@pytest.mark.parametrize("shape", [(128, 256, 128), (256, 512, 1024), (384, 256, 2560)])
def test_gemm_e4m3_small_random_and_against_fp4(cuda, shape):
    M, N, K = shape
    a, b = synth.gemm_operand(M, K, 1), synth.gemm_operand(N, K, 2)
    A, B = mx_operand(a, cuda), mx_operand(b, cuda)
    C = gemm_e4m3(A, B)
    Aq, As, _ = O.mx_quantize(synth.as_f32_numpy(a))
    Bq, Bs, _ = O.mx_quantize(synth.as_f32_numpy(b))
    C64, S = O.gemm_f64(Aq, As, 1.0, Bq, Bs, 1.0, O.MXFP4)
    check(C, C64, S, K=K)
    if K % 256 == 0:  # the FP4 GEMM's stage is 256 values
        C4, ws = fp4.fp4_block_gemm(fp4.MXFP4, A[0], A[1], B[0], B[1])
        assert status_ok(ws)
        diff = np.abs(npy(C.float()).astype(np.float64) - npy(C4.float()).astype(np.float64))
        assert np.all(diff <= 2 * (1e-3 * S + 2.0 ** -8 * np.abs(C64)))


def test_gemm_e4m3_structured_exact_many_tiles(cuda):
    """Single-product operands (see tests/test_gpu_gemm.py) at K = 8192: 64 stages of 128 values
    through the 4-deep ring, 512 tiles of 128 x 256 over 148 CTAs (three or more per CTA).  C must
    equal bf16 of the exact product everywhere."""
    M, N, K = 4096, 4096, 8192
    Aq, sa, Bq, sb = structured_operands(M, N, K, fp4.MXFP4, seed=77)
    want = structured_reference(Aq, sa, Bq, sb, fp4.MXFP4)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(cuda)
    C = gemm_e4m3((dev(Aq), dev(O.scales_to_mma_tiled(sa))), (dev(Bq), dev(O.scales_to_mma_tiled(sb))))
    got = npy(C.float()).astype(np.float64)
    bad = got != want
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} outputs differ (first at {np.argwhere(bad)[0]})"


def test_gemm_e4m3_down_proj_sampled(cuda):
    """The MXFP4 down_proj shape 4096 x 8192 x 28672 on the FP8 route: 8 whole rows and 8 whole
    columns against the fp64 reference, and the whole C against the FP4 GEMM."""
    a, w = synth.swiglu_act(), synth.weight()
    A, B = mx_operand(a, cuda), mx_operand(w, cuda)
    C = gemm_e4m3(A, B)
    rng = np.random.default_rng(43)
    rows, cols = np.sort(rng.choice(4096, 8, replace=False)), np.sort(rng.choice(8192, 8, replace=False))
    check_sampled(C, a, w, fp4.MXFP4, rows, cols)
    C4, ws = fp4.fp4_block_gemm(fp4.MXFP4, A[0], A[1], B[0], B[1])
    assert status_ok(ws)
    rel = (C.float() - C4.float()).abs().max().item() / C4.float().abs().max().item()
    assert rel < 2.0 ** -7

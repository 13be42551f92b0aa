"""GPU parity: the tcgen05 block-scaled GEMM against the fp64 oracle.

Bar: |C_gpu - C64| <= 1e-3 * sum_k |a_k b_k| + ulp(C64)/2 per element, C64 the fp64 dot product of
the exactly dequantised operands and ulp the bf16 unit in the last place: the output is bf16, whose
rounding alone moves it by up to half an ulp (2^-9 |C|), more than 1e-3 * sum |a b| wherever |C| is a
sizeable fraction of sum |a b| (small K).  On zero-mean data the tests also hold the result to one
bf16 rounding step of the exact value plus the fp32 accumulation term: |C_gpu - bf16(C64)| <=
ulp(bf16(C64)) + K * 2^-23 * sum |a b|.  The same-sign test adds 2^-8 |C64| to the first bar.

Structured operands make the pipeline's bookkeeping exact: every output is a single product, so a
dropped, repeated or stale K stage, a wrong barrier phase, an accumulator not reset between the
tiles a CTA takes in turn, or a misplaced scale changes C, and C must equal bf16(C64) bit for bit.
Operands are quantised on the GPU (checked bit-exact against the oracle elsewhere) while the
reference quantises independently on the CPU.
"""
import numpy as np
import pytest
import torch

import block_scaled_fp4_amax_b200 as fp4
import oracle as O
from block_scaled_fp4_amax_b200 import synth

pytestmark = pytest.mark.gpu


def npy(t):
    return t.detach().cpu().numpy()


def status_ok(ws):
    torch.cuda.synchronize()
    return int(ws[:4].view(torch.int32).item()) == 0


def quant(x_cpu, fmt, cuda):
    x = x_cpu.to(cuda)
    if fmt == fp4.NVFP4:
        q, s, g, _ = fp4.nvfp4_quantize(x, layout=fp4.MMA_TILED)
        qo, so, go, _ = O.nvfp4_quantize(synth.as_f32_numpy(x_cpu))
        return (q, s, g), (qo, so, go)
    q, s, _ = fp4.mx_quantize(x, layout=fp4.MMA_TILED)
    qo, so, _ = O.mx_quantize(synth.as_f32_numpy(x_cpu))
    return (q, s, None), (qo, so, 1.0)


def check(C, C64, S, extra_rel=0.0, K=None):
    """The 1e-3 * sum|ab| bar plus the bf16 output rounding (half an ulp; plus `extra_rel` * |C64|
    for same-sign data); with K, also the bf16-aware bar |C - bf16(C64)| <= ulp(bf16(C64)) +
    K * 2^-23 * S."""
    got = npy(C.float()).astype(np.float64)
    err = np.abs(got - C64)
    bound = 1e-3 * S + 0.5 * bf16_ulp(C64) + extra_rel * np.abs(C64)
    bad = err > bound
    assert not bad.any(), f"{bad.sum()} of {bad.size} outside the bound; worst excess {float((err - bound).max())}"
    if K is not None:
        check_bf16_tight(got, C64, S, K)


def bf16_of(C64):
    """Round-to-nearest-even bf16 of fp64 values (through fp32: exact for values with few bits)."""
    return torch.from_numpy(np.ascontiguousarray(C64, dtype=np.float64)).to(torch.bfloat16).double().numpy()


def bf16_ulp(v):
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (e - 7), 2.0 ** -133)


def check_bf16_tight(got, C64, S, K):
    ref = bf16_of(C64)
    err = np.abs(got - ref)
    bound = bf16_ulp(ref) + K * 2.0 ** -23 * S
    bad = err > bound
    assert not bad.any(), f"{bad.sum()} of {bad.size} outside ulp + K 2^-23 S; worst excess {float((err - bound).max())}"


def gemm(fmt, A, B):
    (Aq, As, Ag), (Bq, Bs, Bg) = A, B
    C, ws = fp4.fp4_block_gemm(fmt, Aq, As, Bq, Bs, Ag, Bg)
    assert status_ok(ws)
    return C


def packed_from_codes(codes):
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[:, 0::2] & 15) | ((codes[:, 1::2] & 15) << 4)


@pytest.mark.parametrize("fmt", [fp4.NVFP4, fp4.MXFP4])
@pytest.mark.parametrize("mn", [(128, 256), (256, 256), (512, 768)])  # 1-SM tiles; 2-SM pair tiles
def test_gemm_one_hot_structure(cuda, fmt, mn):
    """A[m, k] = 1 only at k = km(m); B[n, k] = 1 only at k = kn(n); every block scale distinct, so
    C[m, n] = dA[m, km/B] * dB[n, km/B] when km(m) == kn(n), else 0 — an exact bf16 value.  This
    pins the nibble order inside a byte, the K order inside the swizzled tile and the scale-tile
    layout of both operands."""
    M, N = mn
    K = 512
    Bk = 16 if fmt == fp4.NVFP4 else 32
    nb = K // Bk
    km = (np.arange(M) * 7 + 3) % K
    kn = (np.arange(N) * 5 + 1) % K
    ca = np.zeros((M, K), np.uint8)
    ca[np.arange(M), km] = 2  # code 2 = 1.0
    cb = np.zeros((N, K), np.uint8)
    cb[np.arange(N), kn] = 2
    rng = np.random.default_rng(0)
    if fmt == fp4.NVFP4:
        sa = rng.integers(0x20, 0x50, size=(M, nb)).astype(np.uint8)   # E4M3 2^-3 .. 2^3
        sb = rng.integers(0x20, 0x50, size=(N, nb)).astype(np.uint8)
    else:
        sa = rng.integers(120, 134, size=(M, nb)).astype(np.uint8)     # E8M0 2^-7 .. 2^6
        sb = rng.integers(120, 134, size=(N, nb)).astype(np.uint8)
    Aq = torch.from_numpy(packed_from_codes(ca)).to(cuda)
    Bq = torch.from_numpy(packed_from_codes(cb)).to(cuda)
    As = torch.from_numpy(O.scales_to_mma_tiled(sa)).to(cuda)
    Bs = torch.from_numpy(O.scales_to_mma_tiled(sb)).to(cuda)
    one = torch.ones(1, dtype=torch.float32, device=cuda)
    C = gemm(fmt, (Aq, As, one), (Bq, Bs, one))
    C64, S = O.gemm_f64(packed_from_codes(ca), sa, 1.0, packed_from_codes(cb), sb, 1.0, fmt)
    got = npy(C.float()).astype(np.float64)
    assert np.count_nonzero(C64) > 0
    assert np.array_equal(got, C64)


@pytest.mark.parametrize("fmt", [fp4.NVFP4, fp4.MXFP4])
@pytest.mark.parametrize("shape", [(128, 256, 256), (256, 512, 1024), (384, 256, 2560)])
def test_gemm_small_random(cuda, fmt, shape):
    M, N, K = shape
    A, Ao = quant(synth.gemm_operand(M, K, 1), fmt, cuda)
    B, Bo = quant(synth.gemm_operand(N, K, 2), fmt, cuda)
    C = gemm(fmt, A, B)
    C64, S = O.gemm_f64(Ao[0], Ao[1], Ao[2], Bo[0], Bo[1], Bo[2], fmt)
    check(C, C64, S, K=K)


def structured_operands(M, N, K, fmt, seed):
    """Codes and row-major scales with exactly one nonzero product per output.  K = 8192 is 32
    groups of 256 values.  In group g, row m of A holds one nonzero value at 8 ((g - m) mod 32) +
    (g mod 8) and row n of B one at 8 (n mod 32) + (g mod 8): they meet only in the group
    g = (m + n) mod 32, so C[m, n] is that single product (exact in fp32), every output is nonzero,
    and every group and every 16- or 32-value block position takes part somewhere.  Values are
    lattice points of both signs; every block scale is drawn independently."""
    assert K == 8192
    G = K // 256
    rng = np.random.default_rng(seed)
    Bk = 16 if fmt == fp4.NVFP4 else 32
    g = np.arange(G)
    ca = np.zeros((M, K), np.uint8)
    cb = np.zeros((N, K), np.uint8)
    m = np.arange(M)[:, None]
    n = np.arange(N)[:, None]
    pa = g * 256 + 8 * ((g - m) % 32) + (g % 8)
    pb = g * 256 + 8 * (n % 32) + (g % 8)
    code = lambda shape: (rng.integers(1, 8, shape) | (rng.integers(0, 2, shape) << 3)).astype(np.uint8)
    np.put_along_axis(ca, pa, code((M, G)), axis=1)
    np.put_along_axis(cb, np.broadcast_to(pb, (N, G)), code((N, G)), axis=1)
    if fmt == fp4.NVFP4:
        sa = rng.integers(0x20, 0x50, size=(M, K // Bk)).astype(np.uint8)   # E4M3 2^-3 .. 7.5
        sb = rng.integers(0x20, 0x50, size=(N, K // Bk)).astype(np.uint8)
    else:
        sa = rng.integers(120, 134, size=(M, K // Bk)).astype(np.uint8)     # E8M0 2^-7 .. 2^6
        sb = rng.integers(120, 134, size=(N, K // Bk)).astype(np.uint8)
    return packed_from_codes(ca), sa, packed_from_codes(cb), sb


def structured_reference(Aq, sa, Bq, sb, fmt):
    C64, S = O.gemm_f64(Aq, sa, 1.0, Bq, sb, 1.0, fmt)
    assert np.all(C64 != 0) and np.array_equal(np.abs(C64), S)  # one product per output
    return bf16_of(C64)


@pytest.mark.parametrize("fmt", [fp4.NVFP4, fp4.MXFP4])
@pytest.mark.parametrize("M", [4096, 3968])  # 2-SM pair tiles (256 x 256); 1-SM tiles (M % 256 == 128)
def test_gemm_structured_exact_many_tiles(cuda, fmt, M):
    """K = 8192 (32 stages of 256 values through a 4-6 deep ring, so its barriers change phase many
    times per tile); N = 4096, so every cluster (pair kernel: 256 tiles over 74 clusters) or CTA
    (1-SM kernel: 496 tiles over 148 CTAs) computes three or more tiles in turn, re-using its
    accumulator and scale slots.  C must equal bf16 of the exact product everywhere."""
    N, K = 4096, 8192
    Aq, sa, Bq, sb = structured_operands(M, N, K, fmt, seed=M + fmt)
    want = structured_reference(Aq, sa, Bq, sb, fmt)
    one = torch.ones(1, dtype=torch.float32, device=cuda)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(cuda)
    C = gemm(fmt, (dev(Aq), dev(O.scales_to_mma_tiled(sa)), one), (dev(Bq), dev(O.scales_to_mma_tiled(sb)), one))
    got = npy(C.float()).astype(np.float64)
    bad = got != want
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} outputs differ (first at {np.argwhere(bad)[0]})"


def test_gemm_positive_data_bf16_rounding(cuda):
    """Same-sign operands (|C| ~ sum |ab|): the tolerance then includes bf16 output rounding."""
    M, N, K = 128, 256, 1024
    a = synth.normal_f32(M, K, 3).abs().to(torch.bfloat16)
    b = synth.normal_f32(N, K, 4).abs().to(torch.bfloat16)
    A, Ao = quant(a, fp4.NVFP4, cuda)
    B, Bo = quant(b, fp4.NVFP4, cuda)
    C = gemm(fp4.NVFP4, A, B)
    C64, S = O.gemm_f64(Ao[0], Ao[1], Ao[2], Bo[0], Bo[1], Bo[2], fp4.NVFP4)
    check(C, C64, S, extra_rel=2.0 ** -8)


def test_gemm_nvfp4_config4_sampled(cuda):
    """M = N = K = 8192 NVFP4 (A seed 1, B seed 2): 8 whole rows and 8 whole columns of C."""
    M = N = K = 8192
    a, b = synth.gemm_operand(M, K, 1), synth.gemm_operand(N, K, 2)
    A, _ = quant_gpu_only(a, fp4.NVFP4, cuda)
    B, _ = quant_gpu_only(b, fp4.NVFP4, cuda)
    C = gemm(fp4.NVFP4, A, B)
    rng = np.random.default_rng(42)
    rows, cols = np.sort(rng.choice(M, 8, replace=False)), np.sort(rng.choice(N, 8, replace=False))
    check_sampled(C, a, b, fp4.NVFP4, rows, cols)


def test_gemm_mxfp4_config5_sampled(cuda):
    """down_proj shape M = 4096, N = 8192, K = 28672, MXFP4 (E8M0 per 32): activations
    bf16(silu(g) * u) (seed 3), weights N(0, 0.02) (seed 4).  8 rows and 8 columns of C."""
    a, w = synth.swiglu_act(), synth.weight()
    A, _ = quant_gpu_only(a, fp4.MXFP4, cuda)
    B, _ = quant_gpu_only(w, fp4.MXFP4, cuda)
    C = gemm(fp4.MXFP4, A, B)
    rng = np.random.default_rng(43)
    rows, cols = np.sort(rng.choice(4096, 8, replace=False)), np.sort(rng.choice(8192, 8, replace=False))
    check_sampled(C, a, w, fp4.MXFP4, rows, cols)


def quant_gpu_only(x_cpu, fmt, cuda):
    x = x_cpu.to(cuda)
    if fmt == fp4.NVFP4:
        q, s, g, _ = fp4.nvfp4_quantize(x, layout=fp4.MMA_TILED)
        return (q, s, g), None
    q, s, _ = fp4.mx_quantize(x, layout=fp4.MMA_TILED)
    return (q, s, None), None


def check_sampled(C, a_cpu, b_cpu, fmt, rows, cols):
    """Reference for whole sampled rows (all N) and whole sampled columns (all M)."""
    def oq(x):
        if fmt == fp4.NVFP4:
            q, s, g, _ = O.nvfp4_quantize(synth.as_f32_numpy(x))
            return q, s, g
        q, s, _ = O.mx_quantize(synth.as_f32_numpy(x))
        return q, s, 1.0

    # the global scale of each operand comes from its full tensor
    Aq, As, Ag = oq(a_cpu)
    Bq, Bs, Bg = oq(b_cpu)
    Cn = npy(C.float()).astype(np.float64)
    K = 2 * Aq.shape[1]
    C64, S = O.gemm_f64(Aq, As, Ag, Bq, Bs, Bg, fmt, rows=rows)
    err = np.abs(Cn[rows] - C64)
    assert np.all(err <= 1e-3 * S), float((err - 1e-3 * S).max())
    check_bf16_tight(Cn[rows], C64, S, K)
    C64, S = O.gemm_f64(Aq, As, Ag, Bq, Bs, Bg, fmt, cols=cols)
    err = np.abs(Cn[:, cols] - C64)
    assert np.all(err <= 1e-3 * S), float((err - 1e-3 * S).max())
    check_bf16_tight(Cn[:, cols], C64, S, K)


def test_gemm_wait_limit_reports_and_recovers(cuda):
    """Every pipeline wait of the GEMM kernels is bounded.  With a limit of 0 ns the first wait that
    has not completed already gives up: the call returns, the status word names the wait site, and
    the kernel has drained what it issued and freed tensor memory, so the same stream then runs a
    normal GEMM (single-product operands, exact) with the default limit restored."""
    M, N, K = 128, 256, 256           # the 1-SM kernel, one tile, one K stage
    A, _ = quant(synth.gemm_operand(M, K, 5), fp4.NVFP4, cuda)
    B, _ = quant(synth.gemm_operand(N, K, 6), fp4.NVFP4, cuda)
    old = fp4.set_gemm_wait_limit(0)
    try:
        _, ws = fp4.fp4_block_gemm(fp4.NVFP4, A[0], A[1], B[0], B[1], A[2], B[2])
        torch.cuda.synchronize()
    finally:
        assert fp4.set_gemm_wait_limit(old) == 0
    word = int(ws[:4].view(torch.int32).item())
    assert word != 0 and word & ~0x3FF == 0, hex(word)   # one or more of the sites 0-9
    # the context is intact: an exact GEMM on the same stream
    Mx, Nx, Kx = 128, 256, 512
    km = (np.arange(Mx) * 7 + 3) % Kx
    kn = (np.arange(Nx) * 5 + 1) % Kx
    ca = np.zeros((Mx, Kx), np.uint8)
    ca[np.arange(Mx), km] = 2
    cb = np.zeros((Nx, Kx), np.uint8)
    cb[np.arange(Nx), kn] = 2
    rng = np.random.default_rng(1)
    sa = rng.integers(0x20, 0x50, size=(Mx, Kx // 16)).astype(np.uint8)
    sb = rng.integers(0x20, 0x50, size=(Nx, Kx // 16)).astype(np.uint8)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(cuda)
    one = torch.ones(1, dtype=torch.float32, device=cuda)
    C = gemm(fp4.NVFP4, (dev(packed_from_codes(ca)), dev(O.scales_to_mma_tiled(sa)), one),
             (dev(packed_from_codes(cb)), dev(O.scales_to_mma_tiled(sb)), one))
    C64, _ = O.gemm_f64(packed_from_codes(ca), sa, 1.0, packed_from_codes(cb), sb, 1.0, fp4.NVFP4)
    assert np.array_equal(npy(C.float()).astype(np.float64), C64)


def test_gemm_ldc_and_status_word(cuda):
    """A wider output buffer (ldc > N): columns beyond N stay untouched; the status word is 0."""
    M, N, K = 128, 256, 256
    A, Ao = quant(synth.gemm_operand(M, K, 5), fp4.NVFP4, cuda)
    B, Bo = quant(synth.gemm_operand(N, K, 6), fp4.NVFP4, cuda)
    big = torch.full((M, N + 64), 7.0, dtype=torch.bfloat16, device=cuda)
    C, ws = fp4.fp4_block_gemm(fp4.NVFP4, A[0], A[1], B[0], B[1], A[2], B[2], out=big[:, :N])
    assert status_ok(ws)
    assert torch.all(big[:, N:] == 7.0)
    C64, S = O.gemm_f64(Ao[0], Ao[1], Ao[2], Bo[0], Bo[1], Bo[2], fp4.NVFP4)
    check(big[:, :N], C64, S, K=K)


def test_gemm_output_beyond_2p31_elements(cuda):
    """M = 65792, N = 32768, K = 256 NVFP4: 2,155,872,256 bf16 outputs, rows from 65536 on lying
    wholly past element 2^31 of C.  Sampled rows on both sides of the boundary against the fp64
    product of the exactly dequantised operands (1e-3 sum|ab| plus the bf16 rounding term)."""
    M, N, K = 65792, 32768, 256
    a = synth.gemm_operand(M, K, 61)
    b = synth.gemm_operand(N, K, 62)
    qa, sa, ga, _ = fp4.nvfp4_quantize(a.to(cuda), layout=fp4.MMA_TILED)
    qb, sb, gb, _ = fp4.nvfp4_quantize(b.to(cuda), layout=fp4.MMA_TILED)
    C, ws = fp4.fp4_block_gemm(fp4.NVFP4, qa, sa, qb, sb, ga, gb)
    assert status_ok(ws) and C.numel() > 2 ** 31
    rows = [0, 65535, 65536, M - 1]
    qo, so, go, _ = O.nvfp4_quantize(synth.as_f32_numpy(a))        # whole A: its own global scale
    A64 = O.dequantize(qo[rows], so[rows], O.NVFP4, go).astype(np.float64)
    qbo, sbo, gbo, _ = O.nvfp4_quantize(synth.as_f32_numpy(b))
    B64 = O.dequantize(qbo, sbo, O.NVFP4, gbo).astype(np.float64)
    C64 = A64 @ B64.T
    S = np.abs(A64) @ np.abs(B64).T
    check(C[rows], C64, S, K=K)
    del C

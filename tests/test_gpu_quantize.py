"""GPU parity: quantisers, Walsh-Hadamard rotation and dequantiser against the CPU oracle.

Bar: packed nibbles, scale bytes, the global scale and all counters bit-exact (stochastic
rounding included); rotated and dequantised values bit-exact (the stated bar is 1e-6 relative;
both sides follow the same fp32 operation order, so they agree exactly).  Blocks holding Inf or
NaN are rejected: their codes and scales are left open and only the non-finite count covers them
(tests/parity.py).  Every call goes through the C ABI via the thin binding.
"""
import numpy as np
import pytest
import torch

import block_scaled_fp4_amax_b200 as fp4
import oracle as O
from block_scaled_fp4_amax_b200 import synth
from tests.parity import compare_blocks, compare_counts, rowmajor_scales

pytestmark = pytest.mark.gpu


def npy(t):
    return t.detach().cpu().numpy()


def counts_of(c):
    v = [int(x) for x in c.cpu().tolist()]
    return dict(underflow=v[0], saturation=v[1], nonfinite=v[2], blocks_four=v[3])


def f32(t_cpu):
    return synth.as_f32_numpy(t_cpu)


def check_scales(gpu_scales, ora_scales, layout):
    rows, nb = ora_scales.shape
    want = O.scales_to_mma_tiled(ora_scales) if layout == fp4.MMA_TILED else ora_scales.ravel()
    assert np.array_equal(npy(gpu_scales), want)


def run_mx(x_cpu, cuda, policy=fp4.OCP_FLOOR, rnd=fp4.RNE, seed=0, layout=fp4.ROWMAJOR):
    q, s, c = fp4.mx_quantize(x_cpu.to(cuda), policy=policy, round=rnd, seed=seed, layout=layout)
    x = f32(x_cpu)
    qo, so, co, spec = O.mx_quantize(x, policy=policy, round=rnd, seed=seed, spec=True)
    if spec.all():
        assert np.array_equal(npy(q), qo)
        check_scales(s, so, layout)
    else:
        compare_blocks(q, s, qo, so, spec, 32, layout)
    compare_counts(c, co, x, spec, 32)
    return q, s, qo, so


def run_nv(x_cpu, cuda, rnd=fp4.RNE, four_six=False, seed=0, layout=fp4.ROWMAJOR, global_in=None):
    gin = None if global_in is None else torch.tensor([global_in], dtype=torch.float32, device=cuda)
    q, s, g, c = fp4.nvfp4_quantize(x_cpu.to(cuda), round=rnd, four_six=four_six, seed=seed, layout=layout,
                                    global_in=gin)
    x = f32(x_cpu)
    qo, so, go, co, spec = O.nvfp4_quantize(x, round=rnd, four_six=four_six, seed=seed, global_in=global_in,
                                            spec=True)
    assert np.array_equal(np.float32(npy(g)[0]), np.float32(go), equal_nan=True)
    if spec.all():
        assert np.array_equal(npy(q), qo)
        check_scales(s, so, layout)
    else:
        compare_blocks(q, s, qo, so, spec, 16, layout)
    compare_counts(c, co, x, spec, 16)
    return q, s, g, qo, so, go


# ---------------------------------------------------------------------------------------------
# The hardware conversions against the oracle's enumerated encoders

def test_e2m1_encoder_exhaustive_band(cuda):
    """Every fp32 with |y| in [2^-4, 8) (all mantissas, both signs) through the MXFP4 path with a
    4.0 anchor per block (exponent 0, so y = x): nibbles and counters bit-exact."""
    bits = np.arange(123 << 23, 130 << 23, dtype=np.uint32)
    vals = bits.view(np.float32)
    vals = np.concatenate([vals, -vals, np.float32([0.0, -0.0, 1e-30, -1e-30, 2.0 ** -149])])
    n = len(vals)
    nblk = -(-n // 31)
    x = np.zeros((nblk, 32), dtype=np.float32)
    x[:, 0] = 4.0
    flat = np.zeros(nblk * 31, dtype=np.float32)
    flat[:n] = vals
    x[:, 1:] = flat.reshape(nblk, 31)
    rows = nblk // 64 * 64
    xt = torch.from_numpy(x[:rows].reshape(-1, 32 * 64).copy())
    run_mx(xt, cuda)


def test_e4m3_scale_encoder_midpoints(cuda):
    """NVFP4 with s_g = fl(1/6): fl(6 s_g) == 1, so the scale code is the E4M3 encoding of the block
    amax itself.  All E4M3 midpoints (ties) +-2 ulp, every code value, and a dense random set."""
    sg = float(np.float32(1.0 / 6.0))
    assert np.float32(6.0) * np.float32(sg) == np.float32(1.0)
    vals = np.array([O.e4m3_value(c) for c in range(0x7F)])
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    near = np.concatenate([np.nextafter(mids, np.float32(np.inf)), np.nextafter(mids, np.float32(0)), mids])
    u = np.concatenate([near, vals.astype(np.float32), np.float32([448.5, 464, 500, 1e6]),
                        (2.0 ** np.random.default_rng(0).uniform(-11, 9, 200000)).astype(np.float32)])
    n = (len(u) // 64 + 1) * 64
    u = np.concatenate([u, np.full(n - len(u), 1.0, np.float32)])
    x = np.zeros((n, 16), dtype=np.float32)
    x[:, 0] = u
    x[:, 1] = u * np.float32(0.3)
    run_nv(torch.from_numpy(x.reshape(-1, 16 * 64).copy()), cuda, global_in=sg)


# ---------------------------------------------------------------------------------------------
# MXFP4

@pytest.mark.parametrize("policy", [fp4.OCP_FLOOR, fp4.NOSAT_CEIL])
@pytest.mark.parametrize("rnd", [fp4.RNE, fp4.STOCHASTIC])
@pytest.mark.parametrize("layout", [fp4.ROWMAJOR, fp4.MMA_TILED])
def test_mx_config1_fp32(cuda, policy, rnd, layout):
    x = synth.mx_small()  # 256 x 512 fp32 N(0,1), seed 0
    q, s, qo, so = run_mx(x, cuda, policy=policy, rnd=rnd, seed=11, layout=layout)
    out = fp4.fp4_dequantize(q, s, fp4.MXFP4, layout=layout)
    assert np.array_equal(npy(out), O.dequantize(qo, so, O.MXFP4))


@pytest.mark.parametrize("rnd", [fp4.RNE, fp4.STOCHASTIC])
def test_mx_bf16_scaled_and_ragged(cuda, rnd):
    x = (synth.normal_f32(384, 1024, 21) * 37.0).to(torch.bfloat16)
    run_mx(x, cuda, rnd=rnd, seed=5)
    run_mx(synth.normal_bf16(3, 96, 22), cuda, rnd=rnd, seed=5)        # 3 rows, 3 blocks per row
    run_mx(synth.normal_bf16(1, 32, 23), cuda, rnd=rnd)                 # a single block


def test_mx_edge_values(cuda):
    rng = np.random.default_rng(3)
    x = rng.standard_normal((128, 256)).astype(np.float32)
    x[0] = 0.0                                     # all-zero blocks: exponent 0
    x[1] = -0.0
    x[2] = (2.0 ** -140) * np.sign(x[2])           # subnormal block maxima: exponent clamps to -127
    x[3] = x[3] * 2.0 ** 120                        # |x| up to ~2^122
    x[4, :32] = 6.1                                 # the sawtooth block
    x[5] = np.float32(2.0 ** -126) * x[5]
    xt = torch.from_numpy(x)
    for pol in (fp4.OCP_FLOOR, fp4.NOSAT_CEIL):
        run_mx(xt, cuda, policy=pol)


def _bf16_steps_around(center, n, rng):
    """n bf16 values on consecutive bf16 steps centred on bf16(center), random signs (float32)."""
    b = np.array([center], dtype=np.float32).view(np.uint32)[0] >> 16
    bits = (b + np.arange(-(n // 2), n - n // 2)).astype(np.uint32) << 16
    vals = bits.view(np.float32).copy()
    return vals * rng.choice(np.array([-1.0, 1.0], dtype=np.float32), n)


def test_saturation_count_bf16_near_threshold(cuda):
    """Blocks whose maximum saturates, every other value on consecutive bf16 steps around the
    saturation threshold 6*d (NVFP4, caller global scale 1, so the block scale is d) or 6*2^e
    (MXFP4): the saturation counters must equal the oracle's per-element count."""
    rng = np.random.default_rng(11)
    ds = [(1 + m / 8) * 2.0 ** k for k in range(-6, 7) for m in range(8)]
    nv = []
    for _ in range(4096):
        d = ds[rng.integers(len(ds))]
        blk = np.empty(16, dtype=np.float32)
        blk[0] = 6 * d * 1.03           # maps to scale d, normalises above 6
        blk[1:] = _bf16_steps_around(6 * d, 15, rng)
        nv.append(rng.permutation(blk))
    x = torch.from_numpy(np.concatenate(nv).reshape(-1, 512)).to(torch.bfloat16)
    for fs in (False, True):
        run_nv(x, cuda, four_six=fs, global_in=1.0)
    mx = []
    for _ in range(2048):
        e = int(rng.integers(-20, 21))
        blk = np.empty(32, dtype=np.float32)
        blk[0] = 7 * 2.0 ** e           # floor(log2) = e + 2: shared exponent e, normalises to 7
        blk[1:] = _bf16_steps_around(6 * 2.0 ** e, 31, rng)
        mx.append(rng.permutation(blk))
    x = torch.from_numpy(np.concatenate(mx).reshape(-1, 512)).to(torch.bfloat16)
    _, _, c = fp4.mx_quantize(x.to(cuda))
    _, _, co = O.mx_quantize(f32(x))
    assert counts_of(c) == co and co["saturation"] > 0
    run_mx(x, cuda)


def test_mx_empty_and_nonfinite_counts(cuda):
    q, s, c = fp4.mx_quantize(torch.empty((0, 64), dtype=torch.float32, device=cuda))
    assert q.numel() == 0 and counts_of(c)["nonfinite"] == 0
    x = torch.randn(128, 256)
    x[7, 3] = float("nan")
    x[9, 100] = float("inf")
    x[100, 0] = float("-inf")
    _, _, c = fp4.mx_quantize(x.to(cuda))
    assert counts_of(c)["nonfinite"] == 3


def nonfinite_input(dtype, seed):
    """N(0,1) with NaN of both signs, +-Inf, and a block holding both, at fixed positions."""
    x = synth.normal_f32(128, 256, seed)
    b = x.view(torch.int32)
    b[7, 3], b[7, 40], b[9, 100], b[100, 0] = 0x7FC00000, -0x400000, 0x7F800000, -0x800000
    b[64, 16], b[64, 17], b[127, 255] = 0x7FC00000, -0x800000, 0x7F800000
    return x.to(dtype)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rnd", [fp4.RNE, fp4.STOCHASTIC])
def test_nonfinite_inputs_parity(cuda, dtype, rnd):
    """Blocks holding Inf or NaN are rejected: every other block is bit-exact, the counters are
    exact (rejected blocks add only to the non-finite count), and a NaN anywhere makes the two-pass
    global scale NaN, as torch.amax propagates it; every block is then left open.  Dequantisation is
    a total function of (codes, scale bytes, global scale): the GPU's reconstruction of its own
    outputs equals the oracle's reconstruction of them, NaN scale bytes included."""
    x = nonfinite_input(dtype, 36)
    for policy in (fp4.OCP_FLOOR, fp4.NOSAT_CEIL):
        run_mx(x, cuda, policy=policy, rnd=rnd, seed=4)
    for four_six in (False, True):
        q, s, g, qo, so, go = run_nv(x, cuda, rnd=rnd, four_six=four_six, seed=4, global_in=0.01)
        out = fp4.fp4_dequantize(q, s, fp4.NVFP4, g)
        want = O.dequantize(npy(q).reshape(qo.shape), rowmajor_scales(s, *so.shape, fp4.ROWMAJOR), O.NVFP4, 0.01)
        assert np.array_equal(npy(out), want, equal_nan=True)
        q, s, g, qo, so, go = run_nv(x, cuda, rnd=rnd, four_six=four_six, seed=4)
        assert np.isnan(go) and bool(torch.isnan(x.float().abs().amax()))


# ---------------------------------------------------------------------------------------------
# NVFP4

@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rnd", [fp4.RNE, fp4.STOCHASTIC])
@pytest.mark.parametrize("four_six", [False, True])
def test_nvfp4_outliers_small(cuda, dtype, rnd, four_six):
    x = synth.nv_outliers(384, 2048, seed=5)
    x = x if dtype == torch.bfloat16 else x.float()
    for layout in (fp4.ROWMAJOR, fp4.MMA_TILED):
        q, s, g, qo, so, go = run_nv(x, cuda, rnd=rnd, four_six=four_six, seed=9, layout=layout)
    out = fp4.fp4_dequantize(q, s, fp4.NVFP4, g, layout=fp4.MMA_TILED)
    assert np.array_equal(npy(out), O.dequantize(qo, so, O.NVFP4, go))
    outb = fp4.fp4_dequantize(q, s, fp4.NVFP4, g, layout=fp4.MMA_TILED, out_dtype=torch.bfloat16)
    want = torch.from_numpy(O.dequantize(qo, so, O.NVFP4, go)).to(torch.bfloat16)
    assert torch.equal(outb.cpu(), want)


@pytest.mark.parametrize("four_six", [False, True])
def test_nvfp4_caller_global_and_ragged(cuda, four_six):
    x = synth.normal_bf16(5, 48, 31)
    run_nv(x, cuda, four_six=four_six)
    run_nv(x, cuda, four_six=four_six, global_in=0.001)
    run_nv(synth.normal_bf16(256, 512, 32), cuda, four_six=four_six, global_in=1e-4)  # heavy saturation
    run_nv(torch.zeros(64, 64), cuda, four_six=four_six)                               # amax 0 -> s_g = 1


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rnd", [fp4.RNE, fp4.STOCHASTIC])
def test_nvfp4_four_six_near_ties(cuda, dtype, rnd):
    """Blocks of k/8 values: about 2% have candidate error sums too close for the cheap estimate
    to separate, and about 1% would be decided wrongly by it, so this fails unless the exact
    fp32 sums are taken whenever the estimate is inside its error margin."""
    x = synth.lattice_steps(512, 1024, 41)
    x = x if dtype == torch.bfloat16 else x.float()
    run_nv(x, cuda, rnd=rnd, four_six=True, seed=3)
    run_nv(x, cuda, rnd=rnd, four_six=True, seed=3, global_in=1.0 / 256)
    run_nv(x, cuda, rnd=rnd, four_six=True, seed=3, global_in=0.0037)


@pytest.mark.parametrize("four_six", [False, True])
def test_nvfp4_config2_full(cuda, four_six):
    """8192 x 8192 bf16 N(0,1) with 8 outlier columns x U(50,100), seed 5; plain and 4/6."""
    x = synth.nv_outliers()
    run_nv(x, cuda, four_six=four_six, layout=fp4.ROWMAJOR)


# ---------------------------------------------------------------------------------------------
# Walsh-Hadamard rotation fused with the quantisers

@pytest.mark.parametrize("d", [1024, 2048, 4096, 8192, 16384])
@pytest.mark.parametrize("fmt,rnd,four_six", [(fp4.NVFP4, fp4.RNE, False), (fp4.NVFP4, fp4.STOCHASTIC, False),
                                              (fp4.NVFP4, fp4.RNE, True), (fp4.MXFP4, fp4.RNE, False),
                                              (fp4.MXFP4, fp4.STOCHASTIC, False)])
def test_fwht_small(cuda, d, fmt, rnd, four_six):
    rows = 37  # ragged against the row slots per CTA
    x = synth.fwht_laplace(rows, d, seed=6)
    q, s, g, c, rot = fp4.fwht_quantize(x.to(cuda), fmt=fmt, round=rnd, four_six=four_six, seed=7, want_rotated=True)
    y, qo, so, go, co = O.fwht_quantize(f32(x), fmt=fmt, round=rnd, four_six=four_six, seed=7)
    assert np.array_equal(npy(rot), y)
    if fmt == fp4.NVFP4:
        assert np.float32(npy(g)[0]) == np.float32(go)
    assert np.array_equal(npy(q), qo)
    assert np.array_equal(npy(s), so.ravel())
    assert counts_of(c) == co


@pytest.mark.parametrize("d", [1024, 8192, 16384])
@pytest.mark.parametrize("mode", ["sr", "four_six", "if4"])
@pytest.mark.parametrize("gated", [False, True])
def test_fwht_two_pass_routes(cuda, d, mode, gated):
    """The two-pass NVFP4 rotation has two routes with the same bytes: a workspace of
    fp4_workspace_size(FP4_OP_FWHT_QUANTIZE_STORED) keeps the fp32 rotation from the first pass and
    the second pass quantises it; the minimal workspace makes both passes rotate.  Each route is
    compared with the oracle (37 ragged rows; the randomised rotation; SwiGLU inputs when gated)."""
    rows = 37
    kw = dict(round=fp4.STOCHASTIC if mode == "sr" else fp4.RNE, four_six=mode == "four_six", if4=mode == "if4",
              seed=7)
    sg_np = synth.rht_signs(d, 5)
    sg = torch.from_numpy(sg_np.view(np.int32)).to(cuda)
    if gated:
        g, u = synth.swiglu_inputs(rows, d, seed=9)
        want = O.swiglu_fwht_quantize(f32(g), f32(u), signs=sg_np, **kw)
        run = lambda ws: fp4.swiglu_fwht_quantize(g.to(cuda), u.to(cuda), signs=sg, workspace=ws, **kw)
    else:
        x = synth.fwht_laplace(rows, d, seed=8)
        want = O.fwht_quantize(f32(x), signs=sg_np, **kw)
        run = lambda ws: fp4.fwht_quantize(x.to(cuda), signs=sg, workspace=ws, **kw)
    y, qo, so, go, co = want
    small = torch.empty(fp4.workspace_size(fp4.OP_FWHT_QUANTIZE), dtype=torch.uint8, device=cuda)
    big = torch.empty(fp4.workspace_size(fp4.OP_FWHT_QUANTIZE_STORED, rows, d), dtype=torch.uint8, device=cuda)
    assert big.numel() >= rows * d * 4 + 256
    for ws in (small, big):
        q, s, gg, c, _ = run(ws)
        assert np.float32(npy(gg)[0]) == np.float32(go)
        assert np.array_equal(npy(q), qo) and np.array_equal(npy(s), so.ravel())
        assert counts_of(c) == co


def test_fwht_fp32_input_and_tiled_scales(cuda):
    x = synth.fwht_laplace(128, 8192, seed=12).float()
    q, s, g, c, _ = fp4.fwht_quantize(x.to(cuda), layout=fp4.MMA_TILED)
    y, qo, so, go, co = O.fwht_quantize(f32(x))
    assert np.array_equal(npy(q), qo)
    assert np.array_equal(npy(s), O.scales_to_mma_tiled(so))
    assert counts_of(c) == co


def test_fwht_caller_global(cuda):
    x = synth.fwht_laplace(64, 8192, seed=13)
    gin = torch.tensor([0.002], device=cuda)
    q, s, g, c, _ = fp4.fwht_quantize(x.to(cuda), global_in=gin, round=fp4.STOCHASTIC, seed=3)
    y, qo, so, go, co = O.fwht_quantize(f32(x), global_in=0.002, round=fp4.STOCHASTIC, seed=3)
    assert np.array_equal(npy(q), qo) and np.array_equal(npy(s), so.ravel()) and counts_of(c) == co


def test_fwht_config3_full(cuda):
    """16384 tokens x d = 8192 bf16 Laplace(0,1), 8 channels spiked to 120, H_8192 + NVFP4 + SR
    (Philox seed 7, flat element index), global amax of the rotated tensor: full comparison."""
    x = synth.fwht_laplace()
    q, s, g, c, _ = fp4.fwht_quantize(x.to(cuda), fmt=fp4.NVFP4, round=fp4.STOCHASTIC, seed=7)
    y, qo, so, go, co = O.fwht_quantize(f32(x), fmt=O.NVFP4, round=O.STOCHASTIC, seed=7)
    assert np.float32(npy(g)[0]) == np.float32(go)
    assert np.array_equal(npy(q), qo)
    assert np.array_equal(npy(s), so.ravel())
    assert counts_of(c) == co
    # the spikes are spread: 8 spikes contribute at most 8 * 120 / sqrt(8192) ~ 10.6 per value,
    # plus the rotated Laplace noise; the rotated peak stays far below the 120 input spike
    assert float(np.abs(y).max()) < 120.0 / 4


# Randomised rotation (signs D before the butterflies: Q = c H D)

def _signs_dev(d, seed, cuda):
    return torch.from_numpy(synth.rht_signs(d, seed).view(np.int32)).to(cuda)


@pytest.mark.parametrize("d", [1024, 8192, 16384])
@pytest.mark.parametrize("fmt,rnd,four_six", [(fp4.NVFP4, fp4.RNE, False), (fp4.NVFP4, fp4.STOCHASTIC, False),
                                              (fp4.NVFP4, fp4.RNE, True), (fp4.MXFP4, fp4.STOCHASTIC, False)])
def test_rht_small(cuda, d, fmt, rnd, four_six):
    rows = 37
    x = synth.fwht_laplace(rows, d, seed=6)
    sg = synth.rht_signs(d, 31)
    q, s, g, c, rot = fp4.fwht_quantize(x.to(cuda), fmt=fmt, round=rnd, four_six=four_six, seed=7, want_rotated=True,
                                        signs=_signs_dev(d, 31, cuda))
    y, qo, so, go, co = O.fwht_quantize(f32(x), fmt=fmt, round=rnd, four_six=four_six, seed=7, signs=sg)
    assert np.array_equal(npy(rot), y)
    if fmt == fp4.NVFP4:
        assert np.float32(npy(g)[0]) == np.float32(go)
    assert np.array_equal(npy(q), qo)
    assert np.array_equal(npy(s), so.ravel())
    assert counts_of(c) == co


def test_rht_config3_full(cuda):
    """The full fused-rotation workload (16384 x 8192 bf16, NVFP4, stochastic rounding, seed 7)
    with a randomised rotation: bit-exact against the oracle."""
    x = synth.fwht_laplace()
    sg = synth.rht_signs(8192, 32)
    q, s, g, c, _ = fp4.fwht_quantize(x.to(cuda), fmt=fp4.NVFP4, round=fp4.STOCHASTIC, seed=7,
                                      signs=_signs_dev(8192, 32, cuda))
    y, qo, so, go, co = O.fwht_quantize(f32(x), fmt=O.NVFP4, round=O.STOCHASTIC, seed=7, signs=sg)
    assert np.float32(npy(g)[0]) == np.float32(go)
    assert np.array_equal(npy(q), qo)
    assert np.array_equal(npy(s), so.ravel())
    assert counts_of(c) == co


def test_rht_gemm_end_to_end(cuda):
    """(X Q^T)(W Q^T)^T = X W^T for the orthogonal Q = c H D.
    - The GPU's rotated fp32 operands reproduce X W^T in fp64 to fp32 rounding (orthogonality end
      to end through the kernel).
    - Rotating both operands along K with the same signs, quantising to MXFP4 and multiplying on the
      tensor cores approximates X W^T.  With outlier channels in X, the power-of-two 32-value scales
      lose less to the rotated operands than to the raw ones (NVFP4's 16-value E4M3 scales already
      isolate an outlier channel, so the rotation is not expected to help there)."""
    M, N, K = 256, 256, 4096
    X = synth.nv_outliers(M, K, seed=41).float()
    W = synth.normal_bf16(N, K, 42).float()
    ref = X.double() @ W.double().T
    sd = _signs_dev(K, 43, cuda)
    err = lambda C: float(torch.linalg.norm(C - ref) / torch.linalg.norm(ref))

    qa, sa, _, _, ya = fp4.fwht_quantize(X.to(cuda), fmt=fp4.MXFP4, layout=fp4.MMA_TILED, signs=sd, want_rotated=True)
    qb, sb, _, _, yb = fp4.fwht_quantize(W.to(cuda), fmt=fp4.MXFP4, layout=fp4.MMA_TILED, signs=sd, want_rotated=True)
    assert err(ya.double().cpu() @ yb.double().cpu().T) < 1e-5
    C_rht, ws = fp4.fp4_block_gemm(fp4.MXFP4, qa, sa, qb, sb)
    assert int(ws[:4].view(torch.int32).item()) == 0

    pa, ra, _ = fp4.mx_quantize(X.to(cuda), layout=fp4.MMA_TILED)
    pb, rb, _ = fp4.mx_quantize(W.to(cuda), layout=fp4.MMA_TILED)
    C_plain, _ = fp4.fp4_block_gemm(fp4.MXFP4, pa, ra, pb, rb)
    e_rht, e_plain = err(C_rht.double().cpu()), err(C_plain.double().cpu())
    assert e_rht < 0.25 and e_plain < 0.25   # two FP4 operands: ~0.15-0.2 normwise
    assert e_rht < e_plain


# SwiGLU activation fused ahead of the rotation: a = fl(SiLU(g) * u) formed in fp32, never stored

@pytest.mark.parametrize("d", [1024, 8192, 16384])
@pytest.mark.parametrize("fmt,rnd,four_six,rht", [(fp4.NVFP4, fp4.RNE, False, False), (fp4.NVFP4, fp4.STOCHASTIC, False, True),
                                                  (fp4.NVFP4, fp4.RNE, True, False), (fp4.MXFP4, fp4.RNE, False, True)])
def test_swiglu_fwht_small(cuda, d, fmt, rnd, four_six, rht):
    rows = 37
    g, u = synth.swiglu_inputs(rows, d, seed=3)
    sg = synth.rht_signs(d, 34) if rht else None
    q, s, gs, c, rot = fp4.swiglu_fwht_quantize(g.to(cuda), u.to(cuda), fmt=fmt, round=rnd, four_six=four_six,
                                                seed=7, want_rotated=True,
                                                signs=_signs_dev(d, 34, cuda) if rht else None)
    y, qo, so, go, co = O.swiglu_fwht_quantize(f32(g), f32(u), fmt=fmt, round=rnd, four_six=four_six, seed=7,
                                               signs=sg)
    assert np.array_equal(npy(rot), y)       # the activation and the rotation, bit for bit
    if fmt == fp4.NVFP4:
        assert np.float32(npy(gs)[0]) == np.float32(go)
    assert np.array_equal(npy(q), qo)
    assert np.array_equal(npy(s), so.ravel())
    assert counts_of(c) == co


def test_swiglu_fwht_full(cuda):
    """16384 x 8192 bf16 g, u (seed 3 streams): SiLU(g) * u -> H_8192 -> NVFP4 with stochastic
    rounding (seed 7), the global amax over the rotated activation: full comparison."""
    g, u = synth.swiglu_inputs(16384, 8192, seed=3)
    q, s, gs, c, _ = fp4.swiglu_fwht_quantize(g.to(cuda), u.to(cuda), round=fp4.STOCHASTIC, seed=7)
    y, qo, so, go, co = O.swiglu_fwht_quantize(f32(g), f32(u), round=O.STOCHASTIC, seed=7)
    assert np.float32(npy(gs)[0]) == np.float32(go)
    assert np.array_equal(npy(q), qo)
    assert np.array_equal(npy(s), so.ravel())
    assert counts_of(c) == co


# Past 2^31 elements: 64-bit chunk, block, scale and Philox indices

def test_quantise_beyond_2p31_elements(cuda):
    """65537 x 32768 bf16 = 2,147,516,416 elements; the last row lies wholly past element 2^31.  The
    tensor is a seeded 128-row base repeated with a per-row factor (built on the device); sampled rows
    around the 2^31 boundary are compared with the oracle on the same bits."""
    rows, cols = 65537, 32768
    base = synth.normal_bf16(128, cols, 51).to(cuda)
    fac = torch.from_numpy(np.random.default_rng(52).uniform(0.5, 2.0, rows).astype(np.float32)).to(cuda)
    x = torch.empty((rows, cols), dtype=torch.bfloat16, device=cuda)
    for r0 in range(0, rows, 8192):   # chunks keep the temporaries small
        r1 = min(rows, r0 + 8192)
        idx = torch.arange(r0, r1, device=cuda) % 128
        x[r0:r1] = (base[idx].float() * fac[r0:r1, None]).to(torch.bfloat16)
    assert x.numel() > 2 ** 31
    sample = [0, 1, 65535, 65536]      # row 65536 starts at element 2^31 exactly

    q, s, c = fp4.mx_quantize(x, round=fp4.STOCHASTIC, seed=11)
    # stochastic rounding indexes Philox by the flat element index: the oracle quantises each
    # sampled row at its true flat offset
    for r in sample:
        xr = f32(x[r:r + 1].cpu())
        qo, so, _ = O.mx_quantize_rows_at(xr, r * cols, round=O.STOCHASTIC, seed=11)
        assert np.array_equal(npy(q[r:r + 1]), qo)
        assert np.array_equal(npy(s.view(rows, cols // 32)[r:r + 1]), so)

    g = torch.tensor([0.004], dtype=torch.float32, device=cuda)
    q, s, gg, c = fp4.nvfp4_quantize(x, global_in=g)
    for r in sample:
        xr = f32(x[r:r + 1].cpu())
        qo, so, _, _ = O.nvfp4_quantize(xr, global_in=0.004)
        assert np.array_equal(npy(q[r:r + 1]), qo)
        assert np.array_equal(npy(s.view(rows, cols // 16)[r:r + 1]), so)
    out = fp4.fp4_dequantize(q, s, fp4.NVFP4, gg, out_dtype=torch.bfloat16)
    for r in sample:
        want = O.dequantize(npy(q[r:r + 1]), npy(s.view(rows, cols // 16)[r:r + 1]), O.NVFP4, np.float32(0.004))
        assert torch.equal(out[r:r + 1].cpu(), torch.from_numpy(want).to(torch.bfloat16))
    # the two-pass call: the tensor amax over all 2.1 G values sets the global scale
    _, _, g2, _ = fp4.nvfp4_quantize(x)
    amax = float(x.abs().max().float().item())
    assert np.float32(npy(g2)[0]) == np.float32(np.float32(amax) / np.float32(2688.0))
    del x, q, s, out


# ---------------------------------------------------------------------------------------------
# The GEMM workloads' quantisation (MXFP4 activations and weights at the down_proj shape)

def test_mx_swiglu_activation_full(cuda):
    a = synth.swiglu_act()  # 4096 x 28672 bf16
    run_mx(a, cuda, layout=fp4.MMA_TILED)


def test_mx_weight_rows_sampled(cuda):
    w = synth.weight()  # 8192 x 28672 bf16 N(0, 0.02)
    q, s, c = fp4.mx_quantize(w.to(cuda), layout=fp4.ROWMAJOR)
    rows = np.random.default_rng(0).choice(8192, 256, replace=False)
    qo, so, _ = O.mx_quantize(f32(w[torch.from_numpy(rows)]))
    assert np.array_equal(npy(q)[rows], qo)
    assert np.array_equal(npy(s).reshape(8192, -1)[rows], so)


def _offset_by_16(shape, dtype, cuda):
    """A contiguous tensor whose data starts 16 bytes past a 32-byte boundary (the API promises
    16-byte alignment only; 32-byte aligned outputs take the 256-bit store path)."""
    n = int(np.prod(shape)) * torch.empty(0, dtype=dtype).element_size()
    buf = torch.empty(n + 64, dtype=torch.uint8, device=cuda)
    off = (16 - buf.data_ptr()) % 32
    t = buf[off:off + n].view(dtype).view(shape)
    assert t.data_ptr() % 32 == 16
    return t


@pytest.mark.parametrize("fmt", [fp4.MXFP4, fp4.NVFP4, fp4.IF4])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_expansions_on_16_byte_aligned_outputs(cuda, fmt, out_dtype):
    rows, cols = 136, 1056  # ragged against the launch's chunking: 8976 16-blocks
    x = synth.nv_outliers(rows, cols, seed=12).to(cuda)
    if fmt == fp4.MXFP4:
        q, s = fp4.mx_quantize(x)[:2]
        g = None
    else:
        q, s, g = fp4.nvfp4_quantize(x, if4=(fmt == fp4.IF4))[:3]
    want = O.dequantize(npy(q), npy(s), fmt, 1.0 if g is None else float(g.item()))
    want_t = torch.from_numpy(want).to(out_dtype)
    aligned = fp4.fp4_dequantize(q, s, fmt, g, out_dtype=out_dtype)
    assert aligned.data_ptr() % 32 == 0
    shifted = fp4.fp4_dequantize(q, s, fmt, g, out=_offset_by_16((rows, cols), out_dtype, cuda))
    assert torch.equal(aligned.cpu(), want_t)
    assert torch.equal(shifted.cpu(), want_t)
    # the E2M1 -> E4M3 expansion takes the same choice of store
    if fmt == fp4.MXFP4 and out_dtype == torch.float32:
        e_al = fp4.fp4_to_e4m3(q)
        e_sh = fp4.fp4_to_e4m3(q, out=_offset_by_16((rows, cols), torch.uint8, cuda))
        assert np.array_equal(npy(e_al), O.e2m1_to_e4m3(npy(q)))
        assert np.array_equal(npy(e_sh), O.e2m1_to_e4m3(npy(q)))


@pytest.mark.parametrize("mode", ["plain", "four_six", "if4"])
def test_two_pass_workspace_needs_no_initialisation(cuda, mode):
    """The amax pass writes one partial maximum per CTA into the workspace and the quantise pass
    reduces exactly those words, so nothing is zeroed between calls.  A workspace filled with 0xFF
    bytes (NaN patterns, above every finite magnitude) must not leak into the result: the global
    scale, nibbles, scales and counters match the oracle.  Sizes: a one-CTA amax grid, and
    8192 x 2432 (1.2 M 32-byte chunks), whose amax grid is capped at 8 CTAs per SM."""
    kw = dict(four_six=mode == "four_six", if4=mode == "if4")
    for rows, cols in ((37, 1024), (8192, 2432)):
        x_cpu = synth.nv_outliers(rows, cols, seed=21)
        ws = torch.full((fp4.workspace_size(fp4.OP_NVFP4_QUANTIZE),), 0xFF, dtype=torch.uint8, device=cuda)
        q, s, g, c = fp4.nvfp4_quantize(x_cpu.to(cuda), workspace=ws, **kw)
        x = f32(x_cpu)
        qo, so, go, co, spec = O.nvfp4_quantize(x, spec=True, **kw)
        assert spec.all()
        assert np.float32(npy(g)[0]) == np.float32(go)
        assert np.array_equal(npy(q), qo)
        assert np.array_equal(npy(s), so.ravel())
        compare_counts(c, co, x, spec, 16)


def test_four_six_decided_by_upper_bytes_of_each_word(cuda):
    """The four-over-six estimate decodes each packed word in registers, and bytes 2-3 of a word (values
    4-7 and 12-15 of a block) are the ones that once decoded to zeros when the word came straight
    from the encoder.  Blocks whose estimated choice would flip if those values decoded to zero (and
    that the estimate decides by at least four times its margin) are picked from a seeded N(0,1)
    pool; both choices occur among them.  The GPU must choose exactly as the oracle does: nibbles,
    scale bytes and the 4-count.  A caller-fixed global scale (the pool's) keeps the scales the
    selection assumed."""
    rng = np.random.default_rng(41)
    pool = torch.from_numpy(rng.standard_normal((200000, 16), dtype=np.float32)).to(torch.bfloat16)
    x = pool.float().numpy()
    s_g = np.float32(np.float32(np.abs(x).max()) / np.float32(1536.0))
    lat = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])

    def rne(y):  # E2M1 round to nearest, ties to the even code (the selection's own model)
        a = np.minimum(np.abs(y.astype(np.float64)), 6.0)
        i = np.clip(np.searchsorted(lat, a), 1, 7)
        lo, hi = lat[i - 1], lat[i]
        return np.where((a - lo > hi - a) | ((a - lo == hi - a) & (i % 2 == 0)), hi, lo) * (a > 0)

    amax = np.abs(x).max(1)
    upper = np.zeros(16, bool)
    upper[4:8] = upper[12:16] = True
    est, est0 = {}, {}
    for T in (6, 4):
        d = torch.from_numpy(amax * (np.float32(1) / (np.float32(T) * s_g))).to(torch.float8_e4m3fn).float().numpy()
        D = (d * s_g).astype(np.float32)
        y = np.abs(x * (np.float32(1) / D)[:, None]).astype(np.float32)
        r2 = (rne(y) - y) ** 2
        est[T] = D.astype(np.float64) ** 2 * r2.sum(1)
        est0[T] = D.astype(np.float64) ** 2 * np.where(upper, y.astype(np.float64) ** 2, r2).sum(1)
    margin = 2.0 ** -17 * (1.02 * amax.astype(np.float64) ** 2 + 2 * (est[6] + est[4]))
    pick = (np.abs(est[4] - est[6]) > 4 * margin) & (np.sign(est0[4] - est0[6]) != np.sign(est[4] - est[6]))
    blocks = pool[torch.from_numpy(np.nonzero(pick)[0][:8192])]
    assert blocks.shape[0] == 8192
    xs = blocks.reshape(256, 512)
    q, s, g, qo, so, go = run_nv(xs, cuda, four_six=True, global_in=float(s_g))
    co = O.nvfp4_quantize(f32(xs), four_six=True, global_in=float(s_g))[3]
    assert 1000 < co["blocks_four"] < 7000  # both choices are exercised


def test_quantisers_write_into_preallocated_outputs(cuda):
    """`out=` hands the quantisers the caller's buffers: the bytes match the allocating call, and a
    buffer of the wrong size is refused before any launch."""
    x = synth.nv_outliers(64, 2048, seed=31).to(cuda)
    ref = fp4.mx_quantize(x)
    out = (torch.empty_like(ref[0]), torch.empty_like(ref[1]), None, torch.empty_like(ref[2]))
    got = fp4.mx_quantize(x, out=out)
    assert got[0].data_ptr() == out[0].data_ptr()
    assert all(torch.equal(a, b) for a, b in zip(ref, got))
    ref = fp4.nvfp4_quantize(x, four_six=True)
    out = tuple(torch.empty_like(t) for t in ref)
    got = fp4.nvfp4_quantize(x, four_six=True, out=out)
    assert got[1].data_ptr() == out[1].data_ptr()
    assert all(torch.equal(a, b) for a, b in zip(ref, got))
    ref = fp4.fwht_quantize(x, fmt=fp4.NVFP4, round=fp4.STOCHASTIC, seed=3)
    out = tuple(torch.empty_like(t) for t in ref[:4])
    got = fp4.fwht_quantize(x, fmt=fp4.NVFP4, round=fp4.STOCHASTIC, seed=3, out=out)
    assert all(torch.equal(a, b) for a, b in zip(ref[:4], got[:4]))
    bad = (torch.empty(10, dtype=torch.uint8, device=cuda), out[1], out[2], out[3])
    with pytest.raises(ValueError):
        fp4.nvfp4_quantize(x, out=bad)

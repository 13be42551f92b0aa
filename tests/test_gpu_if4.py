"""GPU parity of IF4 (podcast "Adaptive Block-Scaled Data Types for FP4 Training", IF4 segment):
per 16-block E2M1 or sign-magnitude INT4, the choice in the scale byte's bit 7.

Bar: nibbles, scale bytes (flag included), the global scale and all counters bit-exact; the
dequantised values bit-exact.  The choice compares exact fp32 error sums on both sides, so the
near-tie inputs below only pass if the kernel takes every fp32 step in the oracle's order.
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


def run_if4(x_cpu, cuda, layout=fp4.ROWMAJOR, global_in=None, dequant=True):
    gin = None if global_in is None else torch.tensor([global_in], dtype=torch.float32, device=cuda)
    q, s, g, c = fp4.nvfp4_quantize(x_cpu.to(cuda), if4=True, layout=layout, global_in=gin)
    x = synth.as_f32_numpy(x_cpu)
    qo, so, go, co, spec = O.nvfp4_quantize(x, if4=True, global_in=global_in, spec=True)
    assert np.array_equal(np.float32(npy(g)[0]), np.float32(go), equal_nan=True)
    if spec.all():
        assert np.array_equal(npy(q), qo)
        want_s = O.scales_to_mma_tiled(so) if layout == fp4.MMA_TILED else so.ravel()
        assert np.array_equal(npy(s), want_s)
    else:
        compare_blocks(q, s, qo, so, spec, 16, layout)
    compare_counts(c, co, x, spec, 16)
    if dequant:
        # a total function of the stored bytes: the oracle reconstructs the GPU's own outputs
        ref = O.dequantize(npy(q).reshape(qo.shape), rowmajor_scales(s, *so.shape, layout), O.IF4, float(npy(g)[0]))
        out = fp4.fp4_dequantize(q, s, fp4.IF4, g, layout=layout)
        assert np.array_equal(npy(out), ref, equal_nan=True)
        outb = fp4.fp4_dequantize(q, s, fp4.IF4, g, layout=layout, out_dtype=torch.bfloat16)
        want = torch.from_numpy(ref).to(torch.bfloat16)
        assert np.array_equal(npy(outb.float()), npy(want.float()), equal_nan=True)
    return co


def int4_lattice(rows, cols, seed):
    """Values k * fl(6/7) (the INT4 step of scale 1 under s_g = 1), k uniform in -7..7, one |k| = 7
    per block so each block's scale is exactly 1."""
    rng = np.random.default_rng(seed)
    k = rng.integers(-7, 8, size=(rows, cols))
    k[:, ::16] = np.where(rng.random((rows, cols // 16)) < 0.5, -7, 7)
    step = np.float32(6.0) / np.float32(7.0)
    return torch.from_numpy((k.astype(np.float32) * step).astype(np.float32))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("layout", [fp4.ROWMAJOR, fp4.MMA_TILED])
def test_if4_outliers_small(cuda, dtype, layout):
    x = synth.nv_outliers(384, 2048, seed=5)
    co = run_if4(x if dtype == torch.bfloat16 else x.float(), cuda, layout=layout)
    assert 0 < co["blocks_four"] < 384 * 2048 // 16


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_if4_near_ties_and_distributions(cuda, dtype):
    cast = (lambda t: t.to(torch.bfloat16)) if dtype == torch.bfloat16 else (lambda t: t.float())
    rng = np.random.default_rng(21)
    run_if4(cast(synth.lattice_steps(512, 1024, 41)), cuda)
    run_if4(cast(synth.lattice_steps(256, 1024, 42, denom=7, kmax=49)), cuda, global_in=1.0 / 256)
    run_if4(cast(torch.from_numpy(rng.uniform(-1, 1, (256, 1024)).astype(np.float32))), cuda)
    run_if4(cast(torch.from_numpy(rng.laplace(size=(256, 1024)).astype(np.float32))), cuda)
    co = run_if4(int4_lattice(128, 1024, 22).float(), cuda, global_in=1.0)
    assert co["blocks_four"] > 0.9 * 128 * 1024 // 16


def test_if4_edges(cuda):
    run_if4(synth.normal_bf16(5, 48, 31), cuda)                              # ragged: 5 rows, 3 blocks
    run_if4(synth.normal_bf16(5, 48, 31), cuda, global_in=0.001)
    run_if4(synth.normal_bf16(256, 512, 32), cuda, global_in=1e-4)           # clamped scales, saturation
    run_if4(synth.normal_bf16(64, 256, 33), cuda, global_in=1e-30)           # tiny step, still normal
    run_if4(torch.zeros(64, 64), cuda)                                       # amax 0 -> s_g = 1, all ties
    x = synth.normal_f32(64, 256, 34)
    x[3, 5], x[10, 100], x[63, 255] = float("inf"), float("nan"), float("-inf")
    co = run_if4(x, cuda, global_in=0.01)                                    # 3 rejected blocks, the rest exact
    assert co["nonfinite"] == 3 and co["blocks_four"] > 0
    co = run_if4(x, cuda)                                                    # NaN global scale: all open
    assert co["nonfinite"] == 3
    x = synth.normal_f32(64, 256, 35) * 1e-38                               # subnormal inputs
    run_if4(x, cuda)


def test_if4_full_outliers(cuda):
    """8192 x 8192 bf16 N(0,1) with 8 outlier columns x U(50,100), seed 5, two-pass global scale."""
    run_if4(synth.nv_outliers(), cuda, dequant=False)


# ---------------------------------------------------------------------------------------------
# IF4 behind the Walsh-Hadamard rotation (plain and randomised) and the SwiGLU fusion

def _signs_dev(d, seed, cuda):
    return torch.from_numpy(synth.rht_signs(d, seed).view(np.int32)).to(cuda)


@pytest.mark.parametrize("d", [1024, 8192, 16384])
@pytest.mark.parametrize("rht", [False, True])
def test_if4_rotation_small(cuda, d, rht):
    rows = 37
    x = synth.fwht_laplace(rows, d, seed=6)
    sg = synth.rht_signs(d, 31) if rht else None
    q, s, g, c, rot = fp4.fwht_quantize(x.to(cuda), if4=True, want_rotated=True,
                                        signs=_signs_dev(d, 31, cuda) if rht else None)
    y, qo, so, go, co = O.fwht_quantize(synth.as_f32_numpy(x), if4=True, signs=sg)
    assert np.array_equal(npy(rot), y)
    assert np.float32(npy(g)[0]) == np.float32(go)
    assert np.array_equal(npy(q), qo)
    assert np.array_equal(npy(s), so.ravel())
    assert counts_of(c) == co and co["blocks_four"] > 0
    # one pass under a caller-fixed global scale (half the derived one: more saturation)
    gi = float(go) * 0.5
    q, s, _, c, _ = fp4.fwht_quantize(x.to(cuda), if4=True, global_in=torch.tensor([gi], device=cuda),
                                      signs=_signs_dev(d, 31, cuda) if rht else None)
    _, qo, so, _, co = O.fwht_quantize(synth.as_f32_numpy(x), if4=True, signs=sg, global_in=gi)
    assert np.array_equal(npy(q), qo) and np.array_equal(npy(s), so.ravel()) and counts_of(c) == co


@pytest.mark.parametrize("d", [1024, 8192])
def test_if4_swiglu_rotation_small(cuda, d):
    rows = 37
    g, u = synth.swiglu_inputs(rows, d, seed=3)
    q, s, gs, c, _ = fp4.swiglu_fwht_quantize(g.to(cuda), u.to(cuda), if4=True, signs=_signs_dev(d, 34, cuda))
    _, qo, so, go, co = O.swiglu_fwht_quantize(synth.as_f32_numpy(g), synth.as_f32_numpy(u), if4=True,
                                               signs=synth.rht_signs(d, 34))
    assert np.float32(npy(gs)[0]) == np.float32(go)
    assert np.array_equal(npy(q), qo) and np.array_equal(npy(s), so.ravel()) and counts_of(c) == co


def test_if4_rotation_full_sampled_rows(cuda):
    """16384 x 8192 bf16 Laplace with spiked channels (seed 6), randomised rotation, IF4, a
    caller-fixed global scale (so each row quantises on its own): 12 sampled rows bit-exact."""
    x = synth.fwht_laplace()
    d = x.shape[1]
    gi = 0.0125
    q, s, _, c, _ = fp4.fwht_quantize(x.to(cuda), if4=True, global_in=torch.tensor([gi], device=cuda),
                                      signs=_signs_dev(d, 33, cuda))
    rows = np.sort(np.random.default_rng(44).choice(x.shape[0], 12, replace=False))
    _, qo, so, _, _ = O.fwht_quantize(synth.as_f32_numpy(x[rows]), if4=True, signs=synth.rht_signs(d, 33),
                                      global_in=gi)
    assert np.array_equal(npy(q)[rows], qo)
    assert np.array_equal(npy(s).reshape(x.shape[0], d // 16)[rows], so)
    assert counts_of(c)["blocks_four"] > 0

"""Pins of the CPU oracle to facts the source pages and mathematics fix (no GPU).

Each test checks the oracle against something other than itself: a worked example or number the
pages print (fixtures under tests/golden/, each citing its page and section), a closed form, an
invariant, or a special case that reduces to a library routine (torch's float8/bf16 casts, scipy's
Hadamard matrix, numpy's fp64 matmul).
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from tests.conftest import golden_rows

LATTICE = [float(v) for v in golden_rows("e2m1_lattice.txt")[0]]


# ---------------------------------------------------------------------------------------------
# E2M1

def test_e2m1_decode_table_matches_printed_lattice():
    for c in range(8):
        assert O.e2m1_value(c) == LATTICE[c]
        neg = O.e2m1_value(c | 8)
        assert neg == -LATTICE[c] and math.copysign(1.0, neg) == -1.0  # includes -0


def test_e2m1_to_e4m3_identity_all_codes():
    """(q & 0x80808080) | ((q & 0x70707070) >> 2) == E4M3(value * 2^-6) for every nibble."""
    rows = {r[0]: r[1] for r in golden_rows("e2m1_to_e4m3.txt")}
    ms, mm, sh = int(rows["mask_sign"], 16), int(rows["mask_mag"], 16), int(rows["shift"])
    f = 2.0 ** int(rows["factor_log2"])
    for c in range(16):
        q = (c << 4) * 0x01010101  # the nibble in bits 7..4 of every byte
        conv = (q & ms) | ((q & mm) >> sh)
        for byte in range(4):
            b = (conv >> (8 * byte)) & 0xFF
            got = O.e4m3_value(b)
            want = O.e2m1_value(c) * f
            assert got == want and math.copysign(1, got) == math.copysign(1, want), (c, hex(b))


def test_e2m1_to_e4m3_expansion_equals_the_printed_identity():
    """The oracle's expansion (an E4M3 encode of value * 2^-6 per nibble) against the page's bit
    identity applied to every possible packed byte, low nibble first."""
    rows = {r[0]: r[1] for r in golden_rows("e2m1_to_e4m3.txt")}
    ms, mm, sh = int(rows["mask_sign"], 16) & 0xFF, int(rows["mask_mag"], 16) & 0xFF, int(rows["shift"])
    q = np.arange(256, dtype=np.uint8).reshape(8, 32)
    got = O.e2m1_to_e4m3(q)
    for r in range(8):
        for j in range(32):
            byte = int(q[r, j])
            for h, n in enumerate((byte & 15, byte >> 4)):
                b = n << 4
                assert got[r, 2 * j + h] == ((b & ms) | ((b & mm) >> sh)), (byte, h)


def test_e2m1_rne_worked_values_and_ties():
    # exact points stay; ties go to the even mantissa code; >6 saturates; -tiny keeps its sign
    cases = {1.5: 3, 2.5: 4, 0.15: 0, 6.5: 7, 0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 3.5: 6, 5.0: 6,
             6.0: 7, 100.0: 7, 0.2500001: 1, 0.7499999: 1}
    for y, code in cases.items():
        assert O.e2m1_encode_rne(y) == code, y
        assert O.e2m1_encode_rne(-y) == code | 8, -y
    assert O.e2m1_encode_rne(-0.0) == 8
    assert O.e2m1_encode_rne(-1e-30) == 8


def test_e2m1_rne_is_nearest_on_dense_grid():
    """Brute force: the code's value is at minimal distance (a library argmin over the lattice)."""
    ys = np.linspace(0, 6.0, 60001, dtype=np.float32)
    lat = np.array(LATTICE)
    for y in ys[::7]:
        c = O.e2m1_encode_rne(float(y))
        d = np.abs(lat - float(y))
        assert d[c] == d.min()


# ---------------------------------------------------------------------------------------------
# E4M3 and bf16 casts: reduce to torch's library conversions

def test_e4m3_encoder_matches_torch_float8_on_range():
    rng = np.random.default_rng(0)
    u = np.concatenate([rng.uniform(0, 448, 20000), 2.0 ** rng.uniform(-12, 8.8, 20000)]).astype(np.float32)
    # all midpoints between consecutive finite codes (the tie cases)
    vals = np.array([O.e4m3_value(c) for c in range(0x7F)])
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    u = np.concatenate([u, mids, vals.astype(np.float32)])
    u = u[u <= 448]
    ref = torch.from_numpy(u).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([O.e4m3_encode(float(v)) for v in u], dtype=np.uint8)
    assert np.array_equal(ours, ref)


def test_e4m3_decode_known_points_and_saturation():
    assert O.e4m3_value(0x7E) == 448.0
    assert O.e4m3_value(0x38) == 1.0
    assert O.e4m3_value(0x08) == 2.0 ** -6
    assert O.e4m3_value(0x01) == 2.0 ** -9
    assert math.isnan(O.e4m3_value(0x7F))
    assert O.e4m3_encode(449.0) == 0x7E and O.e4m3_encode(1e30) == 0x7E


def test_bf16_rne_matches_torch_cast():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(5000).astype(np.float32),
                        (rng.integers(0, 2 ** 32, 5000, dtype=np.uint64).astype(np.uint32)).view(np.float32)])
    x = x[np.isfinite(x)]
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.bf16_bits(x), ref)


# ---------------------------------------------------------------------------------------------
# Philox and stochastic rounding

def test_philox_known_answers():
    for r in golden_rows("philox4x32_10_kat.txt"):
        h = [int(v, 16) for v in r]
        assert list(O.philox4x32_10(h[0:4], h[4:6])) == h[6:10]


def test_sr_word_mapping():
    seed = 0x0123456789ABCDEF
    for idx in (0, 1, 2, 3, 4, 7, 1 << 33, (1 << 33) + 3):
        blk = idx >> 2
        out = O.philox4x32_10([blk & 0xFFFFFFFF, blk >> 32, 0, 0], [seed & 0xFFFFFFFF, seed >> 32])
        assert O.sr_word(seed, idx) == out[idx & 3]


def test_sr_lattice_points_never_move_and_threshold_is_exact():
    for code in range(16):
        y = O.e2m1_value(code)
        for r in (0, 1, 2 ** 31, 2 ** 32 - 1):
            c = O.e2m1_encode_sr(y, r)
            assert O.e2m1_value(c) == y
    # halfway between 2 and 3: up iff r < 2^31
    assert O.e2m1_encode_sr(2.5, 2 ** 31 - 1) == 5 and O.e2m1_encode_sr(2.5, 2 ** 31) == 4
    # a quarter of the way from 4 to 6: p = 1/4, up iff r < 2^30
    assert O.e2m1_encode_sr(4.5, 2 ** 30 - 1) == 7 and O.e2m1_encode_sr(4.5, 2 ** 30) == 6
    assert O.e2m1_encode_sr(7.0, 0) == 7  # saturates


@pytest.mark.parametrize("y", [0.1, 0.3, 1.2, 2.3, 3.9, 5.1])
def test_sr_is_unbiased(y):
    n = 1 << 15
    vals = np.array([O.e2m1_value(O.e2m1_encode_sr(y, O.sr_word(7, i))) for i in range(n)])
    lat = np.array(LATTICE)
    lo = lat[lat <= y].max()
    hi = lat[lat > y].min()
    p = (y - lo) / (hi - lo)
    sigma = (hi - lo) * math.sqrt(p * (1 - p) / n)
    assert abs(vals.mean() - y) < 4 * sigma


# ---------------------------------------------------------------------------------------------
# MXFP4

def test_bits_per_value():
    B, eb, sb, blk, bpv = golden_rows("bits_per_value.txt")[0]
    B, eb, sb = int(B), int(eb), int(sb)
    assert B * eb + sb == int(blk) and (B * eb + sb) / B == float(bpv)
    x = np.random.default_rng(2).standard_normal((64, 256)).astype(np.float32)
    q, s, _ = O.mx_quantize(x)
    assert (q.nbytes + s.nbytes) * 8 / x.size == float(bpv)


def test_mx_worked_block_13():
    rows = golden_rows("mx_worked_block.txt")
    e_expected = int(rows[0][1])
    x = np.zeros(32, dtype=np.float32)
    srcs = [float(r[0]) for r in rows[1:]]
    x[: len(srcs)] = srcs
    q, s, c = O.mx_quantize(x[None, :])
    assert int(s[0, 0]) - 127 == e_expected
    xh = O.dequantize(q, s, O.MXFP4)[0]
    for i, r in enumerate(rows[1:]):
        assert xh[i] == float(np.float32(r[2])), r
    assert c["underflow"] == 1 and c["saturation"] == 1


def test_mx_ramp_fixtures():
    base = np.array([-2, -1.5, -1, -0.5, 0, 0.5, 1, 1.5, 2] * 4, dtype=np.float32)[:31]
    for appended, e, last, zeros, maxerr, rmse in golden_rows("mx_ramp_fixtures.txt"):
        x = np.append(base, np.float32(appended)).astype(np.float32)
        q, s, _ = O.mx_quantize(x[None, :])
        xh = O.dequantize(q, s, O.MXFP4)[0].astype(np.float64)
        err = xh - x
        assert int(s[0, 0]) - 127 == int(e)
        assert xh[-1] == float(last)
        assert int((xh == 0).sum()) == int(zeros)
        assert np.abs(err).max() == float(maxerr)
        assert round(math.sqrt((err ** 2).mean()), 6) == float(rmse)


def test_e8m0_limits():
    """The E8M0 limits ("MXFP4 Quantization: Audit", "Read the shared E8M0 scale"): exponent -127
    is byte 0 and 127 is byte 254.  A block encoded at each limit exponent and reconstructed from
    the printed byte gives its values back exactly (2^-127 * v and 2^127 * v are representable)."""
    for e, byte in golden_rows("e8m0_limits.txt"):
        e, byte = int(e), int(byte)
        # the whole lattice, both signs; at e = 127 only the magnitudes below 2 (2 * 2^127 overflows fp32)
        lat = [0, 0.5, 1, 1.5] if e == 127 else [0, 0.5, 1, 1.5, 2, 3, 4, 6]
        mags = np.resize(np.array(lat, dtype=np.float64), 16)
        x = (np.concatenate([mags, -mags]) * 2.0 ** e).astype(np.float32)
        codes, c = O.mx_encode_block(x, e)
        q = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)[None, :]
        rec = O.dequantize(q, np.array([[byte]], dtype=np.uint8), O.MXFP4)[0]
        assert np.array_equal(rec, x), (e, rec, x)
        assert c["saturation"] == 0 and c["underflow"] == 0
    # data-driven exponent clamps at -127 (byte 0) and never yields byte 255
    tiny = np.full((1, 32), 2.0 ** -140, dtype=np.float32)
    assert O.mx_quantize(tiny)[1][0, 0] == 0
    huge = np.full((1, 32), 3.0e38, dtype=np.float32)
    assert O.mx_quantize(huge)[1][0, 0] == 125 + 127
    zero = np.zeros((1, 32), dtype=np.float32)
    assert O.mx_quantize(zero)[1][0, 0] == 127  # all-zero policy: exponent 0


def test_mx_exponent_matches_log2_definition():
    rng = np.random.default_rng(3)
    for a in np.concatenate([2.0 ** rng.uniform(-120, 120, 2000), [1.0, 4.0, 6.0, 8.0, 6.1, 13.0]]).astype(np.float32):
        a = float(a)
        assert O.mx_exponent(a, O.OCP_FLOOR) == max(-127, math.floor(math.log2(a / 4)))
        e = O.mx_exponent(a, O.NOSAT_CEIL)
        assert a <= 6 * 2.0 ** e and (e == -127 or a > 6 * 2.0 ** (e - 1))


def test_sawtooth_cliff_6_1():
    """The 6.1-max block: the no-saturation rule doubles the scale (byte 128) and leaves 4 and 6
    unused; the OCP rule keeps byte 127 and saturates."""
    rows = {r[1]: r for r in golden_rows("scale_policies.txt")}
    x = np.linspace(-6.0, 6.1, 32).astype(np.float32)
    x[-1] = np.float32(6.1)
    q, s, c = O.mx_quantize(x[None, :], policy=O.NOSAT_CEIL)
    assert int(s[0, 0]) - 127 == int(rows["nosat_ceil"][2])
    codes = np.stack([q[0] & 15, q[0] >> 4], 1).ravel()
    mags = codes & 7
    assert not np.isin(mags, [6, 7]).any()          # lattice steps 4.0 and 6.0 unused
    assert np.float32(6.1) / 2 == np.float32(rows["nosat_ceil"][3])
    assert c["saturation"] == 0
    q2, s2, c2 = O.mx_quantize(x[None, :], policy=O.OCP_FLOOR)
    assert int(s2[0, 0]) - 127 == int(rows["ocp_floor"][2]) and c2["saturation"] == 1


# ---------------------------------------------------------------------------------------------
# NVFP4

def test_nvfp4_global_scale_closed_forms():
    assert O.nvfp4_global_scale(2688.0) == 1.0
    assert O.nvfp4_global_scale(1536.0, four_six=True) == 1.0
    assert O.nvfp4_global_scale(0.0) == 1.0
    assert O.nvfp4_global_scale(448.0 * 6 * 3) == np.float32(3.0)


def test_nvfp4_exact_block():
    """s_g = 1, block max 6: code 1.0 (0x38), every lattice value reproduces exactly."""
    x = np.array([6, -4, 3, 2, 1.5, 1, 0.5, 0, -0.5, -1, -1.5, -2, -3, 4, 6, -6], dtype=np.float32)[None, :]
    q, s, sg, c = O.nvfp4_quantize(x, global_in=1.0)
    assert sg == 1.0 and s[0, 0] == 0x38
    assert np.array_equal(O.dequantize(q, s, O.NVFP4, sg), x)
    assert c == {"underflow": 0, "saturation": 0, "nonfinite": 0, "blocks_four": 0}


def test_nvfp4_scale_is_amax_over_six_cast_to_e4m3():
    """The block scale is amax_b/(6 s_g) cast to E4M3 (podcast IF4 segment: the block maximum over
    six, in FP8 E4M3) under the FP32 global amax_t/(6*448) ("Sub-4-Bit Microscaling" §2).  Every
    block is compared exactly with the reading's fp32 steps restated in numpy, s_g = fl(amax_t /
    2688), inv6 = fl(1/fl(6 s_g)), u = fl(amax_b * inv6), the code from torch's float8_e4m3fn
    cast; and, through the fp64 ratio, never more than one code from the real amax_b/(6 s_g)."""
    x = O._f32(np.random.default_rng(4).standard_normal((64, 256)) * 3)
    q, s, sg, _ = O.nvfp4_quantize(x)
    f = np.float32
    amax_t = np.abs(x).max()
    assert sg == f(amax_t) / f(2688.0)
    inv6 = f(1.0) / (f(6.0) * f(sg))
    amax_b = np.abs(x.reshape(64, 16, 16)).max(-1).astype(np.float32)
    u = (amax_b * inv6).astype(np.float32)
    code = torch.from_numpy(u).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(s, code)
    ideal = torch.from_numpy((amax_b.astype(np.float64) / (6.0 * float(sg))).astype(np.float32))
    ideal = ideal.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.abs(s.astype(int) - ideal.astype(int)).max() <= 1
    assert s.max() <= 0x7E


def test_nvfp4_block_max_normalises_below_six_times_e4m3_step():
    x = O._f32(np.random.default_rng(5).laplace(size=(128, 512)))
    q, s, sg, c = O.nvfp4_quantize(x)
    d = np.array([O.e4m3_value(int(b)) for b in s.ravel()]).reshape(s.shape)
    top = np.abs(x.reshape(128, 32, 16)).max(-1) / (d * sg)
    assert top.max() <= 6 * (1 + 2 ** -4) + 1e-6


def test_four_over_six_pins():
    gave, usable, cut = golden_rows("four_over_six.txt")[0]
    assert round(1 - 256 / 448, 2) == float(cut)           # M = 256 instead of 448
    assert 2 * 8 - 1 == int(usable)                          # 16 codes, one shared zero
    # a block lying on the 4-scaled lattice: 4/6 picks T=4 with zero error
    x = np.array([4, 3, 2, 1.5, 1, 0.5, 0, -4, -3, -2, -1, -0.5, 4, 3, 2, 1], dtype=np.float32)[None, :] * 0.25
    q, s, sg, c = O.nvfp4_quantize(x, four_six=True, global_in=1.0 / 16)
    assert c["blocks_four"] == 1
    assert np.array_equal(O.dequantize(q, s, O.NVFP4, sg), x)
    # in T=4 blocks the +-6 codes (the two values the segment says are given up) never appear.
    # The T=4 blocks are found independently of the oracle's choice: the stored scale byte equals
    # the E4M3 cast (torch) of fl(amax_b * fl(1/fl(4 s_g))) and differs from the T=6 one.
    y = O._f32(np.random.default_rng(6).standard_normal((256, 256)))
    q, s, sg, c = O.nvfp4_quantize(y, four_six=True)
    f = np.float32
    amax_b = np.abs(y.reshape(256, 16, 16)).max(-1).astype(np.float32)

    def code_for(T):
        u = (amax_b * (f(1.0) / (f(T) * f(sg)))).astype(np.float32)
        return torch.from_numpy(u).to(torch.float8_e4m3fn).view(torch.uint8).numpy()

    c4, c6 = code_for(4.0), code_for(6.0)
    four_blocks = (s == c4) & (c4 != c6)
    assert four_blocks.sum() > 0 and four_blocks.sum() <= c["blocks_four"]
    assert np.all((s == c4) | (s == c6))
    codes = np.stack([q & 15, q >> 4], -1).reshape(256, 16, 16)
    mags = codes[four_blocks] & 7
    assert not (mags == 7).any()                             # no +-6 in a T=4 block
    assert int(gave) == len(set(LATTICE[-1:] + [-v for v in LATTICE[-1:]]))  # the two values: +-6


def test_four_over_six_picks_lower_error_candidate_brute_force():
    """Independent brute force: per block, both candidates from torch's E4M3 cast and a numpy
    nearest-lattice search; the oracle's choice must be the lower-SSE one."""
    rng = np.random.default_rng(7)
    x = O._f32(rng.standard_normal((8, 64)))
    q, s, sg, c = O.nvfp4_quantize(x, four_six=True)
    lat = np.array(LATTICE)
    xh = O.dequantize(q, s, O.NVFP4, sg)
    for r in range(8):
        for b in range(4):
            blk = x[r, 16 * b:16 * b + 16].astype(np.float64)
            sse = {}
            for T in (6.0, 4.0):
                inv = np.float32(1) / (np.float32(T) * np.float32(sg))
                u = np.float32(np.abs(blk).max()) * inv
                code = torch.tensor([u], dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).item()
                d = O.e4m3_value(code)
                if d == 0:
                    rec = np.zeros(16)
                else:
                    R = np.float32(1) / (np.float32(d) * np.float32(sg))
                    y = (blk.astype(np.float32) * R).astype(np.float64)
                    mags = np.array([lat[np.argmin(np.abs(lat - min(abs(v), 6.0)) + (np.arange(8) % 2) * 1e-12)] for v in y])
                    rec = np.sign(y) * mags * d * sg
                sse[T] = float(((blk - rec) ** 2).sum())
            got = float(((blk - xh[r, 16 * b:16 * b + 16]) ** 2).sum())
            assert got <= min(sse.values()) * (1 + 1e-5) + 1e-30


# ---------------------------------------------------------------------------------------------
# Non-finite inputs ("MXFP4 Quantization: Audit", "Publish the MXFP4 audit receipt": non-finite
# input is among the inputs to reject).  A block holding Inf or NaN is rejected: its codes and
# scale byte are left open, its non-finite values are counted, and it adds nothing to the other
# counters.  The tensor maximum propagates NaN as torch.amax does.

def _nonfinite_tensor():
    x = O._f32(np.random.default_rng(14).standard_normal((8, 64)) * 2)
    x[1, 5] = np.nan
    x[2, 40] = -np.inf
    x[5, 0], x[5, 1] = np.inf, -np.nan
    return x


def test_rejected_blocks_and_counts():
    x = _nonfinite_tensor()
    finite16 = np.isfinite(x).reshape(8, 4, 16).all(-1)
    finite32 = np.isfinite(x).reshape(8, 2, 32).all(-1)
    n_bad = int(np.count_nonzero(~np.isfinite(x)))
    clean = np.where(np.repeat(finite16, 16, axis=1), x, np.float32(0)).astype(np.float32)
    clean32 = np.where(np.repeat(finite32, 32, axis=1), x, np.float32(0)).astype(np.float32)
    for mode in ({}, {"four_six": True}, {"if4": True}, {"round": O.STOCHASTIC, "seed": 3}):
        q, s, sg, c, spec = O.nvfp4_quantize(x, global_in=0.01, spec=True, **mode)
        assert np.array_equal(spec, finite16) and c["nonfinite"] == n_bad
        # every other block is encoded as it would be with the rejected blocks' values zeroed (all-zero
        # blocks add no counts), so the blocks are independent and the rejected ones add no counts
        q2, s2, _, c2 = O.nvfp4_quantize(clean, global_in=0.01, **mode)
        assert np.array_equal(s[spec], s2[spec])
        assert np.array_equal(q[np.repeat(spec, 8, axis=1)], q2[np.repeat(spec, 8, axis=1)])
        assert {k: v for k, v in c.items() if k != "nonfinite"} == {k: v for k, v in c2.items() if k != "nonfinite"}
    q, s, c, spec = O.mx_quantize(x, spec=True)
    q2, s2, c2 = O.mx_quantize(clean32)
    assert np.array_equal(spec, finite32) and c["nonfinite"] == n_bad
    assert np.array_equal(s[spec], s2[spec]) and c["underflow"] == c2["underflow"]
    assert c["saturation"] == c2["saturation"]


def test_tensor_scale_of_nonfinite_tensors():
    """The two-pass global scale follows torch.amax: NaN with a NaN present, +Inf with only
    infinities; every block is then left open and only the non-finite values are counted."""
    x = _nonfinite_tensor()
    assert torch.isnan(torch.from_numpy(x).abs().amax())
    q, s, sg, c, spec = O.nvfp4_quantize(x, spec=True)
    assert np.isnan(sg) and not spec.any() and c == {"underflow": 0, "saturation": 0, "nonfinite": 4,
                                                     "blocks_four": 0}
    y = np.where(np.isnan(x), np.float32(1), x).astype(np.float32)
    amax = torch.from_numpy(y).abs().amax().item()
    q, s, sg, c, spec = O.nvfp4_quantize(y, spec=True)
    assert amax == math.inf and sg == math.inf and not spec.any()
    assert c["nonfinite"] == int(np.count_nonzero(~np.isfinite(y))) == 2


def test_encoders_on_infinite_values():
    """Infinities are values beyond the largest magnitude: they saturate (E2M1 to +-6, INT4 to
    +-7, E4M3 scales to 448), with the sign kept."""
    assert O.e2m1_encode_rne(float("-inf")) == 15 and O.e2m1_encode_rne(float("inf")) == 7
    assert O.e2m1_encode_sr(float("inf"), 0) == 7 and O.int4_encode_rne(float("-inf")) == 15
    assert O.e4m3_encode(float("inf")) == 0x7E and O.e4m3_value(0x7E) == 448.0


# ---------------------------------------------------------------------------------------------
# IF4 (E2M1 or INT4 per block, the choice in the scale byte's sign bit)

IF4_ROW = [int(v) for v in golden_rows("if4.txt")[0]]


def _if4_step(sg):
    """fp32 INT4 step of a block with E4M3 scale 1: fl(1 * fl(s_g * fl(num/den)))."""
    n, dd = IF4_ROW[5], IF4_ROW[6]
    return np.float32(np.float32(sg) * (np.float32(n) / np.float32(dd)))


def test_int4_encoder_is_rint_clipped_with_sign_bit():
    """Lattice enumeration against numpy's round-half-even, clipped to the 7 the stretch allows."""
    assert IF4_ROW[1] == 7 and IF4_ROW[2] == 6
    rng = np.random.default_rng(11)
    ys = np.concatenate([rng.uniform(-10, 10, 4000), np.arange(-9, 9.5, 0.5), [0.0, -0.0, 7.4999, -7.5001,
                                                                                np.inf, -np.inf, 1e30]])
    for y in ys.astype(np.float32):
        k = int(np.clip(np.rint(np.abs(np.float64(y))), 0, IF4_ROW[1]))
        want = (8 if np.signbit(y) else 0) | k
        assert O.int4_encode_rne(float(y)) == want, y
    for c in range(16):
        v = O.int4_value(c)
        assert abs(v) == (c & 7) and (math.copysign(1.0, v) < 0) == bool(c & 8)


def test_if4_block_on_the_int4_lattice_is_exact_and_flagged():
    """x_i = k_i * step: the INT4 branch reconstructs exactly, E2M1 cannot (6/7 is off its
    lattice), so the block takes INT4, the flag (scale bit 7) is set and the nibbles are k."""
    step = _if4_step(1.0)
    k = np.array([-7, -6, -5, -4, -3, -2, -1, 0, 1, 2, 3, 4, 5, 6, 7, 3])
    assert k.size == IF4_ROW[0]
    x = (k.astype(np.float32) * step).astype(np.float32)[None, :]
    q, s, sg, c = O.nvfp4_quantize(x, global_in=1.0, if4=True)
    assert s[0, 0] >> 7 == IF4_ROW[4] and O.e4m3_value(int(s[0, 0]) & 0x7F) == 1.0
    assert c["blocks_four"] == 1 and c["saturation"] == 0 and c["underflow"] == 0
    codes = np.stack([q & 15, q >> 4], -1).ravel()
    assert [int(O.int4_value(int(v))) for v in codes] == k.tolist()
    assert np.array_equal(O.dequantize(q, s, O.IF4, sg), x)
    # mixed-pair alignment: an INT4 unit over an E2M1 unit of the same scale is 6/7; two INT4
    # operands multiply to 36/49 of the E2M1 product
    assert abs(float(step) - IF4_ROW[5] / IF4_ROW[6]) < 2 ** -24
    assert abs(float(step) ** 2 - IF4_ROW[7] / IF4_ROW[8]) < 2 ** -22


def test_if4_block_on_the_e2m1_lattice_keeps_fp4():
    """Zero E2M1 error cannot be beaten strictly, and an all-zero block is a tie: both keep E2M1
    with the plain NVFP4 bytes and the flag clear."""
    x = np.array([[6, 4, 3, 2, 1.5, 1, 0.5, 0, -6, -4, -3, -2, -1.5, -1, -0.5, 3],
                  [0] * 16], dtype=np.float32)
    q, s, sg, c = O.nvfp4_quantize(x, global_in=1.0, if4=True)
    q0, s0, _, _ = O.nvfp4_quantize(x, global_in=1.0)
    assert c["blocks_four"] == 0 and (s >> 7 == IF4_ROW[3]).all()
    assert np.array_equal(q, q0) and np.array_equal(s, s0)
    assert np.array_equal(O.dequantize(q, s, O.IF4, sg), x)


def test_if4_saturation_and_clamped_scale():
    """With a small caller global scale the block scale clamps at 448 and elements beyond 7 steps
    saturate to +-7.  s_g = 2^-10 makes the step exactly 0.375 (fl(448 * fl(6/7)) = 384)."""
    sg = 2.0 ** -10
    step = np.float32(np.float32(448.0) * _if4_step(sg))
    assert step == np.float32(0.375)
    k = np.array([1, -2, 3, -4, 5, -6, 6, 5, -4, 3, -2, 1, 2, 4, 10, -12])
    x = (k * 0.375).astype(np.float32)[None, :]
    q, s, _, c = O.nvfp4_quantize(x, global_in=sg, if4=True)
    assert s[0, 0] == (0x80 | 0x7E)  # INT4 flag over E4M3 448
    assert c["saturation"] == 2 and c["underflow"] == 0 and c["blocks_four"] == 1
    codes = np.stack([q & 15, q >> 4], -1).ravel()
    assert [int(O.int4_value(int(v))) for v in codes] == np.clip(k, -7, 7).tolist()


def test_if4_never_worse_than_nvfp4_and_keeps_its_fp4_blocks():
    """Per block the IF4 error (fp64, from the reconstruction) is at most plain NVFP4's; blocks
    that keep E2M1 carry exactly the NVFP4 nibbles and scale; INT4 blocks err by at most half a
    step per unsaturated element; a flat distribution picks INT4 more often than a heavy-tailed
    one, and a rotated Gaussian about as often as a plain one."""
    rng = np.random.default_rng(12)
    frac = {}
    for name, x in [("uniform", rng.uniform(-1, 1, (32, 512))), ("gauss", rng.standard_normal((32, 512))),
                    ("laplace", rng.laplace(size=(32, 512)))]:
        x = O._f32(x)
        q, s, sg, c = O.nvfp4_quantize(x, if4=True)
        q0, s0, sg0, _ = O.nvfp4_quantize(x)
        assert sg == sg0
        flag = (s >> 7).astype(bool)
        frac[name] = flag.mean()
        assert c["blocks_four"] == flag.sum()
        keep = np.repeat(~flag, 8, axis=1)
        assert np.array_equal(q[keep], q0[keep]) and np.array_equal(s[~flag], s0[~flag])
        assert np.array_equal(s[flag] & 0x7F, s0[flag])
        xh = O.dequantize(q, s, O.IF4, sg).astype(np.float64)
        xh0 = O.dequantize(q0, s0, O.NVFP4, sg0).astype(np.float64)
        e = ((x - xh) ** 2).reshape(32, -1, 16).sum(-1)
        e0 = ((x - xh0) ** 2).reshape(32, -1, 16).sum(-1)
        assert (e <= e0 * (1 + 1e-5) + 1e-30).all()
        d = np.array([O.e4m3_value(int(b) & 0x7F) for b in s.ravel()]).reshape(s.shape)
        step = np.repeat(d * float(_if4_step(sg)), 16, axis=1)
        fl16 = np.repeat(flag, 16, axis=1)
        inside = fl16 & (np.abs(x) <= 7 * step)
        assert (np.abs(x - xh)[inside] <= 0.5 * step[inside] * (1 + 2 ** -20)).all()
    assert frac["uniform"] > frac["gauss"] > frac["laplace"] > 0
    xr = O.fwht(O._f32(rng.standard_normal((32, 512))))
    _, s, _, _ = O.nvfp4_quantize(xr, if4=True)
    assert abs((s >> 7).mean() - frac["gauss"]) < 0.1


def test_if4_picks_lower_error_candidate_brute_force():
    """Independent brute force: per block, the E2M1 candidate from torch's E4M3 cast and a numpy
    nearest-lattice search, the INT4 candidate from numpy's round-half-even on the 6/7 step; the
    oracle's reconstruction must be at least as good as the better of the two, and its flag must
    name the candidate whose error it has."""
    rng = np.random.default_rng(15)
    x = O._f32(np.concatenate([rng.standard_normal((4, 64)), rng.uniform(-1, 1, (4, 64))]))
    q, s, sg, c = O.nvfp4_quantize(x, if4=True)
    lat = np.array(LATTICE)
    xh = O.dequantize(q, s, O.IF4, sg).astype(np.float64)
    step7 = np.float32(np.float32(sg) * (np.float32(6) / np.float32(7)))
    for r in range(8):
        for b in range(4):
            blk = x[r, 16 * b:16 * b + 16]
            inv = np.float32(1) / (np.float32(6) * np.float32(sg))
            code = torch.tensor([np.float32(np.abs(blk).max()) * inv]).to(torch.float8_e4m3fn).view(torch.uint8).item()
            d = np.float32(O.e4m3_value(code))
            R = np.float32(1) / (d * np.float32(sg))
            y = (blk * R).astype(np.float64)
            mags = np.array([lat[np.argmin(np.abs(lat - min(abs(v), 6.0)) + (np.arange(8) % 2) * 1e-12)] for v in y])
            rec6 = np.sign(y) * mags * float(d) * sg
            R7 = np.float32(1) / np.float32(d * step7)
            k = np.clip(np.rint(np.abs((blk * R7).astype(np.float64))), 0, 7) * np.sign(blk)
            rec7 = (k * float(d)).astype(np.float32) * step7
            e6 = float(((blk.astype(np.float64) - rec6) ** 2).sum())
            e7 = float(((blk.astype(np.float64) - rec7.astype(np.float64)) ** 2).sum())
            got = float(((blk.astype(np.float64) - xh[r, 16 * b:16 * b + 16]) ** 2).sum())
            assert got <= min(e6, e7) * (1 + 1e-5) + 1e-30
            flagged = bool(s[r, b] & 0x80)
            assert abs(got - (e7 if flagged else e6)) <= 1e-5 * max(got, 1e-30)


def test_if4_rejected_blocks():
    x = O._f32(np.random.default_rng(13).uniform(-1, 1, (1, 64)))
    x[0, 3], x[0, 20], x[0, 40] = np.inf, np.nan, -np.inf
    q, s, _, c, spec = O.nvfp4_quantize(x, global_in=1.0, if4=True, spec=True)
    assert c["nonfinite"] == 3 and spec.tolist() == [[False, False, False, True]]


# ---------------------------------------------------------------------------------------------
# Walsh-Hadamard rotation

def test_fwht_norm_constant():
    assert O.fwht_norm_const(8192) == np.float32(1 / math.sqrt(8192))
    assert O.fwht_norm_const(4096) == 2.0 ** -6


def test_fwht_matches_sylvester_hadamard_matrix():
    from scipy.linalg import hadamard
    rng = np.random.default_rng(8)
    for d in (1024, 2048):
        x = O._f32(rng.standard_normal((3, d)))
        ref = (x.astype(np.float64) @ hadamard(d).T.astype(np.float64)) / math.sqrt(d)
        got = O.fwht(x).astype(np.float64)
        # fp32 butterflies: normwise error within log2(d) roundings of 2^-24 each (doubled)
        assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < math.log2(d) * 2.0 ** -23


def test_fwht_involution_is_exact_on_small_integers():
    """H H^T = I: with d = 4^k, c = 2^-k exactly and all sums of small integers are exact."""
    rng = np.random.default_rng(9)
    for d in (1024, 4096, 16384):
        x = rng.integers(-8, 9, size=(2, d)).astype(np.float32)
        assert np.array_equal(O.fwht(O.fwht(x)), x)
    x = rng.integers(-8, 9, size=(2, 8192)).astype(np.float32)
    assert np.allclose(O.fwht(O.fwht(x)), x, rtol=0, atol=1e-5)


def test_fwht_spike_damping():
    d, spike, damp = golden_rows("hadamard_spike.txt")[0]
    d, spike = int(d), float(spike)
    x = np.zeros((1, d), dtype=np.float32)
    x[0, 1234] = spike
    y = O.fwht(x)[0]
    c = np.float32(O.fwht_norm_const(d))
    assert np.all(np.abs(y) == np.float32(spike) * c)
    assert round(spike / np.abs(y).max(), 1) == float(damp)
    # sign pattern is column 1234 of the Sylvester matrix: (-1)^popcount(i & 1234)
    signs = np.array([(-1) ** bin(i & 1234).count("1") for i in range(d)])
    assert np.array_equal(np.sign(y), signs)


def test_fwht_parseval():
    x = O._f32(np.random.default_rng(10).laplace(size=(4, 8192)))
    y = O.fwht(x)
    n0 = np.linalg.norm(x.astype(np.float64), axis=1)
    n1 = np.linalg.norm(y.astype(np.float64), axis=1)
    assert np.max(np.abs(n1 / n0 - 1)) < 1e-6


def _sign_vector(bits_words, d):
    """+-1 per channel from the packed sign bits (bit i % 32 of word i // 32 set -> -1)."""
    w = np.asarray(bits_words, dtype=np.uint32)
    b = (w[np.arange(d) // 32] >> (np.arange(d) % 32).astype(np.uint32)) & 1
    return np.where(b == 1, -1.0, 1.0)


def test_mx_rows_at_offset_match_the_whole_tensor():
    """Stochastic rounding follows the flat element index: quantising one row at its flat offset
    reproduces that row of the whole-tensor call (used for sampled rows of very large tensors)."""
    from block_scaled_fp4_amax_b200 import synth
    x = synth.as_f32_numpy(synth.mx_small())
    q0, s0, _ = O.mx_quantize(x, round=O.STOCHASTIC, seed=3)
    for r in (0, 5, 255):
        q1, s1, _ = O.mx_quantize_rows_at(x[r:r + 1], r * x.shape[1], round=O.STOCHASTIC, seed=3)
        assert np.array_equal(q0[r:r + 1], q1) and np.array_equal(s0[r:r + 1], s1)


def test_rht_without_signs_is_the_plain_rotation():
    x = O._f32(np.random.default_rng(12).standard_normal((3, 2048)))
    assert np.array_equal(O.fwht(x, np.zeros(64, dtype=np.uint32)), O.fwht(x))


def test_rht_inverse_is_exact_on_small_integers():
    """Q = c H D with Q^-1 = c D H: rotating with the signs, then rotating back without them and
    negating the signed channels, returns small-integer inputs exactly (d = 4^k makes c a power of
    two).  A rotation that applied the signs after the butterflies would not invert this way."""
    from block_scaled_fp4_amax_b200 import synth
    rng = np.random.default_rng(13)
    for d in (1024, 4096):
        sg = synth.rht_signs(d, 21)
        s = _sign_vector(sg, d)
        x = rng.integers(-8, 9, size=(2, d)).astype(np.float32)
        y = O.fwht(x, sg)
        back = (s * O.fwht(y).astype(np.float64)).astype(np.float32)
        assert np.array_equal(back, x)
        assert not np.array_equal(y, O.fwht(x))      # the signs change the rotation


def test_rht_matches_explicit_matrix():
    """c H D x in fp64 from scipy's Hadamard matrix and the decoded signs, within the butterflies'
    fp32 rounding."""
    from scipy.linalg import hadamard
    from block_scaled_fp4_amax_b200 import synth
    d = 1024
    sg = synth.rht_signs(d, 22)
    s = _sign_vector(sg, d)
    x = O._f32(np.random.default_rng(14).standard_normal((3, d)))
    Q = hadamard(d).astype(np.float64) * s[None, :] / math.sqrt(d)
    ref = x.astype(np.float64) @ Q.T
    got = O.fwht(x, sg).astype(np.float64)
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < math.log2(d) * 2.0 ** -23
    assert np.allclose(Q @ Q.T, np.eye(d), atol=1e-12)   # orthogonal


def test_exp_cw_against_the_exponential():
    """The written-out exponential of the SwiGLU path: within 4 units of 2^-24 (relative) of e^x over
    the normal range, exact at 0, and the stated saturation at both ends."""
    xs = np.linspace(-87.0, 88.0, 20001, dtype=np.float32)
    rel = max(abs(O.exp_cw(x) - math.exp(float(x))) / math.exp(float(x)) for x in xs)
    assert rel < 4 * 2.0 ** -24
    assert O.exp_cw(0.0) == 1.0 and O.exp_cw(-0.0) == 1.0
    assert O.exp_cw(88.6) == math.inf and O.exp_cw(-103.5) == 0.0
    assert math.isnan(O.exp_cw(float("nan")))
    # monotone across the reduction boundaries (n changes every ln2)
    ys = [O.exp_cw(x) for x in np.linspace(-5.0, 5.0, 4001, dtype=np.float32)]
    assert all(b >= a for a, b in zip(ys, ys[1:]))


def test_silu_mul_against_fp64():
    rng = np.random.default_rng(15)
    g = rng.standard_normal(20000).astype(np.float32) * 4
    u = rng.standard_normal(20000).astype(np.float32)
    a = O.silu_mul(g, u).astype(np.float64)
    g64, u64 = g.astype(np.float64), u.astype(np.float64)
    ref = g64 / (1.0 + np.exp(-g64)) * u64
    ok = np.abs(ref) > 1e-30
    assert np.max(np.abs(a[ok] - ref[ok]) / np.abs(ref[ok])) < 8 * 2.0 ** -24
    z = O.silu_mul(np.zeros(3, np.float32), np.float32([1, -2, 3]))
    assert np.array_equal(z, np.zeros(3, np.float32))
    big = O.silu_mul(np.float32([40.0]), np.float32([3.0]))   # SiLU(g) = g once e^-g vanishes
    assert big[0] == np.float32(120.0)


def test_swiglu_rotation_composes_the_parts():
    from block_scaled_fp4_amax_b200 import synth
    g, u = (synth.as_f32_numpy(t) for t in synth.swiglu_inputs(4, 1024, 3))
    y, q, s, sg, c = O.swiglu_fwht_quantize(g, u, seed=7)
    y2 = O.fwht(O.silu_mul(g, u))
    assert np.array_equal(y, y2)


# ---------------------------------------------------------------------------------------------
# Dequantisation and the GEMM reference

def test_dequant_f32_equals_exact_value_when_representable():
    x = O._f32(np.random.default_rng(11).standard_normal((32, 128)))
    q, s, sg, _ = O.nvfp4_quantize(x)
    a = O.dequantize(q, s, O.NVFP4, sg).astype(np.float64)
    b = O.dequantize_f64(q, s, O.NVFP4, sg)
    assert np.max(np.abs(a - b) / np.maximum(np.abs(b), 1e-30)) <= 2 ** -24
    q, s, _ = O.mx_quantize(x)
    assert np.array_equal(O.dequantize(q, s, O.MXFP4).astype(np.float64), O.dequantize_f64(q, s, O.MXFP4))


def test_gemm_reference_closed_forms():
    M, N, K = 128, 256, 512
    # every A element = 1 with E8M0 scale 2^1, every B element = 1.5 with 2^-3: C = K * 2 * 1.5/8
    Aq = np.full((M, K // 2), 0x22, dtype=np.uint8)   # code 2 (1.0) in both nibbles
    Bq = np.full((N, K // 2), 0x33, dtype=np.uint8)   # code 3 (1.5)
    As = np.full((M, K // 32), 128, dtype=np.uint8)
    Bs = np.full((N, K // 32), 124, dtype=np.uint8)
    C, S = O.gemm_f64(Aq, As, 1.0, Bq, Bs, 1.0, O.MXFP4)
    assert np.all(C == K * 2 * 1.5 / 8) and np.all(S == C)
    # one-hot: A row m has a single 6.0 at column (m % K); B row n a single -4 at column (n % K)
    Aq = np.zeros((M, K // 2), dtype=np.uint8)
    Bq = np.zeros((N, K // 2), dtype=np.uint8)
    for m in range(M):
        k = (3 * m) % K
        Aq[m, k // 2] |= 7 << (4 * (k & 1))
    for n in range(N):
        k = (3 * n) % K
        Bq[n, k // 2] |= 0xE << (4 * (k & 1))
    As = np.full((M, K // 16), 0x38, dtype=np.uint8)   # E4M3 1.0
    Bs = np.full((N, K // 16), 0x40, dtype=np.uint8)   # E4M3 2.0
    C, _ = O.gemm_f64(Aq, As, 0.5, Bq, Bs, 0.25, O.NVFP4)
    want = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            if (3 * m) % K == (3 * n) % K:
                want[m, n] = 6.0 * 1.0 * 0.5 * (-4.0) * 2.0 * 0.25
    assert np.array_equal(C, want)


def test_if4_gemm_reference_alignment_factors():
    """IF4 block products (podcast IF4 segment, tests/golden/if4.txt): an FP4 x INT4 block pair
    carries six sevenths, an INT4 x INT4 pair thirty-six forty-ninths.  Rows of one 16-block: FP4
    blocks of code 7 (6.0) or 5 (3.0), INT4 blocks of code 7 (+7) or 13 (-5); every product is
    checked against the exact rational value."""
    from fractions import Fraction
    _, _, _, _, _, mix_n, mix_d, ii_n, ii_d = [int(v) for v in golden_rows("if4.txt")[0]]
    rows = [(0x77, 0x38, Fraction(6)), (0x55, 0x38, Fraction(3)),        # FP4 blocks, scale 1.0
            (0x77, 0xB8, Fraction(7)), (0xDD, 0xC0, Fraction(-5))]       # INT4 blocks, scale 1.0 / 2.0
    Aq = np.array([[b] * 8 for b, _, _ in rows], dtype=np.uint8)
    As = np.array([[sb] for _, sb, _ in rows], dtype=np.uint8)
    sga, sgb = 0.5, 0.25
    C, S = O.gemm_f64(Aq, As, sga, Aq, As, sgb, O.IF4)
    for i, (_, sa, va) in enumerate(rows):
        for j, (_, sb, vb) in enumerate(rows):
            int_a, int_b = bool(sa & 0x80), bool(sb & 0x80)
            f = {0: Fraction(1), 1: Fraction(mix_n, mix_d), 2: Fraction(ii_n, ii_d)}[int_a + int_b]
            da = Fraction(O.e4m3_value(sa & 0x7F)).limit_denominator()
            db = Fraction(O.e4m3_value(sb & 0x7F)).limit_denominator()
            want = 16 * va * vb * da * db * f * Fraction(sga) * Fraction(sgb)
            assert abs(C[i, j] - float(want)) <= 1e-12 * abs(float(want)), (i, j, C[i, j], want)
    # the stretch: an INT4 block at its maximum (7) reconstructs an FP4 block at its maximum (6)
    assert C[2, 2] == C[0, 0] == C[0, 2]


def test_scale_tile_layout_is_a_bijection_with_the_documented_offsets():
    rows, nb = 256, 8
    s = np.arange(rows * nb, dtype=np.int64).reshape(rows, nb) % 251
    t = O.scales_to_mma_tiled(s.astype(np.uint8))
    assert np.array_equal(O.scales_from_mma_tiled(t, rows, nb), s.astype(np.uint8))
    # row 37, block 6: tile (0, 1), in-tile (37 % 32) * 16 + (37 // 32) * 4 + 2
    assert t[1 * 512 + 5 * 16 + 1 * 4 + 2] == s[37, 6]
    # row 130, block 1: tile (1, 0) -> 2 * 512, in-tile 2 * 16 + 0 * 4 + 1
    assert t[2 * 512 + 2 * 16 + 1] == s[130, 1]


def test_nvfp4_vs_mxfp4_mse_ratio_reported():
    """Context only (parity unpinned): the Eluvix page claims ~2.4x lower block MSE for NVFP4 with
    no data distribution given; on N(0,1) the ratio is reported, asserting only NVFP4 < MXFP4."""
    x = O._f32(np.random.default_rng(12).standard_normal((128, 1024)))
    q, s, sg, _ = O.nvfp4_quantize(x)
    e_nv = ((O.dequantize(q, s, O.NVFP4, sg) - x) ** 2).mean()
    q, s, _ = O.mx_quantize(x)
    e_mx = ((O.dequantize(q, s, O.MXFP4) - x) ** 2).mean()
    assert e_nv < e_mx

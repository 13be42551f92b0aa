"""Comparison helpers shared by the GPU parity tests.

Codes and scale bytes are compared bit for bit on every block whose outputs the definition fixes
(the oracle's `spec` mask).  The blocks left open are the rejected ones (a value that is Inf or
NaN: "MXFP4 Quantization: Audit the 4.25-Bit Blocks", "Publish the MXFP4 audit receipt", lists
non-finite input among the inputs to reject) and, under a per-tensor scale that is not finite or
too small, blocks whose fp32 steps give a NaN.  Both sides leave a rejected block out of the
underflow, saturation and blocks_four counters, so the counters are compared exactly whenever every
open block is a rejected one; otherwise only the non-finite count is.
"""
from __future__ import annotations

import numpy as np

import block_scaled_fp4_amax_b200 as fp4
import oracle as O


def npy(t):
    return t.detach().cpu().numpy()


def counts_of(c):
    v = [int(x) for x in c.cpu().tolist()]
    return dict(underflow=v[0], saturation=v[1], nonfinite=v[2], blocks_four=v[3])


def rowmajor_scales(gpu_scales, rows: int, nb: int, layout: int) -> np.ndarray:
    s = npy(gpu_scales)
    if layout == fp4.MMA_TILED:
        return O.scales_from_mma_tiled(s, rows, nb)
    return s.reshape(rows, nb)


def compare_blocks(q, s, qo, so, spec, block: int, layout: int) -> None:
    """Nibbles and scale bytes bit-exact on the blocks `spec` marks as defined."""
    rows, nb = so.shape
    qg = npy(q).reshape(qo.shape)
    sg = rowmajor_scales(s, rows, nb, layout)
    qmask = np.repeat(spec, block // 2, axis=1)
    assert np.array_equal(qg[qmask], qo[qmask])
    assert np.array_equal(sg[spec], so[spec])


def compare_counts(c, co, x, spec, block: int) -> None:
    """All four counters exact when every open block holds a non-finite value of `x` (the array
    the blocks were formed from), else the non-finite count alone."""
    got = counts_of(c)
    rows = x.shape[0]
    finite = np.isfinite(x).reshape(rows, -1, block).all(-1)
    if np.array_equal(spec, finite):
        assert got == co, (got, co)
    else:
        assert got["nonfinite"] == co["nonfinite"], (got, co)

"""nvfp4_quantize_noalloc: the NVFP4 quantiser for callers that cannot allocate device memory
(for example a plugin that is handed only its input and output buffers, or a latency-critical loop
that must not call cudaMalloc).  Its scratch word lives in a fixed area of the library's own device
memory, so these checks make sure that (1) its results equal those of nvfp4_quantize with a caller
workspace, and (2) two calls in a row do not see each other's scratch: the second call quantises a
tensor with a much smaller amax, which would come out wrong if the first call's amax were left in
the shared area.  The bar is the one the parity tests use for encodings: bit-exact nibbles, scale
bytes, global scale and counters.

This file is named to be collected last, so that a run stopping at the first failure has already
run every other test.
"""
import numpy as np
import pytest
import torch

import block_scaled_fp4_amax_b200 as fp4
from block_scaled_fp4_amax_b200 import synth

pytestmark = pytest.mark.gpu


def _same(a, b):
    for u, v in zip(a, b):
        assert torch.equal(u.cpu(), v.cpu())


@pytest.mark.parametrize("mode", ["plain", "four_six", "if4"])
@pytest.mark.parametrize("on_stream", [False, True])
def test_noalloc_matches_workspace_entry_point_on_consecutive_calls(cuda, mode, on_stream):
    kw = {"four_six": mode == "four_six", "if4": mode == "if4"}
    big = synth.nv_outliers(512, 2048, seed=5).to(cuda)        # amax ~ 100s (outlier columns)
    small = (synth.normal_f32(512, 2048, 9) * 0.01).to(torch.bfloat16).to(cuda)
    stream = torch.cuda.Stream() if on_stream else None
    fp4.nvfp4_quantize_noalloc(big, stream=stream, **kw)        # warm: the per-device set-up is done
    torch.cuda.synchronize()
    for x in (big, small, big):
        want = fp4.nvfp4_quantize(x, **kw)
        # the outputs are allocated before the free-memory reading: the call itself allocates nothing
        q = torch.empty((x.shape[0], x.shape[1] // 2), dtype=torch.uint8, device=cuda)
        s = torch.empty(x.numel() // 16, dtype=torch.uint8, device=cuda)
        g = torch.empty(1, dtype=torch.float32, device=cuda)
        c = torch.empty(4, dtype=torch.int64, device=cuda)
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        got = fp4.nvfp4_quantize_noalloc(x, stream=stream, out=(q, s, g, c), **kw)
        torch.cuda.synchronize()
        assert torch.cuda.mem_get_info()[0] == free0
        _same(got, want)


def test_noalloc_caller_scale_and_argument_errors(cuda):
    x = synth.normal_bf16(256, 512, 11).to(cuda)
    g = torch.tensor([0.003], device=cuda)
    _same(fp4.nvfp4_quantize_noalloc(x, global_in=g, round=fp4.STOCHASTIC, seed=7),
          fp4.nvfp4_quantize(x, global_in=g, round=fp4.STOCHASTIC, seed=7))
    with pytest.raises(fp4.Fp4Error):
        fp4.nvfp4_quantize_noalloc(x, block=32)   # NVFP4 blocks are 16: rejected, nothing launched
    # the failed call left the shared scratch untouched: the next call is still exact
    _same(fp4.nvfp4_quantize_noalloc(x), fp4.nvfp4_quantize(x))

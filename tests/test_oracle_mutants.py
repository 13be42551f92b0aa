"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source (a dropped term, a wrong constant,
an index or sign slip, a rule left out), compiles the copy, points the oracle module at it, and
checks that the pin named beside it now fails.  The oracle itself is never modified; every
mistake is planted on the CPU.
"""
import ctypes
import os
import subprocess

import pytest

import oracle as O
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(O.__file__), "fp4_oracle.c")

# (name, text in fp4_oracle.c, replacement, pins expected to fail)
MUTANTS = [
    ("T=4 candidate scaled for a maximum of 6", "  float ts = T * s_g;", "  float ts = 6.0f * s_g;",
     [pins.test_four_over_six_pins]),
    ("4/6 keeps the worse candidate", "        if (sse4 < sse6) {", "        if (sse4 > sse6) {",
     [pins.test_four_over_six_pins, pins.test_four_over_six_picks_lower_error_candidate_brute_force]),
    ("E8M0 byte decoded one exponent off", "(float)ldexp(v, (int)sb - 127)", "(float)ldexp(v, (int)sb - 126)",
     [pins.test_e8m0_limits]),
    ("MXFP4 block normalised by 2^-(e+1)", "float inv_scale = ldexpf(1.0f, -e);",
     "float inv_scale = ldexpf(1.0f, -e - 1);", [pins.test_e8m0_limits]),
    ("NVFP4 global constant 6*448 mistyped", "float six_m = four_six ? 1536.0f : 2688.0f;",
     "float six_m = four_six ? 1536.0f : 2668.0f;", [pins.test_nvfp4_scale_is_amax_over_six_cast_to_e4m3]),
    ("block scale argument without the global scale", "  float inv_t = 1.0f / ts;", "  float inv_t = 1.0f / T;",
     [pins.test_nvfp4_scale_is_amax_over_six_cast_to_e4m3]),
    ("blocks holding Inf or NaN encoded instead of rejected", "      int defined = !bad && isfinite(s_g);",
     "      int defined = isfinite(s_g);", [pins.test_rejected_blocks_and_counts]),
    ("non-finite values not counted", "      cnt->nonfinite += (uint64_t)bad;", "",
     [pins.test_rejected_blocks_and_counts]),
    ("E2M1 exponent bias dropped", "ldexp(1.0 + 0.5 * m, e - 1)", "ldexp(1.0 + 0.5 * m, e)",
     [pins.test_e2m1_decode_table_matches_printed_lattice]),
    ("IF4 INT4 blocks without the six-sevenths step in the GEMM reference",
     "(double)s_g * 6.0 / 7.0;", "(double)s_g;", [pins.test_if4_gemm_reference_alignment_factors]),
    ("Hadamard butterfly difference reversed", "        v[i + h] = a - b;", "        v[i + h] = b - a;",
     [pins.test_fwht_matches_sylvester_hadamard_matrix]),
]


def _build_mutant(tmp_path, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
                           "-o", str(so), str(path), "-lm"])
    return O.configure(ctypes.CDLL(str(so)))


@pytest.mark.parametrize("name,old,new,targets", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pin_fails_on_planted_mistake(tmp_path, monkeypatch, name, old, new, targets):
    O.lib()
    for t in targets:  # the real oracle passes the pin
        t()
    monkeypatch.setattr(O, "_lib", _build_mutant(tmp_path, old, new))
    for t in targets:
        with pytest.raises(AssertionError):
            t()

"""The oracle's pins must be able to fail.

Each case plants one plausible mistake in a copy of the oracle's C++ source (a wrong
region boundary, a flipped shift direction, a dropped scale, a wrong head offset, a
missing normalisation, an unbiased variance, eps outside the square root, a dropped
"1 +" in the FiLM gain, an off-by-one wrap strip in the brute force), builds it on the
CPU, and checks that at least one pin in tests/test_oracle.py rejects it.
"""
import os
import subprocess

import pytest

import oracle
from tests import test_oracle as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "swin3d_oracle.cpp")

MUTATIONS = {
    "label_boundary": ("if (pprime < P - s) return 1;", "if (pprime < P - w + s) return 1;"),
    "shift_direction": ("p[a] = (pprime + g.s[a]) % g.P[a];", "p[a] = (pprime + g.P[a] - g.s[a]) % g.P[a];"),
    "scale_dropped": ("logit[j] = scale * dot +", "logit[j] = dot +"),
    "q_head_offset": ("const int64_t qi = t[i] * token_stride + h * head_dim;",
                      "const int64_t qi = t[i] * token_stride;"),
    "no_normalisation": ("for (int64_t j = 0; j < N; ++j) pw[j] /= sum;", ""),
    "unbiased_variance": ("var /= C;", "var /= (C - 1);"),
    "eps_outside_sqrt": ("1.0 / std::sqrt(var + eps)", "1.0 / (std::sqrt(var) + eps)"),
    "film_gain": ("film_form == 0 ? 1.0 + sc : sc", "sc"),
    "strip_off_by_one": ("(p[a] < g.s[a] ? 1 : 0)", "(p[a] <= g.s[a] ? 1 : 0)"),
}

PIN_CALLS = [
    lambda: [pins.test_window_attn_matches_dense_bruteforce(c) for c in pins.CASES],
    lambda: [pins.test_window_attn_matches_torch_route(c) for c in pins.CASES],
    lambda: [pins.test_region_group_sizes_golden(r) for r in pins._golden_rows()],
    lambda: [pins.test_softmax_rows_sum_to_one_and_masked_zero(c) for c in pins.CASES[:4]],
    lambda: pins.test_shift0_equals_block_attention(),
    lambda: [pins.test_adaln_matches_torch_layer_norm(b) for b in (True, False)],
    lambda: pins.test_adaln_constant_row_gives_residual_plus_shift(),
    lambda: pins.test_adaln_zero_film_closed_form(),
]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    mutated = tmp_path / "mutant.cpp"
    mutated.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.run(["g++", "-O1", "-std=c++17", "-fopenmp", "-shared", "-fPIC", str(mutated), "-o", str(so)],
                   check=True)
    saved = oracle._load()
    oracle._lib = oracle._bind(str(so))
    caught = 0
    try:
        for call in PIN_CALLS:
            try:
                call()
            except AssertionError:
                caught += 1
    finally:
        oracle._lib = saved
    assert caught >= 1, f"no pin caught the planted mistake '{name}'"

"""Pins of the fp64 oracle (CPU only).

The oracle is checked against things that are not itself:
  * a pure-Python brute force (complex-number RoPE, per-pair loops),
  * torch's fp64 scaled-dot-product attention (out and LSE) in the special cases
    where bifocal attention reduces to plain RoPE attention: G = 1 and w0 >= L
    (ai-feeds summary, 方法 key modules 1 and 2: the local window keeps the
    unmodified RoPE and G = 1 restores the base model), and w0 = 0 where it is
    linear position interpolation (frequency interpolation) or floor-grouped
    positions (position aliasing),
  * the inclusion-exclusion merge (ai-feeds summary, key module 3; seventnews
    article: no double counting) against the direct masked softmax,
  * shift invariance of RoPE scores, closed-form rotation identities, softmax
    properties, the prefill/decode consistency of the correction rotation,
  * the dynamic-factor table worked by hand from the printed formula.
"""
import itertools

import numpy as np
import pytest

import oracle.bifocal_ref as R
from tests import pins

MODES = ("freq_interp", "pos_alias")


def test_golden_dynamic_factor():
    assert pins.check_golden_factor() == 0


def test_dynamic_factor_rejects_bad_args():
    with pytest.raises(ValueError):
        R.dynamic_factor(10, 0)
    with pytest.raises(ValueError):
        R.dynamic_factor(-1, 4)


def test_rotation_closed_forms():
    assert pins.check_rotation_closed_forms() < 1e-12


def test_far_focus_frequency_scale_half_at_g2():
    # knowledge-base note, 关键实现 / 技术参数: far-focus frequencies beta * theta^(-2d/D), beta = 0.5;
    # in the dynamic reading beta = 1/G, and beta = 0.5 is the G = 2 case (frequency interpolation).
    om = R.rope_omega(128, 1e6)
    pos, w = R.long_branch_rope(np.arange(10), om, 2, "freq_interp")
    assert np.array_equal(pos, np.arange(10, dtype=np.float64))
    assert np.allclose(w, 0.5 * om, rtol=0, atol=0)


BRUTE_GRID = [
    (L, D, hq, hkv, w0, w_pre, mode)
    for L, D, (hq, hkv), w_pre, mode in itertools.product((1, 2, 7, 16, 33), (4, 8), ((1, 1), (4, 2)), (1, 4, 16),
                                                          MODES)
    for w0 in sorted({0, 1, 3, L})
]


@pytest.mark.parametrize("L,D,hq,hkv,w0,w_pre,mode", BRUTE_GRID)
def test_brute_force_grid(L, D, hq, hkv, w0, w_pre, mode):
    assert pins.check_brute(L, D, hq, hkv, w0, w_pre, mode) < 1e-12


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("w0", [0, 5, 48])
def test_brute_force_L48(mode, w0):
    assert pins.check_brute(48, 8, 4, 2, w0, 16, mode) < 1e-12


@pytest.mark.parametrize("mode", MODES)
def test_brute_force_with_offset(mode):
    assert pins.check_brute(12, 8, 2, 1, 3, 4, mode, pos_offset=5) < 1e-12


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("w0", [0, 3, 17, 100])
def test_g1_is_plain_rope_attention(mode, w0):
    # L <= w_pretrained -> G = 1: both branches coincide with the original RoPE.
    assert pins.check_sdpa_case("g1", 40, 8, 4, 2, w0, 40, mode) < 1e-12
    assert pins.check_sdpa_case("g1", 40, 16, 2, 2, w0, 64, mode) < 1e-12


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("w_pre", [1, 3, 8])
def test_wide_window_is_plain_rope_attention(mode, w_pre):
    # w0 >= L: every causal pair is in the local window, for any G.
    assert pins.check_sdpa_case("wide", 37, 8, 4, 2, 37, w_pre, mode) < 1e-12
    assert pins.check_sdpa_case("wide", 37, 8, 2, 1, 1000, w_pre, mode) < 1e-12


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("L,w_pre", [(24, 7), (50, 16), (33, 1)])
def test_w0_zero_is_interpolation_or_grouping(mode, L, w_pre):
    assert pins.check_sdpa_case("w0zero", L, 8, 4, 2, 0, w_pre, mode) < 1e-12


@pytest.mark.parametrize("offset", [0, 17, 100000])
def test_plain_oracle_vs_sdpa(offset):
    assert pins.check_plain_vs_sdpa(30, 8, 4, 2, pos_offset=offset) < 1e-9


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("L,w0,w_pre", [(30, 6, 8), (64, 1, 5), (64, 63, 2), (45, 0, 9), (45, 45, 9)])
def test_inclusion_exclusion_equals_direct(mode, L, w0, w_pre):
    assert pins.check_inclusion_exclusion(L, 8, 2, 1, w0, w_pre, mode) < 1e-10


@pytest.mark.parametrize("c", [1, 17, 100000])
def test_shift_invariance_original_rope(c):
    # w0 >= L and G = 1: the original RoPE only sees i - j.
    assert pins.check_shift(40, 8, 40, 64, "freq_interp", c) < 1e-9


@pytest.mark.parametrize("c", [1, 17, 100000])
def test_shift_invariance_freq_interp_long_branch(c):
    assert pins.check_shift(40, 8, 0, 8, "freq_interp", c) < 1e-9


def test_shift_invariance_pos_alias_only_for_multiples_of_g():
    # G = 5 here; floor(p/G) commutes with shifts by multiples of G only.
    assert pins.check_shift(40, 8, 0, 8, "pos_alias", 10) < 1e-9
    assert pins.check_shift(40, 8, 0, 8, "pos_alias", 100000) < 1e-9
    assert pins.check_shift(40, 8, 0, 8, "pos_alias", 3) > 1e-3


def test_softmax_properties():
    assert pins.check_softmax_properties() < 1e-12
    assert pins.check_softmax_properties(mode="pos_alias") < 1e-12


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("L,w0,w_pre", [(33, 5, 8), (16, 3, 8), (17, 3, 8), (9, 0, 8), (40, 40, 8), (25, 1, 1)])
def test_decode_matches_last_prefill_row(mode, L, w0, w_pre):
    # The correction rotation re-phases cached (original-RoPE) keys: decode at length L
    # equals row L-1 of a prefill of length L, including lengths where G has just changed.
    assert pins.check_decode_consistency(L, 8, 4, 2, w0, w_pre, mode) < 1e-11


def test_rows_subset_matches_full():
    q, k, v = pins.qkv64(7, 50, 4, 2, 8)
    full_o, full_l = R.bifocal_attention(q, k, v, 7, 16, 1e4, "pos_alias")
    rows = [0, 6, 7, 8, 31, 49]
    o, l = R.bifocal_attention(q, k, v, 7, 16, 1e4, "pos_alias", rows=rows, row_chunk=4)
    assert np.array_equal(o[0], full_o[0, rows]) and np.array_equal(l[0], full_l[0][:, rows])


def test_battery_clean():
    for name, fn, tol in pins.battery():
        assert fn() <= tol, name

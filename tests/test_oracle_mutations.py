"""Plant plausible mistakes in the oracle (on the CPU) and check that a pin catches each.

Each mutation patches one function of the oracle module for the duration of the
test; the pin battery must then report at least one failure. This shows the pins
are sharp enough that a dropped term, a flipped sign, a wrong index or a
transposed operand in the oracle would not go unnoticed.
"""
import math

import numpy as np
import pytest

import oracle.bifocal_ref as R
from tests import pins

_orig = {name: getattr(R, name) for name in ("rope_rotate", "rope_omega", "long_branch_rope", "dynamic_factor",
                                             "bifocal_scores", "_softmax_out", "kv_head_for", "cached_key_to_raw")}


def _rot_sign_flipped(x, positions, omega):
    return _orig["rope_rotate"](x, -np.asarray(positions, dtype=np.float64), omega)


def _rot_interleaved(x, positions, omega):
    x = np.asarray(x, dtype=np.float64)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * omega[None, :]
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., 0::2], x[..., 1::2]
    y = np.empty_like(x)
    y[..., 0::2] = a * c - b * s
    y[..., 1::2] = b * c + a * s
    return y


def _rot_dropped_cross_term(x, positions, omega):
    x = np.asarray(x, dtype=np.float64)
    P = x.shape[-1] // 2
    ang = np.asarray(positions, dtype=np.float64)[:, None] * omega[None, :]
    c, s = np.cos(ang), np.sin(ang)
    return np.concatenate([x[..., :P] * c - x[..., P:] * s, x[..., P:] * c], axis=-1)


def _omega_wrong_exponent(head_dim, theta):
    k = np.arange(head_dim // 2, dtype=np.float64)
    return np.power(np.float64(theta), -k / head_dim)


def _long_fi_times_g(positions, omega, G, mode):
    p, w = _orig["long_branch_rope"](positions, omega, G, mode)
    return (p, omega * G) if mode == "freq_interp" else (p, w)


def _long_pa_ceil(positions, omega, G, mode):
    if mode == "pos_alias":
        return (-(-np.asarray(positions, dtype=np.int64) // G)).astype(np.float64), omega
    return _orig["long_branch_rope"](positions, omega, G, mode)


def _long_pa_round(positions, omega, G, mode):
    if mode == "pos_alias":
        return np.round(np.asarray(positions, dtype=np.float64) / G), omega
    return _orig["long_branch_rope"](positions, omega, G, mode)


def _factor_floor(L, w):
    return max(1, L // w)


def _factor_round(L, w):
    return max(1, int(round(L / w)))


def _scores_band_inclusive(q_rows, k_all, rows, w0, G, mode, omega, scale, pos_offset=0):
    return _orig["bifocal_scores"](q_rows, k_all, rows, w0 + 1, G, mode, omega, scale, pos_offset)


def _scores_branches_swapped(q_rows, k_all, rows, w0, G, mode, omega, scale, pos_offset=0):
    # local band scored with the long-range RoPE and vice versa
    L = k_all.shape[0]
    s_band = _orig["bifocal_scores"](q_rows, k_all, rows, 0, G, mode, omega, scale, pos_offset)
    s_orig = _orig["bifocal_scores"](q_rows, k_all, rows, L + 1, G, mode, omega, scale, pos_offset)
    dist = np.asarray(rows)[:, None] - np.arange(L)[None, :]
    return np.where(dist < w0, s_band, s_orig)


def _scores_no_scale(q_rows, k_all, rows, w0, G, mode, omega, scale, pos_offset=0):
    return _orig["bifocal_scores"](q_rows, k_all, rows, w0, G, mode, omega, 1.0, pos_offset)


def _scores_mask_transposed(q_rows, k_all, rows, w0, G, mode, omega, scale, pos_offset=0):
    s = _orig["bifocal_scores"](q_rows, k_all, rows, w0, G, mode, omega, scale, pos_offset)
    if s.shape[0] == s.shape[1]:
        finite = np.where(np.isfinite(s), s, 0.0)
        s = np.where(np.isfinite(s).T, finite.T, -np.inf)
    return s


def _softmax_log2(s, v):
    o, lse = _orig["_softmax_out"](s, v)
    return o, lse / math.log(2.0)


def _softmax_dropped_max(s, v):
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    l = np.sum(e, axis=1, keepdims=True)
    return (e @ v) / l, np.log(l)[:, 0]


def _kv_modulo(h, group):
    return h % group


def _cache_unrotate_wrong_sign(kc, positions, omega):
    return _orig["rope_rotate"](kc, np.asarray(positions, dtype=np.float64), omega)


MUTATIONS = {
    "rope_sign_flipped": ("rope_rotate", _rot_sign_flipped),
    "rope_interleaved_pairs": ("rope_rotate", _rot_interleaved),
    "rope_dropped_cross_term": ("rope_rotate", _rot_dropped_cross_term),
    "omega_wrong_exponent": ("rope_omega", _omega_wrong_exponent),
    "fi_multiplies_by_g": ("long_branch_rope", _long_fi_times_g),
    "pa_ceil_instead_of_floor": ("long_branch_rope", _long_pa_ceil),
    "pa_round_instead_of_floor": ("long_branch_rope", _long_pa_round),
    "factor_floor": ("dynamic_factor", _factor_floor),
    "factor_round": ("dynamic_factor", _factor_round),
    "band_edge_inclusive": ("bifocal_scores", _scores_band_inclusive),
    "branches_swapped": ("bifocal_scores", _scores_branches_swapped),
    "scale_dropped": ("bifocal_scores", _scores_no_scale),
    "causal_mask_transposed": ("bifocal_scores", _scores_mask_transposed),
    "lse_in_log2": ("_softmax_out", _softmax_log2),
    "lse_missing_max": ("_softmax_out", _softmax_dropped_max),
    "gqa_modulo_mapping": ("kv_head_for", _kv_modulo),
    "cache_unrotate_wrong_sign": ("cached_key_to_raw", _cache_unrotate_wrong_sign),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(R, attr, fn)
    failed = []
    for pin_name, check, tol in pins.battery():
        try:
            bad = not (check() <= tol)
        except Exception:
            bad = True
        if bad:
            failed.append(pin_name)
    assert failed, f"mutation {name} passed every pin"

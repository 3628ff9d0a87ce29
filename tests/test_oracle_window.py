"""Pins of the sliding-window oracle (CPU): a window that covers the whole causal range is
plain RoPE attention; a window of 1 is a closed form (row i attends to key i alone, so
out_i = v_i and lse_i = scale <q_i, k_i>, RoPE preserving the dot product at one position);
any window equals torch's fp64 scaled-dot-product attention with the same boolean mask over
RoPE-rotated inputs; and the cached-key form equals the direct one on an exact cache."""
import math

import numpy as np
import pytest
import torch

from oracle import bifocal_ref as R

THETA = 1e4


def _inputs(seed, L, hq, hkv, D):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((1, L, hq, D)), rng.standard_normal((1, L, hkv, D)),
            rng.standard_normal((1, L, hkv, D)))


@pytest.mark.parametrize("L,W", [(1, 1), (17, 17), (17, 40), (40, 64)])
def test_window_covering_everything_is_plain_rope(L, W):
    q, k, v = _inputs(L + W, L, 4, 2, 8)
    wo, wl = R.sliding_window_attention(q, k, v, W, THETA)
    po, pl = R.rope_causal_attention(q, k, v, THETA)
    assert np.abs(wo - po).max() < 1e-12 and np.abs(wl - pl).max() < 1e-12


def test_window_of_one_is_closed_form():
    q, k, v = _inputs(3, 23, 4, 2, 8)
    wo, wl = R.sliding_window_attention(q, k, v, 1, THETA)
    g = 2
    for h in range(4):
        assert np.abs(wo[0, :, h] - v[0, :, h // g]).max() < 1e-12
        lse = np.einsum("ld,ld->l", q[0, :, h], k[0, :, h // g]) / math.sqrt(8)
        assert np.abs(wl[0, h] - lse).max() < 1e-12


@pytest.mark.parametrize("L,W", [(30, 2), (30, 7), (64, 13), (64, 33)])
def test_window_equals_torch_sdpa_with_mask(L, W):
    q, k, v = _inputs(L * 7 + W, L, 4, 2, 8)
    wo, _ = R.sliding_window_attention(q, k, v, W, THETA)
    omega = R.rope_omega(8, THETA)
    pos = np.arange(L)
    for h in range(4):
        qr = torch.from_numpy(R.rope_rotate(q[0, :, h], pos, omega))
        kr = torch.from_numpy(R.rope_rotate(k[0, :, h // 2], pos, omega))
        vv = torch.from_numpy(v[0, :, h // 2])
        d = pos[:, None] - pos[None, :]
        mask = torch.from_numpy((d >= 0) & (d < W))
        ref = torch.nn.functional.scaled_dot_product_attention(qr[None], kr[None], vv[None], attn_mask=mask[None])
        assert np.abs(wo[0, :, h] - ref[0].numpy()).max() < 1e-12


@pytest.mark.parametrize("P0,C,W", [(0, 30, 5), (20, 10, 7), (29, 1, 12), (10, 20, 100)])
def test_cached_form_equals_direct(P0, C, W):
    L = P0 + C
    q, k, v = _inputs(P0 * 3 + C + W, L, 4, 2, 8)
    kc = R.rope_keys_for_cache(k[0], THETA)
    co, cl = R.sliding_window_cached_reference(q[0, P0:], kc, v[0], P0, W, THETA)
    ro, rl = R.sliding_window_attention(q, k, v, W, THETA, rows=range(P0, L))
    assert np.abs(co - ro[0]).max() < 1e-12 and np.abs(cl - rl[0]).max() < 1e-12


def test_planted_mistake_window_off_by_one():
    # a window of W + 1 keys (i - j <= W) must fail the torch pin
    L, W = 30, 5
    q, k, v = _inputs(99, L, 2, 1, 8)
    wrong, _ = R.sliding_window_attention(q, k, v, W + 1, THETA)
    right, _ = R.sliding_window_attention(q, k, v, W, THETA)
    assert np.abs(wrong - right).max() > 1e-6

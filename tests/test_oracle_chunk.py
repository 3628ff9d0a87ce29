"""Pins of the chunked-prefill oracle (CPU).

The chunk reference builds its scores from cached keys (original RoPE, taken back to raw
for the long branch), the path a cache-backed chunk takes. It is pinned to the direct
definition, which is pinned by brute force and the textbook special cases: with a cache
written exactly (fp64) from the raw keys, chunk rows P0..L-1 must equal rows P0..L-1 of the
direct bifocal attention over the whole length. Mistakes planted in a copy of the oracle
(G from the cached length, cached keys used without undoing their RoPE, chunk positions
counted from 0) must fail that pin.
"""
import itertools

import numpy as np
import pytest

from oracle import bifocal_ref as R

THETA = 1e4


def _inputs(seed, L, hq, hkv, D):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((1, L, hq, D)), rng.standard_normal((1, L, hkv, D)),
            rng.standard_normal((1, L, hkv, D)))


def _direct(q, k, v, P0, w0, wp, mode):
    L = q.shape[1]
    return R.bifocal_attention(q, k, v, w0, wp, THETA, mode, rows=range(P0, L))


def _chunk(q, k, v, P0, w0, wp, mode, **kw):
    kc = R.rope_keys_for_cache(k[0], THETA)
    return R.bifocal_chunk_reference(q[0, P0:], kc, v[0], P0, w0, wp, THETA, mode, **kw)


GRID = list(itertools.product(
    [(1, 0), (9, 0), (9, 4), (9, 8), (40, 0), (40, 13), (40, 39)],  # (L, P0)
    [(1, 1, 8), (4, 2, 8), (4, 1, 4)],                               # (hq, hkv, D)
    [0, 3, 100],                                                     # w0
    [1, 4, 16],                                                      # w_pretrained
    R.MODES))


@pytest.mark.parametrize("LP,heads,w0,wp,mode", GRID)
def test_chunk_equals_direct_definition(LP, heads, w0, wp, mode):
    (L, P0), (hq, hkv, D) = LP, heads
    q, k, v = _inputs(L * 100 + P0, L, hq, hkv, D)
    ro, rl = _direct(q, k, v, P0, w0, wp, mode)
    co, cl = _chunk(q, k, v, P0, w0, wp, mode)
    assert np.abs(ro[0] - co).max() < 1e-12
    assert np.abs(rl[0] - cl).max() < 1e-12


@pytest.mark.parametrize("mode", R.MODES)
def test_last_chunk_row_equals_decode_reference(mode):
    L, P0 = 37, 30
    q, k, v = _inputs(7, L, 4, 2, 8)
    kc = R.rope_keys_for_cache(k[0], THETA)
    co, cl = R.bifocal_chunk_reference(q[0, P0:], kc, v[0], P0, 5, 8, THETA, mode)
    do, dl = R.bifocal_decode_reference(q[0, L - 1], kc, v[0], L, 5, 8, THETA, mode)
    assert np.abs(co[-1] - do).max() < 1e-12 and np.abs(cl[:, -1] - dl).max() < 1e-12


@pytest.mark.parametrize("mode", R.MODES)
def test_factor_comes_from_length_after_chunk(mode):
    # L = 40, P0 = 24, w_pre = 8: G(L) = 5 but G(P0) = 3; the pin must reject G(P0)
    L, P0, w0, wp = 40, 24, 3, 8
    q, k, v = _inputs(11, L, 4, 2, 8)
    ro, _ = _direct(q, k, v, P0, w0, wp, mode)
    assert R.dynamic_factor(L, wp) != R.dynamic_factor(P0, wp)
    wrong, _ = _chunk(q, k, v, P0, w0, wp, mode, G=R.dynamic_factor(P0, wp))
    assert np.abs(ro[0] - wrong).max() > 1e-6


@pytest.mark.parametrize("mode", R.MODES)
def test_planted_mistake_cached_keys_not_unrotated(monkeypatch, mode):
    L, P0, w0, wp = 40, 24, 3, 8
    q, k, v = _inputs(12, L, 4, 2, 8)
    ro, _ = _direct(q, k, v, P0, w0, wp, mode)
    monkeypatch.setattr(R, "cached_key_to_raw", lambda kc, positions, omega: kc)
    wrong, _ = _chunk(q, k, v, P0, w0, wp, mode)
    assert np.abs(ro[0] - wrong).max() > 1e-6


@pytest.mark.parametrize("mode", R.MODES)
def test_planted_mistake_chunk_positions_from_zero(monkeypatch, mode):
    # a chunk oracle that forgot its offset is the direct definition over the chunk alone
    L, P0, w0, wp = 40, 24, 3, 8
    q, k, v = _inputs(13, L, 4, 2, 8)
    ro, _ = _direct(q, k, v, P0, w0, wp, mode)
    alone, _ = R.bifocal_attention(q[:, P0:], k[:, P0:], v[:, P0:], w0, wp, THETA, mode)
    assert np.abs(ro[0] - alone[0]).max() > 1e-6

"""Checks that pin the fp64 oracle to things other than itself.

Each ``check_*`` returns the largest deviation it saw; the pin tests assert it is
below the stated tolerance, and the mutation tests assert that a planted mistake in
the oracle pushes at least one of them above it. The oracle module is reached
through its module object so that a test can patch one of its functions.
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch

import oracle.bifocal_ref as R
from seeded_inputs import random_qkv
from tests.brute_force import brute_bifocal, factor_by_search

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def qkv64(seed, L, hq, hkv, D):
    q, k, v = random_qkv(seed, 1, L, hq, hkv, D, dtype="fp32")
    return q.double().numpy(), k.double().numpy(), v.double().numpy()


# --- brute force ------------------------------------------------------------------
def check_brute(L, D, hq, hkv, w0, w_pre, mode, theta=10000.0, seed=0, pos_offset=0):
    q, k, v = qkv64(seed, L, hq, hkv, D)
    out, lse = R.bifocal_attention(q, k, v, w0, w_pre, theta, mode, pos_offset=pos_offset)
    bo, bl = brute_bifocal(q[0].tolist(), k[0].tolist(), v[0].tolist(), w0, w_pre, theta, mode,
                           pos_offset=pos_offset)
    err_o = float(np.max(np.abs(out[0] - np.array(bo))))
    err_l = float(np.max(np.abs(lse[0] - np.array(bl))))
    return max(err_o, err_l)


# --- library scaled-dot-product attention in the special cases -----------------------
def torch_rope(x, positions, theta):
    """RoPE through complex multiplication in torch (independent of the oracle's code).

    x [b, L, H, D] float64 tensor, positions [L] float64 tensor (may be fractional).
    """
    D = x.shape[-1]
    P = D // 2
    freq = torch.tensor(theta, dtype=torch.float64) ** (-2.0 * torch.arange(P, dtype=torch.float64) / D)
    phase = torch.polar(torch.ones(len(positions), P, dtype=torch.float64), positions[:, None] * freq[None, :])
    z = torch.complex(x[..., :P], x[..., P:]) * phase[None, :, None, :]
    return torch.cat([z.real, z.imag], dim=-1)


def sdpa_rope(q, k, v, q_pos, k_pos, theta, scale=None):
    """Causal SDPA (torch's CPU flash kernel, fp64) over RoPE'd q and k; returns out [b,L,H,D], lse [b,H,L]."""
    q, k, v = (torch.from_numpy(np.asarray(t, dtype=np.float64)) for t in (q, k, v))
    D = q.shape[-1]
    g = q.shape[2] // k.shape[2]
    qr = torch_rope(q, torch.as_tensor(q_pos, dtype=torch.float64), theta).transpose(1, 2).contiguous()
    kr = torch_rope(k, torch.as_tensor(k_pos, dtype=torch.float64), theta).repeat_interleave(g, dim=2)
    vv = v.repeat_interleave(g, dim=2).transpose(1, 2).contiguous()
    kr = kr.transpose(1, 2).contiguous()
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    o, lse = torch.ops.aten._scaled_dot_product_flash_attention_for_cpu(qr, kr, vv, 0.0, True, scale=scale)[:2]
    return o.transpose(1, 2).numpy(), lse.numpy()


def check_sdpa_case(case, L, D, hq, hkv, w0, w_pre, mode, theta=10000.0, seed=1):
    """case: 'g1' (L <= w_pre), 'wide' (w0 >= L), 'w0zero' (w0 = 0, pure long branch)."""
    q, k, v = qkv64(seed, L, hq, hkv, D)
    out, lse = R.bifocal_attention(q, k, v, w0, w_pre, theta, mode)
    pos = np.arange(L, dtype=np.float64)
    if case in ("g1", "wide"):
        qp = kp = pos
    elif case == "w0zero":
        G = factor_by_search(L, w_pre)
        qp = kp = (pos / G) if mode == "freq_interp" else np.floor(pos / G)
    else:
        raise ValueError(case)
    so, sl = sdpa_rope(q, k, v, qp, kp, theta)
    return max(float(np.max(np.abs(out - so))), float(np.max(np.abs(lse - sl))))


def check_plain_vs_sdpa(L, D, hq, hkv, theta=10000.0, seed=2, pos_offset=0):
    q, k, v = qkv64(seed, L, hq, hkv, D)
    out, lse = R.rope_causal_attention(q, k, v, theta, pos_offset=pos_offset)
    pos = np.arange(L, dtype=np.float64) + pos_offset
    so, sl = sdpa_rope(q, k, v, pos, pos, theta)
    return max(float(np.max(np.abs(out - so))), float(np.max(np.abs(lse - sl))))


# --- method invariants ------------------------------------------------------------
def check_inclusion_exclusion(L, D, hq, hkv, w0, w_pre, mode, theta=10000.0, seed=3):
    q, k, v = qkv64(seed, L, hq, hkv, D)
    o1, l1 = R.bifocal_attention(q, k, v, w0, w_pre, theta, mode)
    o2, l2 = R.bifocal_attention_ie(q, k, v, w0, w_pre, theta, mode)
    return max(float(np.max(np.abs(o1 - o2) / (1e-300 + np.max(np.abs(o1))))), float(np.max(np.abs(l1 - l2))))


def check_shift(L, D, w0, w_pre, mode, c, theta=10000.0, seed=4):
    """|out(offset c) - out(offset 0)| for the bifocal oracle."""
    q, k, v = qkv64(seed, L, 2, 1, D)
    o0, l0 = R.bifocal_attention(q, k, v, w0, w_pre, theta, mode)
    o1, l1 = R.bifocal_attention(q, k, v, w0, w_pre, theta, mode, pos_offset=c)
    return max(float(np.max(np.abs(o0 - o1))), float(np.max(np.abs(l0 - l1))))


def check_decode_consistency(L, D, hq, hkv, w0, w_pre, mode, theta=10000.0, seed=5):
    """Decode at length L over the cached (original-RoPE) keys == last prefill row."""
    q, k, v = qkv64(seed, L, hq, hkv, D)
    kc = R.rope_keys_for_cache(k[0], theta)
    od, ld = R.bifocal_decode_reference(q[0, L - 1], kc, v[0], L, w0, w_pre, theta, mode)
    op, lp = R.bifocal_attention(q, k, v, w0, w_pre, theta, mode, rows=[L - 1])
    return max(float(np.max(np.abs(od - op[0, 0]))), float(np.max(np.abs(ld - lp[0, :, 0]))))


def check_golden_factor():
    """Max |G_oracle - G_golden| over tests/golden/dynamic_factor.txt."""
    worst = 0
    with open(os.path.join(GOLDEN, "dynamic_factor.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            L, w, G = (int(x) for x in line.split())
            worst = max(worst, abs(R.dynamic_factor(L, w) - G))
    return worst


def check_rotation_closed_forms():
    """Sign convention, pairing and frequencies of the oracle's RoPE against closed forms."""
    errs = []
    # quarter turn of the first pair: e_0 -> e_{P}; rotate-half pairs k with k + D/2
    om = np.array([math.pi / 2, 0.0])
    y = R.rope_rotate(np.array([[1.0, 0.0, 0.0, 0.0]]), np.array([1.0]), om)
    errs.append(np.max(np.abs(y - np.array([[0.0, 0.0, 1.0, 0.0]]))))
    # omega_k = theta^(-2k/D): D=8, theta=16 -> 1, 1/2, 1/4, 1/8
    errs.append(np.max(np.abs(R.rope_omega(8, 16.0) - np.array([1.0, 0.5, 0.25, 0.125]))))
    # R(a) R(b) = R(a + b), norm preserved
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 16))
    om = R.rope_omega(16, 10000.0)
    a, b = rng.integers(0, 1000, 5).astype(np.float64), rng.integers(0, 1000, 5).astype(np.float64)
    errs.append(np.max(np.abs(R.rope_rotate(R.rope_rotate(x, a, om), b, om) - R.rope_rotate(x, a + b, om))))
    errs.append(np.max(np.abs(np.linalg.norm(R.rope_rotate(x, a, om), axis=1) - np.linalg.norm(x, axis=1))))
    # cached keys return to raw values
    errs.append(np.max(np.abs(R.cached_key_to_raw(R.rope_rotate(x, a, om), a, om) - x)))
    return float(max(errs))


def check_softmax_properties(L=40, D=8, w0=5, w_pre=8, mode="freq_interp"):
    """v = 1 gives out = 1 (weights sum to one); outputs lie within [min v, max v] per dim."""
    q, k, v = qkv64(6, L, 2, 1, D)
    o1, _ = R.bifocal_attention(q, k, np.ones_like(v), w0, w_pre, 10000.0, mode)
    err = float(np.max(np.abs(o1 - 1.0)))
    o, _ = R.bifocal_attention(q, k, v, w0, w_pre, 10000.0, mode)
    # row i sees keys 0..i only
    for i in range(L):
        lo, hi = v[0, : i + 1, 0].min(axis=0), v[0, : i + 1, 0].max(axis=0)
        err = max(err, float(np.max(np.maximum(lo - o[0, i, 0], 0))), float(np.max(np.maximum(o[0, i, 0] - hi, 0))))
    return err


# A compact battery for the mutation tests: each entry is (name, callable, tolerance).
def battery():
    return [
        ("golden_factor", check_golden_factor, 0),
        ("rotation_closed_forms", check_rotation_closed_forms, 1e-12),
        ("brute_fi", lambda: check_brute(9, 8, 4, 2, 3, 4, "freq_interp"), 1e-12),
        ("brute_pa", lambda: check_brute(9, 8, 4, 2, 3, 4, "pos_alias"), 1e-12),
        ("brute_w0_1", lambda: check_brute(7, 4, 2, 1, 1, 2, "pos_alias"), 1e-12),
        ("sdpa_g1", lambda: check_sdpa_case("g1", 24, 8, 4, 2, 5, 32, "freq_interp"), 1e-12),
        ("sdpa_w0zero_pa", lambda: check_sdpa_case("w0zero", 24, 8, 2, 1, 0, 7, "pos_alias"), 1e-12),
        ("sdpa_w0zero_fi", lambda: check_sdpa_case("w0zero", 24, 8, 2, 1, 0, 7, "freq_interp"), 1e-12),
        ("plain_sdpa", lambda: check_plain_vs_sdpa(20, 8, 4, 2), 1e-12),
        ("inclusion_exclusion", lambda: check_inclusion_exclusion(30, 8, 2, 1, 6, 8, "pos_alias"), 1e-10),
        ("decode_consistency", lambda: check_decode_consistency(33, 8, 4, 2, 5, 8, "freq_interp"), 1e-11),
        ("softmax", check_softmax_properties, 1e-12),
    ]

"""fp64 CPU oracle for Dynamic Bifocal RoPE attention (Jet-Long, arXiv 2607.07740).

TEST INFRASTRUCTURE, NOT PRODUCT CODE. Only the test suite, the package smoke check
and the benchmark's CPU-baseline / reference leg may import or run this module. The
GPU library never calls it, and this module shares no code, table or constant
generator with the GPU library: its only common ground with the GPU path is the
seeded input module, which holds none of the method's arithmetic.

What it computes is the plain definition, untiled, in float64 with NumPy:

* Dynamic factor (video script "Tom 视频脚本镜像 · arXiv 2607.07740 · Jet-Long",
  storyboard scene-2): G = max(1, ceil(L / w_pretrained)), integer arithmetic.
* RoPE (knowledge-base note "Jet-Long：动态双焦点 RoPE 长上下文扩展", section 设计原理):
  frequencies omega_k = theta^(-2k/D). Pairing is rotate-half (k with k + D/2), the
  layout of the Qwen3 checkpoints the pages evaluate; the pages do not print it.
* Two windows (ai-feeds summary "Jet-Long: 使用动态双焦点RoPE的高效长上下文扩展",
  section 方法, key module 1; seventnews article "L'attention bifocale de Jet-Long ...",
  section "Comment l'attention bifocale contourne ..."): for query row i and key
  j <= i, the score uses the unmodified RoPE when i - j < w0 and the long-range RoPE
  otherwise. Long-range RoPE is frequency interpolation (omega / G at position p) or
  position aliasing (omega at position floor(p / G)); the ablation in the ai-feeds
  summary (section 实验, key findings) names both.
* Inclusion-exclusion merge (ai-feeds summary, key module 3; seventnews article): the
  long branch over all keys, minus the long branch on the local band, plus the local
  branch on the band, in log-sum-exp form. ``bifocal_attention_ie`` writes that form
  out; it must equal the direct masked softmax of ``bifocal_attention``.
* Correction rotation of cached keys (ai-feeds summary, key module 3): the cache holds
  keys under the original RoPE; the long branch re-phases cached key j from the
  original rotation to the long-range rotation. ``bifocal_decode_reference`` does it
  literally: undo R(j * omega), then apply the long-range rotation of position j.

Readings where the pages are silent (each is listed with its reason in the design
notes): one G per call from the full length L (decode: L counts the new token);
positions are 0-based; the band edge is strict (i - j = w0 is long-range); softmax
scale 1/sqrt(D) with no temperature; query head h reads kv head floor(h / (Hq/Hkv));
LSE is the natural log of the sum of exp(scaled score).

Parity pins: tests/test_oracle_pins.py checks every function here against a pure
Python brute force, library scaled-dot-product attention in its special cases,
closed-form rotation identities and the prefill/decode consistency of the method.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence, Tuple

import numpy as np

FREQ_INTERP = "freq_interp"
POS_ALIAS = "pos_alias"
MODES = (FREQ_INTERP, POS_ALIAS)


# ----------------------------------------------------------------------------------
# Dynamic factor and RoPE primitives
# ----------------------------------------------------------------------------------
def dynamic_factor(L: int, w_pretrained: int) -> int:
    """G = max(1, ceil(L / w_pretrained)) (video script, storyboard scene-2).

    Integer ceil-division, so G == 1 exactly when L <= w_pretrained (the ai-feeds
    summary, key module 2: no scaling while the input fits the pretrained window).
    """
    L = int(L)
    w_pretrained = int(w_pretrained)
    if L < 0 or w_pretrained < 1:
        raise ValueError("need L >= 0 and w_pretrained >= 1")
    return max(1, -(-L // w_pretrained))


def rope_omega(head_dim: int, theta: float) -> np.ndarray:
    """omega_k = theta^(-2k/D), k = 0 .. D/2 - 1 (knowledge-base note, 设计原理)."""
    if head_dim % 2:
        raise ValueError("head_dim must be even")
    k = np.arange(head_dim // 2, dtype=np.float64)
    return np.power(np.float64(theta), -2.0 * k / head_dim)


def rope_rotate(x: np.ndarray, positions: np.ndarray, omega: np.ndarray) -> np.ndarray:
    """Rotate-half RoPE of the rows of ``x`` (shape [..., n, D]) at ``positions`` (n,).

    For pair k < D/2 with angle a = p * omega_k:
        y_k       = x_k * cos(a) - x_{k+D/2} * sin(a)
        y_{k+D/2} = x_{k+D/2} * cos(a) + x_k * sin(a)
    """
    x = np.asarray(x, dtype=np.float64)
    P = x.shape[-1] // 2
    ang = np.asarray(positions, dtype=np.float64)[:, None] * np.asarray(omega, dtype=np.float64)[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :P], x[..., P:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def long_branch_rope(positions: np.ndarray, omega: np.ndarray, G: int, mode: str):
    """Positions and frequencies of the long-range RoPE.

    frequency interpolation: (p, omega / G); position aliasing: (floor(p / G), omega).
    Both act on query and key positions alike.
    """
    positions = np.asarray(positions, dtype=np.int64)
    if mode == FREQ_INTERP:
        return positions.astype(np.float64), omega / float(G)
    if mode == POS_ALIAS:
        return np.floor_divide(positions, G).astype(np.float64), omega
    raise ValueError(f"unknown mode {mode!r}")


def kv_head_for(h: int, group: int) -> int:
    """Query head h reads kv head floor(h / group), group = Hq / Hkv (contiguous GQA groups)."""
    return h // group


def cached_key_to_raw(kc: np.ndarray, positions: np.ndarray, omega: np.ndarray) -> np.ndarray:
    """Undo the original RoPE of cached keys: R(-p omega) applied to R(p omega) k."""
    return rope_rotate(kc, -np.asarray(positions, dtype=np.float64), omega)


def _check(q, k, v):
    if q.ndim != 4 or k.ndim != 4 or v.ndim != 4:
        raise ValueError("q, k, v must be [b, L, H, D]")
    b, L, hq, D = q.shape
    if k.shape != (b, L, k.shape[2], D) or v.shape != k.shape:
        raise ValueError("k and v must be [b, L, Hkv, D] matching q")
    if hq % k.shape[2]:
        raise ValueError("Hq must be a multiple of Hkv")
    return b, L, hq, k.shape[2], D


# ----------------------------------------------------------------------------------
# Direct masked-softmax bifocal attention (the definition)
# ----------------------------------------------------------------------------------
def bifocal_scores(q_rows: np.ndarray, k_all: np.ndarray, rows: np.ndarray, w0: int, G: int, mode: str,
                   omega: np.ndarray, scale: float, pos_offset: int = 0) -> np.ndarray:
    """Scaled bifocal scores of query rows ``rows`` against keys 0..L-1 of one head.

    q_rows [n, D] (raw, pre-RoPE query rows), k_all [L, D] (raw keys). Returns [n, L]
    with -inf where j > i. ``pos_offset`` shifts every position (test-only knob for
    the shift-invariance pins); the window test uses the row/key indices.
    """
    L = k_all.shape[0]
    rows = np.asarray(rows, dtype=np.int64)
    pos_k = np.arange(L, dtype=np.int64) + pos_offset
    pos_q = rows + pos_offset
    # local branch: the model's original RoPE
    s_orig = scale * (rope_rotate(q_rows, pos_q, omega) @ rope_rotate(k_all, pos_k, omega).T)
    # long branch: rescaled RoPE
    lq, wq = long_branch_rope(pos_q, omega, G, mode)
    lk, wk = long_branch_rope(pos_k, omega, G, mode)
    s_long = scale * (rope_rotate(q_rows, lq, wq) @ rope_rotate(k_all, lk, wk).T)
    dist = rows[:, None] - np.arange(L, dtype=np.int64)[None, :]
    s = np.where(dist < w0, s_orig, s_long)
    return np.where(dist < 0, -np.inf, s)


def _softmax_out(s: np.ndarray, v: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    l = np.sum(e, axis=1, keepdims=True)
    return (e @ v) / l, (m + np.log(l))[:, 0]


def bifocal_attention(q, k, v, w0: int, w_pretrained: int, theta: float, mode: str = FREQ_INTERP,
                      scale: Optional[float] = None, rows: Optional[Sequence[int]] = None, pos_offset: int = 0,
                      G: Optional[int] = None, row_chunk: int = 128):
    """Bifocal causal attention, direct definition, fp64.

    q [b, L, Hq, D], k and v [b, L, Hkv, D] (raw, pre-RoPE; any float dtype). One G
    for the whole call from the full length L unless ``G`` is given. Returns
    out [b, n, Hq, D] and lse [b, Hq, n] (natural log) for the query rows ``rows``
    (all rows when None).
    """
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    b, L, hq, hkv, D = _check(q, k, v)
    if w0 < 0:
        raise ValueError("w0 must be >= 0")
    if mode not in MODES:
        raise ValueError(f"unknown mode {mode!r}")
    G = dynamic_factor(L, w_pretrained) if G is None else int(G)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    rows = np.arange(L, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    omega = rope_omega(D, theta)
    g = hq // hkv
    out = np.empty((b, len(rows), hq, D))
    lse = np.empty((b, hq, len(rows)))
    for bi in range(b):
        for h in range(hq):
            kv = kv_head_for(h, g)
            for c0 in range(0, len(rows), row_chunk):
                r = rows[c0:c0 + row_chunk]
                s = bifocal_scores(q[bi, r, h], k[bi, :, kv], r, w0, G, mode, omega, scale, pos_offset)
                o, ls = _softmax_out(s, v[bi, :, kv])
                out[bi, c0:c0 + len(r), h] = o
                lse[bi, h, c0:c0 + len(r)] = ls
    return out, lse


def rope_causal_attention(q, k, v, theta: float, scale: Optional[float] = None,
                          rows: Optional[Sequence[int]] = None, pos_offset: int = 0):
    """Plain causal attention under the original RoPE (the comparator's definition).

    Same layouts as :func:`bifocal_attention`.
    """
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    b, L, hq, hkv, D = _check(q, k, v)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    rows = np.arange(L, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    omega = rope_omega(D, theta)
    g = hq // hkv
    pos = np.arange(L, dtype=np.int64) + pos_offset
    out = np.empty((b, len(rows), hq, D))
    lse = np.empty((b, hq, len(rows)))
    for bi in range(b):
        for h in range(hq):
            kvh = kv_head_for(h, g)
            kr = rope_rotate(k[bi, :, kvh], pos, omega)
            qr = rope_rotate(q[bi, rows, h], rows + pos_offset, omega)
            s = scale * (qr @ kr.T)
            s = np.where(rows[:, None] < np.arange(L)[None, :], -np.inf, s)
            o, ls = _softmax_out(s, v[bi, :, kvh])
            out[bi, :, h] = o
            lse[bi, h] = ls
    return out, lse


# ----------------------------------------------------------------------------------
# Inclusion-exclusion form (the merge the pages describe), used as an invariant
# ----------------------------------------------------------------------------------
def bifocal_attention_ie(q, k, v, w0: int, w_pretrained: int, theta: float, mode: str = FREQ_INTERP,
                         scale: Optional[float] = None, G: Optional[int] = None):
    """Bifocal attention through the inclusion-exclusion merge.

    With every exponent taken relative to one common max M per row:
      A = sum_{j<=i} e^{sL_ij},  B = sum_{i-w0<j<=i} e^{sL_ij},  C = sum_{i-w0<j<=i} e^{sO_ij}
    and the same sums weighted by v_j (Av, Bv, Cv); then
      o_i = (Av - Bv + Cv) / (A - B + C),  lse_i = M + ln(A - B + C).
    sL is the long-range score, sO the original-RoPE score.
    """
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    b, L, hq, hkv, D = _check(q, k, v)
    G = dynamic_factor(L, w_pretrained) if G is None else int(G)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    omega = rope_omega(D, theta)
    pos = np.arange(L, dtype=np.int64)
    lp, lw = long_branch_rope(pos, omega, G, mode)
    g = hq // hkv
    dist = pos[:, None] - pos[None, :]
    causal = dist >= 0
    band = causal & (dist < w0)
    out = np.empty((b, L, hq, D))
    lse = np.empty((b, hq, L))
    for bi in range(b):
        for h in range(hq):
            kvh = kv_head_for(h, g)
            sO = scale * (rope_rotate(q[bi, :, h], pos, omega) @ rope_rotate(k[bi, :, kvh], pos, omega).T)
            sL = scale * (rope_rotate(q[bi, :, h], lp, lw) @ rope_rotate(k[bi, :, kvh], lp, lw).T)
            M = np.maximum(np.max(np.where(causal, sL, -np.inf), axis=1),
                           np.max(np.where(band, sO, -np.inf), axis=1))[:, None]
            eL = np.where(causal, np.exp(sL - M), 0.0)
            eLb = np.where(band, eL, 0.0)
            eOb = np.where(band, np.exp(sO - M), 0.0)
            A, B, C = eL.sum(1), eLb.sum(1), eOb.sum(1)
            vv = v[bi, :, kvh]
            num = eL @ vv - eLb @ vv + eOb @ vv
            den = A - B + C
            out[bi, :, h] = num / den[:, None]
            lse[bi, h] = M[:, 0] + np.log(den)
    return out, lse


# ----------------------------------------------------------------------------------
# Decode: one new query against a cache of keys that carry the original RoPE
# ----------------------------------------------------------------------------------
def rope_keys_for_cache(k, theta: float, start: int = 0) -> np.ndarray:
    """Keys as the cache stores them: original RoPE at positions start, start+1, ...

    k [n, Hkv, D] raw -> [n, Hkv, D] fp64.
    """
    k = np.asarray(k, dtype=np.float64)
    n, hkv, D = k.shape
    omega = rope_omega(D, theta)
    pos = np.arange(start, start + n, dtype=np.int64)
    return np.stack([rope_rotate(k[:, h], pos, omega) for h in range(hkv)], axis=1)


def bifocal_decode_reference(q, kcache, vcache, L: int, w0: int, w_pretrained: int, theta: float,
                             mode: str = FREQ_INTERP, scale: Optional[float] = None,
                             G: Optional[int] = None):
    """Output of the newest token p = L - 1 against cache rows 0..L-1.

    q [Hq, D] raw query. kcache [>=L, Hkv, D]: keys already rotated by the original
    RoPE at their own position (what the cache stores). vcache alike. G comes from
    L, the length that includes the new token.

    Local keys (p - j < w0): score = <R(p omega) q, kc_j>.
    Long keys: the cached key is taken back to its raw value with R(-j omega), then
    rotated by the long-range RoPE of position j; the query gets the long-range RoPE
    of position p. Returns out [Hq, D], lse [Hq].
    """
    q = np.asarray(q, dtype=np.float64)
    kc = np.asarray(kcache[:L], dtype=np.float64)
    vc = np.asarray(vcache[:L], dtype=np.float64)
    hq, D = q.shape
    hkv = kc.shape[1]
    g = hq // hkv
    G = dynamic_factor(L, w_pretrained) if G is None else int(G)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    omega = rope_omega(D, theta)
    p = L - 1
    pos = np.arange(L, dtype=np.int64)
    lp, lw = long_branch_rope(pos, omega, G, mode)
    local = (p - pos) < w0
    out = np.empty((hq, D))
    lse = np.empty(hq)
    for kvh in range(hkv):
        raw = cached_key_to_raw(kc[:, kvh], pos, omega)
        k_long = rope_rotate(raw, lp, lw)
        for h in (hh for hh in range(hq) if kv_head_for(hh, g) == kvh):
            qo = rope_rotate(q[h][None], np.array([p]), omega)[0]
            ql = rope_rotate(q[h][None], lp[p:p + 1], lw)[0]
            s = scale * np.where(local, kc[:, kvh] @ qo, k_long @ ql)
            m = s.max()
            e = np.exp(s - m)
            out[h] = (e @ vc[:, kvh]) / e.sum()
            lse[h] = m + math.log(e.sum())
    return out, lse


def bifocal_chunk_reference(q, kcache, vcache, P0: int, w0: int, w_pretrained: int, theta: float,
                            mode: str = FREQ_INTERP, scale: Optional[float] = None,
                            rows: Optional[Sequence[int]] = None, G: Optional[int] = None):
    """Chunked prefill over a cache: chunk rows at positions P0 .. P0+C-1 against cache rows 0..L-1.

    q [C, Hq, D] raw chunk queries. kcache [>=L, Hkv, D] (L = P0 + C) holds every key rotated
    by the original RoPE at its own position - rows 0..P0-1 the cached ones, rows P0.. the
    chunk's own - and vcache the values. G comes from L, the length after the chunk (the
    factor follows the current length: ai-feeds summary, 方法 key module 2). Row i attends
    to keys j <= i. A local key (i - j < w0) scores <R(i omega) q_i, kc_j>; a long-range key is
    taken back to its raw value with R(-j omega) and rotated by the long-range RoPE of j,
    against the long-range RoPE of i (the rotation applied to cached keys, key module 3).
    Returns out [n, Hq, D] and lse [Hq, n] for chunk rows ``rows`` (all C when None).
    """
    q = np.asarray(q, dtype=np.float64)
    C, hq, D = q.shape
    L = P0 + C
    kc = np.asarray(kcache[:L], dtype=np.float64)
    vc = np.asarray(vcache[:L], dtype=np.float64)
    hkv = kc.shape[1]
    g = hq // hkv
    G = dynamic_factor(L, w_pretrained) if G is None else int(G)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    omega = rope_omega(D, theta)
    rows = np.arange(C, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    pos = np.arange(L, dtype=np.int64)
    lp, lw = long_branch_rope(pos, omega, G, mode)
    out = np.empty((len(rows), hq, D))
    lse = np.empty((hq, len(rows)))
    for kvh in range(hkv):
        raw = cached_key_to_raw(kc[:, kvh], pos, omega)
        k_long = rope_rotate(raw, lp, lw)
        for h in (hh for hh in range(hq) if kv_head_for(hh, g) == kvh):
            for n, r in enumerate(rows):
                i = P0 + int(r)
                qo = rope_rotate(q[r, h][None], np.array([i]), omega)[0]
                ql = rope_rotate(q[r, h][None], lp[i:i + 1], lw)[0]
                s = scale * np.where(i - pos < w0, kc[:, kvh] @ qo, k_long @ ql)
                s = np.where(pos > i, -np.inf, s)
                m = s.max()
                e = np.exp(s - m)
                out[n, h] = (e @ vc[:, kvh]) / e.sum()
                lse[h, n] = m + math.log(e.sum())
    return out, lse


# ----------------------------------------------------------------------------------
# Sliding-window attention: the local layers of a hybrid model (Jet-Nemotron, named by the
# ai-feeds summary, 影响 / 局限) keep only the near keys, under the original RoPE
# ----------------------------------------------------------------------------------
def sliding_window_attention(q, k, v, window: int, theta: float, scale: Optional[float] = None,
                             rows: Optional[Sequence[int]] = None):
    """Causal attention restricted to 0 <= i - j < window, original RoPE, fp64.

    Same layouts as :func:`bifocal_attention`; window >= 1.
    """
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    b, L, hq, hkv, D = _check(q, k, v)
    if window < 1:
        raise ValueError("window must be >= 1")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    rows = np.arange(L, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    omega = rope_omega(D, theta)
    g = hq // hkv
    pos = np.arange(L, dtype=np.int64)
    dist = rows[:, None] - pos[None, :]
    keep = (dist >= 0) & (dist < window)
    out = np.empty((b, len(rows), hq, D))
    lse = np.empty((b, hq, len(rows)))
    for bi in range(b):
        for h in range(hq):
            kvh = kv_head_for(h, g)
            kr = rope_rotate(k[bi, :, kvh], pos, omega)
            qr = rope_rotate(q[bi, rows, h], rows, omega)
            s = np.where(keep, scale * (qr @ kr.T), -np.inf)
            o, ls = _softmax_out(s, v[bi, :, kvh])
            out[bi, :, h] = o
            lse[bi, h] = ls
    return out, lse


def sliding_window_cached_reference(q, kcache, vcache, P0: int, window: int, theta: float,
                                    scale: Optional[float] = None, rows: Optional[Sequence[int]] = None):
    """Sliding-window rows at positions P0 .. P0+C-1 against a cache of original-RoPE keys.

    q [C, Hq, D] raw; kcache / vcache [>= P0 + C, Hkv, D] as stored (row j = R(j omega) k_j).
    Covers a chunk over a cache and a decode step (C = 1, P0 = L - 1). Row i scores
    <R(i omega) q_i, kc_j> for 0 <= i - j < window. Returns out [n, Hq, D], lse [Hq, n].
    """
    q = np.asarray(q, dtype=np.float64)
    C, hq, D = q.shape
    L = P0 + C
    kc = np.asarray(kcache[:L], dtype=np.float64)
    vc = np.asarray(vcache[:L], dtype=np.float64)
    g = hq // kc.shape[1]
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    omega = rope_omega(D, theta)
    rows = np.arange(C, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    pos = np.arange(L, dtype=np.int64)
    out = np.empty((len(rows), hq, D))
    lse = np.empty((hq, len(rows)))
    for h in range(hq):
        kvh = kv_head_for(h, g)
        for n, r in enumerate(rows):
            i = P0 + int(r)
            qo = rope_rotate(q[r, h][None], np.array([i]), omega)[0]
            keep = (i - pos >= 0) & (i - pos < window)
            s = np.where(keep, scale * (kc[:, kvh] @ qo), -np.inf)
            m = s.max()
            e = np.exp(s - m)
            out[n, h] = (e @ vc[:, kvh]) / e.sum()
            lse[h, n] = m + math.log(e.sum())
    return out, lse


# ----------------------------------------------------------------------------------
# Per-head RMS norm of q and k (Qwen3's q_norm / k_norm, the step before the path)
# ----------------------------------------------------------------------------------
def qk_rms_norm(x, weight, eps: float):
    """x [..., D] -> x / sqrt(mean_d x^2 + eps) * weight, fp64, over the last axis."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(weight, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * w

"""Helpers for the GPU parity tests: tolerance checks and a process pool for the oracle.

Tolerances (stated for bf16 inputs with fp32 accumulation): output max-abs <= 2e-2,
relative L2 <= 5e-3, per-row |LSE difference| <= 1e-3.
"""
from __future__ import annotations

import concurrent.futures as cf
import multiprocessing as mp
import os

import numpy as np

MAX_ABS = 2e-2
REL_L2 = 5e-3
LSE_ABS = 1e-3


def errors(out_gpu, lse_gpu, out_ref, lse_ref):
    """out_* [..., D] with matching leading dims; lse_* matching shapes. Returns dict."""
    o = np.asarray(out_gpu, dtype=np.float64)
    r = np.asarray(out_ref, dtype=np.float64)
    d = o - r
    res = {
        "max_abs": float(np.max(np.abs(d))) if d.size else 0.0,
        "rel_l2": float(np.linalg.norm(d) / max(np.linalg.norm(r), 1e-300)) if d.size else 0.0,
    }
    if lse_gpu is not None:
        dl = np.asarray(lse_gpu, dtype=np.float64) - np.asarray(lse_ref, dtype=np.float64)
        res["lse_abs"] = float(np.max(np.abs(dl))) if dl.size else 0.0
    return res


def assert_close(out_gpu, lse_gpu, out_ref, lse_ref, what=""):
    e = errors(out_gpu, lse_gpu, out_ref, lse_ref)
    ok = e["max_abs"] <= MAX_ABS and e["rel_l2"] <= REL_L2 and e.get("lse_abs", 0.0) <= LSE_ABS
    assert ok, f"{what}: {e}"
    return e


def _oracle_head(args):
    import oracle.bifocal_ref as R
    q, k, v, w0, w_pre, theta, mode, rows, G = args
    return R.bifocal_attention(q, k, v, w0, w_pre, theta, mode, rows=rows, G=G)


def oracle_rows(q, k, v, w0, w_pre, theta, mode, rows, workers=None):
    """Oracle bifocal attention for `rows`, one query head per task, in a spawn pool.

    q [1, L, Hq, D], k/v [1, L, Hkv, D] numpy. Returns out [1, n, Hq, D], lse [1, Hq, n].
    """
    import oracle.bifocal_ref as R
    L, hq, hkv = q.shape[1], q.shape[2], k.shape[2]
    g = hq // hkv
    G = R.dynamic_factor(L, w_pre)
    tasks = [(q[:, :, h:h + 1], k[:, :, h // g:h // g + 1], v[:, :, h // g:h // g + 1], w0, w_pre, theta, mode,
              rows, G) for h in range(hq)]
    workers = workers or max(1, min(len(tasks), (os.cpu_count() or 2) // 2, 16))
    out = np.empty((1, len(rows), hq, q.shape[3]))
    lse = np.empty((1, hq, len(rows)))
    with cf.ProcessPoolExecutor(max_workers=workers, mp_context=mp.get_context("spawn")) as ex:
        for h, (o, l) in enumerate(ex.map(_oracle_head, tasks)):
            out[:, :, h] = o[:, :, 0]
            lse[:, h] = l[:, 0]
    return out, lse

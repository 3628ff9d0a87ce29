"""GPU parity of the batched chunked prefill over a paged cache (bifocal_prefill_chunk_paged)
against the fp64 chunk oracle, sequence by sequence on the gathered logical cache.

Each sequence has its own cached length, chunk length and so its own G; pages are assigned in a
shuffled order and every pool slot that holds no key is NaN, so the key rows past a sequence's end
(zeroed in the tile loads) and the value rows there (zeroed before P.V) must keep NaN out of every
result. The reference reads each sequence's cache rows as the call left them (bf16, the chunk's own
keys included), the reading of the cache format the decode reference follows too."""
import numpy as np
import pytest
import torch

import oracle.bifocal_ref as R
import rope_context_extension_bifocal_b200 as bfl
import seeded_inputs as si
from tests.gpu_helpers import assert_close

pytestmark = pytest.mark.gpu
THETA = 1e6
FI, PA = si.FREQ_INTERP, si.POS_ALIAS


def bf16_round(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float64)).to(torch.bfloat16).double().numpy()


def build_pool(seed, cached, chunks, hkv, page_size):
    lens = [p0 + c for p0, c in zip(cached, chunks)]
    B = len(lens)
    max_pages = (max(lens) + page_size - 1) // page_size + 1
    g = si.generator(seed)
    pool_pages = sum((L + page_size - 1) // page_size for L in lens) + 5
    perm = torch.randperm(pool_pages, generator=g)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)  # unused entries are never read
    nxt = 0
    for b, L in enumerate(lens):
        n = (L + page_size - 1) // page_size
        table[b, :n] = perm[nxt:nxt + n].to(torch.int32)
        nxt += n
    rows = pool_pages * page_size
    kpool = torch.full((rows, hkv, 128), float("nan"), dtype=torch.bfloat16)
    vpool = torch.full((rows, hkv, 128), float("nan"), dtype=torch.bfloat16)
    return g, lens, table, kpool, vpool


def pool_row(table, b, j, page_size):
    return int(table[b, j // page_size]) * page_size + j % page_size


def run_batch(seed, cached, chunks, hq, hkv, w0, wp, mode, page_size, flags=0, check_rows=None):
    g, lens, table, kpool, vpool = build_pool(seed, cached, chunks, hkv, page_size)
    B = len(lens)
    qs, ks, vs = [], [], []
    for b in range(B):
        q, k, v = si.random_qkv(seed * 100 + b, 1, lens[b], hq, hkv, 128, "bf16")
        prefix = bf16_round(R.rope_keys_for_cache(k[0, :cached[b]].double().numpy(), THETA)) if cached[b] else None
        for j in range(cached[b]):
            r = pool_row(table, b, j, page_size)
            kpool[r] = torch.from_numpy(prefix[j]).to(torch.bfloat16)
            vpool[r] = v[0, j]
        qs.append(q[0, cached[b]:])
        ks.append(k[0, cached[b]:])
        vs.append(v[0, cached[b]:])
    qp, kp_, vp_ = (torch.cat(x).cuda() for x in (qs, ks, vs))
    kpd, vpd = kpool.cuda(), vpool.cuda()
    out, lse = bfl.bifocal_prefill_chunk_paged(qp, kp_, vp_, chunks, cached, kpd, vpd, page_size, table.cuda(),
                                               w0=w0, w_pretrained=wp, theta=THETA, mode=mode, flags=flags)
    torch.cuda.synchronize()
    assert bfl.last_device_error() == 0
    kh, vh = kpd.cpu(), vpd.cpu()
    row0 = 0
    for b in range(B):
        L, C, P0 = lens[b], chunks[b], cached[b]
        idx = [pool_row(table, b, j, page_size) for j in range(L)]
        ref_k = kh[idx].double().numpy()  # the sequence's cache as the call left it
        ref_v = vh[idx].double().numpy()
        assert np.isfinite(ref_k).all() and np.isfinite(ref_v).all()
        # the chunk's rows written: original-RoPE keys within one bf16 step, values copied
        want = R.rope_keys_for_cache(ks[b].double().numpy(), THETA, start=P0)
        assert np.all(np.abs(ref_k[P0:] - want) <= np.abs(want) * 2.0 ** -7 + 1e-5)
        assert np.array_equal(ref_v[P0:], vs[b].double().numpy())
        rows = np.arange(C) if check_rows is None else np.asarray(sorted({r for r in check_rows if r < C}))
        if flags & bfl.FLAG_WINDOW:
            ro, rl = R.sliding_window_cached_reference(qs[b].double().numpy(), ref_k, ref_v, P0, w0, THETA, rows=rows)
        else:
            ro, rl = R.bifocal_chunk_reference(qs[b].double().numpy(), ref_k, ref_v, P0, w0, wp, THETA, mode,
                                               rows=rows)
        go = out[row0:row0 + C].cpu().float().numpy()[rows]
        gl = lse[:, row0:row0 + C].cpu().numpy()[:, rows]
        assert_close(go, gl, ro, rl, f"paged chunk b={b} P0={P0} C={C} G={R.dynamic_factor(L, wp)} page={page_size}")
        row0 += C


@pytest.mark.parametrize("page_size,mode", [(16, FI), (64, PA), (128, FI), (256, PA)])
def test_paged_chunk_batch_matches_oracle(page_size, mode):
    # G per sequence at w_pretrained 512: 1, 3, 5, 2, 1 (and the band edge inside and across tiles)
    cached = [0, 1000, 1777, 700, 20]
    chunks = [300, 129, 333, 1, 100]
    run_batch(80 + page_size, cached, chunks, 4, 2, 100, 512, mode, page_size)


def test_paged_chunk_window():
    run_batch(90, [1500, 0, 333], [400, 257, 64], 4, 2, 300, 128, FI, 32, flags=bfl.FLAG_WINDOW)


def test_paged_chunk_qwen3_8b_heads_sampled():
    rows = list(range(0, 700, 41)) + [699]
    run_batch(95, [9269, 4096, 0], [700, 300, 512], 32, 8, 4096, 2048, FI, 64, check_rows=rows)


def test_paged_chunk_rejects_bad_arguments():
    q = torch.zeros(10, 4, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(10, 2, 128, dtype=torch.bfloat16, device="cuda")
    pool = torch.zeros(256, 2, 128, dtype=torch.bfloat16, device="cuda")
    table = torch.zeros(1, 4, dtype=torch.int32, device="cuda")
    kw = dict(w0=4, w_pretrained=16, theta=1e4)
    with pytest.raises(bfl.BifocalError):  # page size that neither divides 128 nor is a multiple of it
        bfl.bifocal_prefill_chunk_paged(q, k, k, [10], [0], pool, pool, 48, table, **kw)
    with pytest.raises(bfl.BifocalError):  # chunk past the pages the table can address
        bfl.bifocal_prefill_chunk_paged(q, k, k, [10], [250], pool, pool, 64, table, **kw)

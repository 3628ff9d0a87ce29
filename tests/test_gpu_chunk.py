"""GPU parity of the chunked prefill over a cache (bifocal_prefill_chunk) against the fp64
chunk oracle, on seeded inputs. The cached prefix is written by the oracle (original RoPE
of the raw prefix keys, rounded to the cache's bf16); the oracle then reads the cached rows
as stored and the chunk's own keys exact. Cases cover a chunk with no cache, a single row,
band edges inside and across tiles, offsets and chunk lengths that are not tile multiples,
G changing between the cached length and the length after the chunk, w0 = 0, G = 1 and
w0 >= L."""
import numpy as np
import pytest
import torch

import oracle.bifocal_ref as R
import rope_context_extension_bifocal_b200 as bfl
import seeded_inputs as si
from tests.gpu_helpers import assert_close

pytestmark = pytest.mark.gpu

FI, PA = si.FREQ_INTERP, si.POS_ALIAS
THETA = 1e6


def bf16_round(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float64)).to(torch.bfloat16).double().numpy()


def run_chunk(seed, P0, C, hq, hkv, w0, wp, mode, rows=None, cap=None):
    L = P0 + C
    cap = L + 5 if cap is None else cap
    q, k, v = si.random_qkv(seed, 1, L, hq, hkv, 128, "bf16")
    kc_prefix = bf16_round(R.rope_keys_for_cache(k[0, :P0].double().numpy(), THETA)) if P0 else \
        np.zeros((0, hkv, 128))
    kcache = torch.zeros(cap, hkv, 128, dtype=torch.bfloat16, device="cuda")
    vcache = torch.zeros_like(kcache)
    if P0:
        kcache[:P0] = torch.from_numpy(kc_prefix).to(torch.bfloat16).cuda()
        vcache[:P0] = v[0, :P0].cuda()
    out, lse = bfl.bifocal_prefill_chunk(q[0, P0:].cuda(), k[0, P0:].cuda(), v[0, P0:].cuda(), kcache, vcache, P0,
                                         w0=w0, w_pretrained=wp, theta=THETA, mode=mode)
    torch.cuda.synchronize()
    assert bfl.last_device_error() == 0
    chunk_keys = R.rope_keys_for_cache(k[0, P0:].double().numpy(), THETA, start=P0)
    ref_k = np.concatenate([kc_prefix, chunk_keys])
    ref_v = v[0].double().numpy()
    rows = np.arange(C) if rows is None else np.asarray(sorted(set(int(r) for r in rows if 0 <= r < C)))
    ro, rl = R.bifocal_chunk_reference(q[0, P0:].double().numpy(), ref_k, ref_v, P0, w0, wp, THETA, mode, rows=rows)
    e = assert_close(out.cpu().float().numpy()[rows], lse.cpu().numpy()[:, rows], ro, rl,
                     f"chunk P0={P0} C={C} G={R.dynamic_factor(L, wp)}")
    # the chunk's rows of the cache: original-RoPE keys in bf16, values copied. Slack: one bf16
    # step, plus 1e-5 absolute where the rotation cancels (the device rotates in fp32, so a
    # near-zero result can differ from the fp64 one by ~1e-7 before rounding)
    want = bf16_round(chunk_keys)
    got = kcache[P0:L].cpu().double().numpy()
    bad = np.abs(got - want) > np.abs(want) * 2.0 ** -7 + 1e-5
    assert not bad.any(), (np.argwhere(bad)[:4], got[bad][:4], want[bad][:4])
    assert torch.equal(vcache[P0:L].cpu(), v[0, P0:])
    assert torch.count_nonzero(kcache[L:]) == 0  # rows past the chunk untouched
    return e


CASES = [
    # seed, P0, C, hq, hkv, w0, w_pre, mode
    (1, 0, 300, 4, 2, 64, 128, FI),        # no cache: a whole prefill through the chunk entry
    (2, 200, 1, 4, 2, 64, 128, PA),        # one row
    (3, 1000, 300, 8, 2, 100, 512, FI),    # G = 3, band edge inside the chunk's tiles
    (4, 777, 333, 4, 2, 50, 256, PA),      # offset and length not tile multiples, G = 5
    (5, 1024, 300, 4, 2, 64, 512, FI),     # G = 2 for the cached length, 3 after the chunk
    (6, 1024, 300, 4, 2, 64, 512, PA),
    (7, 500, 200, 4, 2, 0, 128, FI),       # w0 = 0: every pair long-range
    (8, 600, 100, 4, 2, 64, 4096, PA),     # G = 1: plain kernel
    (9, 300, 300, 2, 1, 2000, 64, FI),     # w0 >= L: every pair local
]


@pytest.mark.parametrize("seed,P0,C,hq,hkv,w0,wp,mode", CASES)
def test_chunk_matches_oracle(seed, P0, C, hq, hkv, w0, wp, mode):
    run_chunk(seed, P0, C, hq, hkv, w0, wp, mode)


@pytest.mark.parametrize("mode", [FI, PA])
def test_chunk_qwen3_8b_heads_sampled(mode):
    # Qwen3-8B attention heads, 9269 cached rows + a 1000-row chunk, G = 5; sampled rows
    P0, C, w0, wp = 8192 + 1077, 1000, 4096, 2048
    rows = [0, 1, 2, 127, 128, 129, 500, 998, 999] + list(range(250, 1000, 61))
    run_chunk(21, P0, C, 32, 8, w0, wp, mode, rows=rows)


def test_chunk_after_prefill_matches_full_prefill():
    # prefill the first P0 rows (its kcache_out is the cache), then a chunk; against a full
    # prefill of L rows: same G (from L), same keys up to the cache's bf16 rounding
    P0, C, hq, hkv, w0, wp = 1500, 500, 8, 2, 200, 512
    L = P0 + C
    q, k, v = (t.cuda() for t in si.random_qkv(31, 1, L, hq, hkv, 128, "bf16"))
    _, _, kc, vc = bfl.bifocal_prefill(q[:, :P0], k[:, :P0], v[:, :P0], w0=w0, w_pretrained=wp, theta=THETA,
                                       want_cache=True)
    kcache = torch.zeros(L, hkv, 128, dtype=torch.bfloat16, device="cuda")
    vcache = torch.zeros_like(kcache)
    kcache[:P0], vcache[:P0] = kc[0], vc[0]
    out_c, lse_c = bfl.bifocal_prefill_chunk(q[0, P0:], k[0, P0:], v[0, P0:], kcache, vcache, P0, w0=w0,
                                             w_pretrained=wp, theta=THETA)
    out_f, lse_f, _, _ = bfl.bifocal_prefill(q, k, v, w0=w0, w_pretrained=wp, theta=THETA)
    torch.cuda.synchronize()
    assert_close(out_c.cpu().float().numpy(), lse_c.cpu().numpy(), out_f[0, P0:].cpu().float().numpy(),
                 lse_f[0, :, P0:].cpu().numpy(), "chunk vs full prefill")

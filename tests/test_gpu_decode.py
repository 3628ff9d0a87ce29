"""GPU parity of the single-batch decode path (append + split-KV + combine) against the
fp64 oracle, including the steps where G changes and every long-range cached key has
to be re-phased by the correction rotation."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle.bifocal_ref as R
import rope_context_extension_bifocal_b200 as bfl
import seeded_inputs as si
from tests.gpu_helpers import assert_close

pytestmark = pytest.mark.gpu


def bf16_round(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float64)).to(torch.bfloat16).double().numpy()


def session(w: si.DecodeWorkload, check, plain=False, prefix=None, cap=None, steps=None):
    stream = si.DecodeStream(w, prefix_len=prefix, capacity=cap)
    prefix, cap = stream.prefix_len, stream.capacity
    steps = w.steps if steps is None else steps
    kp, vp = stream.cache_prefix()
    kcache = torch.zeros(cap, w.hkv, w.head_dim, dtype=torch.bfloat16, device="cuda")
    vcache = torch.zeros_like(kcache)
    kcache[:prefix] = kp.cuda()
    vcache[:prefix] = vp.cuda()
    ref_k = np.zeros((cap, w.hkv, w.head_dim))
    ref_v = np.zeros((cap, w.hkv, w.head_dim))
    ref_k[:prefix] = kp.float().double().numpy()
    ref_v[:prefix] = vp.float().double().numpy()
    del kp, vp
    results = []
    for t in range(steps):
        q, kn, vn = stream.step()
        L = prefix + t + 1
        p = L - 1
        if plain:
            out, lse = bfl.rope_causal_decode(q.cuda(), kn.cuda(), vn.cuda(), kcache, vcache, L, theta=w.theta)
        else:
            out, lse = bfl.bifocal_decode(q.cuda(), kn.cuda(), vn.cuda(), kcache, vcache, L, w0=w.w0,
                                          w_pretrained=w.w_pretrained, theta=w.theta, mode=w.mode)
        # the cache stores bf16: round the oracle's own fp64 key to the storage format
        ref_k[p] = bf16_round(R.rope_keys_for_cache(kn[None].float().double().numpy(), w.theta, start=p)[0])
        ref_v[p] = vn.float().double().numpy()
        if t in check:
            w0 = L if plain else w.w0
            ro, rl = R.bifocal_decode_reference(q.float().double().numpy(), ref_k, ref_v, L, w0, w.w_pretrained,
                                                w.theta, w.mode)
            e = assert_close(out.cpu().float().numpy(), lse.cpu().numpy(), ro, rl, f"step {t} L={L}")
            results.append((t, L, R.dynamic_factor(L, w.w_pretrained), e))
    torch.cuda.synchronize()
    assert bfl.last_device_error() == 0
    return kcache, ref_k, results


SMALL = dataclasses.replace(si.DECODE_128K, name="small", prefix_len=250, steps=160, capacity=600, hq=8, hkv=2,
                            w0=64, w_pretrained=128, theta=1e4, seed=21)


@pytest.mark.parametrize("mode", [si.FREQ_INTERP, si.POS_ALIAS])
def test_small_session_across_g_changes(mode):
    w = dataclasses.replace(SMALL, mode=mode)
    # L = 251..410: G = 2 up to 256, 3 from 257 to 384, 4 from 385
    check = set(range(0, 160, 7)) | {5, 6, 7, 133, 134, 135}
    _, _, res = session(w, check)
    assert {r[2] for r in res} == {2, 3, 4}


def test_small_session_d64_gqa8():
    w = dataclasses.replace(SMALL, hq=8, hkv=1, head_dim=64, w0=17, seed=22, steps=40, prefix_len=100)
    session(w, set(range(0, 40, 3)))


def test_tiny_lengths():
    # the first steps of a fresh cache: L = 1, 2, ...
    w = dataclasses.replace(SMALL, prefix_len=0, steps=20, capacity=64, w0=3, w_pretrained=4)
    session(w, set(range(20)))


def test_plain_decode_matches_oracle():
    w = dataclasses.replace(SMALL, steps=30)
    session(w, set(range(0, 30, 5)), plain=True)


def test_appended_cache_rows():
    w = dataclasses.replace(SMALL, steps=12)
    kcache, ref_k, _ = session(w, set())
    got = kcache[250:262].cpu().float().double().numpy()
    want = ref_k[250:262]
    assert np.max(np.abs(got - want)) <= 2.0 ** -8 * np.max(np.abs(want)) + 1e-6


def test_qwen3_8b_decode_200_steps_crossing_128k():
    w = si.DECODE_128K
    # G = 4 for L <= 131072 (steps 0..71), G = 5 from step 72
    check = {0, 1, 35, 70, 71, 72, 73, 74, 120, 199}
    _, _, res = session(w, check)
    gs = {t: g for t, _, g, _ in res}
    assert gs[71] == 4 and gs[72] == 5


@pytest.mark.parametrize("w0", [0, 400])
def test_force_bifocal_decode_matches_oracle(w0):
    # BF_FLAG_FORCE_BIFOCAL runs the two-branch split-KV kernel whatever G and w0 are, as in
    # prefill: with G == 1 (L <= w_pretrained) every pair uses the original RoPE; with w0 >= L
    # every pair is local. Either way the result is plain RoPE attention.
    hq, hkv, D, L = 8, 2, 128, 300
    g = si.generator(51 + w0)
    kc = torch.randn(L + 4, hkv, D, generator=g).to(torch.bfloat16)
    vc = torch.randn(L + 4, hkv, D, generator=g).to(torch.bfloat16)
    q = torch.randn(hq, D, generator=g).to(torch.bfloat16)
    kn = torch.randn(hkv, D, generator=g).to(torch.bfloat16)
    vn = torch.randn(hkv, D, generator=g).to(torch.bfloat16)
    w_pre = 512 if w0 == 0 else 128  # G = 1 with w0 = 0 (all long, but the long RoPE is the original one)
    ref_k = kc.float().double().numpy().copy()
    ref_v = vc.float().double().numpy().copy()
    ref_k[L - 1] = bf16_round(R.rope_keys_for_cache(kn[None].float().double().numpy(), 1e4, start=L - 1)[0])
    ref_v[L - 1] = vn.float().double().numpy()
    out, lse = bfl.bifocal_decode(q.cuda(), kn.cuda(), vn.cuda(), kc.cuda(), vc.cuda(), L, w0=w0, w_pretrained=w_pre,
                                  theta=1e4, flags=bfl.FLAG_FORCE_BIFOCAL)
    torch.cuda.synchronize()
    assert bfl.last_device_error() == 0
    ro, rl = R.bifocal_decode_reference(q.float().double().numpy(), ref_k, ref_v, L, w0, w_pre, 1e4, si.FREQ_INTERP)
    assert_close(out.cpu().float().numpy(), lse.cpu().numpy(), ro, rl, f"forced decode w0={w0}")

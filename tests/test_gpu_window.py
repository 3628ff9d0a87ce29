"""GPU parity of sliding-window attention (BF_FLAG_WINDOW: the local layers of a hybrid
model) against the fp64 sliding-window oracle: prefill, chunked prefill over a cache and
decode. Windows of one key, windows off the tile grid, windows wider than the sequence."""
import numpy as np
import pytest
import torch

import oracle.bifocal_ref as R
import rope_context_extension_bifocal_b200 as bfl
import seeded_inputs as si
from tests.gpu_helpers import assert_close

pytestmark = pytest.mark.gpu
THETA = 1e6


def bf16_round(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float64)).to(torch.bfloat16).double().numpy()


@pytest.mark.parametrize("L,hq,hkv,W", [(600, 4, 2, 1), (600, 4, 2, 100), (1000, 8, 2, 128), (1000, 4, 2, 300),
                                        (777, 2, 1, 64), (500, 4, 2, 1000),
                                        # rows whose first visited tile holds no key of their window
                                        (2048, 4, 2, 512), (2048, 4, 2, 1000)])
def test_window_prefill(L, hq, hkv, W):
    q, k, v = si.random_qkv(40 + W, 1, L, hq, hkv, 128, "bf16")
    out, lse, kc, _ = bfl.bifocal_prefill(q.cuda(), k.cuda(), v.cuda(), w0=W, w_pretrained=64, theta=THETA,
                                          flags=bfl.FLAG_WINDOW, want_cache=True)
    torch.cuda.synchronize()
    assert bfl.last_device_error() == 0
    ro, rl = R.sliding_window_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(), W, THETA)
    if W > 1:
        assert_close(out.cpu().float().numpy(), lse.cpu().numpy(), ro, rl, f"window prefill L={L} W={W}")
        return
    # One key per row: the LSE is that pair's score, with nothing to average the rounding of the
    # fp16 QK^T operands. Each rotated operand is rounded once (relative error <= 2^-11), so the
    # product of a pair of elements is off by <= (2^-10 + 2^-22) |q_d k_d|; fp32 accumulation adds
    # ~128 * 2^-24. Bound per row: scale * (2^-10 + 2^-20) * sum_d |q~_d k~_d| (q~, k~ rotated).
    assert_close(out.cpu().float().numpy(), None, ro, None, f"window prefill L={L} W=1 (out)")
    omega = R.rope_omega(128, THETA)
    pos = np.arange(L)
    g = hq // hkv
    for h in range(hq):
        qr = R.rope_rotate(q[0, :, h].double().numpy(), pos, omega)
        kr = R.rope_rotate(k[0, :, h // g].double().numpy(), pos, omega)
        bound = (2.0 ** -10 + 2.0 ** -20) / np.sqrt(128) * np.abs(qr * kr).sum(axis=1)
        err = np.abs(lse[0, h].cpu().double().numpy() - rl[0, h])
        assert np.all(err <= np.maximum(bound, 1e-3)), (h, float(err.max()), float(bound[err.argmax()]))


@pytest.mark.parametrize("P0,C,W", [(1000, 300, 200), (5000, 100, 256), (300, 1, 7), (0, 400, 130)])
def test_window_chunk(P0, C, W):
    hq, hkv = 4, 2
    L = P0 + C
    q, k, v = si.random_qkv(60 + P0, 1, L, hq, hkv, 128, "bf16")
    kc_prefix = bf16_round(R.rope_keys_for_cache(k[0, :P0].double().numpy(), THETA)) if P0 else \
        np.zeros((0, hkv, 128))
    kcache = torch.zeros(L, hkv, 128, dtype=torch.bfloat16, device="cuda")
    vcache = torch.zeros_like(kcache)
    if P0:
        kcache[:P0] = torch.from_numpy(kc_prefix).to(torch.bfloat16).cuda()
        vcache[:P0] = v[0, :P0].cuda()
    out, lse = bfl.bifocal_prefill_chunk(q[0, P0:].cuda(), k[0, P0:].cuda(), v[0, P0:].cuda(), kcache, vcache, P0,
                                         w0=W, w_pretrained=64, theta=THETA, flags=bfl.FLAG_WINDOW)
    torch.cuda.synchronize()
    assert bfl.last_device_error() == 0
    ref_k = np.concatenate([kc_prefix, R.rope_keys_for_cache(k[0, P0:].double().numpy(), THETA, start=P0)])
    ro, rl = R.sliding_window_cached_reference(q[0, P0:].double().numpy(), ref_k, v[0].double().numpy(), P0, W,
                                               THETA)
    assert_close(out.cpu().float().numpy(), lse.cpu().numpy(), ro, rl, f"window chunk P0={P0} C={C} W={W}")


@pytest.mark.parametrize("W", [1, 300, 5000])
def test_window_decode_session(W):
    hq, hkv, prefix, steps = 8, 2, 2000, 12
    cap = prefix + steps
    g = si.generator(70 + W)
    kp = torch.randn(prefix, hkv, 128, generator=g).to(torch.bfloat16)
    vp = torch.randn(prefix, hkv, 128, generator=g).to(torch.bfloat16)
    kcache = torch.zeros(cap, hkv, 128, dtype=torch.bfloat16, device="cuda")
    vcache = torch.zeros_like(kcache)
    kcache[:prefix], vcache[:prefix] = kp.cuda(), vp.cuda()
    ref_k = np.zeros((cap, hkv, 128))
    ref_v = np.zeros((cap, hkv, 128))
    ref_k[:prefix], ref_v[:prefix] = kp.double().numpy(), vp.double().numpy()
    for t in range(steps):
        q = torch.randn(hq, 128, generator=g).to(torch.bfloat16)
        kn = torch.randn(hkv, 128, generator=g).to(torch.bfloat16)
        vn = torch.randn(hkv, 128, generator=g).to(torch.bfloat16)
        L = prefix + t + 1
        out, lse = bfl.bifocal_decode(q.cuda(), kn.cuda(), vn.cuda(), kcache, vcache, L, w0=W, w_pretrained=512,
                                      theta=THETA, flags=bfl.FLAG_WINDOW)
        ref_k[L - 1] = bf16_round(R.rope_keys_for_cache(kn[None].double().numpy(), THETA, start=L - 1)[0])
        ref_v[L - 1] = vn.double().numpy()
        ro, rl = R.sliding_window_cached_reference(q[None].double().numpy(), ref_k, ref_v, L - 1, W, THETA)
        assert_close(out.cpu().float().numpy(), lse.cpu().numpy(), ro[0], rl[:, 0], f"window decode L={L} W={W}")
    torch.cuda.synchronize()
    assert bfl.last_device_error() == 0


def test_window_prefill_many_waves_sampled():
    # 512 CTAs (several waves on 148 SMs), Qwen3-8B heads, sampled rows
    L, hq, hkv, W = 4096, 32, 8, 1000
    q, k, v = si.random_qkv(88, 1, L, hq, hkv, 128, "bf16")
    out, lse, _, _ = bfl.bifocal_prefill(q.cuda(), k.cuda(), v.cuda(), w0=W, w_pretrained=64, theta=THETA,
                                         flags=bfl.FLAG_WINDOW)
    torch.cuda.synchronize()
    assert bfl.last_device_error() == 0
    rows = [0, 1, 127, 128, 999, 1000, 1001, 2047, 2048, 4095] + list(range(300, 4096, 257))
    ro, rl = R.sliding_window_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(), W, THETA,
                                        rows=rows)
    assert_close(out[:, rows].cpu().float().numpy(), lse[:, :, rows].cpu().numpy(), ro, rl, "window 4096 sampled")

"""GPU parity of the fused-load prefill (BF_FLAG_FUSED_ROPE): RoPE and the correction rotation
applied inside the attention kernel's tile loads, with no rotated copy of q or k in HBM.

The same oracle checks as the RoPE-pass path: band edges inside and across tiles, G with and
without the incremental rotation (position aliasing with G = 3, 5 takes exact angles per row),
batch 2, the plain and sliding-window kinds, chunked prefill over a cache (cached keys
re-phased in the tile loads), and sampled rows of the full-size workloads. For the chunk path
the kernel reads the chunk's own keys back from the cache it has just written, so the
reference cache holds them as stored, rounded to bf16 (the reading of the cache format that the
decode reference also follows)."""
import numpy as np
import pytest
import torch

import oracle.bifocal_ref as R
import rope_context_extension_bifocal_b200 as bfl
import seeded_inputs as si
from tests.gpu_helpers import assert_close, oracle_rows

pytestmark = pytest.mark.gpu
FUSED = bfl.FLAG_FUSED_ROPE
FI, PA = si.FREQ_INTERP, si.POS_ALIAS


def np64(t):
    return t.double().numpy() if t.dtype != torch.bfloat16 else t.float().double().numpy()


def bf16_round(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float64)).to(torch.bfloat16).double().numpy()


def run(q, k, v, w0, w_pre, theta, mode, flags=0, want_cache=False):
    out, lse, kc, vc = bfl.bifocal_prefill(q.cuda(), k.cuda(), v.cuda(), w0=w0, w_pretrained=w_pre, theta=theta,
                                           mode=mode, flags=flags | FUSED, want_cache=want_cache)
    torch.cuda.synchronize()
    assert bfl.last_device_error() == 0
    return out, lse, kc, vc


CASES = [
    # L, hq, hkv, w0, w_pre, mode
    (1, 2, 1, 0, 1, FI),
    (127, 4, 2, 1, 32, PA),       # G = 4
    (128, 4, 2, 63, 32, FI),
    (129, 4, 2, 64, 32, PA),      # G = 5: exact angle per row
    (255, 8, 2, 65, 64, FI),
    (600, 8, 4, 600, 100, FI),    # w0 >= L
    (600, 4, 2, 100, 600, PA),    # G = 1
    (1100, 4, 2, 300, 220, PA),   # G = 5
    (1100, 4, 2, 300, 367, FI),   # G = 3
    (1100, 4, 2, 300, 367, PA),   # G = 3: exact angle per row
    (2500, 4, 2, 200, 1250, PA),  # G = 2: incremental
    (2000, 8, 2, 0, 256, FI),     # w0 = 0: all long-range, runs of up to 16 tiles (re-anchoring)
    (2000, 8, 1, 1500, 256, PA),  # G = 8, GQA 8
]


@pytest.mark.parametrize("L,hq,hkv,w0,w_pre,mode", CASES)
def test_fused_prefill_matches_oracle(L, hq, hkv, w0, w_pre, mode):
    q, k, v = si.random_qkv(300 + L, 1, L, hq, hkv, 128, "bf16")
    out, lse, _, _ = run(q, k, v, w0, w_pre, 1e4, mode)
    ro, rl = R.bifocal_attention(np64(q), np64(k), np64(v), w0, w_pre, 1e4, mode)
    assert_close(out.cpu().float().numpy(), lse.cpu().numpy(), ro, rl, f"fused L={L} w0={w0} w_pre={w_pre} {mode}")


def test_fused_matches_rope_pass_path():
    q, k, v = si.random_qkv(13, 1, 3000, 8, 2, 128, "bf16")
    a, la, _, _ = run(q, k, v, 300, 512, 1e6, FI)
    b, lb, _, _ = bfl.bifocal_prefill(q.cuda(), k.cuda(), v.cuda(), w0=300, w_pretrained=512, theta=1e6)
    torch.cuda.synchronize()
    assert (a.float() - b.float()).abs().max().item() < 2e-2
    assert (la - lb).abs().max().item() < 1e-3


def test_fused_batch_two_and_cache_output():
    q, k, v = si.random_qkv(7, 2, 300, 4, 2, 128, "bf16")
    out, lse, kc, vc = run(q, k, v, 50, 100, 1e4, PA, want_cache=True)
    ro, rl = R.bifocal_attention(np64(q), np64(k), np64(v), 50, 100, 1e4, PA)
    assert_close(out.cpu().float().numpy(), lse.cpu().numpy(), ro, rl, "fused batch 2")
    for bb in range(2):
        ref = R.rope_keys_for_cache(np64(k)[bb], 1e4)
        got = kc[bb].cpu().float().double().numpy()
        assert np.max(np.abs(got - ref)) <= 2.0 ** -8 * np.max(np.abs(ref)) + 1e-6
    assert torch.equal(vc.cpu(), v)


def test_fused_plain_comparator():
    q, k, v = si.random_qkv(8, 1, 700, 4, 2, 128, "bf16")
    p = bfl.make_params(4, 2, 128, 0, 1, 1e6, FI, None, FUSED)
    out = torch.empty(1, 700, 4, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(1, 4, 700, dtype=torch.float32, device="cuda")
    assert bfl.prefill_workspace_size(bfl.DTYPE_BF16, 1, 700, p) == 0
    out, lse, _, _ = bfl._prefill("rope_causal_prefill", q.cuda(), k.cuda(), v.cuda(), p, True, False, out, None,
                                  None)
    torch.cuda.synchronize()
    ro, rl = R.rope_causal_attention(np64(q), np64(k), np64(v), 1e6)
    assert_close(out.cpu().float().numpy(), lse.cpu().numpy(), ro, rl, "fused plain")


@pytest.mark.parametrize("W,L", [(1, 300), (100, 1000), (130, 700)])
def test_fused_window(W, L):
    q, k, v = si.random_qkv(500 + W, 1, L, 4, 2, 128, "bf16")
    out, lse, _, _ = run(q, k, v, W, 64, 1e4, FI, flags=bfl.FLAG_WINDOW)
    ro, rl = R.sliding_window_attention(np64(q), np64(k), np64(v), W, 1e4)
    if W == 1:
        # one key per row: the LSE is a single score, bounded by the fp16 rounding of its two
        # operands (the reading of test_gpu_window's W = 1 case)
        assert_close(out.cpu().float().numpy(), None, ro, None, "fused window 1")
        omega = R.rope_omega(128, 1e4)
        pos = np.arange(L)
        for h in range(4):
            qr = R.rope_rotate(q[0, :, h].float().double().numpy(), pos, omega)
            kr = R.rope_rotate(k[0, :, h // 2].float().double().numpy(), pos, omega)
            bound = (2.0 ** -10 + 2.0 ** -20) / np.sqrt(128) * np.abs(qr * kr).sum(axis=1)
            err = np.abs(lse[0, h].cpu().double().numpy() - rl[0, h])
            assert np.all(err <= np.maximum(bound, 1e-3)), (h, float(err.max()))
    else:
        assert_close(out.cpu().float().numpy(), lse.cpu().numpy(), ro, rl, f"fused window {W}")


CHUNK = [
    # seed, P0, C, hq, hkv, w0, w_pre, mode
    (1, 0, 300, 4, 2, 64, 128, FI),
    (2, 200, 1, 4, 2, 64, 128, PA),
    (3, 1000, 300, 8, 2, 100, 512, FI),
    (4, 777, 333, 4, 2, 50, 256, PA),     # G = 5: exact angles
    (5, 1024, 300, 4, 2, 64, 512, FI),
    (6, 1024, 300, 4, 2, 64, 512, PA),
    (7, 500, 200, 4, 2, 0, 128, FI),
    (8, 600, 100, 4, 2, 64, 4096, PA),
    (9, 300, 300, 2, 1, 2000, 64, FI),
    (10, 3000, 500, 4, 2, 0, 256, FI),    # long runs of cached tiles (re-anchoring)
]


def run_chunk(seed, P0, C, hq, hkv, w0, wp, mode, flags=0, rows=None):
    theta = 1e6
    L = P0 + C
    cap = L + 5
    q, k, v = si.random_qkv(seed, 1, L, hq, hkv, 128, "bf16")
    keys = bf16_round(R.rope_keys_for_cache(k[0].double().numpy(), theta))  # every row as the cache stores it
    kcache = torch.zeros(cap, hkv, 128, dtype=torch.bfloat16, device="cuda")
    vcache = torch.zeros_like(kcache)
    if P0:
        kcache[:P0] = torch.from_numpy(keys[:P0]).to(torch.bfloat16).cuda()
        vcache[:P0] = v[0, :P0].cuda()
    p = bfl.make_params(hq, hkv, 128, w0, wp, theta, mode, None, flags | FUSED)
    assert bfl.prefill_chunk_workspace_size(P0, C, p) == 0
    out, lse = bfl.bifocal_prefill_chunk(q[0, P0:].cuda(), k[0, P0:].cuda(), v[0, P0:].cuda(), kcache, vcache, P0,
                                         w0=w0, w_pretrained=wp, theta=theta, mode=mode, flags=flags | FUSED)
    torch.cuda.synchronize()
    assert bfl.last_device_error() == 0
    assert np.max(np.abs(kcache[P0:L].cpu().double().numpy() - keys[P0:])) <= 2.0 ** -7 * np.max(np.abs(keys)) + 1e-5
    assert torch.equal(vcache[P0:L].cpu(), v[0, P0:])
    rows = np.arange(C) if rows is None else np.asarray(sorted(set(int(r) for r in rows if 0 <= r < C)))
    # the reference reads the cache the kernel wrote (every row at bf16)
    ref_k = kcache[:L].cpu().double().numpy()
    if flags & bfl.FLAG_WINDOW:
        ro, rl = R.sliding_window_cached_reference(q[0, P0:].double().numpy(), ref_k, v[0].double().numpy(), P0, w0,
                                                   theta, rows=rows)
    else:
        ro, rl = R.bifocal_chunk_reference(q[0, P0:].double().numpy(), ref_k, v[0].double().numpy(), P0, w0, wp,
                                           theta, mode, rows=rows)
    return assert_close(out.cpu().float().numpy()[rows], lse.cpu().numpy()[:, rows], ro, rl,
                        f"fused chunk P0={P0} C={C} G={R.dynamic_factor(L, wp)}")


@pytest.mark.parametrize("seed,P0,C,hq,hkv,w0,wp,mode", CHUNK)
def test_fused_chunk_matches_oracle(seed, P0, C, hq, hkv, w0, wp, mode):
    run_chunk(seed, P0, C, hq, hkv, w0, wp, mode)


def test_fused_chunk_window():
    run_chunk(21, 1500, 400, 4, 2, 300, 128, FI, flags=bfl.FLAG_WINDOW)


@pytest.mark.parametrize("mode", [FI, PA])
def test_fused_chunk_qwen3_8b_heads_sampled(mode):
    rows = list(range(0, 1000, 37)) + [999]
    run_chunk(31, 9269, 1000, 32, 8, 4096, 2048, mode, rows=rows)


def test_fused_range_guard():
    q, k, v = si.random_qkv(41, 1, 500, 4, 2, 128, "bf16")
    k = (k.float() * 1e5).to(torch.bfloat16)
    bfl.bifocal_prefill(q.cuda(), k.cuda(), v.cuda(), w0=50, w_pretrained=100, theta=1e4, flags=FUSED)
    word = bfl.device_status_word()
    assert word & 0xff == 2 and (word >> 8) == 45, hex(word)  # a row's normaliser was not finite
    assert bfl.last_device_error() == bfl.STATUS_RANGE


# ---------------------------------------------------------------- full-size configs, fused
def sampled_check(w: si.PrefillWorkload, n_rows=512):
    q, k, v = si.prefill_inputs(w)
    out, lse, _, _ = run(q, k, v, w.w0, w.w_pretrained, w.theta, w.mode)
    rows = si.sample_rows(w.seed, w.L, w.w0, w.w_pretrained, n_rows)
    go = out[0, torch.as_tensor(rows, device=out.device)].cpu().float().numpy()
    gl = lse[0][:, torch.as_tensor(rows, device=lse.device)].cpu().numpy()
    del out, lse
    torch.cuda.empty_cache()
    ro, rl = oracle_rows(np64(q), np64(k), np64(v), w.w0, w.w_pretrained, w.theta, w.mode, rows)
    return assert_close(go, gl, ro[0], rl[0], "fused " + w.name)


def test_fused_qwen3_1p7b_32k_g1():
    sampled_check(si.QWEN3_1P7B_32K)


@pytest.mark.parametrize("w", [si.QWEN3_4B_64K_FI, si.QWEN3_4B_64K_PA], ids=lambda w: w.mode)
def test_fused_qwen3_4b_64k(w):
    sampled_check(w)


def test_fused_qwen3_8b_128k():
    sampled_check(si.qwen3_8b_128k(4096))

"""GPU parity of the prefill path (through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle.bifocal_ref as R
import rope_context_extension_bifocal_b200 as bfl
import seeded_inputs as si
from tests.gpu_helpers import assert_close, oracle_rows

pytestmark = pytest.mark.gpu


def run_prefill(q, k, v, w0, w_pre, theta, mode, flags=0, want_cache=False):
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    out, lse, kc, vc = bfl.bifocal_prefill(qd, kd, vd, w0=w0, w_pretrained=w_pre, theta=theta, mode=mode,
                                           flags=flags, want_cache=want_cache)
    torch.cuda.synchronize()
    assert bfl.last_device_error() == 0
    return out, lse, kc, vc


def np64(t):
    return t.double().numpy() if t.dtype != torch.bfloat16 else t.float().double().numpy()


@pytest.mark.parametrize("mode", [si.FREQ_INTERP, si.POS_ALIAS])
def test_tiny_config(mode):
    w = si.TINY
    q, k, v = si.prefill_inputs(w)
    out, lse, _, _ = run_prefill(q, k, v, w.w0, w.w_pretrained, w.theta, mode)
    ro, rl = R.bifocal_attention(np64(q), np64(k), np64(v), w.w0, w.w_pretrained, w.theta, mode)
    assert R.dynamic_factor(w.L, w.w_pretrained) == 4
    assert_close(out.cpu().float().numpy(), lse.cpu().numpy(), ro, rl, f"tiny {mode}")


EDGE = [
    # L, hq, hkv, D, w0, w_pre, mode
    (1, 2, 1, 128, 0, 1, si.FREQ_INTERP),
    (127, 4, 2, 128, 1, 32, si.POS_ALIAS),
    (128, 4, 2, 128, 63, 32, si.FREQ_INTERP),
    (129, 4, 2, 128, 64, 32, si.POS_ALIAS),
    (255, 8, 2, 128, 65, 64, si.FREQ_INTERP),
    (1000, 4, 1, 128, 63, 256, si.POS_ALIAS),
    (1000, 4, 1, 128, 64, 256, si.FREQ_INTERP),
    (1000, 4, 4, 64, 65, 200, si.POS_ALIAS),
    (777, 2, 2, 64, 0, 100, si.FREQ_INTERP),
    (777, 2, 2, 64, 0, 100, si.POS_ALIAS),
    (600, 8, 4, 128, 600, 100, si.FREQ_INTERP),   # w0 >= L: plain RoPE attention for any G
    (600, 4, 2, 128, 100, 600, si.POS_ALIAS),     # G == 1
    (1100, 4, 2, 128, 300, 220, si.POS_ALIAS),    # G == 5
    (1100, 4, 2, 128, 300, 367, si.FREQ_INTERP),  # G == 3
    (1000, 3, 1, 128, 63, 256, si.POS_ALIAS),     # odd GQA group (3): single-tile tcgen05 kernel
    (600, 2, 2, 128, 100, 150, si.FREQ_INTERP),   # MHA (group 1): single-tile tcgen05 kernel
]


@pytest.mark.parametrize("L,hq,hkv,D,w0,w_pre,mode", EDGE)
def test_edge_cases(L, hq, hkv, D, w0, w_pre, mode):
    q, k, v = si.random_qkv(100 + L, 1, L, hq, hkv, D, "bf16")
    out, lse, _, _ = run_prefill(q, k, v, w0, w_pre, 1e4, mode)
    ro, rl = R.bifocal_attention(np64(q), np64(k), np64(v), w0, w_pre, 1e4, mode)
    assert_close(out.cpu().float().numpy(), lse.cpu().numpy(), ro, rl, f"L={L} w0={w0} w_pre={w_pre} {mode}")


@pytest.mark.parametrize("L,hq,hkv,D,w0,w_pre,mode", [EDGE[2], EDGE[5], EDGE[12], EDGE[13]])
def test_edge_cases_mma_sync_path(L, hq, hkv, D, w0, w_pre, mode):
    # the warp-level mma.sync kernel (D = 64 path, and D = 128 on request) against the oracle
    q, k, v = si.random_qkv(100 + L, 1, L, hq, hkv, D, "bf16")
    out, lse, _, _ = run_prefill(q, k, v, w0, w_pre, 1e4, mode, flags=bfl.FLAG_MMA_SYNC)
    ro, rl = R.bifocal_attention(np64(q), np64(k), np64(v), w0, w_pre, 1e4, mode)
    assert_close(out.cpu().float().numpy(), lse.cpu().numpy(), ro, rl, f"mma.sync L={L} w0={w0} {mode}")


def test_tcgen05_and_mma_sync_agree():
    q, k, v = si.random_qkv(13, 1, 2000, 8, 2, 128, "bf16")
    a, la, _, _ = run_prefill(q, k, v, 300, 512, 1e6, si.FREQ_INTERP)
    b, lb, _, _ = run_prefill(q, k, v, 300, 512, 1e6, si.FREQ_INTERP, flags=bfl.FLAG_MMA_SYNC)
    assert (a.float() - b.float()).abs().max().item() < 2e-2
    assert (la - lb).abs().max().item() < 1e-3


def test_batch_two():
    q, k, v = si.random_qkv(7, 2, 300, 4, 2, 128, "bf16")
    out, lse, _, _ = run_prefill(q, k, v, 50, 100, 1e4, si.POS_ALIAS)
    ro, rl = R.bifocal_attention(np64(q), np64(k), np64(v), 50, 100, 1e4, si.POS_ALIAS)
    assert_close(out.cpu().float().numpy(), lse.cpu().numpy(), ro, rl, "batch 2")


def test_plain_comparator_matches_oracle():
    q, k, v = si.random_qkv(8, 1, 700, 4, 2, 128, "bf16")
    out, lse, _, _ = bfl.rope_causal_prefill(q.cuda(), k.cuda(), v.cuda(), theta=1e6)
    ro, rl = R.rope_causal_attention(np64(q), np64(k), np64(v), 1e6)
    assert_close(out.cpu().float().numpy(), lse.cpu().numpy(), ro, rl, "plain")


@pytest.mark.parametrize("mode", [si.FREQ_INTERP, si.POS_ALIAS])
def test_forced_bifocal_equals_shortcut_when_g1(mode):
    # G == 1: both branches coincide, so the two-branch kernel must reproduce the plain kernel up to
    # fp32 summation order (band-edge tiles are accumulated in two visits instead of one)
    q, k, v = si.random_qkv(9, 1, 500, 4, 2, 128, "bf16")
    a, la, _, _ = run_prefill(q, k, v, 64, 512, 1e6, mode)
    b, lb, _, _ = run_prefill(q, k, v, 64, 512, 1e6, mode, flags=bfl.FLAG_FORCE_BIFOCAL)
    assert (a.float() - b.float()).abs().max().item() <= 2.0 ** -7 * max(1.0, a.float().abs().max().item())
    assert (la - lb).abs().max().item() <= 1e-5


def test_kv_cache_output():
    q, k, v = si.random_qkv(10, 1, 333, 4, 2, 128, "bf16")
    _, _, kc, vc = run_prefill(q, k, v, 30, 100, 1e6, si.FREQ_INTERP, want_cache=True)
    ref = R.rope_keys_for_cache(np64(k)[0], 1e6)
    kc = kc.cpu().float().double().numpy()[0]
    assert np.max(np.abs(kc - ref)) <= 2.0 ** -8 * np.max(np.abs(ref)) + 1e-6
    assert torch.equal(vc.cpu(), v)


def test_fp32_inputs_cache_and_v_copy():
    q, k, v = si.random_qkv(11, 1, 200, 2, 1, 64, "fp32")
    out, lse, kc, vc = run_prefill(q, k, v, 20, 64, 1e4, si.FREQ_INTERP, want_cache=True)
    ro, rl = R.bifocal_attention(np64(q), np64(k), np64(v), 20, 64, 1e4, si.FREQ_INTERP)
    assert_close(out.cpu().float().numpy(), lse.cpu().numpy(), ro, rl, "fp32 inputs")
    assert torch.equal(vc.cpu(), v.to(torch.bfloat16))


def test_invalid_arguments_raise():
    q, k, v = (t.cuda() for t in si.random_qkv(12, 1, 64, 4, 2, 128, "bf16"))
    with pytest.raises(bfl.BifocalError):
        bfl.bifocal_prefill(q, k, v, w0=-1, w_pretrained=16, theta=1e4)
    with pytest.raises(bfl.BifocalError):
        bfl.bifocal_prefill(q, k, v, w0=4, w_pretrained=0, theta=1e4)
    q3 = torch.zeros(1, 64, 3, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(bfl.BifocalError):
        bfl.bifocal_prefill(q3, k, v, w0=4, w_pretrained=16, theta=1e4)


# ---------------------------------------------------------------- full-size configs
def sampled_check(w: si.PrefillWorkload, n_rows=512):
    q, k, v = si.prefill_inputs(w)
    out, lse, _, _ = run_prefill(q, k, v, w.w0, w.w_pretrained, w.theta, w.mode)
    rows = si.sample_rows(w.seed, w.L, w.w0, w.w_pretrained, n_rows)
    go = out[0, torch.as_tensor(rows, device=out.device)].cpu().float().numpy()
    gl = lse[0][:, torch.as_tensor(rows, device=lse.device)].cpu().numpy()
    del out, lse
    torch.cuda.empty_cache()
    ro, rl = oracle_rows(np64(q), np64(k), np64(v), w.w0, w.w_pretrained, w.theta, w.mode, rows)
    return assert_close(go, gl, ro[0], rl[0], w.name)


def test_qwen3_1p7b_32k_g1():
    assert R.dynamic_factor(32768, 32768) == 1
    sampled_check(si.QWEN3_1P7B_32K)


@pytest.mark.parametrize("w", [si.QWEN3_4B_64K_FI, si.QWEN3_4B_64K_PA], ids=lambda w: w.mode)
def test_qwen3_4b_64k(w):
    sampled_check(w)


@pytest.mark.parametrize("w0", si.QWEN3_8B_128K_W0)
def test_qwen3_8b_128k(w0):
    sampled_check(si.qwen3_8b_128k(w0))

"""Failure detection on the GPU, without faulting it (GPU).

Two kinds of device-side event set the library's status word instead of trapping:

- a bounded wait that expires. A test-only control makes the producer of one CTA skip a
  whole fill of the prefill kernel (no expect_tx, no copy), or stop issuing the decode kernel's
  stages from a given one on (in a test-only instantiation of that kernel), so the wait for it
  can only run out; with the wait limit shortened to 50 ms the call returns after about that
  long, every role of the CTA leaves through its normal teardown (a producer that saw the expiry
  first waits for each copy it did issue, the MMA issuer for its MMAs, tensor memory is freed),
  and bifocal_last_device_error reports BF_ERR_TIMEOUT with the site of the wait that gave up;
- an fp16 QK^T operand out of range: q scaled by 1e5 makes the rotated queries exceed 65520,
  which fp16 would round to inf; the RoPE pass (prefill) and the query rotation (decode)
  report BF_ERR_RANGE, and a cached key of +-1e6 is caught by the decode kernel's check of its
  final running max and sum.

After each event the next normal call on the same device returns BF_OK and matches the oracle.
"""
import numpy as np
import pytest
import torch

import oracle.bifocal_ref as R
import rope_context_extension_bifocal_b200 as bfl
import seeded_inputs as si
from tests.gpu_helpers import assert_close

pytestmark = pytest.mark.gpu

PREFILL_SITES = set(range(10, 35))  # the bounded waits of the ping-pong prefill kernel
DECODE_SITES = {1, 2, 3, 4, 5}       # the bounded waits of the split-KV decode kernel
LIMIT_NS = 50_000_000


def np64(t):
    return t.float().double().numpy()


@pytest.fixture(autouse=True)
def _clean_status():
    torch.cuda.synchronize()
    bfl.last_device_error()  # start from a clear status word
    yield
    bfl.test_set_fault()     # every injection off, default wait limit
    bfl.last_device_error()


def small_prefill(scale_q=1.0, seed=71, flags=0):
    L, hq, hkv, D, w0, wp = 1000, 4, 2, 128, 100, 256  # D 128, even GQA group: the ping-pong kernel
    q, k, v = si.random_qkv(seed, 1, L, hq, hkv, D, "bf16")
    q = (q.float() * scale_q).to(torch.bfloat16)
    kw = dict(w0=w0, w_pretrained=wp, theta=1e4, mode=si.FREQ_INTERP, flags=flags)
    out, lse, _, _ = bfl.bifocal_prefill(q.cuda(), k.cuda(), v.cuda(), **kw)
    return (q, k, v, kw), out, lse


def check_prefill_parity(case, out, lse):
    q, k, v, kw = case
    ro, rl = R.bifocal_attention(np64(q), np64(k), np64(v), kw["w0"], kw["w_pretrained"], kw["theta"], kw["mode"])
    assert_close(out.cpu().float().numpy(), lse.cpu().numpy(), ro, rl, "prefill after a fault")


@pytest.mark.parametrize("flags", [0, bfl.FLAG_FUSED_ROPE], ids=["rope_pass", "fused_loads"])
@pytest.mark.parametrize("fill", [0, 1, 5])
def test_prefill_skipped_fill_times_out_then_recovers(fill, flags):
    # the fused form's copies are issued by a transform warp between its tiles: a missing K fill
    # leaves the transform warps waiting, a missing V fill the MMA issuer
    bfl.test_set_fault(bfl.FAULT_PREFILL_SKIP_FILL, fill, LIMIT_NS)
    small_prefill(flags=flags)
    word = bfl.device_status_word()
    assert word & 0xff == 1, hex(word)  # a bounded wait expired
    assert (word >> 8) in PREFILL_SITES, hex(word)
    assert bfl.last_device_error() == bfl.STATUS_TIMEOUT
    assert bfl.last_device_error() == 0  # reading cleared it
    bfl.test_set_fault()
    case, out, lse = small_prefill(flags=flags)
    torch.cuda.synchronize()
    assert bfl.last_device_error() == 0
    check_prefill_parity(case, out, lse)


def decode_case(seed=72, scale_q=1.0):
    hq, hkv, D, L = 8, 2, 128, 3000
    g = si.generator(seed)
    kc = torch.randn(L + 8, hkv, D, generator=g).to(torch.bfloat16)
    vc = torch.randn(L + 8, hkv, D, generator=g).to(torch.bfloat16)
    q = (torch.randn(hq, D, generator=g) * scale_q).to(torch.bfloat16)
    kn = torch.randn(hkv, D, generator=g).to(torch.bfloat16)
    vn = torch.randn(hkv, D, generator=g).to(torch.bfloat16)
    return q, kn, vn, kc, vc, L


def run_decode(case):
    q, kn, vn, kc, vc, L = case
    kcd, vcd = kc.cuda(), vc.cuda()
    out, lse = bfl.bifocal_decode(q.cuda(), kn.cuda(), vn.cuda(), kcd, vcd, L, w0=200, w_pretrained=1024,
                                  theta=1e4, mode=si.FREQ_INTERP)
    return out, lse


def check_decode_parity(case, out, lse):
    q, kn, vn, kc, vc, L = case
    ref_k = kc.float().double().numpy().copy()
    ref_v = vc.float().double().numpy().copy()
    row = R.rope_keys_for_cache(kn[None].float().double().numpy(), 1e4, start=L - 1)[0]
    ref_k[L - 1] = torch.from_numpy(row).to(torch.bfloat16).double().numpy()  # the cache's bf16 format
    ref_v[L - 1] = np64(vn)
    ro, rl = R.bifocal_decode_reference(np64(q), ref_k, ref_v, L, 200, 1024, 1e4, si.FREQ_INTERP)
    assert_close(out.cpu().float().numpy(), lse.cpu().numpy(), ro, rl, "decode after a fault")


def test_decode_skipped_stage_times_out_then_recovers():
    case = decode_case()
    bfl.test_set_fault(bfl.FAULT_DECODE_SKIP_STAGE, 0, LIMIT_NS)
    run_decode(case)
    word = bfl.device_status_word()
    assert word & 0xff == 1 and (word >> 8) in DECODE_SITES, hex(word)
    assert bfl.last_device_error() == bfl.STATUS_TIMEOUT
    bfl.test_set_fault()
    out, lse = run_decode(case)
    torch.cuda.synchronize()
    assert bfl.last_device_error() == 0
    check_decode_parity(case, out, lse)


def test_prefill_fp16_range_is_reported_then_recovers():
    small_prefill(scale_q=1e5)
    word = bfl.device_status_word()
    assert word & 0xff == 2 and (word >> 8) == 40, hex(word)  # the RoPE pass saw an operand >= 65520
    assert bfl.last_device_error() == bfl.STATUS_RANGE
    case, out, lse = small_prefill()
    torch.cuda.synchronize()
    assert bfl.last_device_error() == 0
    check_prefill_parity(case, out, lse)


def test_decode_fp16_range_is_reported_then_recovers():
    run_decode(decode_case(scale_q=1e5))
    word = bfl.device_status_word()
    assert word & 0xff == 2 and (word >> 8) == 42, hex(word)  # the rotated query
    assert bfl.last_device_error() == bfl.STATUS_RANGE
    case = decode_case()
    out, lse = run_decode(case)
    torch.cuda.synchronize()
    assert bfl.last_device_error() == 0
    check_decode_parity(case, out, lse)


def test_decode_cached_key_out_of_range_is_reported():
    q, kn, vn, kc, vc, L = decode_case()
    # a cached key no fp16 operand can hold, before or after its rotation, planted with both signs:
    # negating a key negates its score, so one of the two rows scores +inf or NaN for every query
    # head (a score of -inf alone would only give that key weight 0)
    kc[17, 1, 5] = 1e6
    kc[18, 1, 5] = -1e6
    run_decode((q, kn, vn, kc, vc, L))
    word = bfl.device_status_word()
    assert word & 0xff == 2 and (word >> 8) == 43, hex(word)
    assert bfl.last_device_error() == bfl.STATUS_RANGE


def test_fault_control_rejects_bad_arguments():
    with pytest.raises(bfl.BifocalError):
        bfl.test_set_fault(7, 0, 0)
    with pytest.raises(bfl.BifocalError):
        bfl.test_set_fault(bfl.FAULT_PREFILL_SKIP_FILL, -1, 0)
    with pytest.raises(bfl.BifocalError):
        bfl.test_set_fault(bfl.FAULT_NONE, 0, -5)

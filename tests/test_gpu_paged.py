"""GPU parity of the batched decode over a paged cache (bifocal_decode_paged) against the
fp64 decode oracle, sequence by sequence on the gathered logical cache. The sequences have
different lengths and so different G (1, 2, 3 at w_pretrained 4096), the pages are assigned in
a shuffled order, and every pool slot that holds no key is NaN: masked keys and the zeroed
value rows of a stage's tail must keep it out of every result."""
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


@pytest.mark.parametrize("page_size,mode", [(32, si.FREQ_INTERP), (16, si.POS_ALIAS), (64, si.FREQ_INTERP)])
def test_paged_batch_matches_oracle(page_size, mode):
    hq, hkv, D, w0, wp = 8, 2, 128, 300, 4096
    lens = [1, 100, 4096 + 17, 9000, 2000]
    B = len(lens)
    max_len = max(lens) + 3
    max_pages = (max_len + page_size - 1) // page_size
    g = si.generator(500 + page_size)
    pool_pages = sum((L + page_size - 1) // page_size for L in lens) + 7
    perm = torch.randperm(pool_pages, generator=g)
    table = torch.zeros(B, max_pages, dtype=torch.int32)
    nxt = 0
    for b, L in enumerate(lens):
        n = (L + page_size - 1) // page_size
        table[b, :n] = perm[nxt:nxt + n].to(torch.int32)
        nxt += n
    rows = pool_pages * page_size
    kpool = torch.full((rows, hkv, D), float("nan"), dtype=torch.bfloat16)
    vpool = torch.full((rows, hkv, D), float("nan"), dtype=torch.bfloat16)
    logical_k, logical_v = [], []
    for b, L in enumerate(lens):
        kc = torch.randn(L, hkv, D, generator=g).to(torch.bfloat16)  # keys already under the original RoPE
        vc = torch.randn(L, hkv, D, generator=g).to(torch.bfloat16)
        for j in range(L - 1):  # row L-1 is the new token's, written by the call
            r = int(table[b, j // page_size]) * page_size + j % page_size
            kpool[r], vpool[r] = kc[j], vc[j]
        logical_k.append(kc.double().numpy())
        logical_v.append(vc.double().numpy())
    q = torch.randn(B, hq, D, generator=g).to(torch.bfloat16)
    kn = torch.randn(B, hkv, D, generator=g).to(torch.bfloat16)
    vn = torch.randn(B, hkv, D, generator=g).to(torch.bfloat16)
    kp, vp = kpool.cuda(), vpool.cuda()
    out, lse = bfl.bifocal_decode_paged(q.cuda(), kn.cuda(), vn.cuda(), kp, vp, page_size, table.cuda(),
                                        torch.tensor(lens, dtype=torch.int32).cuda(), max_len, w0=w0,
                                        w_pretrained=wp, theta=THETA, mode=mode)
    torch.cuda.synchronize()
    assert bfl.last_device_error() == 0
    kp_h = kp.cpu()
    for b, L in enumerate(lens):
        ref_k, ref_v = logical_k[b].copy(), logical_v[b].copy()
        ref_k[L - 1] = bf16_round(R.rope_keys_for_cache(kn[b][None].double().numpy(), THETA, start=L - 1)[0])
        ref_v[L - 1] = vn[b].double().numpy()
        ro, rl = R.bifocal_decode_reference(q[b].double().numpy(), ref_k, ref_v, L, w0, wp, THETA, mode)
        assert_close(out[b].cpu().float().numpy(), lse[b].cpu().numpy(), ro, rl,
                     f"paged b={b} L={L} G={R.dynamic_factor(L, wp)} page={page_size}")
        r = int(table[b, (L - 1) // page_size]) * page_size + (L - 1) % page_size
        got = kp_h[r].double().numpy()
        assert np.all(np.abs(got - ref_k[L - 1]) <= np.abs(ref_k[L - 1]) * 2.0 ** -7 + 1e-5)

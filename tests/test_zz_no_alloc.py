"""The allocation-free decode entry point against the workspace one (GPU).

bifocal_decode_noalloc serves callers that cannot allocate device memory themselves (a
plug-in inside a runtime that owns all device memory, or a loop where cudaMalloc's device
synchronisation is not acceptable): its split-KV partials live in the library's static
device array. Here two decode sessions run side by side on identical caches, one through
each entry point, and must agree bit for bit on two calls in a row (both run the same
kernels with the same split layout), with no allocation made by the scratch-array call.
The file sorts last so that a run stopping at the first failure has run every other test.
"""
import numpy as np
import pytest
import torch

import rope_context_extension_bifocal_b200 as bfl
import seeded_inputs as si

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mode", [si.FREQ_INTERP, si.POS_ALIAS])
def test_noalloc_decode_matches_workspace_decode(mode):
    hq, hkv, D, cap, prefix = 32, 8, 128, 4200, 4094
    g = si.generator(31)
    kc0 = torch.randn(cap, hkv, D, generator=g).to(torch.bfloat16)
    vc0 = torch.randn(cap, hkv, D, generator=g).to(torch.bfloat16)
    kc_a, vc_a = kc0.cuda(), vc0.cuda()
    kc_b, vc_b = kc0.cuda(), vc0.cuda()
    out_b = torch.empty(hq, D, dtype=torch.bfloat16, device="cuda")
    lse_b = torch.empty(hq, dtype=torch.float32, device="cuda")
    # two calls in a row; L = 4095 (G = 1) then 4096 ... crossing w_pretrained 4095 -> G = 2
    for L in (prefix + 1, prefix + 2):
        q = torch.randn(hq, D, generator=g).to(torch.bfloat16).cuda()
        kn = torch.randn(hkv, D, generator=g).to(torch.bfloat16).cuda()
        vn = torch.randn(hkv, D, generator=g).to(torch.bfloat16).cuda()
        kw = dict(w0=300, w_pretrained=4095, theta=1e6, mode=mode)
        oa, la = bfl.bifocal_decode(q, kn, vn, kc_a, vc_a, L, **kw)
        torch.cuda.synchronize()
        # the call itself allocates nothing: neither through torch's allocator (out and lse are
        # passed in) nor on the device (free device memory is the same before and after)
        alloc0 = torch.cuda.memory_allocated()
        free0 = torch.cuda.mem_get_info()[0]
        ob, lb = bfl.bifocal_decode_noalloc(q, kn, vn, kc_b, vc_b, L, out=out_b, lse=lse_b, **kw)
        torch.cuda.synchronize()
        assert torch.cuda.memory_allocated() == alloc0
        assert torch.cuda.mem_get_info()[0] == free0
        # same kernels, same split layout, same reduction order: the results agree bit for bit,
        # so a wrong offset inside the static scratch cannot hide behind a tolerance
        assert torch.equal(oa, ob) and torch.equal(la, lb)
        assert torch.equal(kc_a[L - 1], kc_b[L - 1]) and torch.equal(vc_a[L - 1], vc_b[L - 1])
    assert bfl.last_device_error() == 0


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 256 query heads of 128: the partials would need more than the 16 MiB static scratch
    p = bfl.make_params(256, 8, 128, 300, 4096, 1e6)
    assert bfl.decode_workspace_size(100000, p) > 16 << 20
    q = torch.zeros(256, 128, dtype=torch.bfloat16, device="cuda")
    kn = torch.zeros(8, 128, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(100000, 8, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(bfl.BifocalError) as e:
        bfl.bifocal_decode_noalloc(q, kn, kn, kc, kc, 100000, w0=300, w_pretrained=4096, theta=1e6)
    assert e.value.status == 5

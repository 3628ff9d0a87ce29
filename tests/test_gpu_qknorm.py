"""GPU parity of the RoPE pass with Qwen3's per-head q/k RMS norm fused in
(bifocal_prefill_rope_qknorm + bifocal_prefill_attention) against the oracle: RMS norm of the
raw q and k in fp64, then the bifocal attention definition; and the cache it writes."""
import numpy as np
import pytest
import torch

import oracle.bifocal_ref as R
import rope_context_extension_bifocal_b200 as bfl
import seeded_inputs as si
from tests.gpu_helpers import assert_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("L,hq,hkv,D,w0,wp,mode,dtype", [
    (1000, 8, 2, 128, 100, 256, si.FREQ_INTERP, "bf16"),
    (777, 4, 2, 128, 64, 128, si.POS_ALIAS, "bf16"),
    (512, 2, 1, 64, 64, 128, si.FREQ_INTERP, "fp32"),
])
def test_qknorm_prefill(L, hq, hkv, D, w0, wp, mode, dtype):
    theta, eps = 1e6, 1e-6
    q, k, v = si.random_qkv(90 + L, 1, L, hq, hkv, D, dtype)
    g = si.generator(91 + L)
    wq = (1.0 + 0.2 * torch.randn(D, generator=g)).to(q.dtype)
    wk = (1.0 + 0.2 * torch.randn(D, generator=g)).to(q.dtype)
    dev = "cuda"
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    p = bfl.make_params(hq, hkv, D, w0, wp, theta, mode)
    ws = torch.empty(bfl.prefill_workspace_size(bfl.DTYPE_BF16 if dtype == "bf16" else bfl.DTYPE_FP32, 1, L, p),
                     dtype=torch.uint8, device=dev)
    kc = torch.empty(1, L, hkv, D, dtype=torch.bfloat16, device=dev)
    bfl.bifocal_prefill_rope_qknorm(qd, kd, vd, p, ws, wq.to(dev), wk.to(dev), eps, kcache=kc)
    out = torch.empty(1, L, hq, D, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(1, hq, L, dtype=torch.float32, device=dev)
    bfl.bifocal_prefill_attention(vd, p, ws, out, lse)
    torch.cuda.synchronize()
    assert bfl.last_device_error() == 0
    qn = R.qk_rms_norm(q.double().numpy(), wq.double().numpy(), eps)
    kn = R.qk_rms_norm(k.double().numpy(), wk.double().numpy(), eps)
    ro, rl = R.bifocal_attention(qn, kn, v.double().numpy(), w0, wp, theta, mode)
    assert_close(out.cpu().float().numpy(), lse.cpu().numpy(), ro, rl, f"qknorm L={L} D={D} {dtype}")
    want = torch.from_numpy(R.rope_keys_for_cache(kn[0], theta)).to(torch.bfloat16).double().numpy()
    got = kc[0].cpu().double().numpy()
    bad = np.abs(got - want) > np.abs(want) * 2.0 ** -7 + 1e-4
    assert not bad.any(), (np.argwhere(bad)[:4], got[bad][:4], want[bad][:4])

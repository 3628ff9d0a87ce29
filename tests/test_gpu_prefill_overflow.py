"""GPU parity of the prefill softmax's overflow paths (the ping-pong kernel, D = 128).

The fast path scores a visit half a row at a time against the row's current reference and sends
the first half of P to the tensor core before the second half is computed. A half whose terms
outgrow the reference (sum above 2^24) takes another route: a first half goes to the exact
two-pass path; a second half, sent after the first, takes a new reference and rescales O once the
first half's P.V has run. Random inputs never reach either route, so this test plants them: every
query row of head 0 is the same vector u on the lowest-frequency pair, and one key is 20 u: key 394
(first half of key tile 3) or key 740 (second half of key tile 5). Rows after the planted key see
a score about 80 units (log2) above the reference of their earlier visits. Head 1 (random queries)
shares the keys and takes whichever routes its scores need. One key at a time: two planted keys
with nearly equal scores would split a row's weight between them by a score difference that the
fp16 rounding of the operands moves (by up to 0.05 in the output, whatever the kernel does).

Tolerance: a row dominated by one key has an LSE that is essentially that key's score, so its
error is the fp16 rounding of the two rotated operands of that product (reading c13), as for a
row with a single key (reading c22): the LSE bound per row is max(1e-3, scale * (2^-10 + 2^-20) *
sum_d |q~_d k~_d|) over the row's largest-score key. Output and relative L2 keep the stated
tolerances (the dominated rows' outputs are the planted keys' values)."""
import math

import numpy as np
import pytest
import torch

import oracle.bifocal_ref as R
import rope_context_extension_bifocal_b200 as bfl
import seeded_inputs as si
from tests.gpu_helpers import MAX_ABS, REL_L2, errors

pytestmark = pytest.mark.gpu


def planted(j, L=1024, theta=1e4, seed=91):
    q, k, v = si.random_qkv(seed, 1, L, 2, 1, 128, "bf16")
    u = torch.zeros(128)
    u[63] = u[127] = 4.0
    q[0, :, 0] = u.to(torch.bfloat16)
    k[0, j, 0] = (20.0 * u).to(torch.bfloat16)
    return q, k, v, theta


def lse_bounds(q, k, theta):
    """Per-row LSE bound for rows dominated by one key (fp16 operand rounding of that product)."""
    qd, kd = q[0].double().numpy(), k[0].double().numpy()
    L = qd.shape[0]
    omega = R.rope_omega(128, theta)
    pos = np.arange(L)
    kr = R.rope_rotate(kd[:, 0], pos, omega)
    scale = 1.0 / math.sqrt(128)
    out = np.empty((2, L))
    for h in range(2):
        qr = R.rope_rotate(qd[:, h], pos, omega)
        s = qr @ kr.T
        s = np.where(pos[:, None] < pos[None, :], -np.inf, s)
        jstar = np.argmax(s, axis=1)
        mag = np.sum(np.abs(qr * kr[jstar]), axis=1)
        out[h] = np.maximum(1e-3, scale * (2.0 ** -10 + 2.0 ** -20) * mag)
    return out


@pytest.mark.parametrize("j", [394, 740])
@pytest.mark.parametrize("fused", [False, True])
def test_planted_key_takes_the_overflow_route(fused, j):
    q, k, v, theta = planted(j)
    flags = bfl.FLAG_FUSED_ROPE if fused else 0
    if fused:
        out, lse, _, _ = bfl.bifocal_prefill(q.cuda(), k.cuda(), v.cuda(), w0=q.shape[1], w_pretrained=1 << 20,
                                             theta=theta, flags=flags)
    else:
        out, lse, _, _ = bfl.rope_causal_prefill(q.cuda(), k.cuda(), v.cuda(), theta=theta)
    torch.cuda.synchronize()
    assert bfl.last_device_error() == 0
    ro, rl = R.rope_causal_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(), theta)
    go, gl = out.cpu().float().numpy(), lse.cpu().numpy()
    e = errors(go, None, ro, None)
    assert e["max_abs"] <= MAX_ABS and e["rel_l2"] <= REL_L2, e
    d = np.abs(gl[0] - rl[0])
    bound = lse_bounds(q, k, theta)
    assert np.all(d <= bound), (float(np.max(d - bound)), int(np.argmax(d - bound)))
    # the planted key dominates the rows after it (the route was taken, not skipped)
    assert np.all(rl[0, 0, j + 5:] > 50.0)


@pytest.mark.parametrize("j", [394, 740])
def test_bifocal_planted_key_long_branch(j):
    # the same planted rows through the two-branch kind: w0 = 200 puts the planted key in the
    # long-range branch (frequency interpolation, G = 4) for the rows 200 and more after it
    q, k, v, theta = planted(j)
    out, lse, _, _ = bfl.bifocal_prefill(q.cuda(), k.cuda(), v.cuda(), w0=200, w_pretrained=256, theta=theta)
    torch.cuda.synchronize()
    assert bfl.last_device_error() == 0
    ro, rl = R.bifocal_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(), 200, 256, theta)
    e = errors(out.cpu().float().numpy(), None, ro, None)
    assert e["max_abs"] <= MAX_ABS and e["rel_l2"] <= REL_L2, e
    # LSE: the rows' dominating products use the branch's operands, so bound sum_d |q~_d k~_d| by
    # |q_i| |k_j| (Cauchy-Schwarz; every RoPE form is a rotation, which keeps the norms), over the
    # row's largest-score key j
    qd, kd = q[0].double().numpy(), k[0].double().numpy()
    G = R.dynamic_factor(qd.shape[0], 256)
    omega, scale = R.rope_omega(128, theta), 1.0 / math.sqrt(128)
    s = np.stack([R.bifocal_scores(qd[:, h], kd[:, 0], np.arange(qd.shape[0]), 200, G, si.FREQ_INTERP, omega, scale)
                  for h in range(2)])
    jstar = np.argmax(s, axis=2)
    norm = np.linalg.norm(qd, axis=2).T * np.linalg.norm(kd[:, 0], axis=1)[jstar]
    bound = np.maximum(1e-3, scale * (2.0 ** -10 + 2.0 ** -20) * norm)
    d = np.abs(lse.cpu().numpy()[0] - rl[0])
    assert np.all(d <= bound), float(np.max(d - bound))

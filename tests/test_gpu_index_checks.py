"""Device-side index checks of the paged entry points (GPU; nothing faults).

The sequence lengths of a paged decode and the block tables of both paged entry points live in
device memory, where the host cannot validate them. A length outside [1, max_len] or a table
entry outside [0, pool_pages) is reported as STATUS_INDEX with the site of the check, and the
kernels neither read nor write the cache rows it would address.

Every bad input here is chosen so that even an unchecked access would stay inside memory the test
owns: the bad length belongs to sequence 0, so its table row and partial rows are followed by
sequence 1's, and the bad page index is one past the declared pool, inside two spare pages that
the pool tensor carries beyond what the call is told. The tests check that the spare pages are
untouched, that the other sequences still match the oracle, and that the next call is clean."""
import numpy as np
import torch

import oracle.bifocal_ref as R
import rope_context_extension_bifocal_b200 as bfl
import seeded_inputs as si
from tests.gpu_helpers import assert_close
import pytest

pytestmark = pytest.mark.gpu
THETA = 1e6
HQ, HKV, D, W0, WP, PAGE = 8, 2, 128, 300, 256, 16
SPARE = 2  # pages past the declared pool


def bf16_round(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float64)).to(torch.bfloat16).double().numpy()


def build_decode(seed, lens):
    B = len(lens)
    max_len = max(lens) + 3
    max_pages = (max_len + PAGE - 1) // PAGE
    g = si.generator(seed)
    pool_pages = sum((L + PAGE - 1) // PAGE for L in lens) + 3
    perm = torch.randperm(pool_pages, generator=g)
    table = torch.zeros(B, max_pages, dtype=torch.int32)
    nxt = 0
    for b, L in enumerate(lens):
        n = (L + PAGE - 1) // PAGE
        table[b, :n] = perm[nxt:nxt + n].to(torch.int32)
        nxt += n
    rows = (pool_pages + SPARE) * PAGE
    kfull = torch.randn(rows, HKV, D, generator=g).to(torch.bfloat16)
    vfull = torch.randn(rows, HKV, D, generator=g).to(torch.bfloat16)
    q = torch.randn(B, HQ, D, generator=g).to(torch.bfloat16)
    kn = torch.randn(B, HKV, D, generator=g).to(torch.bfloat16)
    vn = torch.randn(B, HKV, D, generator=g).to(torch.bfloat16)
    return dict(lens=lens, max_len=max_len, table=table, pool_pages=pool_pages, kfull=kfull, vfull=vfull, q=q,
                kn=kn, vn=vn)


def run_decode(c, lens_dev, table):
    kf, vf = c["kfull"].cuda(), c["vfull"].cuda()
    n = c["pool_pages"] * PAGE  # the pool the call is told about; the spare pages follow it
    out, lse = bfl.bifocal_decode_paged(c["q"].cuda(), c["kn"].cuda(), c["vn"].cuda(), kf[:n], vf[:n], PAGE,
                                        table.cuda(), torch.tensor(lens_dev, dtype=torch.int32).cuda(),
                                        c["max_len"], w0=W0, w_pretrained=WP, theta=THETA)
    torch.cuda.synchronize()
    return out, lse, kf.cpu(), vf.cpu()


def check_sequence(c, b, out, lse, kpool):
    L, t = c["lens"][b], c["table"]
    idx = [int(t[b, j // PAGE]) * PAGE + j % PAGE for j in range(L)]
    ref_k = c["kfull"][idx].double().numpy()
    ref_v = c["vfull"][idx].double().numpy()
    ref_k[L - 1] = bf16_round(R.rope_keys_for_cache(c["kn"][b][None].double().numpy(), THETA, start=L - 1)[0])
    ref_v[L - 1] = c["vn"][b].double().numpy()
    ro, rl = R.bifocal_decode_reference(c["q"][b].double().numpy(), ref_k, ref_v, L, W0, WP, THETA, si.FREQ_INTERP)
    assert_close(out[b].cpu().float().numpy(), lse[b].cpu().numpy(), ro, rl, f"paged b={b} L={L}")


def assert_clean_next_call():
    c = build_decode(77, [40, 500])
    out, lse, kp, _ = run_decode(c, c["lens"], c["table"])
    assert bfl.last_device_error() == 0
    for b in range(2):
        check_sequence(c, b, out, lse, kp)


def test_paged_decode_length_out_of_range():
    c = build_decode(70, [300, 900, 41])
    bad = list(c["lens"])
    bad[0] = c["max_len"] + 5  # past max_len, inside the table rows and partial rows of sequence 1
    out, lse, kp, vp = run_decode(c, bad, c["table"])
    word = bfl.device_status_word()
    assert word & 0xff == 3 and (word >> 8) in (50, 52), hex(word)  # the append or the partial saw it first
    assert bfl.last_device_error() == bfl.STATUS_INDEX
    assert torch.isnan(out[0].float()).all()  # nothing merged for the bad sequence
    for b in (1, 2):
        check_sequence(c, b, out, lse, kp)
    # the bad sequence appended nothing: every pool row other than the two appended ones is as built
    t = c["table"]
    written = {int(t[b, (c["lens"][b] - 1) // PAGE]) * PAGE + (c["lens"][b] - 1) % PAGE for b in (1, 2)}
    keep = [r for r in range(kp.shape[0]) if r not in written]
    assert torch.equal(kp[keep], c["kfull"][keep]) and torch.equal(vp[keep], c["vfull"][keep])
    assert_clean_next_call()


def test_paged_decode_table_entry_out_of_range():
    c = build_decode(71, [300, 900, 41])
    table = c["table"].clone()
    last = (c["lens"][1] - 1) // PAGE
    table[1, last] = c["pool_pages"]  # one past the declared pool: the first spare page
    out, lse, kp, vp = run_decode(c, c["lens"], table)
    word = bfl.device_status_word()
    assert word & 0xff == 3 and (word >> 8) in (51, 53), hex(word)  # the append or the partial's producer
    assert bfl.last_device_error() == bfl.STATUS_INDEX
    spare = slice(c["pool_pages"] * PAGE, None)
    assert torch.equal(kp[spare], c["kfull"][spare]) and torch.equal(vp[spare], c["vfull"][spare])
    for b in (0, 2):
        check_sequence(c, b, out, lse, kp)
    assert_clean_next_call()


def test_paged_chunk_table_entry_out_of_range():
    hq, hkv, wp, w0 = 4, 2, 512, 100
    cached, chunks = [200, 37], [150, 90]
    lens = [p + cc for p, cc in zip(cached, chunks)]
    B = 2
    max_pages = (max(lens) + PAGE - 1) // PAGE
    g = si.generator(72)
    pool_pages = sum((L + PAGE - 1) // PAGE for L in lens) + 1
    perm = torch.randperm(pool_pages, generator=g)
    table = torch.zeros(B, max_pages, dtype=torch.int32)
    nxt = 0
    for b, L in enumerate(lens):
        n = (L + PAGE - 1) // PAGE
        table[b, :n] = perm[nxt:nxt + n].to(torch.int32)
        nxt += n
    rows = (pool_pages + SPARE) * PAGE
    kfull = torch.zeros(rows, hkv, 128, dtype=torch.bfloat16)
    vfull = torch.zeros(rows, hkv, 128, dtype=torch.bfloat16)
    qs, ks, vs = [], [], []
    for b in range(B):
        q, k, v = si.random_qkv(720 + b, 1, lens[b], hq, hkv, 128, "bf16")
        pref = bf16_round(R.rope_keys_for_cache(k[0, :cached[b]].double().numpy(), THETA))
        for j in range(cached[b]):
            r = int(table[b, j // PAGE]) * PAGE + j % PAGE
            kfull[r] = torch.from_numpy(pref[j]).to(torch.bfloat16)
            vfull[r] = v[0, j]
        qs.append(q[0, cached[b]:])
        ks.append(k[0, cached[b]:])
        vs.append(v[0, cached[b]:])
    kfull[pool_pages * PAGE:] = 7.0  # sentinel in the spare pages
    vfull[pool_pages * PAGE:] = 7.0
    bad = table.clone()
    bad[0, (cached[0] + 5) // PAGE] = pool_pages  # a page that holds chunk rows of sequence 0
    kf, vf = kfull.cuda(), vfull.cuda()
    n = pool_pages * PAGE
    qp, kp_, vp_ = (torch.cat(x).cuda() for x in (qs, ks, vs))
    out, lse = bfl.bifocal_prefill_chunk_paged(qp, kp_, vp_, chunks, cached, kf[:n], vf[:n], PAGE, bad.cuda(),
                                               w0=w0, w_pretrained=wp, theta=THETA)
    torch.cuda.synchronize()
    word = bfl.device_status_word()
    assert word & 0xff == 3 and (word >> 8) in (54, 55), hex(word)  # the pool write or the tile load
    assert bfl.last_device_error() == bfl.STATUS_INDEX
    kh, vh = kf.cpu(), vf.cpu()
    assert torch.equal(kh[n:], kfull[n:]) and torch.equal(vh[n:], vfull[n:])
    # sequence 1 never touches the bad entry: it still matches the chunk oracle
    L, C, P0 = lens[1], chunks[1], cached[1]
    idx = [int(table[1, j // PAGE]) * PAGE + j % PAGE for j in range(L)]
    ro, rl = R.bifocal_chunk_reference(qs[1].double().numpy(), kh[idx].double().numpy(), vh[idx].double().numpy(),
                                       P0, w0, wp, THETA, si.FREQ_INTERP)
    assert_close(out[chunks[0]:].cpu().float().numpy(), lse[:, chunks[0]:].cpu().numpy(), ro, rl, "paged chunk b=1")
    assert_clean_next_call()

"""Run one prefill or decode case a few times on cuda:0 (for profilers and quick timing).

    python -m rope_context_extension_bifocal_b200.run_case prefill --L 32768 --hq 32 --hkv 8 --reps 3
    python -m rope_context_extension_bifocal_b200.run_case decode --L 131072 --reps 20

Inputs follow the seeded recipe (iid N(0,1) bf16). Prints the mean device time per call.
"""
from __future__ import annotations

import argparse
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main():
    import torch

    import rope_context_extension_bifocal_b200 as bfl
    import seeded_inputs as si

    ap = argparse.ArgumentParser()
    ap.add_argument("kind", choices=["prefill", "prefill_plain", "decode", "decode_plain"])
    ap.add_argument("--L", type=int, default=32768)
    ap.add_argument("--hq", type=int, default=32)
    ap.add_argument("--hkv", type=int, default=8)
    ap.add_argument("--D", type=int, default=128)
    ap.add_argument("--w0", type=int, default=4096)
    ap.add_argument("--w-pretrained", type=int, default=8192)
    ap.add_argument("--theta", type=float, default=1e6)
    ap.add_argument("--mode", default=si.FREQ_INTERP)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--flags", type=int, default=0, help="BF_FLAG_* bits for the bifocal calls")
    ap.add_argument("--no-warm", action="store_true", help="skip the untimed first call")
    a = ap.parse_args()
    dev = torch.device("cuda", 0)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if a.kind.startswith("prefill"):
        q, k, v = (t.to(dev) for t in si.random_qkv(3, 1, a.L, a.hq, a.hkv, a.D, "bf16"))
        p = bfl.make_params(a.hq, a.hkv, a.D, a.w0, a.w_pretrained, a.theta, a.mode)
        ws = torch.empty(bfl.prefill_workspace_size(bfl.DTYPE_BF16, 1, a.L, p), dtype=torch.uint8, device=dev)
        out = torch.empty(1, a.L, a.hq, a.D, dtype=torch.bfloat16, device=dev)

        def call():
            if a.kind == "prefill":
                bfl.bifocal_prefill(q, k, v, w0=a.w0, w_pretrained=a.w_pretrained, theta=a.theta, mode=a.mode,
                                    flags=a.flags, out=out, workspace=ws)
            else:
                bfl.rope_causal_prefill(q, k, v, theta=a.theta, out=out, workspace=ws)
        flops = 4.0 * a.L * a.L / 2 * a.D * a.hq
    else:
        cap = a.L + 16
        kc = torch.randn(cap, a.hkv, a.D, device=dev).to(torch.bfloat16)
        vc = torch.randn(cap, a.hkv, a.D, device=dev).to(torch.bfloat16)
        q = torch.randn(a.hq, a.D, device=dev).to(torch.bfloat16)
        kn = torch.randn(a.hkv, a.D, device=dev).to(torch.bfloat16)
        vn = torch.randn(a.hkv, a.D, device=dev).to(torch.bfloat16)
        p = bfl.make_params(a.hq, a.hkv, a.D, a.w0, a.w_pretrained, a.theta, a.mode)
        ws = torch.empty(bfl.decode_workspace_size(cap, p), dtype=torch.uint8, device=dev)
        out = torch.empty(a.hq, a.D, dtype=torch.bfloat16, device=dev)

        def call():
            if a.kind == "decode":
                bfl.bifocal_decode(q, kn, vn, kc, vc, a.L, w0=a.w0, w_pretrained=a.w_pretrained, theta=a.theta,
                                   mode=a.mode, out=out, workspace=ws)
            else:
                bfl.rope_causal_decode(q, kn, vn, kc, vc, a.L, theta=a.theta, out=out, workspace=ws)
        flops = 2.0 * 2 * a.L * a.hkv * a.D * 2  # bytes, reported as GB/s below
    if not a.no_warm:
        call()
    torch.cuda.synchronize()
    s.record()
    for _ in range(a.reps):
        call()
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / a.reps
    word = bfl.device_status_word()
    print(f"device status word: {word:#x}")
    if a.kind.startswith("prefill"):
        print(f"{a.kind} L={a.L}: {ms:.3f} ms/call, {flops / ms / 1e9:.1f} TFLOP/s")
    else:
        print(f"{a.kind} L={a.L}: {ms * 1e3:.1f} us/call, {flops / ms / 1e6:.1f} GB/s")
    assert word == 0, f"a bounded wait expired at site {word >> 8}"


if __name__ == "__main__":
    main()

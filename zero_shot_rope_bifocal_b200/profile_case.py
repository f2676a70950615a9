"""Run one hot-path kernel configuration a few times, for profilers.

    python -m zero_shot_rope_bifocal_b200.profile_case --case prefill --workload qwen3_8b_64k --L 16384
    python -m zero_shot_rope_bifocal_b200.profile_case --case decode --workload decode_8b_32k
    python -m zero_shot_rope_bifocal_b200.profile_case --case decode --two-form ...

Inputs are the seeded synthetic ones of ``synth``; sizes default to the named
workload, ``--L`` overrides the sequence length (keep captures small: a
profiler replays each captured launch many times).  Prints the mean
CUDA-event time per repetition of the timed call.
"""
from __future__ import annotations

import argparse
import sys

import torch

from . import jetlong as jl
from .synth import WORKLOADS, decode_inputs, prefill_inputs


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--case", choices=["prefill", "decode"], required=True)
    ap.add_argument("--workload", default=None)
    ap.add_argument("--L", type=int, default=None)
    ap.add_argument("--w0", type=int, default=None)
    ap.add_argument("--w-pretrained", type=int, default=None)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--two-form", action="store_true",
                    help="decode: read remote keys from the FP16 remote form of the cache")
    args = ap.parse_args(argv)
    name = args.workload or ("qwen3_8b_64k" if args.case == "prefill" else "decode_8b_32k")
    w = WORKLOADS[name]
    if args.L is not None:
        w = w.with_(L=args.L)
    if args.w0 is not None:
        w = w.with_(w0=args.w0)
    if args.w_pretrained is not None:
        w = w.with_(w_pretrained=args.w_pretrained)
    dev = torch.device("cuda", 0)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if args.case == "prefill":
        x = prefill_inputs(w, device=dev)
        out = torch.empty((w.B, w.L, w.Hq, w.D), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((w.B, w.Hq, w.L), dtype=torch.float32, device=dev)
        ws = torch.empty(jl.jetlong_prefill_workspace_size(w.B, w.Hq, w.Hkv, w.L, w.D),
                         dtype=torch.uint8, device=dev)
        jl.jetlong_prefill_rotate(x.k, x.v, w.w_pretrained, w.theta, ws)

        def call():
            jl.jetlong_prefill_attend(x.q, out, lse, w.Hkv, w.w_pretrained, w.w0, w.theta, ws)
    else:
        d = decode_inputs(w, device=dev)
        kc = torch.empty_like(d.k_raw)
        jl.jetlong_rope_cache(d.k_raw, kc, 0, w.theta)
        out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)
        ws = torch.empty(jl.jetlong_decode_workspace_size(w.B, w.Hq, w.Hkv, w.L, w.D),
                         dtype=torch.uint8, device=dev)

        if args.two_form:
            kr = torch.empty(kc.shape, dtype=torch.float16, device=dev)
            jl.jetlong_remote_cache(kc, kr, 0, w.L, w.L, w.w_pretrained, w.theta)

            def call():
                jl.jetlong_decode_two_form(d.q, kc, kr, d.v, w.L, w.w_pretrained, w.w0, w.theta,
                                           out=out, lse=lse, workspace=ws)
        else:
            def call():
                jl.jetlong_decode(d.q, kc, d.v, w.L, w.w_pretrained, w.w0, w.theta, out=out,
                                  lse=lse, workspace=ws)
    call()
    torch.cuda.synchronize()
    ev0.record()
    for _ in range(args.reps):
        call()
    ev1.record()
    torch.cuda.synchronize()
    st = jl.jetlong_device_status()
    print(f"{args.case} {name} L={w.L} w_pretrained={w.w_pretrained} w0={w.w0}: "
          f"{ev0.elapsed_time(ev1) / args.reps:.3f} ms/rep, "
          f"status {st}")
    return 0 if st == jl.JL_OK else 1


if __name__ == "__main__":
    sys.exit(main())

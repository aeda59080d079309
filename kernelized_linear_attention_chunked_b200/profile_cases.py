"""Small, self-contained launches of each kernel for Nsight Compute captures.

    python -m kernelized_linear_attention_chunked_b200.profile_cases CASE [--launches N]

Each case allocates its inputs once (a few hundred MB at most, but more than
the 126 MB L2 where DRAM traffic is the point), runs two warm-up launches and
then N profiled launches of one kernel, and exits. Cases:

  prefill_headline  kata_prefill, B=4 H=8 T=2048 d=32 bf16 chunk 64, output only
                    (the quadratic form: quad_kernel)
  prefill_headline_chunked  the same call in the chunked form (state_kernel,
                    readout_kernel)
  prefill_long      kata_prefill, B=2 H=16 T=4096 d=64 bf16 chunk 128
  decode            kata_decode_step, B=16 H=16 d=64 (state 138 MB > L2)
  sre               lola_sre_score_topk + merge, B=16 H=16 d=64, 192 candidates
"""
from __future__ import annotations

import argparse

import torch

import kernelized_linear_attention_chunked_b200 as kata
from kernelized_linear_attention_chunked_b200.inputs import (
    candidate_inputs, decode_inputs, prefill_inputs)


def case_prefill(B, H, T, d, chunk, n, form="auto"):
    q, k, v = (x.cuda() for x in prefill_inputs(B, H, T, d, dtype="bf16", seed=1))
    o = torch.empty(B, H, T, d, device="cuda")
    for _ in range(2 + n):
        kata.prefill(q, k, v, chunk=chunk, state=False, o=o, form=form)


def case_decode(n):
    B, H, d = 16, 16, 64
    _, _, q, k, v = decode_inputs(B, H, d, 1, 1, dtype="bf16", seed=3)
    D = d * (d + 1) // 2
    Hst = torch.randn(B, H, D, d, device="cuda") * 0.01
    s = torch.rand(B, H, D, device="cuda")
    q, k, v = q[0].cuda(), k[0].cuda(), v[0].cuda()
    o = torch.empty(B, H, d, device="cuda")
    for _ in range(2 + n):
        kata.decode_step(q, k, v, Hst, s, o=o)


def case_sre(n):
    B, H, d, m = 16, 16, 64, 192
    D = d * (d + 1) // 2
    Hst = torch.randn(B, H, D, d, device="cuda") * 0.01
    s = torch.rand(B, H, D, device="cuda")
    kc, vc, pos = (x.cuda() for x in candidate_inputs(B, H, m, d, dtype="bf16", seed=5))
    for _ in range(2 + n):
        kata.sre_score_topk(Hst, s, kc, vc, pos, keep=128, merge=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["prefill_headline", "prefill_headline_chunked",
                                     "prefill_long", "decode", "sre"])
    ap.add_argument("--launches", type=int, default=3)
    a = ap.parse_args()
    if a.case == "prefill_headline":
        case_prefill(4, 8, 2048, 32, 64, a.launches)
    elif a.case == "prefill_headline_chunked":
        case_prefill(4, 8, 2048, 32, 64, a.launches, form="chunked")
    elif a.case == "prefill_long":
        case_prefill(2, 16, 4096, 64, 128, a.launches, form="chunked")
    elif a.case == "decode":
        case_decode(a.launches)
    else:
        case_sre(a.launches)
    torch.cuda.synchronize()
    kata.sync_status()


if __name__ == "__main__":
    main()
